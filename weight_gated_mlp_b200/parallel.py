"""Context parallelism of the fast-weight MLP prefill: one sequence split into
G contiguous segments of whole chunks, segment r on rank r.

The chunk updates are additive, so the recurrence splits into three steps
around one exchange (the prefix-sum scheme of the pages: forum summary,
"Three Core Designs" item 2; iplexlaw review section 6, Algorithm 1 — the
deltas in parallel, an exclusive prefix sum, the application in parallel;
here a rank plays the part of a chunk):

1. delta:  rank r computes Z and the (clipped) targets of its segment and
   S_r, the sum of its chunk deltas.  With sequence-end padding it first
   receives the first k-1 rows of X0 of rank r+1, the look-ahead of its last
   tokens (the halo; a send/recv of (k-1) x d values);
2. prefix: P_r = S_0 + ... + S_{r-1}.  Exchange by all-to-all slices: rank q
   owns slice q of the flattened d x f matrix, receives that slice of every
   S_r, forms all G exclusive prefixes of it with the library's prefix
   kernel and returns row r to rank r.  Each rank sends and receives
   2 (G-1)/G x 4 d f bytes, where an all-gather of whole S_r moves
   (G-1) x 4 d f;
3. apply:  rank r runs the chunk recurrence of its segment from
   W_down0 + P_r: O of its tokens and W_end = W_down0 + P_r + S_r, the state
   after its segment (W_down_final of the sequence on the last rank).

The compute steps are an `ops` object (`CudaSegmentOps`: the CUDA library
through its C ABI); the exchange is torch.distributed (NCCL over NVLink).
`emulate_ranks` runs all G segments in turn on one device, with the prefix
over the stacked S_r, the same arithmetic without an exchange.
"""

from __future__ import annotations

from typing import Optional, Tuple

import weight_gated_mlp_b200 as ittt


class CudaSegmentOps:
    """The three compute steps of one segment on the GPU (CUDA library)."""

    def __init__(self, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float, C: int,
                 clip: float = 0.0, pad: str = "sequence"):
        if pad not in ("sequence", "chunk"):
            raise ValueError(f"pad must be 'sequence' or 'chunk', not {pad!r}")
        self.W_gate, self.W_up, self.W_down0 = W_gate, W_up, W_down0
        self.conv_kernel, self.W_target = conv_kernel, W_target
        self.eta, self.C, self.clip, self.pad = float(eta), int(C), float(clip), pad
        self.k = int(conv_kernel.shape[1])

    def delta(self, H, X0x, S_out=None):
        return ittt.cp_delta(H, X0x, self.W_gate, self.W_up, self.conv_kernel, self.W_target,
                             self.eta, self.C, clip=self.clip, pad=self.pad, S=S_out)

    def prefix(self, S_all):
        return ittt.cp_prefix(S_all)

    def apply(self, state, P):
        return ittt.cp_apply(state, self.W_down0, P)


def _halo_needed(ops, world: int) -> bool:
    return ops.pad == "sequence" and world > 1 and ops.k > 1


def exchange_halo(X0, T: int, k: int, group=None):
    """X0 of this rank's segment of T tokens with the first k-1 rows of the
    next rank's segment appended ([B, T + k - 1, d]); the last rank's X0
    unchanged.

    Every rank sends its first k-1 rows to rank - 1 and receives rank + 1's.
    X0 is [B, T, d], or [B, T + k - 1, d] with room for the halo (the extra
    rows are overwritten, which saves a copy of the segment)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    B, Tin, d = X0.shape
    if Tin not in (T, T + k - 1):
        raise ValueError(f"X0 has {Tin} rows, expected {T} or {T + k - 1}")
    last = rank == world - 1
    halo = torch.empty((B, k - 1, d), dtype=X0.dtype, device=X0.device)
    reqs = []
    if rank > 0:
        reqs.append(dist.isend(X0[:, : k - 1].contiguous(), _global(group, rank - 1), group=group))
    if not last:
        reqs.append(dist.irecv(halo, _global(group, rank + 1), group=group))
    for r in reqs:
        r.wait()
    if last:
        return X0[:, :T].contiguous() if Tin != T else X0
    if Tin == T + k - 1:
        X0[:, T:].copy_(halo)
        return X0
    out = torch.empty((B, T + k - 1, d), dtype=X0.dtype, device=X0.device)
    out[:, :T].copy_(X0)
    out[:, T:].copy_(halo)
    return out


def _global(group, rank: int) -> int:
    import torch.distributed as dist

    if group is None:
        return rank
    return dist.get_global_rank(group, rank)


def slice_len(total: int, world: int) -> int:
    """Length of one rank's slice of a flattened [B, d, f] matrix: total / G
    rounded up to a multiple of 64 floats (256-byte aligned slices)."""
    per = -(-total // world)
    return -(-per // 64) * 64


def exchange_prefix(S_padded, ops, group=None):
    """P_r (flattened, padded like S_padded) of this rank from every rank's S.

    S_padded: [G * slice] float32, this rank's S_r flattened and zero-padded.
    Collective over `group`: all-to-all of the slices, the prefix kernel on
    the G rows of the owned slice, all-to-all of the rows back."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    if world == 1:
        return torch.zeros_like(S_padded)
    sl = S_padded.numel() // world
    recv = torch.empty_like(S_padded)
    # row q of recv: slice `rank` of rank q's S
    dist.all_to_all_single(recv, S_padded, group=group)
    owned = ops.prefix(recv.view(world, sl))
    P = torch.empty_like(S_padded)
    # row q of owned (the prefix of ranks < q on this slice) goes to rank q
    dist.all_to_all_single(P, owned.reshape(-1).contiguous(), group=group)
    return P


def context_parallel_forward(H, X0, ops, group=None, final: str = "last"
                             ) -> Tuple[object, object]:
    """(O [B, T_r, d] of this rank's segment, W [B, d, f] fp32).

    H, X0: [B, T_r, d], this rank's segment of B sequences (rank order is
    sequence order; T_r a multiple of C; segments may differ in length).  X0
    may hold k-1 more rows as room for the halo.  W is this rank's W_end (the
    state after its segment: the sequence's W_down_final on the last rank)
    with final="last", or W_down_final on every rank with final="all" (one
    broadcast more).
    Collective: every rank of `group` calls it."""
    import torch
    import torch.distributed as dist

    if final not in ("last", "all"):
        raise ValueError(f"final must be 'last' or 'all', not {final!r}")
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T = H.shape[1]
    if _halo_needed(ops, world):
        X0x = exchange_halo(X0, T, ops.k, group)
    else:
        X0x = X0[:, :T].contiguous() if X0.shape[1] != T else X0
    B = H.shape[0]
    d, f = ops.W_down0.shape
    total = B * d * f
    sl = slice_len(total, world)
    S_padded = torch.empty(world * sl, dtype=torch.float32, device=H.device)
    S_padded[total:].zero_()
    S, state = ops.delta(H, X0x, S_out=S_padded[:total].view(B, d, f))
    P = exchange_prefix(S_padded, ops, group)
    O, W_end = ops.apply(state, P[:total].view(B, d, f))
    if final == "all" and world > 1:
        dist.broadcast(W_end, _global(group, world - 1), group=group)
    return O, W_end


def emulate_ranks(H, X0, ops, segments: int) -> Tuple[object, object]:
    """All `segments` segments of B sequences [B, T, d] on one device, in
    turn: every delta, the prefix over the stacked S_r (row r = P_r), every
    apply.  Returns (O [B, T, d], W_down_final [B, d, f])."""
    import torch

    B, T, d = H.shape
    if T % segments:
        raise ValueError("T must split into equal segments")
    Tr = T // segments
    k = ops.k
    dd, f = ops.W_down0.shape
    S_all = torch.empty((segments, B, dd, f), dtype=torch.float32, device=H.device)
    states = []
    for r in range(segments):
        s, e = r * Tr, (r + 1) * Tr
        stop = e + (k - 1 if (_halo_needed(ops, segments) and r < segments - 1) else 0)
        _, st = ops.delta(H[:, s:e].contiguous(), X0[:, s:stop].contiguous(), S_out=S_all[r])
        states.append(st)
    P_all = ops.prefix(S_all)
    outs = []
    W_end: Optional[object] = None
    for r, st in enumerate(states):
        O, W_end = ops.apply(st, P_all[r])
        outs.append(O)
    return torch.cat(outs, dim=1), W_end
