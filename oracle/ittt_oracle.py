"""CPU fp64 oracle for the In-Place TTT fast-weight MLP layer forward (prefill).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
module: only the tests, the smoke check and the benchmark's CPU-baseline leg
call it.  It shares no code with the CUDA library; the only shared module is
the seeded input generator (``synthetic``), which holds none of the layer's
arithmetic.

Sources (web pages about "In-Place Test-Time Training", Feng et al.):

* [notes]  "论文精读：In-Place Test-Time Training" (jindou-blog deep-read notes),
  sections "In-Place 设计：复用 MLP 的 W_down" (gated-MLP equation),
  "Chunk-Wise 更新机制" (update equation), "LM-Aligned 目标函数" (target eq.).
* [forum]  "In-Place TTT: ByteDance Seed's Test-Time Training Framework Gives
  LLMs On-the-Fly Memory", section "Three Core Designs", items 1-3.
* [review] iplexlaw blog review of "In-Place Test-Time Training"
  (2604.06169), sections 2 (W_down as fast weight), 3 (apply then update),
  4 (LM-aligned target), 6 (context parallelism, Algorithm 1).

What is computed, per sequence b (each starts from the shared W_down0: the
fast weight is reset at document boundaries, [review] section 6):

    Z      = silu(H W_gate^T) * (H W_up^T)                  [notes] gated MLP
    Y[t,c] = sum_j conv[c, j] * X0[t + j, c], X0 = 0 past T  [forum] 3, [review] 4
    Vhat   = Y W_target                                      [notes] target eq.
    for chunk i:   O_i = Z_i W^(i)^T                        [review] 3 (apply)
                   W^(i+1) = W^(i) + eta Vhat_i^T Z_i       [notes] update eq.
    W_down_final = W^(n)

Readings where the pages are silent or garbled (each one is listed in the
design notes of the repository):

* phi is SiLU, x * sigmoid(x) (the pages only write "phi").
* W_gate, W_up are [f, d] and W_down is [d, f] (the equations use H W^T and
  Z W_down^T); W_target is [d, d] applied untransposed as Y W_target.
* tap j of the depthwise kernel multiplies X0 at offset +j, so the kernel
  e_1 = [0, 1, 0, ...] with W_target = I gives Vhat_t = X0_{t+1}, the
  next-token special case of [forum] item 3; the sequence is zero-padded
  past its end only.
* the update is +eta Vhat_i^T Z_i with no 1/C normalisation; optional
  update-norm clipping rescales each chunk's delta to Frobenius norm <= tau.
* a ragged last chunk (T not a multiple of C) is simply shorter.
* padding of the conv: zero past the sequence end (default), or, as an
  option, zero past each chunk's end (no look-ahead across chunks); a
  continued segment may supply the next segment's first k-1 rows of X0.

Parity pins: every function here is pinned by tests under ``tests/``
(brute-force scalar loops, the eta = 0 plain-MLP special case against
torch, the next-token special case, sequential = prefix-scan = dual = hybrid form,
closed forms for C = 1 and C = T, affinity in eta, causality, batch
independence).  No function is "parity unpinned".
"""

from __future__ import annotations

from typing import Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=F64)


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x), evaluated without overflow for large |x|."""
    x = _f64(x)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = x[pos] / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = x[~pos] * ex / (1.0 + ex)
    return out


def gated_activations(H: np.ndarray, W_gate: np.ndarray, W_up: np.ndarray) -> np.ndarray:
    """Z = silu(H W_gate^T) * (H W_up^T): the gated-MLP hidden activations.

    [notes] "In-Place 设计" gated-MLP equation; [review] section 2.  H is [T, d],
    W_gate and W_up are [f, d]; returns Z [T, f] in fp64.
    """
    H = _f64(H)
    return silu(H @ _f64(W_gate).T) * (H @ _f64(W_up).T)


def lookahead_conv(X0: np.ndarray, conv_kernel: np.ndarray) -> np.ndarray:
    """Depthwise Conv1D over time that looks ahead: Y[t,c] = sum_j K[c,j] X0[t+j,c].

    X0 is taken as zero for t + j >= T.  [forum] "Three Core Designs" item 3
    (kernel [0,1,0,...] recovers the next token), [review] section 4.
    X0 is [T, d], conv_kernel [d, k]; returns Y [T, d] in fp64.
    """
    X0 = _f64(X0)
    K = _f64(conv_kernel)
    T, d = X0.shape
    k = K.shape[1]
    Y = np.zeros((T, d), dtype=F64)
    for j in range(k):
        if j >= T:
            break
        Y[: T - j] += X0[j:] * K[:, j][None, :]
    return Y


def lm_target(X0: np.ndarray, conv_kernel: np.ndarray, W_target: np.ndarray) -> np.ndarray:
    """Vhat = Conv1D(X0) W_target, the LM-aligned value target.

    [notes] "LM-Aligned 目标函数" equation; [review] section 4.  Returns [T, d].
    """
    return lookahead_conv(X0, conv_kernel) @ _f64(W_target)


def conv_rows(X0: np.ndarray, conv_kernel: np.ndarray, C: int, pad: str = "sequence",
              X0_next: Optional[np.ndarray] = None) -> np.ndarray:
    """The look-ahead conv of a whole sequence under a padding rule.

    pad = "sequence": X0 is zero past the end of the sequence, or continues with
    X0_next ([k-1, d], the next segment's first rows) when given.
    pad = "chunk": the look-ahead stops at the end of each chunk; X0 is zero
    past it ([review] section 6: chunk boundaries manage the padding so the
    target-generating convolution pulls no information from other chunks).
    """
    X0 = _f64(X0)
    T = X0.shape[0]
    if pad == "chunk":
        return np.concatenate([lookahead_conv(X0[s:e], conv_kernel)
                               for s, e in chunk_bounds(T, C)])
    if X0_next is not None:
        ext = np.concatenate([X0, _f64(X0_next)])
        return lookahead_conv(ext, conv_kernel)[:T]
    return lookahead_conv(X0, conv_kernel)


def chunk_bounds(T: int, C: int) -> list:
    """Non-overlapping chunks [iC, min((i+1)C, T)) ([notes] "Chunk-Wise 更新机制")."""
    if C <= 0:
        raise ValueError("chunk size must be positive")
    return [(s, min(s + C, T)) for s in range(0, T, C)]


def _sequence(inputs: Dict[str, np.ndarray], b: int):
    return (inputs["H"][b], inputs["X0"][b], inputs["W_gate"], inputs["W_up"],
            inputs["W_down0"], inputs["conv_kernel"], inputs["W_target"])


def forward_sequential_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float,
                           C: int, upto_chunk: Optional[int] = None, clip: float = 0.0,
                           pad: str = "sequence", X0_next: Optional[np.ndarray] = None
                           ) -> Tuple[np.ndarray, np.ndarray]:
    """The definition: chunk by chunk, apply with the current W, then update.

    [review] section 3 (apply-then-update: chunk i's output uses the state
    before chunk i's own update); [notes] "Chunk-Wise 更新机制" update
    W^(i+1) = W^(i) + eta Vhat_i^T Z_i.  One sequence: H, X0 are [T, d].
    Vhat_i reads X0 up to k-1 rows past the chunk end (zero past T).

    With ``upto_chunk`` the loop stops after that chunk: rows of later chunks
    of O are left zero and the returned W is W^(upto_chunk + 1).
    Returns (O [T, d], W_final [d, f]) in fp64.
    """
    T, d = H.shape
    k = conv_kernel.shape[1]
    W = _f64(W_down0).copy()
    O = np.zeros((T, d), dtype=F64)
    Wt = _f64(W_target)
    X0x = X0 if (X0_next is None or pad == "chunk") else np.concatenate([X0, X0_next])
    for i, (s, e) in enumerate(chunk_bounds(T, C)):
        if upto_chunk is not None and i > upto_chunk:
            break
        Z_i = gated_activations(H[s:e], W_gate, W_up)
        # the target of the chunk's tokens needs X0[s : e + k - 1] (X0[s : e]
        # when the look-ahead stops at the chunk end)
        stop = e if pad == "chunk" else min(e + k - 1, X0x.shape[0])
        win = lookahead_conv(X0x[s:stop], conv_kernel)[: e - s]
        O[s:e], W = apply_then_update(Z_i, win @ Wt, W, eta, clip)
    return O, W


def clip_delta(dW: np.ndarray, tau: float) -> np.ndarray:
    """Update-norm clipping: dW scaled to Frobenius norm <= tau (tau <= 0: off).

    [review] section 6 (the Frobenius norm of the update delta is limited to
    a threshold).  Reading: each chunk's delta dW_i = eta Vhat_i^T Z_i is
    rescaled on its own, dW_i * min(1, tau / ||dW_i||_F); tau is a parameter.
    """
    if tau <= 0:
        return dW
    nrm = float(np.linalg.norm(dW))
    return dW * (tau / nrm) if nrm > tau else dW


def apply_then_update(Z_i: np.ndarray, V_i: np.ndarray, W: np.ndarray, eta: float,
                      clip: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """One chunk: O_i = Z_i W^T with the current state, then W + eta V_i^T Z_i.

    [review] section 3 (apply first, update after); [notes] "Chunk-Wise 更新机制".
    Z_i is [c, f], V_i is [c, d], W is [d, f].  clip > 0 bounds the delta's
    Frobenius norm (see clip_delta).
    """
    Z_i, V_i, W = _f64(Z_i), _f64(V_i), _f64(W)
    return Z_i @ W.T, W + clip_delta(eta * (V_i.T @ Z_i), clip)


def chunk_recurrence(Z: np.ndarray, V: np.ndarray, W_down0: np.ndarray, eta: float, C: int,
                     clip: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """The chunk loop on given activations Z [T, f] and targets V [T, d]."""
    T = Z.shape[0]
    W = _f64(W_down0).copy()
    O = np.zeros((T, W.shape[0]), dtype=F64)
    for s, e in chunk_bounds(T, C):
        O[s:e], W = apply_then_update(Z[s:e], V[s:e], W, eta, clip)
    return O, W


def forward_sequential(inputs: Dict[str, np.ndarray], eta: float, C: int, clip: float = 0.0,
                       pad: str = "sequence", W_start: Optional[np.ndarray] = None
                       ) -> Tuple[np.ndarray, np.ndarray]:
    """Batched definition: every sequence b starts from the shared W_down0.

    Returns (O [B, T, d], W_final [B, d, f]) in fp64.  inputs may hold
    "X0_next" [B, k-1, d] (the next segment's first rows); W_start [B, d, f]
    replaces W_down0 per sequence (a continued segment).
    """
    B = inputs["H"].shape[0]
    outs = []
    for b in range(B):
        args = list(_sequence(inputs, b))
        if W_start is not None:
            args[4] = W_start[b]
        nxt = inputs["X0_next"][b] if "X0_next" in inputs else None
        outs.append(forward_sequential_one(*args, eta, C, clip=clip, pad=pad, X0_next=nxt))
    return np.stack([o for o, _ in outs]), np.stack([w for _, w in outs])


def forward_prefix_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float, C: int,
                       clip: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """The parallel form ([review] section 6, Algorithm 1; [forum] item 2).

    Step 1: every chunk's activations and update delta, independently.
    Step 2: exclusive prefix sum of the deltas over chunks.
    Step 3: effective fast weight of chunk i = W_down0 + that prefix.
    Step 4: every chunk's output with its effective weight.
    """
    T, _ = H.shape
    Z = gated_activations(H, W_gate, W_up)
    V = lm_target(X0, conv_kernel, W_target)
    bounds = chunk_bounds(T, C)
    deltas = [clip_delta(eta * (V[s:e].T @ Z[s:e]), clip) for s, e in bounds]   # step 1
    prefix = []                                                        # step 2
    acc = np.zeros_like(_f64(W_down0))
    for dW in deltas:
        prefix.append(acc.copy())
        acc = acc + dW
    O = np.zeros((T, H.shape[1]), dtype=F64)
    for (s, e), P in zip(bounds, prefix):
        W_eff = _f64(W_down0) + P                                      # step 3
        O[s:e] = Z[s:e] @ W_eff.T                                      # step 4
    return O, _f64(W_down0) + acc


def forward_dual_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float, C: int,
                     clip: float = 0.0) -> Tuple[np.ndarray, np.ndarray]:
    """The dual form, an exact rewrite of the recurrence (not printed on the pages).

    Expanding W^(i) = W_down0 + eta sum_{j<i} Vhat_j^T Z_j inside O_i = Z_i W^(i)^T
    gives O_i = Z_i W_down0^T + eta sum_{j<i} (Z_i Z_j^T) Vhat_j, and
    W_final = W_down0 + eta Vhat^T Z over the whole sequence.  Clipping scales
    chunk j's delta by s_j, i.e. replaces Vhat_j by s_j Vhat_j.
    """
    T, _ = H.shape
    Z = gated_activations(H, W_gate, W_up)
    V = lm_target(X0, conv_kernel, W_target)
    W0 = _f64(W_down0)
    if clip > 0:
        for s, e in chunk_bounds(T, C):
            nrm = abs(eta) * float(np.linalg.norm(V[s:e].T @ Z[s:e]))
            if nrm > clip:
                V[s:e] *= clip / nrm
    O = Z @ W0.T
    for i, (s, e) in enumerate(chunk_bounds(T, C)):
        if s == 0:
            continue
        O[s:e] += eta * ((Z[s:e] @ Z[:s].T) @ V[:s])
    return O, W0 + eta * (V.T @ Z)


def forward_hybrid_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float, C: int,
                       clip: float = 0.0, m: int = 2) -> Tuple[np.ndarray, np.ndarray]:
    """Groups of m chunks: the fast weight at each group's first chunk, the
    dual rewrite inside the group (an exact rewrite, not printed on the pages).

    With g the first chunk of the group holding chunk i,
    W^(g) = W_down0 + eta sum_{j<g} Vhat_j^T Z_j, and expanding the
    recurrence from W^(g) instead of W_down0 gives
    O_i = Z_i W^(g)^T + eta sum_{g<=j<i} (Z_i Z_j^T) Vhat_j.  m = 1 is the
    prefix form, m >= n the dual form; the last group may be shorter.
    Clipping replaces Vhat_j by s_j Vhat_j as in the dual form.
    """
    if m < 1:
        raise ValueError("m >= 1")
    T, _ = H.shape
    Z = gated_activations(H, W_gate, W_up)
    V = lm_target(X0, conv_kernel, W_target)
    bounds = chunk_bounds(T, C)
    if clip > 0:
        for s, e in bounds:
            nrm = abs(eta) * float(np.linalg.norm(V[s:e].T @ Z[s:e]))
            if nrm > clip:
                V[s:e] *= clip / nrm
    W0 = _f64(W_down0)
    O = np.zeros((T, H.shape[1]), dtype=F64)
    for g in range(0, len(bounds), m):
        gs = bounds[g][0]                                  # first token of the group
        W_g = W0 + eta * (V[:gs].T @ Z[:gs])               # fast weight at the group's start
        for s, e in bounds[g:g + m]:
            O[s:e] = Z[s:e] @ W_g.T
            if s > gs:
                O[s:e] += eta * ((Z[s:e] @ Z[gs:s].T) @ V[gs:s])
    return O, W0 + eta * (V.T @ Z)


def forward(inputs: Dict[str, np.ndarray], eta: float, C: int, form: str = "sequential",
            clip: float = 0.0, m: int = 2) -> Tuple[np.ndarray, np.ndarray]:
    """Batched forward in one of the four forms ("sequential", "prefix",
    "dual", "hybrid" with groups of m chunks)."""
    fn = dict(sequential=forward_sequential_one, prefix=forward_prefix_one,
              dual=forward_dual_one, hybrid=forward_hybrid_one)[form]
    kw = dict(clip=clip, m=m) if form == "hybrid" else dict(clip=clip)
    B = inputs["H"].shape[0]
    outs = [fn(*_sequence(inputs, b), eta, C, **kw) for b in range(B)]
    return np.stack([o for o, _ in outs]), np.stack([w for _, w in outs])


# --------------------------------------------------------------------------
# Sampled evaluation for full-size workloads: only what a test samples.
# --------------------------------------------------------------------------

def w_final_block(inputs: Dict[str, np.ndarray], b: int, eta: float,
                  rows: Sequence[int], cols: Sequence[int]) -> np.ndarray:
    """W_final[rows][:, cols] of sequence b.

    W_final = W_down0 + eta sum_i Vhat_i^T Z_i = W_down0 + eta Vhat^T Z (the
    chunk sums add up to the whole-sequence sum).  Only the needed columns of
    Vhat ([T, |rows|]) and of Z ([T, |cols|]) are formed.
    """
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    H, X0, W_gate, W_up, W0, K, Wt = _sequence(inputs, b)
    Zc = gated_activations(H, W_gate[cols], W_up[cols])               # [T, |cols|]
    Vr = lookahead_conv(X0, K) @ _f64(Wt)[:, rows]                     # [T, |rows|]
    return _f64(W0)[np.ix_(rows, cols)] + eta * (Vr.T @ Zc)


def output_rows(inputs: Dict[str, np.ndarray], b: int, eta: float, C: int,
                tokens: Iterable[int], clip: float = 0.0) -> np.ndarray:
    """O[tokens] of sequence b, running the definition only as far as needed."""
    tokens = sorted(set(int(t) for t in tokens))
    last_chunk = max(tokens) // C
    H, X0, W_gate, W_up, W0, K, Wt = _sequence(inputs, b)
    T, d = H.shape
    k = K.shape[1]
    W = _f64(W0).copy()
    out = {}
    for i, (s, e) in enumerate(chunk_bounds(T, C)):
        if i > last_chunk:
            break
        want = [t for t in tokens if s <= t < e]
        if want:
            Zw = gated_activations(H[want], W_gate, W_up)
            for t, z in zip(want, Zw @ W.T):
                out[t] = z
        if i < last_chunk:
            Z_i = gated_activations(H[s:e], W_gate, W_up)
            V_i = lookahead_conv(X0[s:min(e + k - 1, T)], K)[: e - s] @ _f64(Wt)
            W = W + clip_delta(eta * (V_i.T @ Z_i), clip)
    return np.stack([out[t] for t in tokens])


# --------------------------------------------------------------------------
# Closed form of single rows of O, for late chunks of long sequences.
# --------------------------------------------------------------------------

def target_rows(inputs: Dict[str, np.ndarray], b: int, s0: int, s1: int,
                pad: str = "sequence", C: Optional[int] = None) -> np.ndarray:
    """Vhat[s0:s1] of sequence b (the rows of lm_target / conv_rows @ W_target).

    Row t reads X0[t .. t+k-1]; past the sequence end X0 is zero, and with
    pad = "chunk" also past the end of t's chunk ([review] section 6).
    """
    H, X0, _, _, _, K, Wt = _sequence(inputs, b)
    T = X0.shape[0]
    k = K.shape[1]
    pieces = [(s0, s1)]
    if pad == "chunk":
        pieces = [(max(s, s0), min(e, s1)) for s, e in chunk_bounds(T, C) if s < s1 and e > s0]
    out = []
    for a, e in pieces:
        stop = min(e + k - 1, T)
        if pad == "chunk":
            stop = min(stop, (a // C + 1) * C)
        out.append(lookahead_conv(X0[a:stop], K)[: e - a])
    return np.concatenate(out) @ _f64(Wt)


def update_terms(inputs: Dict[str, np.ndarray], b: int, tokens: Sequence[int],
                 bounds: Sequence[int], pad: str = "sequence", C: Optional[int] = None,
                 block: int = 1024) -> Dict[int, np.ndarray]:
    """U[S] = sum_{s < S} (Z_t . Z_s) Vhat_s for the rows t of `tokens`, at
    every token boundary S of `bounds`: a dict S -> [len(tokens), d] (fp64).

    This is the update's contribution to O_t when every token before S has
    updated the state: expanding W = W_down0 + eta sum_{s<S} Vhat_s^T Z_s
    (the chunk sums of the update equation, [notes] "Chunk-Wise 更新机制")
    inside O_t = Z_t W^T gives O_t = Z_t W_down0^T + eta U[S]_t.  Z_s and
    Vhat_s are formed block by block, so memory stays O(block (d + f)).
    """
    H, _, W_gate, W_up, _, _, _ = _sequence(inputs, b)
    Zt = gated_activations(H[list(tokens)], W_gate, W_up)          # [m, f]
    d = inputs["W_down0"].shape[0]
    acc = np.zeros((len(tokens), d), dtype=F64)
    out = {}
    s = 0
    for S in sorted(set(int(x) for x in bounds)):
        while s < S:
            e = min(s + block, S)
            Zs = gated_activations(H[s:e], W_gate, W_up)              # [e - s, f]
            acc += (Zt @ Zs.T) @ target_rows(inputs, b, s, e, pad, C)
            s = e
        out[S] = acc.copy()
    return out


def output_rows_closed_form(inputs: Dict[str, np.ndarray], b: int, eta: float, C: int,
                            tokens: Sequence[int], pad: str = "sequence",
                            U: Optional[Dict[int, np.ndarray]] = None,
                            tokens_of_U: Optional[Sequence[int]] = None
                            ) -> Tuple[np.ndarray, np.ndarray]:
    """O[tokens] of sequence b from the closed form of the recurrence.

    Token t of chunk i is applied with W^(i) = W_down0 + eta sum_{s < iC}
    Vhat_s^T Z_s ([review] section 3: the chunk's own update comes after its
    output), so O_t = Z_t W_down0^T + eta sum_{s < iC} (Z_t . Z_s) Vhat_s.
    A ragged last chunk starts at iC as well.  U (from update_terms over the
    rows tokens_of_U, a superset of tokens) may be passed in to share the
    sums between chunk sizes.  Returns (O rows, Z_t W_down0^T rows), the
    second being the output without any update.  No clipping.
    """
    tokens = [int(t) for t in tokens]
    starts = [(t // C) * C for t in tokens]
    if U is None:
        U = update_terms(inputs, b, tokens, starts, pad, C)
        tokens_of_U = tokens
    where = {t: j for j, t in enumerate(tokens_of_U)}
    H, _, W_gate, W_up, W0, _, _ = _sequence(inputs, b)
    plain = gated_activations(H[tokens], W_gate, W_up) @ _f64(W0).T
    upd = np.stack([U[S][where[t]] for t, S in zip(tokens, starts)])
    return plain + eta * upd, plain
