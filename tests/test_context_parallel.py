"""Context parallelism on the CPU: gloo ranks run the orchestration of
weight_gated_mlp_b200.parallel (halo exchange, all-to-all slices, prefix,
rows back) with the oracle as the compute, and the concatenated outputs and
the last rank's state must equal the oracle's forward of the whole sequence.
The CUDA steps behind the same interface are checked on the GPU
(test_gpu_context_parallel.py)."""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from oracle import ittt_oracle as orc  # noqa: E402
from synthetic import make_inputs, small_case  # noqa: E402
from weight_gated_mlp_b200 import parallel  # noqa: E402

from _cp_oracle_ops import OracleSegmentOps  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case(T, C, d, f, k, B, seed=3):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.2, dtype="f32")
    return make_inputs(w, seed=seed)


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _worker(rank, world, port, cfg, out):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        inp = _case(*cfg["shape"])
        ops = OracleSegmentOps(inp, 0.2, cfg["C"], clip=cfg["clip"], pad=cfg["pad"])
        bounds = np.cumsum([0] + cfg["lengths"])
        s, e = int(bounds[rank]), int(bounds[rank + 1])
        H = torch.from_numpy(inp["H"][:, s:e].copy())
        X0 = inp["X0"][:, s:e]
        if cfg["room"]:          # room for the halo, filled with junk
            X0 = np.concatenate([X0, np.full((X0.shape[0], ops.k - 1, X0.shape[2]), 7.0)], 1)
        O, W = parallel.context_parallel_forward(H, torch.from_numpy(X0.copy()), ops,
                                                 final=cfg["final"])
        out[rank] = (O.numpy(), W.numpy())
    finally:
        dist.destroy_process_group()


def _run(world, cfg):
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, cfg, out), nprocs=world, join=True)
        return dict(out)


CFGS = [
    # world, lengths (tokens per rank), C, pad, clip, room, final
    (2, [16, 16], 8, "sequence", 0.0, False, "last"),
    (3, [16, 8, 24], 8, "sequence", 0.0, True, "all"),
    (3, [8, 16, 16], 8, "chunk", 0.0, False, "last"),
    (2, [24, 16], 8, "sequence", 0.05, False, "all"),
    (4, [8, 16, 8, 24], 8, "sequence", 0.0, True, "last"),
]


@pytest.mark.parametrize("world,lengths,C,pad,clip,room,final", CFGS)
def test_gloo_ranks_reproduce_the_whole_sequence(world, lengths, C, pad, clip, room, final):
    T = sum(lengths)
    # d * f * B = 5 * 12 * 2 = 120: not a multiple of the slice count
    shape = (T, C, 5, 12, 4, 2)
    cfg = dict(shape=shape, C=C, pad=pad, clip=clip, lengths=lengths, room=room, final=final)
    res = _run(world, cfg)
    inp = _case(*shape)
    Oref, Wref = orc.forward_sequential(inp, 0.2, C, clip=clip, pad=pad)
    O = np.concatenate([res[r][0] for r in range(world)], axis=1)
    assert _rel(O, Oref) < 1e-6
    assert _rel(res[world - 1][1], Wref) < 1e-6
    if final == "all":
        for r in range(world):
            assert np.array_equal(res[r][1], res[world - 1][1])
    else:
        # W_end of rank r: the state after its segment
        for r in range(world - 1):
            upto = sum(lengths[: r + 1]) // C - 1
            _, Wr = orc.forward_sequential_one(*[inp[k][0] if k in ("H", "X0") else inp[k] for k in (
                "H", "X0", "W_gate", "W_up", "W_down0", "conv_kernel", "W_target")], 0.2, C,
                upto_chunk=upto, clip=clip, pad=pad)
            assert _rel(res[r][1][0], Wr) < 1e-6
    if clip > 0:  # clipping is active in this case
        _, Wfree = orc.forward_sequential(inp, 0.2, C, pad=pad)
        W0 = inp["W_down0"].astype(np.float64)
        assert _rel(Wfree - W0, Wref - W0) > 0.05


def test_slice_len_covers_and_aligns():
    for total in (1, 63, 64, 120, 2560 * 9728):
        for world in (1, 2, 3, 8):
            sl = parallel.slice_len(total, world)
            assert sl % 64 == 0 and sl * world >= total and (sl - 64) * world < total


@pytest.mark.parametrize("segments,pad,clip", [(2, "sequence", 0.0), (4, "sequence", 0.05),
                                               (4, "chunk", 0.0)])
def test_emulated_ranks_reproduce_the_whole_sequence(segments, pad, clip):
    T, C = 32, 8
    inp = _case(T, C, 6, 10, 3, 2)
    ops = OracleSegmentOps(inp, 0.2, C, clip=clip, pad=pad)
    O, W = parallel.emulate_ranks(torch.from_numpy(inp["H"]), torch.from_numpy(inp["X0"]), ops,
                                  segments)
    Oref, Wref = orc.forward_sequential(inp, 0.2, C, clip=clip, pad=pad)
    assert _rel(O.numpy(), Oref) < 1e-6
    assert _rel(W.numpy(), Wref) < 1e-6


def test_dropped_halo_is_detected():
    """A wrong halo (zeros instead of the next segment's rows) changes the
    answer under sequence-end padding: the halo exchange is not vacuous."""
    T, C = 32, 8
    inp = _case(T, C, 6, 10, 3, 1)
    ops = OracleSegmentOps(inp, 0.2, C)
    H = torch.from_numpy(inp["H"])
    X0 = inp["X0"]
    Sa, sa = ops.delta(H[:, :16], torch.from_numpy(np.concatenate(
        [X0[:, :16], np.zeros((1, 2, 6))], 1)))
    Sb, sb = ops.delta(H[:, 16:], torch.from_numpy(X0[:, 16:].copy()))
    P = ops.prefix(torch.stack([Sa, Sb]))
    Oa, _ = ops.apply(sa, P[0])
    Ob, Wb = ops.apply(sb, P[1])
    Oref, Wref = orc.forward_sequential(inp, 0.2, C)
    assert _rel(Wb.numpy(), Wref) > 1e-4


def _leaver(rank, world, port, out):
    """Rank 1 leaves before the exchange (between steps, nothing in flight);
    rank 0 must get an error from its next collective, not wait for ever."""
    import time

    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=10))
    if rank == 1:
        dist.destroy_process_group()
        out[rank] = "left"
        return
    inp = _case(16, 8, 5, 12, 4, 1)
    ops = OracleSegmentOps(inp, 0.2, 8)
    t0 = time.monotonic()
    try:
        parallel.context_parallel_forward(torch.from_numpy(inp["H"][:, :8].copy()),
                                          torch.from_numpy(inp["X0"][:, :8].copy()), ops)
        out[rank] = ("returned", time.monotonic() - t0)
    except Exception as e:  # the dead peer surfaces as an error
        out[rank] = (type(e).__name__, time.monotonic() - t0)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_a_rank_that_leaves_is_an_error_on_its_peer():
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_leaver, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[1] == "left"
    outcome, secs = res[0]
    assert outcome != "returned" and secs < 60
