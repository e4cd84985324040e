"""GPU parity of the context-parallel steps (ittt_cp_delta, ittt_cp_prefix,
ittt_cp_apply): G segments of one sequence run in turn on one GPU, the
prefix over the stacked segment sums, and the concatenated outputs and the
last segment's state must match the oracle's forward of the whole sequence.
Ranks that exchange over NCCL are covered on the CPU (test_context_parallel.py);
a one-rank NCCL group runs the same entry point here."""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case, workload
from weight_gated_mlp_b200 import parallel

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu


def _ops(dev, eta, C, clip=0.0, pad="sequence"):
    return parallel.CudaSegmentOps(dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
                                   dev["W_target"], eta, C, clip=clip, pad=pad)


CASES = [
    # dtype, T, C, d, f, k, B, segments, pad, clip
    ("bf16", 2048, 256, 320, 1000, 4, 1, 2, "sequence", 0.0),
    ("bf16", 2048, 256, 320, 1000, 4, 2, 4, "sequence", 0.0),
    ("bf16", 1536, 128, 256, 776, 5, 1, 3, "chunk", 0.0),
    ("bf16", 2048, 256, 192, 512, 4, 2, 2, "sequence", "clip"),
    ("f32", 512, 64, 64, 256, 4, 2, 4, "sequence", 0.0),
    ("f32", 512, 64, 64, 256, 3, 1, 2, "chunk", "clip"),
]


def _tau(inp, eta, C):
    Z = orc.gated_activations(inp["H"][0], inp["W_gate"], inp["W_up"])
    V = orc.lm_target(inp["X0"][0], inp["conv_kernel"], inp["W_target"])
    norms = [abs(eta) * np.linalg.norm(V[s:e].T @ Z[s:e]) for s, e in orc.chunk_bounds(Z.shape[0], C)]
    return 0.5 * float(np.median(norms))


@pytest.mark.parametrize("dtype,T,C,d,f,k,B,segments,pad,clip", CASES)
def test_emulated_ranks_match_the_oracle(dtype, T, C, d, f, k, B, segments, pad, clip):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype=dtype)
    inp = make_inputs(w)
    tau = _tau(inp, w.eta, C) if clip == "clip" else 0.0
    dev = to_device(inp, dtype)
    O, Wf = parallel.emulate_ranks(dev["H"], dev["X0"], _ops(dev, w.eta, C, tau, pad), segments)
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, clip=tau, pad=pad)
    assert rel_err(host(O), Oref) <= TOL[dtype]
    assert rel_err(host(Wf), Wref) <= TOL[dtype]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(host(Wf) - W0, Wref - W0) <= (1e-2 if dtype == "bf16" else 1e-4)


@pytest.mark.parametrize("G,n,offset", [(5, 4099, 0), (7, 1 << 16, 0), (3, 1 << 12, 1), (1, 64, 0)])
def test_prefix_is_the_ordered_fp32_sum(G, n, offset):
    """Row g = S[0] + ... + S[g-1] added in that order in fp32: the same adds
    on the host give the same bits (n % 4 == 0 and aligned: the float4 path;
    otherwise the scalar one)."""
    rng = np.random.default_rng(G * 31 + n)
    S = rng.standard_normal((G, n)).astype(np.float32)
    want = np.zeros_like(S)
    for g in range(1, G):
        want[g] = want[g - 1] + S[g - 1]
    buf = torch.empty(G * n + offset, dtype=torch.float32, device="cuda")
    dS = buf[offset:].view(G, n)
    dS.copy_(torch.from_numpy(S))
    P = ittt.cp_prefix(dS)
    assert ittt.get_last_error() == ittt.OK
    assert np.array_equal(P.cpu().numpy(), want)


def test_cp_entry_points_reject_bad_arguments():
    w = small_case(T=512, C=128, d=64, f=128, k=4, B=1, eta=0.01, dtype="bf16")
    dev = to_device(make_inputs(w), "bf16")
    S, st = ittt.cp_delta(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["conv_kernel"],
                          dev["W_target"], w.eta, w.C)
    lib = ittt.load_library()
    S2 = torch.empty((2, 8), dtype=torch.float32, device="cuda")
    # overlapping input and output
    assert lib.ittt_cp_prefix(S2.data_ptr(), 2, 8, S2.data_ptr() + 4, None) == ittt.ERR_INVALID_ARG
    assert lib.ittt_cp_prefix(S2.data_ptr(), 0, 8, S2.data_ptr(), None) == ittt.ERR_INVALID_ARG
    # workspace too small for the apply step
    p = st.p
    P = torch.zeros_like(S)
    O = torch.empty((1, 512, 64), dtype=torch.bfloat16, device="cuda")
    We = torch.empty_like(S)
    import ctypes
    assert lib.ittt_cp_apply(ctypes.byref(p), dev["W_down0"].data_ptr(), P.data_ptr(),
                             S.data_ptr(), O.data_ptr(), We.data_ptr(), st.workspace.data_ptr(),
                             16, None) == ittt.ERR_WORKSPACE
    # S missing
    assert lib.ittt_cp_apply(ctypes.byref(p), dev["W_down0"].data_ptr(), P.data_ptr(), None,
                             O.data_ptr(), We.data_ptr(), st.workspace.data_ptr(),
                             st.workspace.numel(), None) == ittt.ERR_INVALID_ARG
    assert ittt.get_last_error() == ittt.OK


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_group_equals_the_forward():
    import torch.distributed as dist

    w = small_case(T=1024, C=256, d=256, f=512, k=4, B=1, eta=0.01, dtype="bf16")
    inp = make_inputs(w)
    dev = to_device(inp, "bf16")
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    try:
        O, W = parallel.context_parallel_forward(dev["H"], dev["X0"], _ops(dev, w.eta, w.C))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C)
    assert rel_err(host(O), Oref) <= TOL["bf16"]
    assert rel_err(host(W), Wref) <= TOL["bf16"]


def test_full_size_two_segments_sampled():
    """qwen3-4b (T = 8192, C = 512) as two segments of 4096 tokens: blocks of
    W_down_final and rows of O of both segments against the oracle."""
    w = workload("qwen3-4b")
    inp = make_inputs(w, seed=0)
    dev = to_device(inp, "bf16")
    O, Wf = parallel.emulate_ranks(dev["H"], dev["X0"], _ops(dev, w.eta, w.C), 2)
    assert ittt.get_last_error() == ittt.OK
    del dev
    rng = np.random.default_rng(99)
    rows = np.sort(rng.choice(w.d, 12, replace=False))
    cols = np.sort(rng.choice(w.f, 24, replace=False))
    ref = orc.w_final_block(inp, 0, w.eta, rows, cols)
    got = host(Wf[0])[np.ix_(rows, cols)]
    assert rel_err(got, ref) <= TOL["bf16"]
    W0 = inp["W_down0"].astype(np.float64)[np.ix_(rows, cols)]
    assert rel_err(got - W0, ref - W0) <= 1e-2
    # the last rows of segment 0, the first rows of segment 1, one late chunk
    toks = [4095 - 511, 4095, 4096, 4096 + 100, 8191 - 600, 8191]
    ref_rows = orc.output_rows(inp, 0, w.eta, w.C, toks)
    got_rows = host(O[0])[toks]
    assert rel_err(got_rows, ref_rows) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_uneven_segments_through_the_three_steps(dtype):
    """Segments of different lengths (one, four and two chunks), driven
    through the entry points directly: the order of ranks, each rank's own
    problem size and the halo rows are what make the result exact."""
    C = 256 if dtype == "bf16" else 64
    lengths = [C, 4 * C, 2 * C]
    T = sum(lengths)
    w = small_case(T=T, C=C, d=192, f=384, k=4, B=2, eta=0.01, dtype=dtype)
    inp = make_inputs(w)
    dev = to_device(inp, dtype)
    ops = _ops(dev, w.eta, C)
    bounds = np.cumsum([0] + lengths)
    S_all = torch.empty((len(lengths), 2, w.d, w.f), dtype=torch.float32, device="cuda")
    states = []
    for r in range(len(lengths)):
        s0, s1 = int(bounds[r]), int(bounds[r + 1])
        stop = s1 + (w.k - 1 if r < len(lengths) - 1 else 0)
        _, st = ops.delta(dev["H"][:, s0:s1].contiguous(), dev["X0"][:, s0:stop].contiguous(),
                          S_out=S_all[r])
        states.append(st)
    P_all = ops.prefix(S_all)
    res = [ops.apply(st, P_all[r]) for r, st in enumerate(states)]
    outs, W_end = [o for o, _ in res], res[-1][1]
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, C)
    assert rel_err(host(torch.cat(outs, dim=1)), Oref) <= TOL[dtype]
    assert rel_err(host(W_end), Wref) <= TOL[dtype]
