"""GPU parity: the CUDA path through the C ABI against the CPU fp64 oracle,
element by element on the same seeded inputs.

Tolerance (normwise relative error, ||x - x_oracle||_F / ||x_oracle||_F):
5e-3 for the bf16 path (bf16 storage, fp32 accumulation) and 1e-5 for the
fp32 path, on O and on W_down_final.
"""

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case, workload

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu


def _run(w, seed=0, form="auto", eta=None):
    inp = make_inputs(w, seed=seed)
    dev = to_device(inp, w.dtype)
    eta = w.eta if eta is None else eta
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                                  dev["conv_kernel"], dev["W_target"], eta, w.C, form=form)
    assert ittt.get_last_error() == ittt.OK
    return inp, dev, host(O), host(Wf)


def _oracle_plain(inp):
    Z = np.stack([orc.gated_activations(inp["H"][b], inp["W_gate"], inp["W_up"])
                  for b in range(inp["H"].shape[0])])
    return Z, Z @ inp["W_down0"].astype(np.float64).T


# ------------------------------------------------------------------ fp32 path

def test_tiny_fp32_workload():
    w = workload("tiny-fp32")
    inp, _, O, Wf = _run(w)
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C)
    assert rel_err(O, Oref) <= TOL["f32"]
    assert rel_err(Wf, Wref) <= TOL["f32"]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(Wf - W0, Wref - W0) <= 1e-4


@pytest.mark.parametrize("T,C,d,f,k,B", [(96, 32, 33, 70, 3, 2), (64, 64, 20, 40, 1, 1),
                                         (96, 48, 24, 40, 11, 1),
                                         (200, 8, 17, 9, 5, 1)])
def test_fp32_ragged_shapes(T, C, d, f, k, B):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.02)
    inp, _, O, Wf = _run(w)
    Oref, Wref = orc.forward_sequential(inp, w.eta, C)
    assert rel_err(O, Oref) <= TOL["f32"]
    assert rel_err(Wf, Wref) <= TOL["f32"]


def test_fp32_steps_match_oracle_intermediates():
    w = workload("tiny-fp32")
    inp = make_inputs(w)
    dev = to_device(inp, "f32")
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=w.C)
    Zr = orc.gated_activations(inp["H"][0], inp["W_gate"], inp["W_up"])
    Vr = orc.lm_target(inp["X0"][0], inp["conv_kernel"], inp["W_target"])
    assert rel_err(host(Z), Zr) <= TOL["f32"]
    assert rel_err(host(V), Vr) <= TOL["f32"]
    stack, wf = ittt.fast_weight_scan(V, Z, dev["W_down0"], 1, w.T, w.C, w.eta)
    W = inp["W_down0"].astype(np.float64)
    for i in range(w.n_chunks - 1):
        W = W + w.eta * Vr[i * w.C:(i + 1) * w.C].T @ Zr[i * w.C:(i + 1) * w.C]
        assert rel_err(host(stack[0, i]), W) <= TOL["f32"]
    O = ittt.apply(Z, dev["W_down0"], stack, 1, w.T, w.C)
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C)
    assert rel_err(host(wf), Wref) <= TOL["f32"]
    assert rel_err(host(O), Oref[0]) <= TOL["f32"]


# ------------------------------------------------------------------ bf16 path

BF16_CASES = [
    # T, C, d, f, k, B : several tiles in every dimension, ragged d/f tails
    (512, 128, 256, 512, 4, 1),
    (1024, 256, 320, 1000, 4, 2),
    (768, 384, 200, 776, 5, 1),
    (384, 128, 136, 264, 1, 3),
    (256, 256, 512, 1536, 8, 1),    # one chunk: the plain gated MLP
    (768, 256, 200, 776, 4, 3),     # three chunks: chunks 0-1 by the dual kernels, 2 by apply
    (512, 256, 256, 512, 16, 2),    # the widest conv (k = 16: the generic conv kernel)
    # C >= 512: the scan stores 128-row snapshot boxes; d, f multiples of 64 with
    # ragged 256-wide tiles (3-D operand boxes), then widths that are not
    (1536, 512, 320, 704, 4, 2),
    (2048, 512, 200, 776, 4, 1),
    (2048, 1024, 256, 512, 4, 1),
]


@pytest.mark.parametrize("T,C,d,f,k,B", BF16_CASES)
def test_bf16_small_cases(T, C, d, f, k, B):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype="bf16")
    inp, _, O, Wf = _run(w)
    Oref, Wref = orc.forward_sequential(inp, w.eta, C)
    assert rel_err(O, Oref) <= TOL["bf16"], rel_err(O, Oref)
    assert rel_err(Wf, Wref) <= TOL["bf16"], rel_err(Wf, Wref)
    # diagnostics of the update itself (stricter views, looser bars)
    W0 = inp["W_down0"].astype(np.float64)
    if T > C:
        assert rel_err(Wf - W0, Wref - W0) <= 1e-2
        _, plain = _oracle_plain(inp)
        assert rel_err(O - plain, Oref - plain) <= 5e-2


@pytest.mark.parametrize("T,C,d,f,k,B", BF16_CASES + [(640, 128, 128, 384, 4, 2)])
def test_bf16_dual_form(T, C, d, f, k, B):
    """The dual rewrite O_i = Z_i W0^T + eta sum_{j<i} (Z_i Z_j^T) Vhat_j on the GPU."""
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype="bf16")
    inp, _, O, Wf = _run(w, form="dual")
    Oref, Wref = orc.forward_sequential(inp, w.eta, C)
    assert rel_err(O, Oref) <= TOL["bf16"], rel_err(O, Oref)
    assert rel_err(Wf, Wref) <= TOL["bf16"], rel_err(Wf, Wref)
    W0 = inp["W_down0"].astype(np.float64)
    if T > C:
        assert rel_err(Wf - W0, Wref - W0) <= 1e-2
        _, plain = _oracle_plain(inp)
        # P = eta Z Z^T is stored in bf16: the update's share of O keeps ~2^-9 accuracy
        assert rel_err(O - plain, Oref - plain) <= 2e-2


def test_forms_agree_and_workspace_follows_form():
    w = small_case(T=1024, C=256, d=256, f=512, k=4, B=2, eta=0.01, dtype="bf16")
    inp, _, Op, Wp = _run(w, form="prefix")
    _, _, Od, Wd = _run(w, form="dual")
    assert rel_err(Od, Op) <= TOL["bf16"] and rel_err(Wd, Wp) <= TOL["bf16"]
    pre = ittt.workspace_size(ittt.make_problem(2, 1024, 256, 512, 256, 4, 0.01, "bf16", "prefix"))
    dual = ittt.workspace_size(ittt.make_problem(2, 1024, 256, 512, 256, 4, 0.01, "bf16", "dual"))
    assert pre != dual


def test_bf16_intermediates_match_oracle():
    w = small_case(T=512, C=128, d=256, f=640, k=4, B=2, eta=0.01, dtype="bf16")
    inp = make_inputs(w)
    dev = to_device(inp, "bf16")
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    Y = ittt.lookahead_conv(dev["X0"], dev["conv_kernel"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=w.C)
    for b in range(2):
        Zr = orc.gated_activations(inp["H"][b], inp["W_gate"], inp["W_up"])
        Yr = orc.lookahead_conv(inp["X0"][b], inp["conv_kernel"])
        Vr = orc.lm_target(inp["X0"][b], inp["conv_kernel"], inp["W_target"])
        assert rel_err(host(Z)[b * 512:(b + 1) * 512], Zr) <= TOL["bf16"]
        assert rel_err(host(Y)[b], Yr) <= TOL["bf16"]
        assert rel_err(host(V)[b * 512:(b + 1) * 512], Vr) <= TOL["bf16"]
    stack, wf = ittt.fast_weight_scan(V, Z, dev["W_down0"], 2, w.T, w.C, w.eta)
    O = ittt.apply(Z, dev["W_down0"], stack, 2, w.T, w.C)
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C)
    assert rel_err(host(wf), Wref) <= TOL["bf16"]
    assert rel_err(host(O).reshape(2, 512, 256), Oref) <= TOL["bf16"]
    # every W^(i) of the stack against the definition's state before chunk i
    for b in range(2):
        Wb = inp["W_down0"].astype(np.float64)
        Zb = orc.gated_activations(inp["H"][b], inp["W_gate"], inp["W_up"])
        Vb = orc.lm_target(inp["X0"][b], inp["conv_kernel"], inp["W_target"])
        for i in range(w.n_chunks - 1):
            Wb = Wb + w.eta * Vb[i * 128:(i + 1) * 128].T @ Zb[i * 128:(i + 1) * 128]
            assert rel_err(host(stack[b, i]), Wb) <= TOL["bf16"]


def test_bf16_eta_zero_is_plain_mlp():
    w = small_case(T=512, C=128, d=256, f=512, k=4, B=2, eta=0.0, dtype="bf16")
    inp, _, O, Wf = _run(w)
    _, plain = _oracle_plain(inp)
    assert rel_err(O, plain) <= TOL["bf16"]
    for b in range(2):
        assert np.array_equal(Wf[b], inp["W_down0"].astype(np.float64))


def test_bf16_chunk0_rows_are_plain_mlp():
    w = small_case(T=512, C=256, d=256, f=512, k=4, B=1, eta=0.5, dtype="bf16")
    inp, _, O, _ = _run(w)
    _, plain = _oracle_plain(inp)
    assert rel_err(O[0, :256], plain[0, :256]) <= TOL["bf16"]
    assert rel_err(O[0, 256:], plain[0, 256:]) > 1e-2  # the update is visible after chunk 0


def test_bf16_next_token_special_case():
    """conv = e_1, W_target = I: Vhat is X0 shifted by one token (exact in bf16)."""
    w = small_case(T=256, C=128, d=128, f=256, k=4, B=2, dtype="bf16")
    inp = make_inputs(w)
    K = np.zeros((128, 4), np.float32)
    K[:, 1] = 1.0
    dev = to_device(dict(X0=inp["X0"], K=K, I=np.eye(128, dtype=np.float32)), "bf16")
    V = host(ittt.lm_target(dev["X0"], dev["K"], dev["I"], C=128)).reshape(2, 256, 128)
    X0 = inp["X0"].astype(np.float64)
    assert np.array_equal(V[:, :-1], X0[:, 1:])
    assert np.all(V[:, -1] == 0)


def test_repeatable_bitwise():
    w = small_case(T=1024, C=256, d=320, f=1000, k=4, B=2, eta=0.01, dtype="bf16")
    inp = make_inputs(w)
    dev = to_device(inp, "bf16")
    args = (dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
            dev["W_target"], w.eta, w.C)
    O1, W1 = ittt.fast_mlp_forward(*args)
    O2, W2 = ittt.fast_mlp_forward(*args)
    assert torch.equal(O1, O2) and torch.equal(W1, W2)


def test_timeout_path_reports_and_recovers():
    ittt.selftest_wait_timeout(20_000_000)   # 20 ms wait on a barrier nobody signals
    assert ittt.get_last_error() == ittt.ERR_TIMEOUT
    assert ittt.get_last_error() == ittt.OK  # cleared
    # the context is still usable
    w = small_case(T=256, C=128, d=128, f=256, k=4, B=1, eta=0.01, dtype="bf16")
    inp, _, O, Wf = _run(w)
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C)
    assert rel_err(O, Oref) <= TOL["bf16"]


def test_device_index_check_skips_the_unit_and_reports():
    """The apply kernel checks each unit's weight-slice index against the
    stack's extent before loading anything: told the stack holds one slice
    fewer, it skips the last sequence's last chunk (those rows stay as they
    were), reports ITTT_ERR_DEVICE_FAULT, and computes every other row with
    the same bits as a plain apply."""
    w = small_case(T=1024, C=256, d=256, f=512, k=4, B=2, eta=0.01, dtype="bf16")
    dev = to_device(make_inputs(w), "bf16")
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=w.C)
    stack, _ = ittt.fast_weight_scan(V, Z, dev["W_down0"], w.B, w.T, w.C, w.eta)
    ref = ittt.apply(Z, dev["W_down0"], stack, w.B, w.T, w.C)
    assert ittt.get_last_error() == ittt.OK
    O = torch.full_like(ref, float("nan"))
    ittt.selftest_device_check(Z, dev["W_down0"], stack, O, w.B, w.T, w.C)
    assert ittt.get_last_error() == ittt.ERR_DEVICE_FAULT
    assert ittt.get_last_error() == ittt.OK  # cleared
    skipped = torch.zeros(w.B * w.T, dtype=torch.bool, device="cuda")
    skipped[(w.B - 1) * w.T + (w.n_chunks - 1) * w.C:] = True
    assert torch.isnan(O[skipped]).all()
    assert torch.equal(O[~skipped], ref[~skipped])
    # the context is still usable
    again = ittt.apply(Z, dev["W_down0"], stack, w.B, w.T, w.C)
    assert torch.equal(again, ref) and ittt.get_last_error() == ittt.OK


def test_probe_times_the_gate_up_gemm_of_each_forward():
    w = small_case(T=1024, C=256, d=256, f=512, k=4, B=1, eta=0.01, dtype="bf16")
    dev = to_device(make_inputs(w), "bf16")
    args = (dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
            dev["W_target"], w.eta, w.C)
    ittt.probe_start(3)
    for _ in range(5):                       # two calls more than probed
        ittt.fast_mlp_forward(*args)
    ms = ittt.probe_read(8)
    assert len(ms) == 3 and all(0.0 < t < 100.0 for t in ms)
    assert ittt.probe_read(8) == []         # reading turned the probe off
    assert ittt.get_last_error() == ittt.OK


def test_buffer_check_decisions():
    """ittt_check_buffer on buffers whose outcome is certain (no launch)."""
    lib = ittt.load_library()
    dev_buf = torch.empty(64 << 20, dtype=torch.uint8, device="cuda")
    host_buf = torch.empty(4096, dtype=torch.uint8)
    assert lib.ittt_check_buffer(dev_buf.data_ptr(), dev_buf.numel()) == ittt.OK
    assert lib.ittt_check_buffer(dev_buf.data_ptr() + 1024, 4096) == ittt.OK
    assert lib.ittt_check_buffer(dev_buf.data_ptr(), 1 << 45) == ittt.ERR_INVALID_ARG
    assert lib.ittt_check_buffer(host_buf.data_ptr(), 16) == ittt.ERR_INVALID_ARG


def test_forward_with_buffer_checks_on_is_unchanged():
    """With the buffer checks on, a forward on correctly sized buffers gives the
    same bits (the refusals themselves are tested without a launch above)."""
    w = small_case(T=1024, C=256, d=320, f=1000, k=4, B=2, eta=0.01, dtype="bf16")
    dev = to_device(make_inputs(w), "bf16")
    args = (dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
            dev["W_target"], w.eta, w.C)
    O0, W0 = ittt.fast_mlp_forward(*args)
    ittt.set_checks(1)
    try:
        O1, W1 = ittt.fast_mlp_forward(*args)
    finally:
        ittt.set_checks(0)
    torch.cuda.synchronize()
    assert ittt.get_last_error() == ittt.OK
    assert torch.equal(O0, O1) and torch.equal(W0, W1)


def test_forward_records_into_a_cuda_graph():
    """The forward (with its side-stream fork and join) records into a CUDA
    graph; replays on new inputs give the eager call's bits."""
    w = small_case(T=1024, C=256, d=256, f=512, k=4, B=1, eta=0.01, dtype="bf16")
    inp = make_inputs(w, seed=1)
    dev = to_device(inp, "bf16")
    p = ittt.problem_from(dev["H"], dev["W_gate"], dev["conv_kernel"], w.eta, w.C)
    ws = torch.empty(ittt.workspace_size(p), dtype=torch.uint8, device="cuda")
    O = torch.empty((1, w.T, w.d), dtype=torch.bfloat16, device="cuda")
    Wf = torch.empty((1, w.d, w.f), dtype=torch.float32, device="cuda")
    H = dev["H"].clone()

    def fwd():
        ittt.fast_mlp_forward(H, dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                              dev["conv_kernel"], dev["W_target"], w.eta, w.C, workspace=ws,
                              out=O, w_final=Wf)

    fwd()                                   # first call: per-device set-up outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=side):
        fwd()
    for seed in (2, 3):
        H.copy_(to_device(make_inputs(w, seed=seed), "bf16")["H"])
        g.replay()
        torch.cuda.synchronize()
        O_graph, W_graph = O.clone(), Wf.clone()
        fwd()
        torch.cuda.synchronize()
        assert torch.equal(O_graph, O) and torch.equal(W_graph, Wf)
    assert ittt.get_last_error() == ittt.OK


def test_auto_dual_at_a_wide_short_shape():
    """d = 4096, f = 14336, T = 2048, C = 256: AUTO takes the dual form (measured
    faster there); sampled rows of O and a block of W_down_final against the
    oracle, and the whole output against the prefix form."""
    w = workload("llama3.1-8b").with_(T=2048, C=256)
    inp = make_inputs(w, seed=0)
    dev = to_device(inp, "bf16")
    args = (dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
            dev["W_target"], w.eta, w.C)
    O, Wf = ittt.fast_mlp_forward(*args)                    # AUTO
    Op, Wp = ittt.fast_mlp_forward(*args, form="prefix")
    assert ittt.get_last_error() == ittt.OK
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(w.d, 12, replace=False))
    cols = np.sort(rng.choice(w.f, 24, replace=False))
    ref = orc.w_final_block(inp, 0, w.eta, rows, cols)
    got = host(Wf[0])[np.ix_(rows, cols)]
    assert rel_err(got, ref) <= TOL["bf16"]
    toks = [0, 255, 256, 700, 1300, 2047]
    ref_rows = orc.output_rows(inp, 0, w.eta, w.C, toks)
    assert rel_err(host(O[0])[toks], ref_rows) <= TOL["bf16"]
    assert rel_err(host(O), host(Op)) <= TOL["bf16"]
    assert rel_err(host(Wf), host(Wp)) <= TOL["bf16"]


HYBRID_CASES = [
    # T, C, d, f, k, B (groups of max(2, 1024 / C) chunks)
    (2048, 256, 256, 512, 4, 2),     # 4 chunks a group, 2 groups
    (4096, 512, 200, 776, 4, 1),     # 2 chunks a group, 4 groups, ragged d, f
    (3072, 256, 320, 1000, 5, 3),    # 3 groups
    (1536, 128, 256, 512, 4, 1),     # 12 chunks, not whole groups of 8: the prefix form runs
]


@pytest.mark.parametrize("T,C,d,f,k,B", HYBRID_CASES)
@pytest.mark.parametrize("clipped", [False, True])
def test_bf16_hybrid_form(T, C, d, f, k, B, clipped):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype="bf16")
    inp = make_inputs(w)
    clip = 0.0
    if clipped:
        Z = orc.gated_activations(inp["H"][0], inp["W_gate"], inp["W_up"])
        V = orc.lm_target(inp["X0"][0], inp["conv_kernel"], inp["W_target"])
        clip = 0.5 * w.eta * float(np.median([np.linalg.norm(V[s:e].T @ Z[s:e])
                                              for s, e in orc.chunk_bounds(T, C)]))
    dev = to_device(inp, "bf16")
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                                  dev["conv_kernel"], dev["W_target"], w.eta, C, form="hybrid",
                                  clip=clip)
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, clip=clip)
    assert rel_err(host(O), Oref) <= TOL["bf16"]
    assert rel_err(host(Wf), Wref) <= TOL["bf16"]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(host(Wf) - W0, Wref - W0) <= 1e-2
