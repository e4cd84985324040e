"""GPU parity of update-norm clipping (every chunk's delta rescaled to
Frobenius norm <= tau) against the oracle, bf16 and fp32, both forms."""

import numpy as np
import pytest

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case, workload

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu


def _delta_norms(inp, eta, C):
    out = []
    for b in range(inp["H"].shape[0]):
        Z = orc.gated_activations(inp["H"][b], inp["W_gate"], inp["W_up"])
        V = orc.lm_target(inp["X0"][b], inp["conv_kernel"], inp["W_target"])
        out.append([abs(eta) * np.linalg.norm(V[s:e].T @ Z[s:e]) for s, e in
                    orc.chunk_bounds(Z.shape[0], C)])
    return np.array(out)


CASES = [
    (1024, 256, 320, 1000, 4, 2),   # C % 256 == 0: chunks 0-1 by the dual kernels
    (768, 384, 200, 776, 5, 1),     # 256-token tiles straddle chunks in the norm kernel
    (512, 128, 256, 512, 4, 3),
]


@pytest.mark.parametrize("form", ["prefix", "dual"])
@pytest.mark.parametrize("T,C,d,f,k,B", CASES)
def test_bf16_clipped_forward(T, C, d, f, k, B, form):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype="bf16")
    inp = make_inputs(w)
    norms = _delta_norms(inp, w.eta, C)
    tau = 0.5 * float(np.median(norms))       # most chunks clipped, to about half
    dev = to_device(inp, "bf16")
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                                  dev["conv_kernel"], dev["W_target"], w.eta, C, form=form, clip=tau)
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, clip=tau)
    assert rel_err(host(O), Oref) <= TOL["bf16"]
    assert rel_err(host(Wf), Wref) <= TOL["bf16"]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(host(Wf) - W0, Wref - W0) <= 1e-2
    # clipping changed the answer (the case is not vacuous)
    _, Wfree = orc.forward_sequential(inp, w.eta, C)
    assert rel_err(Wfree - W0, Wref - W0) > 0.05


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_clip_step_entry_point_norms_and_targets(dtype):
    T, C = (512, 128) if dtype == "bf16" else (256, 64)
    w = small_case(T=T, C=C, d=192, f=320, k=4, B=2, eta=0.02, dtype=dtype)
    inp = make_inputs(w)
    dev = to_device(inp, dtype)
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=C)
    ref = _delta_norms(inp, w.eta, C)
    tau = float(np.median(ref))
    Vin = host(V).copy()
    norms = ittt.clip_update_targets(Z, V, 2, T, C, w.eta, tau)
    assert ittt.get_last_error() == ittt.OK
    tol = TOL[dtype]
    assert rel_err(host(norms), ref) <= tol
    # rows of clipped chunks scaled by tau / norm, the others untouched
    scale = np.where(ref > tau, tau / ref, 1.0)
    want = Vin.reshape(2, T // C, C, -1) * scale[:, :, None, None]
    assert rel_err(host(V).reshape(2, T // C, C, -1), want) <= tol


def test_f32_tiny_workload_clipped():
    w = workload("tiny-fp32")
    inp = make_inputs(w)
    tau = float(np.median(_delta_norms(inp, w.eta, w.C)))
    dev = to_device(inp, "f32")
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                                  dev["conv_kernel"], dev["W_target"], w.eta, w.C, clip=tau)
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C, clip=tau)
    assert rel_err(host(O), Oref) <= TOL["f32"]
    assert rel_err(host(Wf), Wref) <= TOL["f32"]
