"""Pins of the oracle's update-norm clipping (each chunk's delta rescaled to
Frobenius norm <= tau; iplexlaw review section 6), against scalar loops,
the other forms, and properties the reading fixes."""

import numpy as np
import pytest

from oracle import brute
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case


def _inputs(T=48, C=16, d=6, f=10, k=4, B=1, seed=5):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B)
    return w, make_inputs(w, seed=seed)


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


def _deltas(inp, eta, C, clip):
    """The per-chunk state changes W^(i+1) - W^(i) seen by the definition."""
    T = inp["H"].shape[1]
    prev = inp["W_down0"].astype(np.float64)
    out = []
    for i in range(-(-T // C)):
        _, W = orc.forward_sequential_one(*[inp[k][0] if k in ("H", "X0") else inp[k] for k in (
            "H", "X0", "W_gate", "W_up", "W_down0", "conv_kernel", "W_target")], eta, C,
            upto_chunk=i, clip=clip)
        out.append(W - prev)
        prev = W
    return out


def test_clip_off_and_loose_change_nothing():
    w, inp = _inputs()
    O0, W0 = orc.forward_sequential(inp, 0.1, 16)
    O1, W1 = orc.forward_sequential(inp, 0.1, 16, clip=0.0)
    O2, W2 = orc.forward_sequential(inp, 0.1, 16, clip=1e9)
    assert np.array_equal(O0, O1) and np.array_equal(W0, W1)
    assert np.array_equal(O0, O2) and np.array_equal(W0, W2)


def test_every_applied_delta_respects_the_bound():
    w, inp = _inputs(T=64, C=16)
    eta = 0.2
    free = [np.linalg.norm(x) for x in _deltas(inp, eta, 16, 0.0)]
    tau = float(np.median(free))          # about half the chunks get clipped
    got = [np.linalg.norm(x) for x in _deltas(inp, eta, 16, tau)]
    for g, f in zip(got[:-1], free[:-1]):
        if f > tau:
            assert g == pytest.approx(tau, rel=1e-12)
    # unclipped chunks keep their own delta only while the history is identical:
    # the first chunk's delta depends on no earlier clipping
    assert got[0] == pytest.approx(min(free[0], tau), rel=1e-12)
    assert all(g <= tau * (1 + 1e-12) for g in got)


@pytest.mark.parametrize("T,C,d,f,k", [(12, 4, 3, 5, 2), (13, 4, 4, 6, 3), (16, 3, 5, 8, 5)])
def test_clip_brute_force_agreement(T, C, d, f, k):
    w, inp = _inputs(T=T, C=C, d=d, f=f, k=k, seed=T)
    eta = 0.3
    free = [np.linalg.norm(x) for x in _deltas(inp, eta, C, 0.0)]
    tau = 0.5 * float(np.mean(free))
    O, W = orc.forward_sequential(inp, eta, C, clip=tau)
    Ob, Wb = brute.forward_one(inp["H"][0], inp["X0"][0], inp["W_gate"], inp["W_up"],
                               inp["W_down0"], inp["conv_kernel"], inp["W_target"], eta, C,
                               clip=tau)
    assert _rel(O[0], np.array(Ob)) < 1e-13
    assert _rel(W[0], np.array(Wb)) < 1e-13


@pytest.mark.parametrize("T,C", [(48, 16), (50, 16)])
def test_clip_sequential_equals_prefix_equals_dual(T, C):
    w, inp = _inputs(T=T, C=C, B=2)
    eta = 0.2
    free = [np.linalg.norm(x) for x in _deltas({k: (v[:1] if k in ("H", "X0") else v)
                                                for k, v in inp.items()}, eta, C, 0.0)]
    tau = float(np.median(free))
    Os, Ws = orc.forward(inp, eta, C, "sequential", clip=tau)
    Op, Wp = orc.forward(inp, eta, C, "prefix", clip=tau)
    Od, Wd = orc.forward(inp, eta, C, "dual", clip=tau)
    Oh, Wh = orc.forward(inp, eta, C, "hybrid", clip=tau, m=2)
    assert _rel(Op, Os) < 1e-12 and _rel(Od, Os) < 1e-12 and _rel(Oh, Os) < 1e-12
    assert _rel(Wp, Ws) < 1e-12 and _rel(Wd, Ws) < 1e-12 and _rel(Wh, Ws) < 1e-12


def test_tiny_tau_freezes_the_fast_weight():
    w, inp = _inputs(T=64, C=16)
    tau = 1e-9
    _, W = orc.forward_sequential(inp, 0.2, 16, clip=tau)
    W0 = inp["W_down0"].astype(np.float64)
    assert np.linalg.norm(W[0] - W0) <= 4 * tau * (1 + 1e-9)


def test_gram_identity_for_the_delta_norm():
    """||Vhat_i^T Z_i||_F^2 = sum((Z_i Z_i^T) * (Vhat_i Vhat_i^T)): the way the
    GPU path gets each chunk's norm without forming the delta."""
    rng = np.random.default_rng(0)
    Z = rng.standard_normal((40, 13))
    V = rng.standard_normal((40, 7))
    direct = np.linalg.norm(V.T @ Z) ** 2
    gram = float(np.sum((Z @ Z.T) * (V @ V.T)))
    assert gram == pytest.approx(direct, rel=1e-12)
