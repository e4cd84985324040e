"""Pins of the CPU oracle to facts the pages and the mathematics fix.

None of these compares the oracle with itself: each check uses a different
computation (torch library routines, scalar loops, hand-derived values,
closed forms, or structural invariants of the recurrence).
"""

import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import brute
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(T=48, C=16, d=6, f=10, k=4, B=1, seed=3, dtype="f32"):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, dtype=dtype)
    return w, make_inputs(w, seed=seed)


def _rel(a, b):
    return float(np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300))


# -- worked examples -------------------------------------------------------

def test_golden_update_recurrence():
    g = json.load(open(os.path.join(GOLDEN, "update_recurrence_d2f2.json")))
    O, W = orc.chunk_recurrence(np.array(g["Z"], float), np.array(g["Vhat"], float),
                                np.array(g["W_down0"], float), g["eta"], g["C"])
    assert np.array_equal(O, np.array(g["O"], float))
    assert np.array_equal(W, np.array(g["W_down_final"], float))


def test_golden_next_token_and_reconstruction_targets():
    g = json.load(open(os.path.join(GOLDEN, "next_token_target.json")))
    X0 = np.array(g["X0"], float)
    T, d = X0.shape
    I = np.eye(d)
    for tap, key in ((g["next_token_kernel_tap"], "Vhat_next_token"),
                     (g["reconstruction_kernel_tap"], "Vhat_reconstruction")):
        K = np.zeros((d, g["k"]))
        K[:, tap] = 1.0
        assert np.array_equal(orc.lm_target(X0, K, I), np.array(g[key], float))


# -- special cases that reduce to library routines -------------------------

def _torch_plain_mlp(inp):
    H = torch.from_numpy(inp["H"]).double()
    Wg = torch.from_numpy(inp["W_gate"]).double()
    Wu = torch.from_numpy(inp["W_up"]).double()
    W0 = torch.from_numpy(inp["W_down0"]).double()
    return (F.silu(H @ Wg.T) * (H @ Wu.T) @ W0.T).numpy()


def _torch_target(inp):
    """Vhat via torch's depthwise conv1d (cross-correlation) with right zero padding."""
    X0 = torch.from_numpy(inp["X0"]).double()          # [B, T, d]
    K = torch.from_numpy(inp["conv_kernel"]).double()   # [d, k]
    d, k = K.shape
    x = F.pad(X0.transpose(1, 2), (0, k - 1))           # [B, d, T + k - 1]
    y = F.conv1d(x, K[:, None, :], groups=d)            # [B, d, T]
    return (y.transpose(1, 2) @ torch.from_numpy(inp["W_target"]).double()).numpy()


def test_eta_zero_is_plain_gated_mlp():
    w, inp = _inputs(B=2)
    O, W = orc.forward_sequential(inp, 0.0, w.C)
    assert _rel(O, _torch_plain_mlp(inp)) < 1e-13
    for b in range(2):
        assert np.array_equal(W[b], inp["W_down0"].astype(np.float64))


def test_target_matches_torch_depthwise_conv():
    w, inp = _inputs(k=5, B=2)
    ref = _torch_target(inp)
    for b in range(2):
        got = orc.lm_target(inp["X0"][b], inp["conv_kernel"], inp["W_target"])
        assert _rel(got, ref[b]) < 1e-13


def test_gated_activations_match_torch():
    _, inp = _inputs()
    H = torch.from_numpy(inp["H"][0]).double()
    ref = (F.silu(H @ torch.from_numpy(inp["W_gate"]).double().T)
           * (H @ torch.from_numpy(inp["W_up"]).double().T)).numpy()
    assert _rel(orc.gated_activations(inp["H"][0], inp["W_gate"], inp["W_up"]), ref) < 1e-14


def test_silu_extremes():
    x = np.array([-1000.0, -50.0, -1.0, 0.0, 1.0, 50.0, 1000.0])
    ref = F.silu(torch.from_numpy(x)).numpy()
    assert np.allclose(orc.silu(x), ref, rtol=1e-15, atol=0)


# -- structure of the recurrence ---------------------------------------------

def test_chunk0_never_sees_an_update():
    w, inp = _inputs()
    O1, _ = orc.forward_sequential(inp, 0.05, w.C)
    inp2 = dict(inp)
    rng = np.random.default_rng(9)
    inp2["X0"] = rng.standard_normal(inp["X0"].shape).astype(np.float32)
    inp2["conv_kernel"] = rng.standard_normal(inp["conv_kernel"].shape).astype(np.float32)
    inp2["W_target"] = rng.standard_normal(inp["W_target"].shape).astype(np.float32)
    O2, _ = orc.forward_sequential(inp2, -3.0, w.C)
    assert np.array_equal(O1[:, : w.C], O2[:, : w.C])
    assert not np.allclose(O1[:, w.C:], O2[:, w.C:])


@pytest.mark.parametrize("T,C", [(48, 16), (50, 16), (33, 7), (40, 40), (40, 64)])
def test_sequential_equals_prefix_scan_equals_dual(T, C):
    w, inp = _inputs(T=T, C=C, B=2)
    Os, Ws = orc.forward(inp, 0.07, C, "sequential")
    Op, Wp = orc.forward(inp, 0.07, C, "prefix")
    Od, Wd = orc.forward(inp, 0.07, C, "dual")
    assert _rel(Op, Os) < 1e-12 and _rel(Od, Os) < 1e-12
    assert _rel(Wp, Ws) < 1e-12 and _rel(Wd, Ws) < 1e-12


@pytest.mark.parametrize("T,C,m", [(64, 8, 2), (64, 8, 3), (50, 8, 4), (33, 7, 2), (40, 40, 2)])
def test_hybrid_groups_equal_the_sequential_loop(T, C, m):
    """Groups of m chunks (a shorter last group and a ragged last chunk among
    the cases) give the sequential loop's outputs and state."""
    w, inp = _inputs(T=T, C=C, B=2)
    Os, Ws = orc.forward(inp, 0.07, C, "sequential")
    Oh, Wh = orc.forward(inp, 0.07, C, "hybrid", m=m)
    assert _rel(Oh, Os) < 1e-12 and _rel(Wh, Ws) < 1e-12


def test_hybrid_reduces_to_the_prefix_and_dual_forms():
    """m = 1 stores every chunk's weight (the prefix form); m >= n stores only
    W_down0 (the dual form): the same terms, so equal up to rounding."""
    w, inp = _inputs(T=48, C=8, B=1)
    Op, Wp = orc.forward(inp, 0.07, 8, "prefix")
    Od, Wd = orc.forward(inp, 0.07, 8, "dual")
    O1, W1 = orc.forward(inp, 0.07, 8, "hybrid", m=1)
    On, Wn = orc.forward(inp, 0.07, 8, "hybrid", m=6)
    assert _rel(O1, Op) < 1e-13 and _rel(On, Od) < 1e-13 and _rel(Wn, Wd) < 1e-13
    # a group's first chunk sees only the group's stored weight: changing a
    # later chunk's inputs inside the group leaves it alone
    Oa, _ = orc.forward(inp, 0.07, 8, "hybrid", m=3)
    inp2 = dict(inp)
    H2 = inp["H"].copy()
    H2[:, 40:48] += 1.0                                  # chunk 5, second of group 1
    inp2["H"] = H2
    Ob, _ = orc.forward(inp2, 0.07, 8, "hybrid", m=3)
    assert np.array_equal(Oa[:, :40], Ob[:, :40]) and not np.allclose(Oa[:, 40:], Ob[:, 40:])


def test_w_final_is_independent_of_chunk_size():
    w, inp = _inputs(T=48)
    ref = None
    for C in (1, 5, 16, 48, 100):
        _, W = orc.forward_sequential(inp, 0.05, C)
        if ref is None:
            ref = W
        assert _rel(W, ref) < 1e-12


def test_single_chunk_is_plain_mlp():
    w, inp = _inputs(T=48)
    O, _ = orc.forward_sequential(inp, 0.5, 48)
    assert _rel(O[0], _torch_plain_mlp(inp)[0]) < 1e-13


def test_chunk_size_one_closed_form():
    """C = 1: O_t = Z_t W0^T + eta sum_{s<t} (Z_t . Z_s) Vhat_s, with Z, Vhat from torch."""
    w, inp = _inputs(T=20, d=5, f=7)
    eta = 0.03
    H = torch.from_numpy(inp["H"][0]).double()
    Z = (F.silu(H @ torch.from_numpy(inp["W_gate"]).double().T)
         * (H @ torch.from_numpy(inp["W_up"]).double().T)).numpy()
    V = _torch_target(inp)[0]
    W0 = inp["W_down0"].astype(np.float64)
    ref = np.zeros((20, 5))
    for t in range(20):
        ref[t] = Z[t] @ W0.T
        for s in range(t):
            ref[t] += eta * float(Z[t] @ Z[s]) * V[s]
    O, W = orc.forward_sequential(inp, eta, 1)
    assert _rel(O[0], ref) < 1e-12
    Wref = W0 + eta * sum(np.outer(V[s], Z[s]) for s in range(20))
    assert _rel(W[0], Wref) < 1e-12


def test_affine_in_eta():
    w, inp = _inputs()
    a = 0.02
    O0, W0 = orc.forward_sequential(inp, 0.0, w.C)
    O1, W1 = orc.forward_sequential(inp, a, w.C)
    O2, W2 = orc.forward_sequential(inp, 2 * a, w.C)
    assert np.abs(O2 - 2 * O1 + O0).max() < 1e-12 * np.abs(O1).max()
    assert np.abs(W2 - 2 * W1 + W0).max() < 1e-12 * np.abs(W1).max()
    # the update part is linear in W_target
    inp3 = dict(inp)
    inp3["W_target"] = (3.0 * inp["W_target"].astype(np.float64))
    O3, _ = orc.forward_sequential(inp3, a, w.C)
    assert np.abs((O3 - O0) - 3 * (O1 - O0)).max() < 1e-12 * np.abs(O1).max()


def test_causality_of_h_and_x0():
    w, inp = _inputs(T=64, C=16, k=4)
    O, _ = orc.forward_sequential(inp, 0.1, 16)
    # H perturbed in chunk 2 leaves chunks 0..1 unchanged
    inp2 = dict(inp)
    H = inp["H"].copy()
    H[:, 40] += 1.0
    inp2["H"] = H
    O2, _ = orc.forward_sequential(inp2, 0.1, 16)
    assert np.array_equal(O[:, :32], O2[:, :32]) and not np.allclose(O[:, 32:], O2[:, 32:])
    # X0 perturbed at p = 35 changes Vhat rows 32..35: chunks 0..2 unchanged, chunk 3 changes
    inp3 = dict(inp)
    X0 = inp["X0"].copy()
    X0[:, 35] += 1.0
    inp3["X0"] = X0
    O3, _ = orc.forward_sequential(inp3, 0.1, 16)
    assert np.array_equal(O[:, :48], O3[:, :48]) and not np.allclose(O[:, 48:], O3[:, 48:])
    # p = 33 with k = 4 reaches back to Vhat row 30 (chunk 1): chunk 2 changes
    X0 = inp["X0"].copy()
    X0[:, 33] += 1.0
    inp3["X0"] = X0
    O4, _ = orc.forward_sequential(inp3, 0.1, 16)
    assert np.array_equal(O[:, :32], O4[:, :32]) and not np.allclose(O[:, 32:48], O4[:, 32:48])


def test_lookahead_crosses_chunk_boundary_but_not_sequence_end():
    """Vhat at the end of a chunk reads X0 of the next chunk; nothing past T."""
    w, inp = _inputs(T=32, C=8, d=4, f=6, k=3)
    V = orc.lm_target(inp["X0"][0], inp["conv_kernel"], inp["W_target"])
    X0 = inp["X0"][0].astype(np.float64)
    K = inp["conv_kernel"].astype(np.float64)
    y7 = K[:, 0] * X0[7] + K[:, 1] * X0[8] + K[:, 2] * X0[9]
    assert np.allclose(V[7], y7 @ inp["W_target"].astype(np.float64), rtol=1e-14, atol=1e-15)
    y31 = K[:, 0] * X0[31]
    assert np.allclose(V[31], y31 @ inp["W_target"].astype(np.float64), rtol=1e-14, atol=1e-15)


def test_batch_sequences_are_independent():
    w, inp = _inputs(B=3)
    O, W = orc.forward_sequential(inp, 0.05, w.C)
    for b in range(3):
        one = {key: (v[b:b + 1] if key in ("H", "X0") else v) for key, v in inp.items()}
        Ob, Wb = orc.forward_sequential(one, 0.05, w.C)
        assert np.array_equal(O[b], Ob[0]) and np.array_equal(W[b], Wb[0])


# -- brute force -------------------------------------------------------------

@pytest.mark.parametrize("T,C,d,f,k", [(12, 4, 3, 5, 2), (13, 4, 4, 6, 3), (9, 9, 2, 3, 1),
                                       (16, 3, 5, 8, 5), (7, 1, 3, 4, 4)])
def test_brute_force_agreement(T, C, d, f, k):
    w, inp = _inputs(T=T, C=C, d=d, f=f, k=k, seed=T + d)
    eta = 0.11
    O, W = orc.forward_sequential(inp, eta, C)
    Ob, Wb = brute.forward_one(inp["H"][0], inp["X0"][0], inp["W_gate"], inp["W_up"],
                               inp["W_down0"], inp["conv_kernel"], inp["W_target"], eta, C)
    assert _rel(O[0], np.array(Ob)) < 1e-13
    assert _rel(W[0], np.array(Wb)) < 1e-13


# -- sampled evaluation used by full-size GPU parity -------------------------

def test_sampled_helpers_match_full_oracle():
    w, inp = _inputs(T=64, C=16, d=8, f=12, B=2)
    eta = 0.04
    O, W = orc.forward_sequential(inp, eta, 16)
    rows, cols = [0, 3, 7], [1, 2, 11]
    for b in range(2):
        blk = orc.w_final_block(inp, b, eta, rows, cols)
        assert _rel(blk, W[b][np.ix_(rows, cols)]) < 1e-13
        toks = [0, 15, 16, 40, 63]
        assert _rel(orc.output_rows(inp, b, eta, 16, toks), O[b][toks]) < 1e-13


@pytest.mark.parametrize("T,C,k,pad,B", [(50, 8, 3, "sequence", 1), (53, 8, 4, "sequence", 2),
                                         (40, 1, 2, "sequence", 1), (48, 8, 5, "chunk", 1),
                                         (45, 16, 11, "chunk", 2), (13, 4, 3, "sequence", 1)])
def test_closed_form_rows_equal_the_sequential_loop(T, C, k, pad, B):
    """O_t = Z_t W0^T + eta sum_{s < start of t's chunk} (Z_t . Z_s) Vhat_s,
    the recurrence expanded, reproduces the chunk loop row by row: ragged last
    chunk, C = 1, a look-ahead wider than a chunk, chunk-end padding, and
    block sizes that do and do not divide the chunks.  Its no-update part is
    torch's gated MLP with W_down0, and on the smallest shape it equals the
    scalar loops."""
    w, inp = _inputs(T=T, C=C, d=6, f=10, k=k, B=B, seed=T + k)
    eta = 0.07
    O, _ = orc.forward_sequential(inp, eta, C, pad=pad)
    b = B - 1
    toks = list(range(T))
    starts = sorted({(t // C) * C for t in toks})
    for block in (1, 5, 1024):
        U = orc.update_terms(inp, b, toks, starts, pad, C, block=block)
        got, plain = orc.output_rows_closed_form(inp, b, eta, C, toks, pad=pad, U=U,
                                                 tokens_of_U=toks)
        assert _rel(got, O[b]) < 1e-13, block
    Ht = torch.from_numpy(inp["H"][b]).double()
    Zt = F.silu(Ht @ torch.from_numpy(inp["W_gate"]).double().T) * \
        (Ht @ torch.from_numpy(inp["W_up"]).double().T)
    assert _rel(plain, (Zt @ torch.from_numpy(inp["W_down0"]).double().T).numpy()) < 1e-13
    if T <= 16 and pad == "sequence":
        Ob, _ = brute.forward_one(inp["H"][b], inp["X0"][b], inp["W_gate"], inp["W_up"],
                                  inp["W_down0"], inp["conv_kernel"], inp["W_target"], eta, C)
        assert _rel(got, np.array(Ob)) < 1e-13
    # a subset of rows, evaluated on its own, gives the same rows
    sub = [T - 1, 0, C, T // 2]
    alone, _ = orc.output_rows_closed_form(inp, b, eta, C, sub, pad=pad)
    assert _rel(alone, O[b][sub]) < 1e-13


def test_generator_is_seeded_and_bf16_rounded():
    w = small_case(T=16, C=8, d=8, f=16, dtype="bf16")
    a = make_inputs(w, seed=0)
    b = make_inputs(w, seed=0)
    for key in a:
        assert np.array_equal(a[key], b[key])
        t = torch.from_numpy(a[key])
        assert torch.equal(t.to(torch.bfloat16).float(), t)
