"""The chunk recurrence step (ittt_chunk_recurrence) on the GPU: O and
W_down_final from Z and Vhat, against the CPU fp64 oracle's chunk loop on
the same (bf16-rounded) Z and Vhat, and against the scan and apply step entry
points run one after the other.

On the bf16 prefix form the step is one persistent kernel whose work queue
holds the fused scan's tile pairs and the apply units; the shapes below give
one and several d-tiles and f-tiles (odd tile counts leave a one-tile pair),
ragged d and f, several sequences, two chunks only, and C = 128 (an apply tile
spans two chunks).
"""

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu

CASES = [
    # T, C, d, f, B
    (512, 256, 256, 512, 1),       # one d-tile, two f-tiles: one scan pair
    (1024, 256, 320, 1000, 2),     # ragged d, f; 2 x 4 tiles
    (768, 256, 200, 776, 3),       # ragged, odd tile count per sequence
    (512, 128, 256, 768, 1),       # C = 128, three f-tiles (a one-tile pair)
    (1024, 512, 512, 256, 2),      # two chunks
    (2048, 256, 768, 1280, 1),     # 3 x 5 tiles, 8 chunks
    (1536, 512, 320, 704, 2),      # C = 512 (128-row snapshot stores), ragged 256-wide tiles
]


def _inputs(T, C, d, f, B, seed=0):
    w = small_case(T=T, C=C, d=d, f=f, k=4, B=B, eta=0.01, dtype="bf16")
    inp = make_inputs(w, seed=seed)
    dev = to_device(inp, "bf16")
    Z = ittt.gated_activations(dev["H"], dev["W_gate"], dev["W_up"])
    V = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=C)
    return w, inp, dev, Z, V


@pytest.mark.parametrize("T,C,d,f,B", CASES)
def test_recurrence_matches_oracle_chunk_loop(T, C, d, f, B):
    w, inp, dev, Z, V = _inputs(T, C, d, f, B)
    O, Wf = ittt.chunk_recurrence(Z, V, dev["W_down0"], B, T, C, w.eta, form="prefix")
    assert ittt.get_last_error() == ittt.OK
    Zh, Vh = host(Z).reshape(B, T, f), host(V).reshape(B, T, d)
    W0 = inp["W_down0"].astype(np.float64)
    for b in range(B):
        Oref, Wref = orc.chunk_recurrence(Zh[b], Vh[b], W0, w.eta, C)
        assert rel_err(host(O[b]), Oref) <= TOL["bf16"]
        assert rel_err(host(Wf[b]), Wref) <= TOL["bf16"]
        assert rel_err(host(Wf[b]) - W0, Wref - W0) <= 1e-2


@pytest.mark.parametrize("T,C,d,f,B", CASES)
def test_recurrence_equals_scan_then_apply(T, C, d, f, B):
    """The one-launch recurrence and the two step kernels store the same
    effective weights and outputs: every tile accumulates its chunks and its
    k-blocks in the same order."""
    w, inp, dev, Z, V = _inputs(T, C, d, f, B, seed=1)
    O, Wf = ittt.chunk_recurrence(Z, V, dev["W_down0"], B, T, C, w.eta, form="prefix")
    stack, wf2 = ittt.fast_weight_scan(V, Z, dev["W_down0"], B, T, C, w.eta)
    O2 = ittt.apply(Z, dev["W_down0"], stack, B, T, C)
    assert ittt.get_last_error() == ittt.OK
    assert rel_err(host(Wf), host(wf2)) <= 1e-6
    assert rel_err(host(O).reshape(B * T, d), host(O2)) <= 1e-6


def test_recurrence_is_repeatable_and_reuses_its_workspace():
    """Two calls on the same workspace (whose counter and flags are cleared by
    each call) give identical bits, also after the workspace was scribbled on."""
    T, C, d, f, B = 2048, 256, 768, 1280, 2
    w, inp, dev, Z, V = _inputs(T, C, d, f, B, seed=2)
    p = ittt.make_problem(B, T, d, f, C, 1, w.eta, "bf16", "prefix")
    ws = torch.full((ittt.workspace_size(p),), 0x5A, dtype=torch.uint8, device="cuda")
    O1, W1 = ittt.chunk_recurrence(Z, V, dev["W_down0"], B, T, C, w.eta, form="prefix", workspace=ws)
    ws.fill_(0xFF)
    O2, W2 = ittt.chunk_recurrence(Z, V, dev["W_down0"], B, T, C, w.eta, form="prefix", workspace=ws)
    assert ittt.get_last_error() == ittt.OK
    assert torch.equal(O1, O2) and torch.equal(W1, W2)
