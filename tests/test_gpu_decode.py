"""GPU parity of the decode step: tokens fed one at a time reproduce the
prefill recurrence with chunk-end padding (outputs of every token and the
fast weight after each completed chunk), bf16 and fp32, with and without
update-norm clipping."""

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,T,C,d,f,k,B", [
    ("bf16", 384, 128, 128, 256, 4, 3),
    ("bf16", 256, 128, 256, 512, 4, 1),    # two rows per warp in both GEMVs
    ("bf16", 256, 128, 200, 776, 4, 8),    # d not a multiple of a warp's 256-element step
    ("bf16", 256, 128, 224, 776, 4, 8),    # warp MMAs: 7 steps of 32 inputs, f % 16 = 8
    ("bf16", 256, 128, 1024, 520, 4, 5),   # warp MMAs: two unrolled rounds per warp
    ("f32", 96, 32, 48, 80, 3, 2),
    ("f32", 64, 32, 50, 82, 3, 1),         # d, f not multiples of 4: the scalar GEMVs
])
@pytest.mark.parametrize("clipped", [False, True])
def test_decode_matches_prefill(dtype, T, C, d, f, k, B, clipped):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.02, dtype=dtype)
    inp = make_inputs(w)
    clip = 0.0
    if clipped:
        Z = orc.gated_activations(inp["H"][0], inp["W_gate"], inp["W_up"])
        V = orc.conv_rows(inp["X0"][0], inp["conv_kernel"], C, "chunk") @ inp["W_target"]
        clip = 0.5 * abs(w.eta) * float(np.linalg.norm(V[:C].T @ Z[:C]))
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, clip=clip, pad="chunk")
    dev = to_device(inp, dtype)
    dec = ittt.Decoder(dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
                       dev["W_target"], B, w.eta, C, clip=clip)
    outs = []
    for t in range(T):
        outs.append(dec.step(dev["H"][:, t].contiguous(), dev["X0"][:, t].contiguous()).clone())
    assert ittt.get_last_error() == ittt.OK
    O = torch.stack(outs, dim=1)
    assert rel_err(host(O), Oref) <= TOL[dtype]
    assert rel_err(host(dec.state), Wref) <= TOL[dtype]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(host(dec.state) - W0, Wref - W0) <= (1e-2 if dtype == "bf16" else 1e-4)


@pytest.mark.parametrize("dtype,B", [("bf16", 2), ("f32", 1)])
def test_graph_replay_matches_the_plain_step(dtype, B):
    """The steps recorded as CUDA graphs (one per chunk position) give the
    same bits as the plain calls, across two chunk ends."""
    T, C = (384, 128) if dtype == "bf16" else (96, 32)
    w = small_case(T=T, C=C, d=128, f=256, k=4, B=B, eta=0.02, dtype=dtype)
    inp = make_inputs(w)
    dev = to_device(inp, dtype)
    args = (dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"], dev["W_target"], B,
            w.eta, C)
    plain, graphed = ittt.Decoder(*args), ittt.Decoder(*args)
    graphed.capture()
    for t in range(T):
        a = plain.step(dev["H"][:, t].contiguous(), dev["X0"][:, t].contiguous())
        b = graphed.replay(dev["H"][:, t], dev["X0"][:, t])
        assert torch.equal(a, b), t
    torch.cuda.synchronize()
    assert ittt.get_last_error() == ittt.OK
    assert torch.equal(plain.state, graphed.state)
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, pad="chunk")
    assert rel_err(host(graphed.state), Wref) <= TOL[dtype]


@pytest.mark.parametrize("B", [1, 4])
def test_decode_at_qwen3_4b_widths(B):
    """d = 2560, f = 9728, C = 512: the GEMVs' batched loads run over many
    steps per row (B = 4: the gated GEMV on warp MMAs), and a chunk end goes
    through the tcgen05 update; every output of two chunks and the state after
    them against the oracle."""
    from synthetic import workload

    w = workload("qwen3-4b").with_(T=1024, B=B)
    inp = make_inputs(w, seed=0)
    dev = to_device(inp, "bf16")
    dec = ittt.Decoder(dev["W_gate"], dev["W_up"], dev["W_down0"], dev["conv_kernel"],
                       dev["W_target"], B, w.eta, w.C)
    outs = [dec.step(dev["H"][:, t].contiguous(), dev["X0"][:, t].contiguous()).clone()
            for t in range(w.T)]
    assert ittt.get_last_error() == ittt.OK
    Oref, Wref = orc.forward_sequential(inp, w.eta, w.C, pad="chunk")
    assert rel_err(host(torch.stack(outs, dim=1)), Oref) <= TOL["bf16"]
    assert rel_err(host(dec.state), Wref) <= TOL["bf16"]
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(host(dec.state) - W0, Wref - W0) <= 1e-2
