"""GPU parity of the conv padding rules and of segment continuation
(a document processed as consecutive calls, the fast weight carried)."""

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, small_case

from _helpers import TOL, host, rel_err, to_device

pytestmark = pytest.mark.gpu


def _fwd(dev, eta, C, **kw):
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"], dev["W_down0"],
                                  dev["conv_kernel"], dev["W_target"], eta, C, **kw)
    assert ittt.get_last_error() == ittt.OK
    return O, Wf


@pytest.mark.parametrize("dtype,T,C,d,f,k,B", [("bf16", 1024, 256, 320, 1000, 4, 2),
                                               ("bf16", 768, 384, 200, 776, 5, 1),
                                               ("f32", 256, 64, 64, 256, 4, 1)])
@pytest.mark.parametrize("form", ["prefix", "dual"])
def test_chunk_end_padding(dtype, T, C, d, f, k, B, form):
    w = small_case(T=T, C=C, d=d, f=f, k=k, B=B, eta=0.01, dtype=dtype)
    inp = make_inputs(w)
    O, Wf = _fwd(to_device(inp, dtype), w.eta, C, pad="chunk", form=form)
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, pad="chunk")
    assert rel_err(host(O), Oref) <= TOL[dtype]
    assert rel_err(host(Wf), Wref) <= TOL[dtype]
    # the rule matters here: sequence-end padding gives a different fast weight
    _, Wseq = orc.forward_sequential(inp, w.eta, C)
    W0 = inp["W_down0"].astype(np.float64)
    assert rel_err(Wseq - W0, Wref - W0) > 1e-3


@pytest.mark.parametrize("dtype,pad", [("bf16", "sequence"), ("bf16", "chunk"),
                                       ("f32", "sequence"), ("f32", "chunk")])
def test_segment_continuation(dtype, pad):
    """Two calls ([0, T1) then [T1, T) from the carried W) reproduce one call."""
    T, C, T1 = (1024, 256, 512) if dtype == "bf16" else (256, 64, 128)
    w = small_case(T=T, C=C, d=192, f=384, k=4, B=1, eta=0.01, dtype=dtype)
    inp = make_inputs(w)
    Oref, Wref = orc.forward_sequential(inp, w.eta, C, pad=pad)
    dev = to_device(inp, dtype)
    first = dict(dev, H=dev["H"][:, :T1].contiguous())
    # sequence-end padding: segment 1 carries the next segment's first k-1 rows
    first["X0"] = dev["X0"][:, :T1 + (w.k - 1 if pad == "sequence" else 0)].contiguous()
    O1, W1 = _fwd(first, w.eta, C, pad=pad)
    second = dict(dev, H=dev["H"][:, T1:].contiguous(), X0=dev["X0"][:, T1:].contiguous())
    second["W_down0"] = W1[0].to(dev["W_down0"].dtype).contiguous()   # carried fast weight
    O2, W2 = _fwd(second, w.eta, C, pad=pad)
    O = torch.cat([O1, O2], dim=1)
    assert rel_err(host(O), Oref) <= TOL[dtype]
    assert rel_err(host(W2), Wref) <= TOL[dtype]
