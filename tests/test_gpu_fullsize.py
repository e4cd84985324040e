"""Full-size parity: every model-shaped workload, in the launch configuration
bench.py times (whole forward, form AUTO), checked against the CPU fp64
oracle on sampled outputs the oracle can compute one by one:

* blocks of W_down_final (W0 + eta Vhat^T Z over the whole sequence: needs
  only the sampled columns of Vhat and Z);
* rows of O from the first chunks (the recurrence is run only as far as the
  sampled tokens' chunk); for qwen3-4b, rows from every chunk.

Tolerance: normwise relative error <= 5e-3 on each sampled set (bf16 path).
"""

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from oracle import ittt_oracle as orc
from synthetic import make_inputs, workload

from _helpers import TOL, rel_err

pytestmark = pytest.mark.gpu

CASES = [
    # workload, sequences to sample, chunks whose rows are sampled (None = all)
    ("qwen3-4b", [0], None),
    ("llama3.1-8b", [0], [0, 1, 2]),
    ("qwen3-14b-b4", [0, 3], [0, 1]),
    ("qwen3-4b-128k-c256", [0], [0, 1, 2, 3]),
    ("qwen3-4b-128k-c512", [0], [0, 1, 2]),
    ("qwen3-4b-128k-c1024", [0], [0, 1, 2]),
    ("qwen3-4b-128k-c2048", [0], [0, 1]),
]


@pytest.mark.parametrize("name,seqs,chunks", CASES)
def test_full_size_workload(name, seqs, chunks):
    w = workload(name)
    inp = make_inputs(w, seed=0)
    dev = {k: torch.from_numpy(v).to("cuda", torch.bfloat16) for k, v in inp.items()}
    O, Wf = ittt.fast_mlp_forward(dev["H"], dev["X0"], dev["W_gate"], dev["W_up"],
                                  dev["W_down0"], dev["conv_kernel"], dev["W_target"], w.eta, w.C)
    assert ittt.get_last_error() == ittt.OK
    del dev
    rng = np.random.default_rng(1234)
    n = w.n_chunks
    for b in seqs:
        # W_down_final blocks
        rows = np.sort(rng.choice(w.d, 12, replace=False))
        cols = np.sort(rng.choice(w.f, 24, replace=False))
        ref = orc.w_final_block(inp, b, w.eta, rows, cols)
        ri = torch.from_numpy(rows).cuda()
        ci = torch.from_numpy(cols).cuda()
        got = Wf[b].index_select(0, ri).index_select(1, ci).double().cpu().numpy()
        assert rel_err(got, ref) <= TOL["bf16"], (name, b, rel_err(got, ref))
        W0 = inp["W_down0"].astype(np.float64)[np.ix_(rows, cols)]
        assert rel_err(got - W0, ref - W0) <= 1e-2, (name, b, rel_err(got - W0, ref - W0))
        # rows of O: first and last token of each sampled chunk, plus one inside
        use = range(n) if chunks is None else chunks
        toks = sorted({t for i in use for t in (i * w.C, i * w.C + w.C // 3, (i + 1) * w.C - 1)})
        ref_rows = orc.output_rows(inp, b, w.eta, w.C, toks)
        got_rows = O[b].index_select(0, torch.tensor(toks, device="cuda")).double().cpu().numpy()
        assert rel_err(got_rows, ref_rows) <= TOL["bf16"], (name, b, rel_err(got_rows, ref_rows))
