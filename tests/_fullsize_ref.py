"""Oracle references for the full-size parity tests, computed once per
workload shape and shared between the tests that sample it.

For sampled rows t of a sequence the closed form
O_t = Z_t W_down0^T + eta sum_{s < S} (Z_t . Z_s) Vhat_s with S the start of
t's chunk needs Z and Vhat of every earlier token: the oracle streams them in
blocks once (update_terms) and keeps the sums at every boundary S asked for.
The 128k workloads differ only in C, so one pass serves all four chunk sizes
and the hybrid form's test (an exact rewrite: the same reference); besides each row's own chunk start, the sums at
the neighbouring chunks' starts are kept, so a test can check that a row was
applied with its own chunk's state and not a neighbour's.
"""

from __future__ import annotations

import numpy as np

from oracle import ittt_oracle as orc
from synthetic import make_inputs, workload

LONG = [f"qwen3-4b-128k-c{C}" for C in (256, 512, 1024, 2048)]

_inputs = {}
_terms = {}


def shape_key(w):
    return (w.B, w.T, w.d, w.f, w.k, w.dtype, w.tiny_distributions)


def inputs(name: str):
    """The workload's seeded inputs (seed 0), upcast once to fp64."""
    w = workload(name)
    key = shape_key(w)
    if key not in _inputs:
        _inputs.clear()  # one full-size input set in memory at a time
        _terms.clear()
        _inputs[key] = {k: v.astype(np.float64) for k, v in make_inputs(w, seed=0).items()}
    return _inputs[key]


def sample_tokens(T: int, C: int):
    """First, an inner and the last token of chunks 0, 1, 2, the middle one and
    the last two (every chunk when there are at most six)."""
    n = T // C
    chunks = sorted({i for i in (0, 1, 2, n // 2, n - 2, n - 1) if 0 <= i < n})
    return sorted({t for i in chunks for t in (i * C, i * C + C // 3, (i + 1) * C - 1)})


def _plan(name: str):
    """Rows and boundaries every test of this shape needs."""
    w = workload(name)
    names = LONG if name in LONG else [name]
    rows, bounds = set(), set()
    for nm in names:
        C = workload(nm).C
        for t in sample_tokens(w.T, C):
            rows.add(t)
            i = t // C
            for j in (i - 1, i, i + 1):       # own chunk start and the neighbours'
                if 0 <= j:
                    bounds.add(min(j * C, w.T))
    return sorted(rows), sorted(bounds)


def update_terms(name: str, b: int):
    """(rows, U): U[S] = sum_{s<S} (Z_t . Z_s) Vhat_s for the planned rows t."""
    w = workload(name)
    key = shape_key(w) + (b,)
    if key not in _terms:
        rows, bounds = _plan(name)
        _terms[key] = (rows, orc.update_terms(inputs(name), b, rows, bounds, block=2048))
    return _terms[key]


def output_rows(name: str, b: int, tokens, state_shift: int = 0):
    """Oracle O[tokens] of sequence b and the no-update part Z_t W_down0^T.
    state_shift = +1 / -1 applies each row with the state of the chunk after /
    before its own (a wrong-state reference, for discrimination checks)."""
    w = workload(name)
    rows, U = update_terms(name, b)
    inp = inputs(name)
    if state_shift == 0:
        return orc.output_rows_closed_form(inp, b, w.eta, w.C, tokens, U=U, tokens_of_U=rows)
    where = {t: j for j, t in enumerate(rows)}
    plain = orc.gated_activations(inp["H"][b][list(tokens)], inp["W_gate"], inp["W_up"]) @ \
        inp["W_down0"].T
    S = [min(max((t // w.C + state_shift) * w.C, 0), w.T) for t in tokens]
    return plain + w.eta * np.stack([U[s][where[t]] for t, s in zip(tokens, S)]), plain
