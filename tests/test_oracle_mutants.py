"""Planted mistakes in the oracle, on the CPU.

Each mutant below is a plausible error in writing the oracle (a dropped term,
a wrong sign, an index off by one, a transposed operand, the update before
the apply, an inclusive prefix, a clipping or padding rule misread, state
carried across sequences).  It is planted consistently in every place the
oracle computes that step, as a real mistake would be, so that comparing the
oracle's forms with one another cannot catch it by itself.  At least one pin
(the tests of test_oracle_pins.py, test_oracle_clip.py and
test_oracle_segments.py, called directly) must then fail.  The unchanged
oracle passes every pin in the ordinary test run."""

import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from oracle import ittt_oracle as orc  # noqa: E402

import test_oracle_clip as clip  # noqa: E402
import test_oracle_pins as pins  # noqa: E402
import test_oracle_segments as seg  # noqa: E402

PINS = [
    ("golden recurrence", pins.test_golden_update_recurrence),
    ("golden targets", pins.test_golden_next_token_and_reconstruction_targets),
    ("eta = 0 against torch", pins.test_eta_zero_is_plain_gated_mlp),
    ("conv against torch", pins.test_target_matches_torch_depthwise_conv),
    ("gating against torch", pins.test_gated_activations_match_torch),
    ("silu extremes", pins.test_silu_extremes),
    ("scalar loops, ragged", lambda: pins.test_brute_force_agreement(13, 4, 4, 6, 3)),
    ("scalar loops", lambda: pins.test_brute_force_agreement(12, 4, 3, 5, 2)),
    ("forms agree", lambda: pins.test_sequential_equals_prefix_scan_equals_dual(50, 16)),
    ("hybrid agrees", lambda: pins.test_hybrid_groups_equal_the_sequential_loop(64, 8, 3)),
    ("chunk 0 sees no update", pins.test_chunk0_never_sees_an_update),
    ("C = 1 closed form", pins.test_chunk_size_one_closed_form),
    ("affine in eta", pins.test_affine_in_eta),
    ("causality", pins.test_causality_of_h_and_x0),
    ("look-ahead at boundaries", pins.test_lookahead_crosses_chunk_boundary_but_not_sequence_end),
    ("batch independence", pins.test_batch_sequences_are_independent),
    ("clip off or loose", clip.test_clip_off_and_loose_change_nothing),
    ("clip bound", clip.test_every_applied_delta_respects_the_bound),
    ("clip scalar loops", lambda: clip.test_clip_brute_force_agreement(13, 4, 4, 6, 3)),
    ("chunk padding next token", seg.test_chunk_padding_next_token_case),
    ("chunk padding scalar loops", lambda: seg.test_chunk_padding_brute_force(12, 4, 3, 5, 3)),
    ("segments compose", lambda: seg.test_segments_compose_exactly("sequence")),
    ("closed-form rows", lambda: pins.test_closed_form_rows_equal_the_sequential_loop(
        53, 8, 4, "sequence", 2)),
]

_silu = orc.silu
_seq_one = orc.forward_sequential_one
_prefix_one = orc.forward_prefix_one
_dual_one = orc.forward_dual_one
_hybrid_one = orc.forward_hybrid_one
_conv_rows = orc.conv_rows
_rows_closed = orc.output_rows_closed_form
_target_rows = orc.target_rows


def _f(a):
    return np.asarray(a, dtype=np.float64)


def _conv_shifted(shift, reverse=False, back=False):
    """The look-ahead conv with tap j at offset j + shift, taps reversed, or
    looking back instead of ahead."""
    def conv(X0, K):
        X0, K = _f(X0), _f(K)
        T, d = X0.shape
        k = K.shape[1]
        Y = np.zeros((T, d))
        for j in range(k):
            kj = K[:, k - 1 - j] if reverse else K[:, j]
            o = j + shift
            if o >= T:
                continue
            if back:
                Y[o:] += X0[: T - o] * kj
            else:
                Y[: T - o] += X0[o:] * kj
        return Y
    return conv


def _eta_map(fn):
    """Every form and the chunk step with eta replaced by fn(eta)."""
    def patch(mp):
        def step(Z_i, V_i, W, eta, clip=0.0):
            Z_i, V_i, W = _f(Z_i), _f(V_i), _f(W)
            return Z_i @ W.T, W + orc.clip_delta(fn(eta) * (V_i.T @ Z_i), clip)
        mp.setattr(orc, "apply_then_update", step)
        for name, orig in (("forward_prefix_one", _prefix_one), ("forward_dual_one", _dual_one),
                           ("forward_hybrid_one", _hybrid_one)):
            mp.setattr(orc, name, lambda *a, _o=orig, **kw: _o(*a[:7], fn(a[7]), *a[8:], **kw))
    return patch


def _update_before_apply(mp):
    def step(Z_i, V_i, W, eta, clip=0.0):
        Z_i, V_i, W = _f(Z_i), _f(V_i), _f(W)
        W = W + orc.clip_delta(eta * (V_i.T @ Z_i), clip)
        return Z_i @ W.T, W
    mp.setattr(orc, "apply_then_update", step)


def _w_target_transposed(mp):
    mp.setattr(orc, "lm_target", lambda X0, K, Wt: orc.lookahead_conv(X0, K) @ _f(Wt).T)
    mp.setattr(orc, "forward_sequential_one",
               lambda H, X0, Wg, Wu, W0, K, Wt, *a, **kw: _seq_one(H, X0, Wg, Wu, W0, K, _f(Wt).T,
                                                                  *a, **kw))


def _inclusive_prefix(mp):
    def prefix_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta, C, clip=0.0):
        Z = orc.gated_activations(H, W_gate, W_up)
        V = orc.lm_target(X0, conv_kernel, W_target)
        acc = _f(W_down0).copy()
        O = np.zeros((H.shape[0], H.shape[1]))
        for s, e in orc.chunk_bounds(H.shape[0], C):
            acc = acc + orc.clip_delta(eta * (V[s:e].T @ Z[s:e]), clip)
            O[s:e] = Z[s:e] @ acc.T
        return O, acc
    mp.setattr(orc, "forward_prefix_one", prefix_one)


def _dual_own_chunk(mp):
    def dual_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta, C, clip=0.0):
        O, W = _dual_one(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta, C, clip)
        Z = orc.gated_activations(H, W_gate, W_up)
        V = orc.lm_target(X0, conv_kernel, W_target)
        for s, e in orc.chunk_bounds(H.shape[0], C):
            O[s:e] += eta * ((Z[s:e] @ Z[s:e].T) @ V[s:e])   # j <= i instead of j < i
        return O, W
    mp.setattr(orc, "forward_dual_one", dual_one)


def _chunks_overlap(mp):
    mp.setattr(orc, "chunk_bounds", lambda T, C: [(s, min(s + C + 1, T)) for s in range(0, T, C)])


def _ragged_tail_dropped(mp):
    mp.setattr(orc, "chunk_bounds", lambda T, C: [(s, s + C) for s in range(0, T - C + 1, C)])


def _clip_always(mp):
    def cd(dW, tau):
        return dW if tau <= 0 else dW * (tau / float(np.linalg.norm(dW)))
    mp.setattr(orc, "clip_delta", cd)


def _clip_max_abs(mp):
    def cd(dW, tau):
        if tau <= 0:
            return dW
        nrm = float(np.abs(dW).max())
        return dW * (tau / nrm) if nrm > tau else dW
    mp.setattr(orc, "clip_delta", cd)


def _chunk_padding_ignored(mp):
    mp.setattr(orc, "conv_rows", lambda X0, K, C, pad="sequence", X0_next=None:
               _conv_rows(X0, K, C, "sequence", X0_next))
    mp.setattr(orc, "forward_sequential_one",
               lambda *a, pad="sequence", **kw: _seq_one(*a, pad="sequence", **kw))


def _state_carried_across_sequences(mp):
    def fwd(inputs, eta, C, clip=0.0, pad="sequence", W_start=None):
        B = inputs["H"].shape[0]
        W = _f(inputs["W_down0"]) if W_start is None else _f(W_start[0])
        outs = []
        for b in range(B):
            args = [inputs["H"][b], inputs["X0"][b], inputs["W_gate"], inputs["W_up"], W,
                    inputs["conv_kernel"], inputs["W_target"]]
            nxt = inputs["X0_next"][b] if "X0_next" in inputs else None
            O, W = orc.forward_sequential_one(*args, eta, C, clip=clip, pad=pad, X0_next=nxt)
            outs.append((O, W))
        return np.stack([o for o, _ in outs]), np.stack([w for _, w in outs])
    mp.setattr(orc, "forward_sequential", fwd)


def _final_state_misses_last_chunk(mp):
    def seq_one(H, X0, *a, upto_chunk=None, **kw):
        O, W = _seq_one(H, X0, *a, upto_chunk=upto_chunk, **kw)
        n = len(orc.chunk_bounds(H.shape[0], a[6]))
        if upto_chunk is None and n > 1:
            _, W = _seq_one(H, X0, *a, upto_chunk=n - 2, **kw)
        return O, W

    def recurrence(Z, V, W_down0, eta, C, clip=0.0):
        W = _f(W_down0).copy()
        O = np.zeros((Z.shape[0], W.shape[0]))
        for s, e in orc.chunk_bounds(Z.shape[0], C):
            O[s:e], W_next = orc.apply_then_update(Z[s:e], V[s:e], W, eta, clip)
            if e < Z.shape[0]:
                W = W_next
        return O, W
    mp.setattr(orc, "forward_sequential_one", seq_one)
    mp.setattr(orc, "chunk_recurrence", recurrence)


def _closed_form_own_chunk(mp):
    """The closed form summing up to the end of the row's chunk (its own
    update applied before its output)."""
    def rows(inputs, b, eta, C, tokens, pad="sequence", U=None, tokens_of_U=None):
        tokens = [int(t) for t in tokens]
        T = inputs["H"].shape[1]
        ends = [min((t // C + 1) * C, T) for t in tokens]
        U = orc.update_terms(inputs, b, tokens, ends, pad, C)
        Zt = orc.gated_activations(inputs["H"][b][tokens], inputs["W_gate"], inputs["W_up"])
        plain = Zt @ _f(inputs["W_down0"]).T
        return plain + eta * np.stack([U[e][j] for j, e in enumerate(ends)]), plain
    mp.setattr(orc, "output_rows_closed_form", rows)


def _closed_form_without_eta(mp):
    def rows(inputs, b, eta, C, tokens, **kw):
        O, plain = _rows_closed(inputs, b, eta, C, tokens, **kw)
        return plain + (O - plain) / eta, plain
    mp.setattr(orc, "output_rows_closed_form", rows)


def _closed_form_target_transposed(mp):
    def tr(inputs, b, s0, s1, pad="sequence", C=None):
        w = dict(inputs, W_target=np.ascontiguousarray(_f(inputs["W_target"]).T))
        return _target_rows(w, b, s0, s1, pad, C)
    mp.setattr(orc, "target_rows", tr)


MUTANTS = {
    "silu is the sigmoid": lambda mp: mp.setattr(orc, "silu", lambda x: 1.0 / (1.0 + np.exp(-_f(x)))),
    "silu with the sign flipped": lambda mp: mp.setattr(orc, "silu",
                                                         lambda x: _f(x) / (1.0 + np.exp(_f(x)))),
    "gate and up swapped": lambda mp: mp.setattr(
        orc, "gated_activations", lambda H, Wg, Wu: _silu(_f(H) @ _f(Wu).T) * (_f(H) @ _f(Wg).T)),
    "conv looks back": lambda mp: mp.setattr(orc, "lookahead_conv", _conv_shifted(0, back=True)),
    "conv tap one further": lambda mp: mp.setattr(orc, "lookahead_conv", _conv_shifted(1)),
    "conv taps reversed": lambda mp: mp.setattr(orc, "lookahead_conv", _conv_shifted(0, True)),
    "W_target transposed": _w_target_transposed,
    "update before apply": _update_before_apply,
    "update sign flipped": _eta_map(lambda eta: -eta),
    "eta dropped": _eta_map(lambda eta: 1.0),
    "eta doubled": _eta_map(lambda eta: 2.0 * eta),
    "inclusive prefix": _inclusive_prefix,
    "dual includes its own chunk": _dual_own_chunk,
    "chunks overlap by one token": _chunks_overlap,
    "ragged last chunk dropped": _ragged_tail_dropped,
    "clip always rescales": _clip_always,
    "clip by the largest entry": _clip_max_abs,
    "chunk padding ignored": _chunk_padding_ignored,
    "state carried across sequences": _state_carried_across_sequences,
    "final state misses the last chunk": _final_state_misses_last_chunk,
    "closed form includes the row's own chunk": _closed_form_own_chunk,
    "closed form without eta": _closed_form_without_eta,
    "closed form with W_target transposed": _closed_form_target_transposed,
}


def _caught(patch):
    """Name of the first pin that fails under the planted mistake, or None."""
    with pytest.MonkeyPatch.context() as mp:
        patch(mp)
        for name, pin in PINS:
            try:
                pin()
            except AssertionError:  # anything else is a fault of the mutant itself
                return name
    return None


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_a_planted_mistake_fails_a_pin(mutant):
    assert _caught(MUTANTS[mutant]) is not None, f"no pin catches: {mutant}"


def test_the_unchanged_oracle_passes_every_pin():
    assert _caught(lambda mp: None) is None
