"""C ABI of libittt.so without a GPU: it loads, exports every declared entry
point, and its host-side argument checks answer before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

import weight_gated_mlp_b200 as ittt
from weight_gated_mlp_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return ittt.load_library()


def _declared():
    src = open(os.path.join(ROOT, "include", "ittt.h")).read()
    return sorted(set(re.findall(r"\b(ittt_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 10
    out = subprocess.run(["nm", "-D", "--defined-only", ittt.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(ittt_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    assert set(ittt.EXPORTED) == set(names)


def test_library_targets_sm100a(lib):
    assert lib.ittt_version() >= 100
    # the build command names the Blackwell target explicitly
    cmd = " ".join(_build.command())
    assert "arch=compute_100a,code=sm_100a" in cmd


def test_status_strings(lib):
    for s in range(7):
        assert ittt.status_string(s)
    assert ittt.status_string(99) == "unknown status"


def _ws(p):
    n = ctypes.c_size_t(0)
    return ittt.load_library().ittt_workspace_size(ctypes.byref(p), ctypes.byref(n)), n.value


@pytest.mark.parametrize("kw,status", [
    (dict(B=0), ittt.ERR_INVALID_ARG),
    (dict(T=-1), ittt.ERR_INVALID_ARG),
    (dict(k=0), ittt.ERR_INVALID_ARG),
    (dict(k=17), ittt.ERR_UNSUPPORTED),
    (dict(C=100), ittt.ERR_UNSUPPORTED),          # T % C != 0
    (dict(d=100), ittt.ERR_UNSUPPORTED),          # bf16 needs d % 8 == 0
    (dict(f=1001), ittt.ERR_UNSUPPORTED),
    (dict(C=64, T=256), ittt.ERR_UNSUPPORTED),    # bf16 needs C % 128 == 0
    (dict(eta=float("nan")), ittt.ERR_INVALID_ARG),
    (dict(eta=1e-35), ittt.ERR_UNSUPPORTED),      # bf16: 0 < |eta| < 1e-30
    (dict(eta=-1e-31), ittt.ERR_UNSUPPORTED),
    (dict(eta=1e-35, dtype="f32"), ittt.OK),     # f32: any finite eta
    (dict(eta=1e-30), ittt.OK),
    (dict(eta=0.0), ittt.OK),
    (dict(clip=-1.0), ittt.ERR_INVALID_ARG),
    (dict(clip=float("inf")), ittt.ERR_INVALID_ARG),
])
def test_invalid_problems_rejected(lib, kw, status):
    base = dict(B=1, T=512, d=256, f=512, C=128, k=4, eta=1e-3, dtype="bf16")
    base.update(kw)
    p = ittt.make_problem(**base)
    assert _ws(p)[0] == status


def test_bad_enums_and_flags(lib):
    p = ittt.make_problem(1, 512, 256, 512, 128, 4, 1e-3)
    p.dtype = 7
    assert _ws(p)[0] == ittt.ERR_INVALID_ARG
    p = ittt.make_problem(1, 512, 256, 512, 128, 4, 1e-3)
    p.form = 9
    assert _ws(p)[0] == ittt.ERR_INVALID_ARG
    p = ittt.make_problem(1, 512, 256, 512, 128, 4, 1e-3)
    p.flags = 4
    assert _ws(p)[0] == ittt.ERR_INVALID_ARG
    for fl in (ittt.FLAG_PAD_CHUNK_END, ittt.FLAG_X0_LOOKAHEAD, 3):
        p.flags = fl
        assert _ws(p)[0] == ittt.OK
    p = ittt.make_problem(1, 512, 256, 512, 128, 4, 1e-3)
    p.reserved = 3
    assert _ws(p)[0] == ittt.ERR_INVALID_ARG
    assert lib.ittt_workspace_size(None, None) == ittt.ERR_INVALID_ARG


def test_fp32_accepts_any_width(lib):
    p = ittt.make_problem(1, 256, 63, 250, 64, 4, 0.01, dtype="f32")
    st, n = _ws(p)
    assert st == ittt.OK
    # Z, Y, Vhat and a (n-1)-deep stack of fp32 d x f weights
    assert n >= 4 * (256 * 250 + 2 * 256 * 63 + 3 * 63 * 250)


def test_workspace_grows_with_chunks(lib):
    a = _ws(ittt.make_problem(1, 4096, 256, 512, 1024, 4, 1e-3))[1]
    b = _ws(ittt.make_problem(1, 4096, 256, 512, 256, 4, 1e-3))[1]
    # bf16 weight stack of n - 1 slices, plus the [B, 2C, C] gram block of the
    # two chunks the prefix forward computes with the dual kernels; the one-launch
    # recurrence's work counter and readiness flags (256 bytes + 4 per d-tile and
    # chunk) fit one 512-byte block at both chunk sizes
    stack = (15 - 3) * 256 * 512 * 2
    gram = 2 * 256 * 256 * 2 - 2 * 1024 * 1024 * 2
    assert b - a == stack + gram
    # eta = 0 runs no recurrence: no flags, no gram block
    z = _ws(ittt.make_problem(1, 4096, 256, 512, 256, 4, 0.0))[1]
    assert b - z == 512 + 2 * 256 * 256 * 2


def test_forward_argument_checks_precede_cuda(lib):
    p = ittt.make_problem(1, 512, 256, 512, 128, 4, 1e-3)
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: the checks fail first
    args = [fake] * 9
    # null pointer
    assert lib.ittt_fast_mlp_forward(ctypes.byref(p), None, *args[1:], None, 0, None) == \
        ittt.ERR_INVALID_ARG
    # missing workspace
    assert lib.ittt_fast_mlp_forward(ctypes.byref(p), *args, None, 0, None) == ittt.ERR_WORKSPACE
    # too small workspace
    assert lib.ittt_fast_mlp_forward(ctypes.byref(p), *args, fake, 16, None) == ittt.ERR_WORKSPACE
    # misaligned bf16 operand
    need = _ws(p)[1]
    bad = [ctypes.c_void_p((1 << 20) + 2)] + args[1:]
    assert lib.ittt_fast_mlp_forward(ctypes.byref(p), *bad, fake, need, None) == ittt.ERR_UNSUPPORTED
    # step entry points check their pointers too
    assert lib.ittt_apply(ctypes.byref(p), None, fake, fake, fake, None) == ittt.ERR_INVALID_ARG
    assert lib.ittt_fast_weight_scan(ctypes.byref(p), fake, fake, fake, None, fake, None) == \
        ittt.ERR_INVALID_ARG


def test_wait_limit_arguments(lib):
    assert lib.ittt_set_wait_limit_ns(0) == ittt.ERR_INVALID_ARG
    assert lib.ittt_selftest_wait_timeout(0, None) == ittt.ERR_INVALID_ARG
    assert lib.ittt_selftest_wait_timeout(10 ** 12, None) == ittt.ERR_INVALID_ARG
    assert lib.ittt_set_wait_limit_ns(4_000_000_000) == ittt.OK


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "weight_gated_mlp_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, fn


def test_probe_argument_checks(lib):
    got = ctypes.c_int(-1)
    assert lib.ittt_probe_start(0) == ittt.ERR_INVALID_ARG
    assert lib.ittt_probe_start(65537) == ittt.ERR_INVALID_ARG
    assert lib.ittt_probe_read(None, 4, ctypes.byref(got)) == ittt.ERR_INVALID_ARG
    assert lib.ittt_probe_read(None, 0, None) == ittt.ERR_INVALID_ARG
    # nothing probed: nothing to read, no CUDA call needed
    assert lib.ittt_probe_read(None, 0, ctypes.byref(got)) == ittt.OK and got.value == 0


def test_checks_argument_checks(lib):
    assert lib.ittt_set_checks(2) == ittt.ERR_INVALID_ARG
    assert lib.ittt_set_checks(-1) == ittt.ERR_INVALID_ARG
    assert lib.ittt_set_checks(0) == ittt.OK
    assert lib.ittt_check_buffer(None, 16) == ittt.ERR_INVALID_ARG


# (B, T, C, d, f, faster form): points of bench.py --sweep-forms on B200 where
# one form was more than 3% faster and the rule agrees, at three widths, B in
# {1, 2, 4} and T off the powers of two; AUTO must pick that form there.  (Of
# the sweep's 162 points the rule misses 16, e.g. B = 1, T = 1536, C = 256 at
# d = 2560: dual 0.336 vs prefix 0.354 ms with T C (d + f) = 194 d f.)
SWEEP_POINTS = [
    (1, 2048, 256, 2560, 9728, "prefix"),    # dual 0.455 vs prefix 0.432 ms
    (1, 1024, 512, 2560, 9728, "prefix"),    # 0.245 vs 0.287
    (4, 8192, 256, 2560, 9728, "hybrid"),    # 6.686 vs 9.318; the hybrid rule (T d >= 2^24)
    (1, 8192, 512, 2560, 9728, "prefix"),    # qwen3-4b: 1.347 vs 1.935
    (1, 1024, 256, 4096, 14336, "dual"),     # 0.530 vs 0.565
    (4, 1536, 256, 4096, 14336, "dual"),     # 2.592 vs 2.809
    (2, 2048, 256, 4096, 14336, "dual"),     # 1.710 vs 1.802
    (4, 3072, 256, 4096, 14336, "prefix"),   # 5.641 vs 6.043
    (1, 2048, 512, 4096, 14336, "prefix"),   # 0.819 vs 0.874
    (1, 8192, 1024, 4096, 14336, "prefix"),  # 3.131 vs 4.054
    (1, 1536, 256, 5120, 17408, "dual"),     # 1.024 vs 1.155
    (2, 2048, 256, 5120, 17408, "dual"),     # 2.556 vs 2.802
    (4, 1024, 256, 5120, 17408, "dual"),     # 2.687 vs 2.942
    (4, 3072, 256, 5120, 17408, "prefix"),   # 8.651 vs 10.790
    (1, 4096, 1024, 5120, 17408, "prefix"),  # 2.376 vs 2.540
]


# (B, T, C, d, f, faster form) of bench.py --compare-forms prefix,hybrid --paired
# on B200 at C = 256 (hybrid / prefix time in the comment)
HYBRID_POINTS = [
    (1, 2048, 256, 2560, 9728, "prefix"),     # 1.038
    (1, 4096, 256, 2560, 9728, "prefix"),     # 1.004 (T d = 2^23.3: below the cut)
    (1, 8192, 256, 2560, 9728, "hybrid"),     # 0.930
    (1, 131072, 256, 2560, 9728, "hybrid"),   # 0.924 (qwen3-4b-128k-c256)
    (1, 131072, 512, 2560, 9728, "prefix"),   # 0.994 (C = 512)
    (1, 4096, 256, 4096, 14336, "hybrid"),    # 0.909
    (1, 32768, 256, 4096, 14336, "hybrid"),   # 0.922
    (1, 4096, 256, 5120, 17408, "hybrid"),    # 0.960
    (1, 16384, 256, 5120, 17408, "hybrid"),   # 0.943
    (2, 16384, 256, 2560, 9728, "hybrid"),    # 0.954
]


@pytest.mark.parametrize("B,T,C,d,f,want", SWEEP_POINTS + HYBRID_POINTS + [
    (1, 16384, 512, 2560, 9728, "prefix"),   # long sequences, C = 512: the prefix form
    (1, 2048, 128, 4096, 14336, "dual"),     # C = 128, inside the threshold
])
def test_auto_form_follows_the_measured_crossover(lib, B, T, C, d, f, want):
    """AUTO's pick (and its workspace) is the form the sweep measured faster."""
    def ws(form):
        p = ittt.make_problem(B, T, d, f, C, 4, 1e-3, "bf16", form)
        n = ctypes.c_size_t(0)
        assert lib.ittt_workspace_size(ctypes.byref(p), ctypes.byref(n)) == ittt.OK
        return n.value
    assert ws("auto") == ws(want)
    assert ws("dual") != ws("prefix")
    assert ittt.resolve_form(ittt.make_problem(B, T, d, f, C, 4, 1e-3, "bf16", "auto")) == want


def test_auto_hybrid_rule(lib):
    """Past the dual threshold, the hybrid form exactly when C = 256, T d >= 2^24
    and the hybrid's groups fit (C = 256: groups of four chunks, at least two)."""
    for B, T, C, d, f in [(1, 6144, 256, 2560, 9728), (1, 6656, 256, 2560, 9728),
                          (3, 4096, 256, 4096, 14336), (1, 4096, 256, 4096, 14336),
                          (1, 3072, 256, 5120, 17408), (1, 3584, 256, 5120, 17408),
                          (1, 131072, 512, 2560, 9728), (1, 65536, 128, 2560, 9728),
                          (1, 7168, 256, 2560, 9728)]:
        n = T // C
        fits = C % 256 == 0 and n % 4 == 0 and n // 4 >= 2
        dual = C <= 256 and T * C * (d + f) <= 170 * d * f
        want = "dual" if dual else ("hybrid" if C == 256 and T * d >= 2 ** 24 and fits else "prefix")
        got = ittt.resolve_form(ittt.make_problem(B, T, d, f, C, 4, 1e-3, "bf16", "auto"))
        assert got == want, (B, T, C, d, f, got, want)


def test_auto_rule_is_the_fitted_threshold(lib):
    """The dual form exactly when C <= 256 and T C (d + f) <= 170 d f."""
    for B, T, C, d, f in [(1, 2048, 256, 4096, 14336), (1, 2560, 256, 4096, 14336),
                          (3, 1280, 256, 5120, 17408), (1, 1024, 512, 5120, 17408),
                          (2, 4096, 128, 2560, 9728), (1, 6144, 128, 2560, 9728)]:
        want = "dual" if C <= 256 and T * C * (d + f) <= 170 * d * f else "prefix"
        assert ittt.resolve_form(ittt.make_problem(B, T, d, f, C, 4, 1e-3, "bf16", "auto")) == want


@pytest.mark.parametrize("B,T,C,dtype,form,want", [
    (1, 2048, 256, "bf16", "hybrid", "hybrid"),
    (2, 4096, 512, "bf16", "hybrid", "hybrid"),
    (1, 1536, 128, "bf16", "hybrid", "prefix"),   # 12 chunks: not whole groups of 8
    (1, 2048, 128, "bf16", "hybrid", "prefix"),   # C = 128: the prefix form
    (1, 3072, 768, "bf16", "hybrid", "hybrid"),   # 4 chunks of 768: two groups of 2
    (1, 1024, 256, "bf16", "hybrid", "prefix"),   # one group
    (1, 2048, 256, "f32", "dual", "prefix"),      # fp32 has the prefix form only
    (1, 2048, 256, "f32", "hybrid", "prefix"),
    (1, 2048, 256, "bf16", "dual", "dual"),
    (1, 2048, 256, "bf16", "prefix", "prefix"),
])
def test_resolve_form(lib, B, T, C, dtype, form, want):
    p = ittt.make_problem(B, T, 256, 512, C, 4, 1e-3, dtype, form)
    assert ittt.resolve_form(p) == want
    v = ctypes.c_int32(-7)
    assert lib.ittt_resolve_form(ctypes.byref(p), None) == ittt.ERR_INVALID_ARG
    p.form = 9
    assert lib.ittt_resolve_form(ctypes.byref(p), ctypes.byref(v)) == ittt.ERR_INVALID_ARG
    assert v.value == -7                          # not written on an error


def test_hybrid_workspace_and_fallback(lib):
    def ws(T, C, form, d=256, f=512):
        p = ittt.make_problem(1, T, d, f, C, 4, 1e-3, "bf16", form)
        n = ctypes.c_size_t(0)
        assert lib.ittt_workspace_size(ctypes.byref(p), ctypes.byref(n)) == ittt.OK
        return n.value
    # groups of 4 chunks at C = 256 and qwen3-4b widths: 2 stored weights instead
    # of 7 (the in-group Gram blocks, 3 MB, cost far less than 5 weights of 50 MB)
    assert ws(2048, 256, "hybrid", 2560, 9728) < ws(2048, 256, "prefix", 2560, 9728)
    assert ws(2048, 256, "hybrid") != ws(2048, 256, "prefix")
    # 12 chunks of 128 do not make whole groups of 8: the prefix form runs
    assert ws(1536, 128, "hybrid") == ws(1536, 128, "prefix")
    # one group only: the prefix form runs
    assert ws(1024, 256, "hybrid") == ws(1024, 256, "prefix")


def test_no_cpu_fallback(monkeypatch):
    """Without the built library the package raises instead of computing, and
    host tensors are refused before any library call."""
    import torch

    monkeypatch.setattr(ittt, "_lib", None)
    with pytest.raises(RuntimeError, match="CUDA library missing"):
        ittt.load_library(os.path.join(os.path.dirname(ittt.LIB_PATH), "no_such_libittt.so"))
    monkeypatch.undo()
    d, f, T, C, k = 16, 32, 64, 16, 4
    H = torch.zeros((1, T, d), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        ittt.fast_mlp_forward(H, H.clone(), torch.zeros((f, d), dtype=torch.bfloat16),
                              torch.zeros((f, d), dtype=torch.bfloat16),
                              torch.zeros((d, f), dtype=torch.bfloat16),
                              torch.zeros((d, k), dtype=torch.bfloat16),
                              torch.zeros((d, d), dtype=torch.bfloat16), 0.01, C)
