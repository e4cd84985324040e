"""The target entry point that allocates nothing (ittt_lm_target_noalloc).

Some callers cannot allocate device memory: a plugin whose host framework
owns all device memory through its own pool, or a latency-critical loop that
cannot afford the implicit synchronisation of cudaMalloc, and neither has a
workspace to lend.  For them the library keeps the conv intermediate in a
built-in 16 MiB device array.  These tests check, through the C ABI, that the
variant gives the same Vhat as the workspace entry point on two calls in a
row (the shared array keeps the previous call's contents), and that a problem
too large for the array is refused before anything runs.

This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

import weight_gated_mlp_b200 as ittt
from weight_gated_mlp_b200 import _build
from synthetic import make_inputs, small_case

from _helpers import TOL, host, rel_err, to_device


def _call_noalloc(p, dev, V):
    lib = ittt.load_library()
    stream = int(torch.cuda.current_stream().cuda_stream) or None
    return lib.ittt_lm_target_noalloc(ctypes.byref(p), dev["X0"].data_ptr(),
                                      dev["conv_kernel"].data_ptr(), dev["W_target"].data_ptr(),
                                      V.data_ptr(), stream)


def test_noalloc_refuses_problems_beyond_its_scratch():
    _build.build()
    lib = ittt.load_library()
    # Y = B*T*d bf16 = 42 MB > 16 MiB: refused before any CUDA call
    p = ittt.make_problem(1, 8192, 2560, 9728, 512, 4, 1e-3)
    fake = ctypes.c_void_p(1 << 20)
    assert lib.ittt_lm_target_noalloc(ctypes.byref(p), fake, fake, fake, fake, None) == \
        ittt.ERR_WORKSPACE
    assert lib.ittt_lm_target_noalloc(ctypes.byref(p), None, fake, fake, fake, None) == \
        ittt.ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("dtype,T,d,k", [("bf16", 1024, 1024, 4), ("f32", 512, 320, 5)])
def test_noalloc_matches_workspace_entry_point_twice(dtype, T, d, k):
    _build.build()
    torch.cuda.set_device(0)
    C = 128 if dtype == "bf16" else 64
    for call, (seed, B) in enumerate(((11, 2), (12, 3))):
        w = small_case(T=T, C=C, d=d, f=64, k=k, B=B, eta=0.0, dtype=dtype)
        assert B * T * d * (2 if dtype == "bf16" else 4) <= ittt.NOALLOC_SCRATCH_BYTES
        dev = to_device(make_inputs(w, seed=seed), dtype)
        p = ittt.make_problem(B, T, d, 64, C, k, 0.0, dtype)
        V = torch.full((B * T, d), float("nan"), dtype=dev["X0"].dtype, device="cuda")
        assert _call_noalloc(p, dev, V) == ittt.OK, f"call {call}"
        assert ittt.get_last_error() == ittt.OK
        ref = ittt.lm_target(dev["X0"], dev["conv_kernel"], dev["W_target"], C=C)
        assert ittt.get_last_error() == ittt.OK
        got, want = host(V), host(ref)
        assert np.isfinite(got).all(), f"call {call}"
        assert rel_err(got, want) <= TOL[dtype], f"call {call}: {rel_err(got, want)}"
