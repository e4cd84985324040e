"""Python binding of ``libittt.so``, the B200 (sm_100a) In-Place TTT fast-weight MLP layer.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI of ``include/ittt.h``.  torch supplies device
memory and streams.  The library must have been built
(``python -m weight_gated_mlp_b200._build``); importing this module without
it raises, and there is no CPU fallback.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libittt.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_FAULT = range(7)
FLAG_PAD_CHUNK_END, FLAG_X0_LOOKAHEAD = 1, 2
F32, BF16 = 0, 1
FORM_AUTO, FORM_PREFIX, FORM_DUAL, FORM_HYBRID = 0, 1, 2, 3
_FORMS = {"auto": FORM_AUTO, "prefix": FORM_PREFIX, "dual": FORM_DUAL, "hybrid": FORM_HYBRID}

# every entry point include/ittt.h declares
EXPORTED = (
    "ittt_version", "ittt_status_string", "ittt_workspace_size", "ittt_fast_mlp_forward",
    "ittt_gated_activations", "ittt_lookahead_conv", "ittt_lm_target", "ittt_fast_weight_scan",
    "ittt_apply", "ittt_get_last_error", "ittt_set_wait_limit_ns", "ittt_selftest_wait_timeout",
    "ittt_lm_target_noalloc", "ittt_clip_update_targets", "ittt_decode_workspace_size",
    "ittt_decode_step", "ittt_cp_workspace_size", "ittt_cp_delta", "ittt_cp_apply",
    "ittt_cp_prefix", "ittt_probe_start", "ittt_probe_read", "ittt_set_checks",
    "ittt_check_buffer", "ittt_resolve_form", "ittt_selftest_device_check",
    "ittt_chunk_recurrence", "ittt_probe_read2",
)
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class IttTError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("d", ctypes.c_int64),
                ("f", ctypes.c_int64), ("C", ctypes.c_int32), ("k", ctypes.c_int32),
                ("eta", ctypes.c_float), ("dtype", ctypes.c_int32), ("form", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("clip", ctypes.c_float), ("reserved", ctypes.c_int32)]


_lib: Optional[ctypes.CDLL] = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libittt.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library missing: {path} (run python -m weight_gated_mlp_b200._build)")
    lib = ctypes.CDLL(path)
    vp, i32, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64
    P = ctypes.POINTER(Problem)
    sig = {
        "ittt_version": ([], i32),
        "ittt_status_string": ([i32], ctypes.c_char_p),
        "ittt_workspace_size": ([P, ctypes.POINTER(ctypes.c_size_t)], i32),
        "ittt_fast_mlp_forward": ([P] + [vp] * 10 + [ctypes.c_size_t, vp], i32),
        "ittt_gated_activations": ([P, vp, vp, vp, vp, vp], i32),
        "ittt_lookahead_conv": ([P, vp, vp, vp, vp], i32),
        "ittt_lm_target": ([P, vp, vp, vp, vp, vp, ctypes.c_size_t, vp], i32),
        "ittt_fast_weight_scan": ([P, vp, vp, vp, vp, vp, vp], i32),
        "ittt_apply": ([P, vp, vp, vp, vp, vp], i32),
        "ittt_get_last_error": ([vp], i32),
        "ittt_set_wait_limit_ns": ([u64], i32),
        "ittt_selftest_wait_timeout": ([u64, vp], i32),
        "ittt_selftest_device_check": ([P, vp, vp, vp, vp, vp], i32),
        "ittt_chunk_recurrence": ([P, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp], i32),
        "ittt_lm_target_noalloc": ([P, vp, vp, vp, vp, vp], i32),
        "ittt_clip_update_targets": ([P, vp, vp, vp, vp], i32),
        "ittt_decode_workspace_size": ([P, ctypes.POINTER(ctypes.c_size_t)], i32),
        "ittt_decode_step": ([P, ctypes.c_int64] + [vp] * 11 + [ctypes.c_size_t, vp], i32),
        "ittt_cp_workspace_size": ([P, ctypes.POINTER(ctypes.c_size_t)], i32),
        "ittt_cp_delta": ([P] + [vp] * 8 + [ctypes.c_size_t, vp], i32),
        "ittt_cp_apply": ([P] + [vp] * 6 + [ctypes.c_size_t, vp], i32),
        "ittt_cp_prefix": ([vp, ctypes.c_int64, ctypes.c_int64, vp, vp], i32),
        "ittt_probe_start": ([i32], i32),
        "ittt_set_checks": ([i32], i32),
        "ittt_check_buffer": ([vp, ctypes.c_size_t], i32),
        "ittt_resolve_form": ([P, ctypes.POINTER(ctypes.c_int32)], i32),
        "ittt_probe_read": ([vp, i32, ctypes.POINTER(ctypes.c_int)], i32),
        "ittt_probe_read2": ([vp, vp, i32, ctypes.POINTER(ctypes.c_int)], i32),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().ittt_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != OK:
        raise IttTError(status, where)


def make_problem(B: int, T: int, d: int, f: int, C: int, k: int, eta: float, dtype: str = "bf16",
                 form: str = "auto", clip: float = 0.0, flags: int = 0) -> Problem:
    return Problem(B, T, d, f, C, k, float(eta), BF16 if dtype == "bf16" else F32, _FORMS[form],
                   int(flags), float(clip), 0)


def workspace_size(p: Problem) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().ittt_workspace_size(ctypes.byref(p), ctypes.byref(n)), "ittt_workspace_size")
    return int(n.value)


def resolve_form(p: Problem) -> str:
    """Name of the form the forward takes for *p ("prefix", "dual" or "hybrid")."""
    v = ctypes.c_int32(-1)
    _check(load_library().ittt_resolve_form(ctypes.byref(p), ctypes.byref(v)), "ittt_resolve_form")
    return {FORM_PREFIX: "prefix", FORM_DUAL: "dual", FORM_HYBRID: "hybrid"}[v.value]


# --------------------------------------------------------------- torch helpers

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


def _dtype_name(t) -> str:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return "bf16"
    if t.dtype == torch.float32:
        return "f32"
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_tensor(t, name: str, shape, dtype) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def problem_from(H, W_gate, conv_kernel, eta: float, C: int, form: str = "auto",
                 clip: float = 0.0, flags: int = 0) -> Problem:
    B, T, d = H.shape
    f = W_gate.shape[0]
    return make_problem(B, T, d, f, C, conv_kernel.shape[1], eta, _dtype_name(H), form, clip, flags)


def fast_mlp_forward(H, X0, W_gate, W_up, W_down0, conv_kernel, W_target, eta: float, C: int,
                     form: str = "auto", workspace=None, out=None, w_final=None,
                     stream=None, clip: float = 0.0, pad: str = "sequence"
                     ) -> Tuple["object", "object"]:
    """(O [B,T,d], W_down_final [B,d,f] fp32) of the fast-weight MLP prefill.

    H: [B, T, d]; X0: [B, T, d], or [B, T + k - 1, d] with the next segment's
    first k - 1 rows appended (segment continuation); W_gate, W_up: [f, d];
    W_down0: [d, f] (a carried W_down_final of one sequence for a continued
    segment); conv_kernel: [d, k]; W_target: [d, d]; all of one dtype (bf16 or
    fp32) on one device.  clip > 0 bounds the Frobenius norm of every chunk's
    update delta; pad = "chunk" stops the conv's look-ahead at chunk ends.
    """
    torch = _torch()
    k = conv_kernel.shape[1]
    flags = FLAG_PAD_CHUNK_END if pad == "chunk" else 0
    if X0.shape[1] == H.shape[1] + k - 1 and k > 1:
        flags |= FLAG_X0_LOOKAHEAD
    p = problem_from(H, W_gate, conv_kernel, eta, C, form, clip, flags)
    B, T, d, f = p.B, p.T, p.d, p.f
    dt = H.dtype
    Tx = T + (k - 1 if flags & FLAG_X0_LOOKAHEAD else 0)
    for t, name, shape in ((H, "H", (B, T, d)), (X0, "X0", (B, Tx, d)), (W_gate, "W_gate", (f, d)),
                           (W_up, "W_up", (f, d)), (W_down0, "W_down0", (d, f)),
                           (conv_kernel, "conv_kernel", (d, k)), (W_target, "W_target", (d, d))):
        _check_tensor(t, name, shape, dt)
    ws_bytes = workspace_size(p)
    if workspace is None or workspace.numel() < ws_bytes:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=H.device)
    if out is None:
        out = torch.empty((B, T, d), dtype=dt, device=H.device)
    if w_final is None:
        w_final = torch.empty((B, d, f), dtype=torch.float32, device=H.device)
    lib = load_library()
    st = lib.ittt_fast_mlp_forward(ctypes.byref(p), _ptr(H), _ptr(X0), _ptr(W_gate), _ptr(W_up),
                                   _ptr(W_down0), _ptr(conv_kernel), _ptr(W_target), _ptr(out),
                                   _ptr(w_final), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "ittt_fast_mlp_forward")
    return out, w_final


def gated_activations(H, W_gate, W_up, stream=None):
    """Z [B*T, f] = silu(H W_gate^T) * (H W_up^T)."""
    torch = _torch()
    B, T, d = H.shape
    f = W_gate.shape[0]
    p = make_problem(B, T, d, f, T, 1, 0.0, _dtype_name(H))
    Z = torch.empty((B * T, f), dtype=H.dtype, device=H.device)
    _check(load_library().ittt_gated_activations(ctypes.byref(p), _ptr(H), _ptr(W_gate), _ptr(W_up),
                                                 _ptr(Z), _stream(stream)), "ittt_gated_activations")
    return Z


def lookahead_conv(X0, conv_kernel, stream=None):
    """Y [B, T, d] = depthwise look-ahead Conv1D of X0 (zero past each sequence end)."""
    torch = _torch()
    B, T, d = X0.shape
    p = make_problem(B, T, d, 8, T, conv_kernel.shape[1], 0.0, _dtype_name(X0))
    Y = torch.empty_like(X0)
    _check(load_library().ittt_lookahead_conv(ctypes.byref(p), _ptr(X0), _ptr(conv_kernel), _ptr(Y),
                                              _stream(stream)), "ittt_lookahead_conv")
    return Y


def lm_target(X0, conv_kernel, W_target, C: Optional[int] = None, stream=None):
    """Vhat [B*T, d] = Conv1D(X0) W_target."""
    torch = _torch()
    B, T, d = X0.shape
    p = make_problem(B, T, d, 8, C or T, conv_kernel.shape[1], 0.0, _dtype_name(X0))
    ws = torch.empty(max(workspace_size(p), 1), dtype=torch.uint8, device=X0.device)
    V = torch.empty((B * T, d), dtype=X0.dtype, device=X0.device)
    _check(load_library().ittt_lm_target(ctypes.byref(p), _ptr(X0), _ptr(conv_kernel), _ptr(W_target),
                                         _ptr(V), _ptr(ws), ws.numel(), _stream(stream)),
           "ittt_lm_target")
    return V


def lm_target_noalloc(X0, conv_kernel, W_target, C: Optional[int] = None, stream=None):
    """Vhat [B*T, d] = Conv1D(X0) W_target without any device allocation by the library.

    For callers that cannot allocate device memory (see ittt_lm_target_noalloc
    in include/ittt.h): the intermediate lives in the library's built-in
    16 MiB scratch array, shared by all calls on a device, so calls that may
    overlap on the GPU must be serialised.  Only the output is allocated here,
    by torch, for convenience; pass-through C callers allocate nothing.
    """
    torch = _torch()
    B, T, d = X0.shape
    p = make_problem(B, T, d, 8, C or T, conv_kernel.shape[1], 0.0, _dtype_name(X0))
    V = torch.empty((B * T, d), dtype=X0.dtype, device=X0.device)
    _check(load_library().ittt_lm_target_noalloc(ctypes.byref(p), _ptr(X0), _ptr(conv_kernel),
                                                 _ptr(W_target), _ptr(V), _stream(stream)),
           "ittt_lm_target_noalloc")
    return V


def fast_weight_scan(Vhat, Z, W_down0, B: int, T: int, C: int, eta: float, stream=None):
    """(W_stack [B, n-1, d, f] of the input dtype, W_down_final [B, d, f] fp32)."""
    torch = _torch()
    d, f = W_down0.shape
    n = T // C
    p = make_problem(B, T, d, f, C, 1, eta, _dtype_name(Z))
    stack = torch.empty((B, max(n - 1, 0), d, f), dtype=Z.dtype, device=Z.device)
    wf = torch.empty((B, d, f), dtype=torch.float32, device=Z.device)
    _check(load_library().ittt_fast_weight_scan(ctypes.byref(p), _ptr(Vhat), _ptr(Z), _ptr(W_down0),
                                                _ptr(stack) if n > 1 else None, _ptr(wf),
                                                _stream(stream)), "ittt_fast_weight_scan")
    return stack, wf


def chunk_recurrence(Z, Vhat, W_down0, B: int, T: int, C: int, eta: float, form: str = "auto",
                     workspace=None, stream=None):
    """(O [B, T, d], W_down_final [B, d, f] fp32) from Z [B*T, f] and Vhat [B*T, d]
    by the chunk recurrence (the form *form* resolves to; no clipping)."""
    torch = _torch()
    d, f = W_down0.shape
    p = make_problem(B, T, d, f, C, 1, eta, _dtype_name(Z), form)
    if workspace is None:
        workspace = torch.empty(workspace_size(p), dtype=torch.uint8, device=Z.device)
    O = torch.empty((B, T, d), dtype=Z.dtype, device=Z.device)
    wf = torch.empty((B, d, f), dtype=torch.float32, device=Z.device)
    _check(load_library().ittt_chunk_recurrence(ctypes.byref(p), _ptr(Z), _ptr(Vhat), _ptr(W_down0),
                                                _ptr(O), _ptr(wf), _ptr(workspace),
                                                workspace.numel(), _stream(stream)),
           "ittt_chunk_recurrence")
    return O, wf


def apply(Z, W_down0, W_stack, B: int, T: int, C: int, stream=None):
    """O [B*T, d] with O_i = Z_i W^(i)^T."""
    torch = _torch()
    d, f = W_down0.shape
    n = T // C
    p = make_problem(B, T, d, f, C, 1, 0.0, _dtype_name(Z))
    O = torch.empty((B * T, d), dtype=Z.dtype, device=Z.device)
    _check(load_library().ittt_apply(ctypes.byref(p), _ptr(Z), _ptr(W_down0),
                                     _ptr(W_stack) if n > 1 else None, _ptr(O), _stream(stream)),
           "ittt_apply")
    return O


def clip_update_targets(Z, Vhat, B: int, T: int, C: int, eta: float, clip: float, stream=None):
    """Per-chunk delta norms [B, T/C] (before clipping); Vhat is rescaled in place."""
    torch = _torch()
    d = Vhat.shape[1]
    f = Z.shape[1]
    p = make_problem(B, T, d, f, C, 1, eta, _dtype_name(Z), clip=clip)
    norms = torch.empty((B, T // C), dtype=torch.float32, device=Z.device)
    _check(load_library().ittt_clip_update_targets(ctypes.byref(p), _ptr(Z), _ptr(Vhat),
                                                   _ptr(norms), _stream(stream)),
           "ittt_clip_update_targets")
    return norms


class Decoder:
    """Token-by-token decoding of B <= 8 sequences in lockstep (chunk-end padding).

    Holds the fp32 fast-weight state [B, d, f] and the current chunk's Z and X0
    rows; step(H_tok, X0_tok) returns O_tok [B, d] and, after every C-th
    token, applies that chunk's update to the state.  On the bf16 path the
    per-token product uses the state rounded to bf16 (kept in the workspace,
    rebuilt at each chunk's first token), as the prefill does.
    """

    def __init__(self, W_gate, W_up, W_down0, conv_kernel, W_target, B: int, eta: float, C: int,
                 clip: float = 0.0):
        torch = _torch()
        f, d = W_gate.shape
        self.w = (W_gate, W_up, conv_kernel, W_target)
        self.p = make_problem(B, C, d, f, C, conv_kernel.shape[1], eta, _dtype_name(W_gate),
                              clip=clip, flags=FLAG_PAD_CHUNK_END)
        n = ctypes.c_size_t(0)
        _check(load_library().ittt_decode_workspace_size(ctypes.byref(self.p), ctypes.byref(n)),
               "ittt_decode_workspace_size")
        dev, dt = W_gate.device, W_gate.dtype
        self.ws = torch.empty(max(int(n.value), 1), dtype=torch.uint8, device=dev)
        self.state = W_down0.float().unsqueeze(0).repeat(B, 1, 1).contiguous()
        self.Z = torch.zeros((B, C, f), dtype=dt, device=dev)
        self.X0 = torch.zeros((B, C, d), dtype=dt, device=dev)
        self.pos = 0
        # the arguments that stay the same from token to token, marshalled once
        Wg, Wu, K, Wt = self.w
        self._fixed = (_ptr(Wg), _ptr(Wu), _ptr(K), _ptr(Wt), _ptr(self.state), _ptr(self.Z),
                       _ptr(self.X0))
        self._fn = load_library().ittt_decode_step
        self._pref = ctypes.byref(self.p)

    def step(self, H_tok, X0_tok, out=None, stream=None):
        if out is None:
            out = _torch().empty_like(H_tok)
        _check(self._fn(self._pref, self.pos, H_tok.data_ptr(), X0_tok.data_ptr(), *self._fixed,
                        out.data_ptr(), self.ws.data_ptr(), self.ws.numel(), _stream(stream)),
               "ittt_decode_step")
        self.pos += 1
        return out

    def capture(self):
        """Record the step of every position of a chunk as one CUDA graph each,
        over static buffers H_in, X0_in (inputs) and O_out (output); replay()
        then runs a step with a single graph launch.  Recording runs nothing:
        the state and the chunk buffers are untouched.  Call between chunks or
        before the first token."""
        torch = _torch()
        B, d, C = self.p.B, self.p.d, self.p.C
        dev, dt = self.state.device, self.Z.dtype
        self.H_in = torch.zeros((B, d), dtype=dt, device=dev)
        self.X0_in = torch.zeros((B, d), dtype=dt, device=dev)
        self.O_out = torch.empty((B, d), dtype=dt, device=dev)
        lib = load_library()
        Wg, Wu, K, Wt = self.w
        side = torch.cuda.Stream(device=dev)
        graphs = []
        for slot in range(C):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                _check(lib.ittt_decode_step(
                    ctypes.byref(self.p), slot, _ptr(self.H_in), _ptr(self.X0_in), _ptr(Wg),
                    _ptr(Wu), _ptr(K), _ptr(Wt), _ptr(self.state), _ptr(self.Z), _ptr(self.X0),
                    _ptr(self.O_out), _ptr(self.ws), self.ws.numel(), _stream(side)),
                    "ittt_decode_step")
            graphs.append(g)
        self.graphs = graphs

    def replay(self, H_tok=None, X0_tok=None):
        """One step through the recorded graphs: copies the token's rows into
        H_in / X0_in when given (or the caller has written them), returns O_out
        (overwritten by the next step)."""
        if H_tok is not None:
            self.H_in.copy_(H_tok)
        if X0_tok is not None:
            self.X0_in.copy_(X0_tok)
        self.graphs[self.pos % self.p.C].replay()
        self.pos += 1
        return self.O_out


# ------------------------------------------------------------ context parallel

class CpState:
    """What ittt_cp_delta leaves for ittt_cp_apply of the same segment: the
    problem, the workspace (Z and the segment's running sums) and S."""

    def __init__(self, p: Problem, workspace, dtype, S):
        self.p, self.workspace, self.dtype, self.S = p, workspace, dtype, S


def cp_delta(H, X0, W_gate, W_up, conv_kernel, W_target, eta: float, C: int, clip: float = 0.0,
             pad: str = "sequence", S=None, stream=None):
    """(S [B, d, f] fp32, CpState): one segment's summed (clipped) chunk deltas.

    H: [B, T, d] (segment r of each sequence); X0: [B, T, d], or [B, T + k - 1, d]
    with the next segment's first k - 1 rows appended (sequence-end padding,
    every rank but the last)."""
    torch = _torch()
    k = conv_kernel.shape[1]
    flags = FLAG_PAD_CHUNK_END if pad == "chunk" else 0
    if X0.shape[1] == H.shape[1] + k - 1 and k > 1:
        flags |= FLAG_X0_LOOKAHEAD
    p = problem_from(H, W_gate, conv_kernel, eta, C, "auto", clip, flags)
    B, T, d, f = p.B, p.T, p.d, p.f
    Tx = T + (k - 1 if flags & FLAG_X0_LOOKAHEAD else 0)
    for t, name, shape in ((H, "H", (B, T, d)), (X0, "X0", (B, Tx, d)), (W_gate, "W_gate", (f, d)),
                           (W_up, "W_up", (f, d)), (conv_kernel, "conv_kernel", (d, k)),
                           (W_target, "W_target", (d, d))):
        _check_tensor(t, name, shape, H.dtype)
    n = ctypes.c_size_t(0)
    lib = load_library()
    _check(lib.ittt_cp_workspace_size(ctypes.byref(p), ctypes.byref(n)), "ittt_cp_workspace_size")
    ws = torch.empty(max(int(n.value), 1), dtype=torch.uint8, device=H.device)
    if S is None:
        S = torch.empty((B, d, f), dtype=torch.float32, device=H.device)
    _check_tensor(S, "S", (B, d, f), torch.float32)
    _check(lib.ittt_cp_delta(ctypes.byref(p), _ptr(H), _ptr(X0), _ptr(W_gate), _ptr(W_up),
                             _ptr(conv_kernel), _ptr(W_target), _ptr(S), _ptr(ws), ws.numel(),
                             _stream(stream)), "ittt_cp_delta")
    return S, CpState(p, ws, H.dtype, S)


def cp_prefix(S_all, out=None, stream=None):
    """P_all[g] = S_all[0] + ... + S_all[g-1] (row 0 zeros) for S_all [G, ...] fp32."""
    torch = _torch()
    if out is None:
        out = torch.empty_like(S_all)
    _check_tensor(S_all, "S_all", tuple(S_all.shape), torch.float32)
    _check_tensor(out, "out", tuple(S_all.shape), torch.float32)
    G = S_all.shape[0]
    n = S_all.numel() // max(G, 1)
    _check(load_library().ittt_cp_prefix(_ptr(S_all), G, n, _ptr(out), _stream(stream)),
           "ittt_cp_prefix")
    return out


def cp_apply(state: CpState, W_down0, P, out=None, w_end=None, stream=None):
    """(O [B, T, d], W_end [B, d, f] fp32) of the segment from W_down0 + P (S: the
    segment's sum returned by cp_delta, which must still hold it).  Once per
    cp_delta: the running sums in the workspace become the effective weights."""
    torch = _torch()
    p = state.p
    B, T, d, f = p.B, p.T, p.d, p.f
    dev = state.workspace.device
    _check_tensor(W_down0, "W_down0", (d, f), state.dtype)
    _check_tensor(P, "P", (B, d, f), torch.float32)
    if out is None:
        out = torch.empty((B, T, d), dtype=state.dtype, device=dev)
    if w_end is None:
        w_end = torch.empty((B, d, f), dtype=torch.float32, device=dev)
    _check(load_library().ittt_cp_apply(ctypes.byref(p), _ptr(W_down0), _ptr(P), _ptr(state.S),
                                        _ptr(out), _ptr(w_end), _ptr(state.workspace),
                                        state.workspace.numel(), _stream(stream)), "ittt_cp_apply")
    return out, w_end


def set_checks(level: int) -> None:
    """1: every compute call first checks its buffers against their device
    allocations (see ittt_set_checks); 0: off (the default)."""
    _check(load_library().ittt_set_checks(int(level)), "ittt_set_checks")


def probe_start(n: int) -> None:
    """Time the gate/up GEMM of the next n forwards on this thread (CUDA events
    around its launch; see ittt_probe_start)."""
    _check(load_library().ittt_probe_start(int(n)), "ittt_probe_start")


def probe_read(capacity: int):
    """The probed kernel times in ms of the forwards since probe_start."""
    buf = (ctypes.c_float * max(int(capacity), 1))()
    got = ctypes.c_int(0)
    _check(load_library().ittt_probe_read(buf, int(capacity), ctypes.byref(got)), "ittt_probe_read")
    return [float(buf[i]) for i in range(got.value)]


def probe_read2(capacity: int):
    """(gate/up GEMM ms, chunk recurrence ms) lists of the forwards since probe_start."""
    n = max(int(capacity), 1)
    g, r = (ctypes.c_float * n)(), (ctypes.c_float * n)()
    got = ctypes.c_int(0)
    _check(load_library().ittt_probe_read2(g, r, int(capacity), ctypes.byref(got)),
           "ittt_probe_read2")
    return [float(g[i]) for i in range(got.value)], [float(r[i]) for i in range(got.value)]


def get_last_error(stream=None) -> int:
    return int(load_library().ittt_get_last_error(_stream(stream)))


def set_wait_limit_ns(ns: int) -> None:
    _check(load_library().ittt_set_wait_limit_ns(int(ns)), "ittt_set_wait_limit_ns")


def selftest_device_check(Z, W_down0, W_stack, O, B: int, T: int, C: int, stream=None) -> None:
    """ittt_apply into O with the kernel told that W_stack holds one slice fewer
    than it does (the device-side index check skips the last sequence's last
    chunk and reports ITTT_ERR_DEVICE_FAULT through get_last_error)."""
    d, f = W_down0.shape
    p = make_problem(B, T, d, f, C, 1, 0.0, _dtype_name(Z))
    _check(load_library().ittt_selftest_device_check(ctypes.byref(p), _ptr(Z), _ptr(W_down0),
                                                     _ptr(W_stack), _ptr(O), _stream(stream)),
           "ittt_selftest_device_check")


def selftest_wait_timeout(ns: int, stream=None) -> None:
    _check(load_library().ittt_selftest_wait_timeout(int(ns), _stream(stream)),
           "ittt_selftest_wait_timeout")
