"""Workload shapes and the seeded input generator.

Shapes follow the model widths the In-Place TTT pages evaluate (Qwen3-4B,
LLaMA-3.1-8B, Qwen3-14B; "In-Place Test-Time Training" deep-read notes and
the iplexlaw review, section 7) at the prefill lengths of the efficiency
figure (8k / 32k / 128k, review section 7.5, Figure 4) and the chunk sizes of
the ablation (512-1024, review section 7.4).  Weights are random: there are
no trained checkpoints here.

Distribution recipe ("N(0, v)" means variance v):

* tiny fp32 case: H, X0 ~ N(0, 1); W_gate, W_up, W_down0, W_target ~
  N(0, 1/fan_in); conv kernel ~ N(0, 0.1).
* model-shaped bf16 cases: H rows ~ N(0, 1) then RMS-normalised
  (h / sqrt(mean(h^2))); X0 ~ N(0, 0.02); W_gate, W_up, W_down0 ~
  N(0, 1/fan_in); W_target ~ N(0, 1e-2 / d_model); conv kernel ~ N(0, 0.1).

fan_in is the contracted dimension: d for W_gate/W_up ([f, d]) and for
W_target ([d, d]); f for W_down0 ([d, f]).

One numpy Generator(seed) draws float32 normals in the fixed order H, X0,
W_gate, W_up, W_down0, W_target, conv_kernel; the B sequences of a batch are
one [B, T, d] draw.  bf16 workloads are rounded once (round to nearest even)
and both the GPU path and the oracle consume exactly those rounded values.
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dtype: str  # "f32" or "bf16"
    B: int
    T: int
    d: int
    f: int
    C: int
    k: int
    eta: float
    tiny_distributions: bool  # True: the tiny fp32 recipe; False: model-shaped recipe

    @property
    def n_chunks(self) -> int:
        return self.T // self.C

    def flops(self) -> float:
        """Algorithmic FLOP of one forward pass, prefix form: B(8Tdf + 2Td^2 + 2Tdk)."""
        B, T, d, f, k = self.B, self.T, self.d, self.f, self.k
        return float(B) * (8.0 * T * d * f + 2.0 * T * d * d + 2.0 * T * d * k)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny-fp32": Workload("tiny-fp32", "f32", 1, 256, 64, 256, 64, 4, 0.01, True),
    "qwen3-4b": Workload("qwen3-4b", "bf16", 1, 8192, 2560, 9728, 512, 4, 1e-3, False),
    "llama3.1-8b": Workload("llama3.1-8b", "bf16", 1, 32768, 4096, 14336, 1024, 4, 1e-3, False),
    "qwen3-14b-b4": Workload("qwen3-14b-b4", "bf16", 4, 16384, 5120, 17408, 1024, 4, 1e-3, False),
}
for _C in (256, 512, 1024, 2048):
    WORKLOADS[f"qwen3-4b-128k-c{_C}"] = Workload(
        f"qwen3-4b-128k-c{_C}", "bf16", 1, 131072, 2560, 9728, _C, 4, 1e-3, False)


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    r = ((u + bias) & np.uint64(0xFFFF0000)).astype(np.uint32)
    # NaN/Inf are never produced by the recipes; keep them untouched anyway.
    special = (u & np.uint64(0x7F800000)) == np.uint64(0x7F800000)
    r = np.where(special, x.view(np.uint32), r)
    return r.view(np.float32)


def make_inputs(w: Workload, seed: int = 0) -> Dict[str, np.ndarray]:
    """Draw one workload's inputs.  All arrays are float32 C-contiguous.

    Keys and shapes: H [B,T,d], X0 [B,T,d], W_gate [f,d], W_up [f,d],
    W_down0 [d,f], W_target [d,d] (applied as Y @ W_target), conv_kernel [d,k]
    (tap j of channel c multiplies X0[t+j, c]).
    """
    rng = np.random.default_rng(seed)
    B, T, d, f, k = w.B, w.T, w.d, w.f, w.k

    def normal(shape, var: float) -> np.ndarray:
        a = rng.standard_normal(shape, dtype=np.float32)
        if var != 1.0:
            a *= np.float32(np.sqrt(var))
        return a

    if w.tiny_distributions:
        H = normal((B, T, d), 1.0)
        X0 = normal((B, T, d), 1.0)
        W_gate = normal((f, d), 1.0 / d)
        W_up = normal((f, d), 1.0 / d)
        W_down0 = normal((d, f), 1.0 / f)
        W_target = normal((d, d), 1.0 / d)
        conv = normal((d, k), 0.1)
    else:
        H = normal((B, T, d), 1.0)
        ms = np.mean(np.square(H, dtype=np.float32), axis=-1, keepdims=True, dtype=np.float32)
        H /= np.sqrt(np.maximum(ms, np.float32(1e-12)))
        X0 = normal((B, T, d), 0.02)
        W_gate = normal((f, d), 1.0 / d)
        W_up = normal((f, d), 1.0 / d)
        W_down0 = normal((d, f), 1.0 / f)
        W_target = normal((d, d), 1e-2 / d)
        conv = normal((d, k), 0.1)

    out = dict(H=H, X0=X0, W_gate=W_gate, W_up=W_up, W_down0=W_down0,
               W_target=W_target, conv_kernel=conv)
    if w.dtype == "bf16":
        out = {key: round_to_bf16(v) for key, v in out.items()}
    return {key: np.ascontiguousarray(v) for key, v in out.items()}


def small_case(T: int, C: int, d: int, f: int, k: int = 4, B: int = 1, eta: float = 0.01,
               dtype: str = "f32", name: Optional[str] = None) -> Workload:
    """An ad-hoc small workload with the tiny recipe's distributions."""
    return Workload(name or f"small-T{T}-C{C}-d{d}-f{f}-k{k}-B{B}-{dtype}", dtype, B, T, d, f, C,
                    k, eta, True)
