"""The three compute steps of a context-parallel segment, on the CPU oracle
(fp64), for testing the orchestration of weight_gated_mlp_b200.parallel
without a GPU.  Interface of parallel.CudaSegmentOps: delta, prefix, apply,
and the attributes k, pad, W_down0."""

import numpy as np
import torch

from oracle import ittt_oracle as orc


class OracleSegmentOps:
    def __init__(self, inp, eta, C, clip=0.0, pad="sequence"):
        self.inp = inp                       # the shared weights (numpy)
        self.eta, self.C, self.clip, self.pad = eta, C, clip, pad
        self.k = inp["conv_kernel"].shape[1]
        self.W_down0 = torch.from_numpy(np.ascontiguousarray(inp["W_down0"]))

    def _segment(self, H, X0x):
        T = H.shape[1]
        seg = {k: self.inp[k] for k in ("W_gate", "W_up", "W_down0", "conv_kernel", "W_target")}
        seg["H"] = H.numpy()
        seg["X0"] = X0x[:, :T].numpy()
        if X0x.shape[1] > T:
            seg["X0_next"] = X0x[:, T:].numpy()
        return seg

    def delta(self, H, X0x, S_out=None):
        seg = self._segment(H, X0x)
        B, d, f = H.shape[0], *self.inp["W_down0"].shape
        # the state after the segment when it starts from zero: the sum of its
        # (clipped) deltas, which do not depend on the state
        _, S = orc.forward_sequential(seg, self.eta, self.C, clip=self.clip, pad=self.pad,
                                      W_start=np.zeros((B, d, f)))
        if S_out is None:
            S_out = torch.empty((B, d, f), dtype=torch.float32)
        S_out.copy_(torch.from_numpy(S))
        return S_out, seg

    def prefix(self, S_all):
        out = torch.zeros_like(S_all)
        for g in range(1, S_all.shape[0]):
            out[g] = out[g - 1] + S_all[g - 1]
        return out

    def apply(self, seg, P):
        W_start = self.inp["W_down0"].astype(np.float64)[None] + P.double().numpy()
        O, W = orc.forward_sequential(seg, self.eta, self.C, clip=self.clip, pad=self.pad,
                                      W_start=W_start)
        return torch.from_numpy(O), torch.from_numpy(W)
