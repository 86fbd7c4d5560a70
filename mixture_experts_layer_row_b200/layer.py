"""Buffer management around the C ABI: one MoE expert layer (forward + backward) on one GPU.

PyTorch only allocates device memory here; every step runs in libmoe_b200's kernels through
`moe_layer_fwd` / `moe_layer_bwd`.
"""
from __future__ import annotations

import torch

from . import _lib as L

_DT = {"fp32": (L.DTYPE_FP32, torch.float32), "bf16": (L.DTYPE_BF16, torch.bfloat16)}


class MoELayer:
    """Holds every caller-owned buffer of one layer configuration.

    Args:
        T, d, F, E, k: tokens, model width, expert hidden width, experts, experts per token.
        dtype: "bf16" (bf16 storage, fp32 accumulate) or "fp32" (GEMMs on tf32 tensor cores).
        learned_router: allocate router buffers (scores, score gradients, dW_r).
    """

    def __init__(self, T, d, F, E, k, dtype="bf16", device="cuda", learned_router=True, renorm=True):
        if dtype not in _DT:
            raise ValueError(f"unsupported dtype {dtype}")
        code, self.act = _DT[dtype]
        self.cfg = L.make_config(T, d, F, E, k, code, 1 if renorm else 0)
        self.T, self.d, self.F, self.E, self.k = T, d, F, E, k
        self.device = torch.device(device)
        self.R = L.max_rows(self.cfg)
        if self.R <= 0:
            raise L.MoEError("invalid layer configuration")
        dev, act, R = self.device, self.act, self.R
        i32, f32 = torch.int32, torch.float32

        def z(shape, dt):
            return torch.zeros(shape, dtype=dt, device=dev)

        self.ws = z(L.workspace_size(self.cfg), torch.uint8)
        self.learned_router = learned_router
        self.logits = z((T, E), f32) if learned_router else None
        self.idx, self.gates = z((T, k), i32), z((T, k), f32)
        self.counts, self.offsets, self.poff = z(E, i32), z(E + 1, i32), z(E + 1, i32)
        self.perm, self.prow, self.row_token = z(T * k, i32), z(T * k, i32), z(R, i32)
        self.x_perm, self.h13, self.a, self.y = z((R, d), act), z((R, 2 * F), act), z((R, F), act), z((R, d), act)
        self.out = z((T, d), act)
        self.dx = z((T, d), act)
        self.dW13, self.dW2 = z((E, 2 * F, d), act), z((E, d, F), act)
        self.dW_r = z((E, d), act) if learned_router else None
        self.dgates = z((T, k), f32)
        self.dy, self.dh13, self.dx_perm = z((R, d), act), z((R, 2 * F), act), z((R, d), act)
        self.saved = L.Saved(*[L.ptr(t) for t in (self.logits, self.idx, self.gates, self.counts,
                                                  self.offsets, self.poff, self.perm, self.prow,
                                                  self.row_token, self.x_perm, self.h13, self.a,
                                                  self.y)])
        self.grads = L.Grads(*[L.ptr(t) for t in (self.dW_r, self.dW13, self.dW2, self.dgates, self.dy,
                                                  self.dh13, self.dx_perm)])
        self._w = None

    def set_weights(self, W13, W2, W_r=None):
        for t, shape in ((W13, (self.E, 2 * self.F, self.d)), (W2, (self.E, self.d, self.F))):
            if tuple(t.shape) != shape or t.dtype != self.act or not t.is_contiguous():
                raise ValueError("weight shape/dtype/layout mismatch")
        if self.learned_router and W_r is None:
            raise ValueError("learned router needs W_r")
        self._keep = (W13, W2, W_r)
        self._w = L.Weights(L.ptr(W_r) if self.learned_router else None, L.ptr(W13), L.ptr(W2))

    def forward(self, x, bias=None, idx=None, gates=None, stream=None):
        """out = layer(x). With a learned router, routing comes from x W_r^T (+ bias); otherwise
        `idx` [T,k] int32 and `gates` [T,k] fp32 are copied in as the routing."""
        if self._w is None:
            raise RuntimeError("set_weights first")
        if not self.learned_router:
            self.idx.copy_(idx)
            self.gates.copy_(gates)
        self._x = x
        L.layer_fwd(self.cfg, self._w, x, bias, self.out, self.saved, self.ws, stream)
        return self.out

    def backward(self, dout, stream=None):
        """Fills dx, dW13, dW2 (and dW_r, dgates)."""
        L.layer_bwd(self.cfg, self._w, self.saved, self._x, dout, self.dx, self.grads, self.ws, stream)
        return self.dx

    def error_flags(self, stream=None) -> int:
        return L.get_error(self.ws, stream)
