"""Buffer management around the C ABI: one MoE expert layer (forward + backward) on one GPU.

PyTorch only allocates device memory here; every step runs in libmoe_b200's kernels through
`moe_layer_fwd` / `moe_layer_bwd`.
"""
from __future__ import annotations

import torch

from . import _lib as L

_DT = {"fp32": (L.DTYPE_FP32, torch.float32), "bf16": (L.DTYPE_BF16, torch.bfloat16),
       "mxfp8": (L.DTYPE_MXFP8, torch.bfloat16)}


class MoELayer:
    """Holds every caller-owned buffer of one layer configuration.

    Args:
        T, d, F, E, k: tokens, model width, expert hidden width, experts, experts per token.
        dtype: "bf16" (bf16 storage, fp32 accumulate), "fp32" (GEMMs on tf32 tensor cores) or
            "mxfp8" (bf16 storage, expert GEMMs on E4M3 operands with UE8M0 block scales).
        learned_router: allocate router buffers (scores, score gradients, dW_r).
    """

    def __init__(self, T, d, F, E, k, dtype="bf16", device="cuda", learned_router=True, renorm=True,
                 recompute=False):
        """recompute: keep no h13 between the passes; the backward regenerates it with one more GEMM1
        (bf16 / fp32 layers)."""
        if dtype not in _DT:
            raise ValueError(f"unsupported dtype {dtype}")
        if recompute and dtype == "mxfp8":
            raise ValueError("activation recompute is implemented for the bf16 / fp32 layer")
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
        self.recompute = recompute
        self.mx = dtype == "mxfp8"
        # MXFP8: the routed input, a, dy and dh13 exist only as their two quantised forms (qa_t)
        self.x_perm = None if self.mx else z((R, d), act)
        self.a = None if self.mx else z((R, F), act)
        self.y = z((R, d), act)
        self.h13 = None if recompute else z((R, 2 * F), act)
        self.out = z((T, d), act)
        self.dx = z((T, d), act)
        self.dW13, self.dW2 = z((E, 2 * F, d), act), z((E, d, F), act)
        self.dW_r = z((E, d), act) if learned_router else None
        self.dgates = z((T, k), f32)
        self.dy = None if self.mx else z((R, d), act)
        self.dh13 = None if self.mx else z((R, 2 * F), act)
        self.dx_perm = z((R, d), act)
        if self.mx:
            u8 = torch.uint8
            self.qw_t = {  # quantised weights
                "W13q": z((E * 2 * F, d), u8), "W13s": z((E * 2 * F, d // 32), u8),
                "W13tq": z((E * 2 * F, d), u8), "W13ts": z((d, E * 2 * F // 32), u8),
                "W2q": z((E * d, F), u8), "W2s": z((E * d, F // 32), u8),
                "W2tq": z((E * d, F), u8), "W2ts": z((F, E * d // 32), u8)}
            self.qa_t = {}
            for nm, cols in (("x", d), ("a", F), ("dy", d), ("dh", 2 * F)):
                self.qa_t[nm + "q"] = z((R, cols), u8)
                self.qa_t[nm + "s"] = z((R, cols // 32), u8)
                self.qa_t[nm + "tq"] = z((R, cols), u8)
                self.qa_t[nm + "ts"] = z((cols, R // 32), u8)
            self.qw = L.MxWeights(*[L.ptr(self.qw_t[n]) for n, _ in L.MxWeights._fields_])
            order = ["xq", "xs", "xtq", "xts", "aq", "as", "atq", "ats", "dyq", "dys", "dytq", "dyts",
                     "dhq", "dhs", "dhtq", "dhts"]
            self.qa = L.MxActs(*[L.ptr(self.qa_t[n]) for n in order])
            self.q_ops = {nm: L.mx_operand(self.qa_t[nm + "q"], self.qa_t[nm + "s"], self.qa_t[nm + "tq"],
                                           self.qa_t[nm + "ts"]) for nm in ("x", "a", "dy", "dh")}
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
        if self.mx:
            self.quantize_weights()

    def quantize_weights(self, stream=None):
        """Refresh the MXFP8 weight copies (after every weight update)."""
        L.quantize_weights_mxfp8(self.cfg, self._w, self.qw, stream)

    def _result(self, t, own):
        """The caller's output buffer (any [T, d] contiguous tensor of the activation dtype on this
        layer's device), or the layer's own."""
        if t is None:
            return own
        if tuple(t.shape) != (self.T, self.d) or t.dtype != self.act or not t.is_contiguous() \
                or t.device != own.device:
            raise ValueError("output buffer shape/dtype/layout/device mismatch")
        return t

    def forward(self, x, bias=None, idx=None, gates=None, stream=None, out=None):
        """out = layer(x). With a learned router, routing comes from x W_r^T (+ bias); otherwise
        `idx` [T,k] int32 and `gates` [T,k] fp32 are copied in as the routing. `out`: where to write
        the result (default: the layer's own buffer), e.g. to let a host copy of the previous step's
        result run on while this step computes."""
        if self._w is None:
            raise RuntimeError("set_weights first")
        out = self._result(out, self.out)
        if not self.learned_router:
            self.idx.copy_(idx)
            self.gates.copy_(gates)
        self._x = x
        if self.mx:
            L.layer_fwd_mxfp8(self.cfg, self._w, self.qw, x, bias, out, self.saved, self.qa,
                              self.ws, stream)
        else:
            L.layer_fwd(self.cfg, self._w, x, bias, out, self.saved, self.ws, stream)
        return out

    def backward(self, dout, stream=None, dx=None):
        """Fills dx (the layer's own buffer, or `dx`), dW13, dW2 (and dW_r, dgates)."""
        dx = self._result(dx, self.dx)
        if self.mx:
            L.layer_bwd_mxfp8(self.cfg, self._w, self.qw, self.saved, self.qa, self._x, dout, dx,
                              self.grads, self.ws, stream)
        else:
            L.layer_bwd(self.cfg, self._w, self.saved, self._x, dout, dx, self.grads, self.ws,
                        stream)
        return dx

    def error_flags(self, stream=None) -> int:
        return L.get_error(self.ws, stream)
