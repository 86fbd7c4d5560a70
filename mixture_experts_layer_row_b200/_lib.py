"""ctypes binding of libmoe_b200.so: argument marshalling only (torch tensors -> device pointers).

Every computation runs in the library's CUDA kernels. If the shared library is missing this module
raises at import time: there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_OK = 0
ERRORS = {-1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_WORKSPACE",
          -4: "MOE_ERR_CUDA"}
DEVERR_ROUTING, DEVERR_TIMEOUT, DEVERR_NONFINITE = 1, 2, 4
DTYPE_FP32, DTYPE_BF16, DTYPE_MXFP8 = 0, 1, 2
GEMM_FWD1_SWIGLU, GEMM_FWD2, GEMM_DGRAD2_SWIGLU, GEMM_DGRAD1, GEMM_WGRAD2, GEMM_WGRAD1 = range(6)

# Every symbol include/moe_b200.h declares.
EXPORTS = [
    "moe_max_rows", "moe_workspace_size", "moe_get_error", "moe_clear_error", "moe_router_logits",
    "moe_route_topk", "moe_route_metadata", "moe_dispatch", "moe_combine", "moe_combine_bwd",
    "moe_token_reduce", "moe_grouped_gemm", "moe_router_wgrad", "moe_layer_fwd", "moe_layer_bwd",
    "moe_test_bounded_wait", "moe_version", "moe_launch_count", "moe_route_metadata_noalloc",
    "moe_quantize_mxfp8", "moe_quantize_mxfp8_rowcol", "moe_grouped_gemm_mxfp8", "moe_quantize_weights_mxfp8",
    "moe_layer_fwd_mxfp8", "moe_layer_bwd_mxfp8", "moe_dispatch_mxfp8", "moe_combine_bwd_mxfp8",
    "moe_grouped_gemm_mxfp8_quant", "moe_ep_max_rows", "moe_ep_layout", "moe_ep_zero_pad",
    "moe_ep_dispatch", "moe_ep_combine", "moe_ep_combine_bwd", "moe_ep_token_reduce",
]


class MoEError(RuntimeError):
    pass


class Config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("d", ctypes.c_int), ("F", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("dtype", ctypes.c_int), ("renorm", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [("W_r", ctypes.c_void_p), ("W13", ctypes.c_void_p), ("W2", ctypes.c_void_p)]


class Saved(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "idx", "gates", "counts", "offsets", "poff", "perm", "prow", "row_token",
                 "x_perm", "h13", "a", "y")]


class Grads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("dW_r", "dW13", "dW2", "dgates", "dy", "dh13", "dx_perm")]


class MxWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("W13q", "W13s", "W13tq", "W13ts", "W2q", "W2s", "W2tq", "W2ts")]


class MxOperand(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("q_row", "s_row", "q_col", "s_col")]


class MxActs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("xq", "xs", "xtq", "xts", "aq", "as_", "atq", "ats", "dyq", "dys", "dytq", "dyts",
                 "dhq", "dhs", "dhtq", "dhts")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmoe_b200.so not built ({LIB_PATH}); run "
                          "`python mixture_experts_layer_row_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    cfgp = ctypes.POINTER(Config)
    sig = {
        "moe_max_rows": ([cfgp], ctypes.c_int64),
        "moe_workspace_size": ([cfgp, ctypes.POINTER(ctypes.c_size_t)], i),
        "moe_get_error": ([vp, ctypes.POINTER(ctypes.c_uint32), vp], i),
        "moe_clear_error": ([vp, vp], i),
        "moe_router_logits": ([cfgp, vp, vp, vp, vp, vp, sz, vp], i),
        "moe_route_topk": ([cfgp, vp, vp, vp, vp, vp, sz, vp], i),
        "moe_route_metadata": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i),
        "moe_dispatch": ([cfgp, vp, vp, vp, vp, vp, vp], i),
        "moe_combine": ([cfgp, vp, vp, vp, vp, vp], i),
        "moe_combine_bwd": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp], i),
        "moe_token_reduce": ([cfgp, vp, vp, vp, vp, vp, vp, vp], i),
        "moe_grouped_gemm": ([cfgp, i, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i),
        "moe_router_wgrad": ([cfgp, vp, vp, vp, vp, sz, vp], i),
        "moe_layer_fwd": ([cfgp, ctypes.POINTER(Weights), vp, vp, vp, ctypes.POINTER(Saved), vp, sz,
                           vp], i),
        "moe_layer_bwd": ([cfgp, ctypes.POINTER(Weights), ctypes.POINTER(Saved), vp, vp, vp,
                           ctypes.POINTER(Grads), vp, sz, vp], i),
        "moe_test_bounded_wait": ([vp, u64, vp], i),
        "moe_version": ([], ctypes.c_char_p),
        "moe_launch_count": ([], ctypes.c_uint64),
        "moe_route_metadata_noalloc": ([cfgp, vp, vp, vp, vp, vp, vp, vp, vp], i),
        "moe_quantize_mxfp8": ([vp, ctypes.c_int64, i, i, ctypes.c_int64, vp, vp, vp], i),
        "moe_quantize_mxfp8_rowcol": ([vp, ctypes.c_int64, i, vp, vp, vp, vp, vp], i),
        "moe_grouped_gemm_mxfp8": ([cfgp, i, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp], i),
        "moe_quantize_weights_mxfp8": ([cfgp, ctypes.POINTER(Weights), ctypes.POINTER(MxWeights), vp], i),
        "moe_layer_fwd_mxfp8": ([cfgp, ctypes.POINTER(Weights), ctypes.POINTER(MxWeights), vp, vp, vp,
                                 ctypes.POINTER(Saved), ctypes.POINTER(MxActs), vp, sz, vp], i),
        "moe_layer_bwd_mxfp8": ([cfgp, ctypes.POINTER(Weights), ctypes.POINTER(MxWeights),
                                 ctypes.POINTER(Saved), ctypes.POINTER(MxActs), vp, vp, vp,
                                 ctypes.POINTER(Grads), vp, sz, vp], i),
        "moe_dispatch_mxfp8": ([cfgp, vp, vp, vp, ctypes.POINTER(MxOperand), vp], i),
        "moe_combine_bwd_mxfp8": ([cfgp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(MxOperand), vp], i),
        "moe_grouped_gemm_mxfp8_quant": ([cfgp, i, vp, vp, vp, vp, vp, vp, ctypes.POINTER(MxOperand),
                                          vp, vp, vp, sz, vp], i),
        "moe_ep_max_rows": ([cfgp, i], ctypes.c_int64),
        "moe_ep_layout": ([cfgp, i, i, vp, vp, vp, vp, vp, vp, vp, vp, vp], i),
        "moe_ep_zero_pad": ([cfgp, i, vp, vp, vp, vp], i),
        "moe_ep_dispatch": ([cfgp, i, vp, vp, vp, ctypes.POINTER(vp), vp], i),
        "moe_ep_combine": ([cfgp, i, ctypes.POINTER(vp), vp, vp, vp, vp, vp], i),
        "moe_ep_combine_bwd": ([cfgp, i, vp, ctypes.POINTER(vp), vp, vp, vp, ctypes.POINTER(vp), vp,
                                vp], i),
        "moe_ep_token_reduce": ([cfgp, i, ctypes.POINTER(vp), vp, vp, vp, vp], i),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def ptr(t) -> int | None:
    """Device pointer of a tensor (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def stream_handle(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def check(rc: int, what: str = "") -> None:
    if rc != MOE_OK:
        raise MoEError(f"{what}: {ERRORS.get(rc, rc)}")


def make_config(T, d, F, E, k, dtype=DTYPE_BF16, renorm=1) -> Config:
    return Config(T, d, F, E, k, dtype, renorm)


def max_rows(cfg: Config) -> int:
    return int(lib.moe_max_rows(ctypes.byref(cfg)))


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t(0)
    check(lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_workspace_size")
    return int(n.value)


def get_error(ws, stream=None) -> int:
    f = ctypes.c_uint32(0)
    check(lib.moe_get_error(ptr(ws), ctypes.byref(f), stream_handle(stream)), "moe_get_error")
    return int(f.value)


def clear_error(ws, stream=None) -> None:
    check(lib.moe_clear_error(ptr(ws), stream_handle(stream)), "moe_clear_error")


def _ws(ws):
    return ptr(ws), ws.numel() * ws.element_size()


def router_logits(cfg, x, W_r, bias, logits, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_router_logits(ctypes.byref(cfg), ptr(x), ptr(W_r), ptr(bias), ptr(logits), w, n,
                                stream_handle(stream)), "moe_router_logits")


def route_topk(cfg, logits, bias, idx, gates, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_route_topk(ctypes.byref(cfg), ptr(logits), ptr(bias), ptr(idx), ptr(gates), w, n,
                             stream_handle(stream)), "moe_route_topk")


def route_metadata(cfg, idx, counts, offsets, poff, perm, prow, row_token, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_route_metadata(ctypes.byref(cfg), ptr(idx), ptr(counts), ptr(offsets), ptr(poff),
                                 ptr(perm), ptr(prow), ptr(row_token), w, n, stream_handle(stream)),
          "moe_route_metadata")


def route_metadata_noalloc(cfg, idx, counts, offsets, poff, perm, prow, row_token, stream=None):
    """moe_route_metadata without a workspace (scratch in a static device array of the library)."""
    check(lib.moe_route_metadata_noalloc(ctypes.byref(cfg), ptr(idx), ptr(counts), ptr(offsets),
                                         ptr(poff), ptr(perm), ptr(prow), ptr(row_token),
                                         stream_handle(stream)), "moe_route_metadata_noalloc")


def dispatch(cfg, x, prow, counts, poff, x_perm, stream=None):
    check(lib.moe_dispatch(ctypes.byref(cfg), ptr(x), ptr(prow), ptr(counts), ptr(poff), ptr(x_perm),
                           stream_handle(stream)), "moe_dispatch")


def combine(cfg, y, gates, prow, out, stream=None):
    check(lib.moe_combine(ctypes.byref(cfg), ptr(y), ptr(gates), ptr(prow), ptr(out),
                          stream_handle(stream)), "moe_combine")


def combine_bwd(cfg, dout, y, gates, prow, idx, counts, poff, dy, dgates, dlsel=None, dlogits=None,
                stream=None):
    check(lib.moe_combine_bwd(ctypes.byref(cfg), ptr(dout), ptr(y), ptr(gates), ptr(prow), ptr(idx),
                              ptr(counts), ptr(poff), ptr(dy), ptr(dgates), ptr(dlsel), ptr(dlogits),
                              stream_handle(stream)), "moe_combine_bwd")


def token_reduce(cfg, dx_perm, prow, dx, dlsel=None, idx=None, W_r=None, stream=None):
    check(lib.moe_token_reduce(ctypes.byref(cfg), ptr(dx_perm), ptr(prow), ptr(dlsel), ptr(idx),
                               ptr(W_r), ptr(dx), stream_handle(stream)), "moe_token_reduce")


def grouped_gemm(cfg, op, A, B, C, C2, aux, counts, poff, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_grouped_gemm(ctypes.byref(cfg), int(op), ptr(A), ptr(B), ptr(C), ptr(C2), ptr(aux),
                               ptr(counts), ptr(poff), w, n, stream_handle(stream)),
          "moe_grouped_gemm")


def router_wgrad(cfg, dlogits, x, dW_r, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_router_wgrad(ctypes.byref(cfg), ptr(dlogits), ptr(x), ptr(dW_r), w, n,
                               stream_handle(stream)), "moe_router_wgrad")


def test_bounded_wait(ws, limit_ns: int, stream=None):
    check(lib.moe_test_bounded_wait(ptr(ws), int(limit_ns), stream_handle(stream)),
          "moe_test_bounded_wait")


def layer_fwd(cfg, weights: Weights, x, bias, out, saved: Saved, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_layer_fwd(ctypes.byref(cfg), ctypes.byref(weights), ptr(x), ptr(bias), ptr(out),
                            ctypes.byref(saved), w, n, stream_handle(stream)), "moe_layer_fwd")


def layer_bwd(cfg, weights: Weights, saved: Saved, x, dout, dx, grads: Grads, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_layer_bwd(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(saved), ptr(x),
                            ptr(dout), ptr(dx), ctypes.byref(grads), w, n, stream_handle(stream)),
          "moe_layer_bwd")


QUANT_ROW, QUANT_COL, QUANT_ROW_TILED, QUANT_COL_TILED, QUANT_ROW_TILED_GATEUP = range(5)


def quantize_mxfp8(src, q, s, mode, G=0, stream=None):
    """MXFP8 quantisation of a bf16 matrix src [rows, cols] into codes q and scales s."""
    rows, cols = src.shape
    check(lib.moe_quantize_mxfp8(ptr(src), rows, cols, mode, int(G), ptr(q), ptr(s),
                                 stream_handle(stream)), "moe_quantize_mxfp8")


def quantize_mxfp8_rowcol(src, q_row, s_row, q_col, s_col, stream=None):
    """Row-block and column-block tiled MXFP8 quantisations of src [rows, cols] in one pass."""
    rows, cols = src.shape
    check(lib.moe_quantize_mxfp8_rowcol(ptr(src), rows, cols, ptr(q_row), ptr(s_row), ptr(q_col),
                                        ptr(s_col), stream_handle(stream)), "moe_quantize_mxfp8_rowcol")


def grouped_gemm_mxfp8(cfg, op, Aq, As, Bq, Bs, C, C2, aux, counts, poff, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_grouped_gemm_mxfp8(ctypes.byref(cfg), int(op), ptr(Aq), ptr(As), ptr(Bq), ptr(Bs),
                                     ptr(C), ptr(C2), ptr(aux), ptr(counts), ptr(poff), w, n,
                                     stream_handle(stream)), "moe_grouped_gemm_mxfp8")


def mx_operand(q_row, s_row, q_col, s_col) -> MxOperand:
    """Both tiled MXFP8 forms of one routed-row activation (device buffers)."""
    return MxOperand(ptr(q_row), ptr(s_row), ptr(q_col), ptr(s_col))


def dispatch_mxfp8(cfg, x, row_token, poff, out: MxOperand, stream=None):
    """Row-wise dispatch of x into the routed buffer's two MXFP8 forms (no bf16 copy)."""
    check(lib.moe_dispatch_mxfp8(ctypes.byref(cfg), ptr(x), ptr(row_token), ptr(poff), ctypes.byref(out),
                                 stream_handle(stream)), "moe_dispatch_mxfp8")


def combine_bwd_mxfp8(cfg, dout, y, gates, row_token, poff, dgates, dy: MxOperand, stream=None):
    """Combine backward into dy's two MXFP8 forms (no bf16 dy) and the gate gradients."""
    check(lib.moe_combine_bwd_mxfp8(ctypes.byref(cfg), ptr(dout), ptr(y), ptr(gates), ptr(row_token),
                                    ptr(poff), ptr(dgates), ctypes.byref(dy), stream_handle(stream)),
          "moe_combine_bwd_mxfp8")


def grouped_gemm_mxfp8_quant(cfg, op, Aq, As, Bq, Bs, C, aux, out: MxOperand, counts, poff, ws,
                             stream=None):
    """The MXFP8 SwiGLU GEMMs with their activation output quantised in the epilogue."""
    w, n = _ws(ws)
    check(lib.moe_grouped_gemm_mxfp8_quant(ctypes.byref(cfg), int(op), ptr(Aq), ptr(As), ptr(Bq),
                                           ptr(Bs), ptr(C), ptr(aux), ctypes.byref(out), ptr(counts),
                                           ptr(poff), w, n, stream_handle(stream)),
          "moe_grouped_gemm_mxfp8_quant")


def quantize_weights_mxfp8(cfg, weights: Weights, qw: MxWeights, stream=None):
    check(lib.moe_quantize_weights_mxfp8(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(qw),
                                         stream_handle(stream)), "moe_quantize_weights_mxfp8")


def layer_fwd_mxfp8(cfg, weights, qw, x, bias, out, saved, qa, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_layer_fwd_mxfp8(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(qw), ptr(x),
                                  ptr(bias), ptr(out), ctypes.byref(saved), ctypes.byref(qa), w, n,
                                  stream_handle(stream)), "moe_layer_fwd_mxfp8")


def layer_bwd_mxfp8(cfg, weights, qw, saved, qa, x, dout, dx, grads, ws, stream=None):
    w, n = _ws(ws)
    check(lib.moe_layer_bwd_mxfp8(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(qw),
                                  ctypes.byref(saved), ctypes.byref(qa), ptr(x), ptr(dout), ptr(dx),
                                  ctypes.byref(grads), w, n, stream_handle(stream)),
          "moe_layer_bwd_mxfp8")


# ---- expert parallelism across the GPUs of one node -----------------------------------------------

def peer_array(ptrs) -> ctypes.Array:
    """A host array of device pointers (one per rank) for the *_peers arguments."""
    return (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(int(p)) for p in ptrs])


def ep_max_rows(cfg, world) -> int:
    return int(lib.moe_ep_max_rows(ctypes.byref(cfg), int(world)))


def ep_layout(cfg, rank, world, all_counts, idx, perm, offsets, src_base, counts_loc, poff_loc, dst_row,
              stream=None):
    check(lib.moe_ep_layout(ctypes.byref(cfg), int(rank), int(world), ptr(all_counts), ptr(idx), ptr(perm),
                            ptr(offsets), ptr(src_base), ptr(counts_loc), ptr(poff_loc), ptr(dst_row),
                            stream_handle(stream)), "moe_ep_layout")


def ep_zero_pad(cfg, world, buf, counts_loc, poff_loc, stream=None):
    check(lib.moe_ep_zero_pad(ctypes.byref(cfg), int(world), ptr(buf), ptr(counts_loc), ptr(poff_loc),
                              stream_handle(stream)), "moe_ep_zero_pad")


def ep_dispatch(cfg, world, x, idx, dst_row, x_perm_peers, stream=None):
    check(lib.moe_ep_dispatch(ctypes.byref(cfg), int(world), ptr(x), ptr(idx), ptr(dst_row),
                              x_perm_peers, stream_handle(stream)), "moe_ep_dispatch")


def ep_combine(cfg, world, y_peers, gates, idx, dst_row, out, stream=None):
    check(lib.moe_ep_combine(ctypes.byref(cfg), int(world), y_peers, ptr(gates), ptr(idx), ptr(dst_row),
                             ptr(out), stream_handle(stream)), "moe_ep_combine")


def ep_combine_bwd(cfg, world, dout, y_peers, gates, idx, dst_row, dy_peers, dgates, stream=None):
    check(lib.moe_ep_combine_bwd(ctypes.byref(cfg), int(world), ptr(dout), y_peers, ptr(gates), ptr(idx),
                                 ptr(dst_row), dy_peers, ptr(dgates), stream_handle(stream)),
          "moe_ep_combine_bwd")


def ep_token_reduce(cfg, world, dx_perm_peers, idx, dst_row, dx, stream=None):
    check(lib.moe_ep_token_reduce(ctypes.byref(cfg), int(world), dx_perm_peers, ptr(idx), ptr(dst_row),
                                  ptr(dx), stream_handle(stream)), "moe_ep_token_reduce")


def version() -> str:
    return lib.moe_version().decode()


def launch_count() -> int:
    """Kernels this library has enqueued in this process so far."""
    return int(lib.moe_launch_count())
