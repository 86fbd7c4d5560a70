"""The C-ABI library loads, exports every symbol include/moe_b200.h declares, has the struct layout
the header defines, and rejects bad arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    from mixture_experts_layer_row_b200 import _lib
    return _lib


def header_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src, flags=re.M)))


def test_exports_match_header(L):
    declared = header_functions()
    assert len(declared) >= 17
    assert sorted(L.EXPORTS) == declared
    for name in declared:
        assert hasattr(L.lib, name), name
    # exported from the shared object itself, visible to any C caller
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True, text=True)
    if out.returncode == 0:
        syms = set(re.findall(r"\bT (moe_\w+)", out.stdout))
        assert set(declared) <= syms


def test_struct_layout_matches_c(tmp_path, L):
    prog = tmp_path / "layout.c"
    prog.write_text(r'''
#include <stdio.h>
#include <stddef.h>
#include "moe_b200.h"
int main(void) {
  printf("%zu %zu %zu %zu\n", sizeof(moe_config_t), sizeof(moe_weights_t), sizeof(moe_saved_t),
         sizeof(moe_grads_t));
  printf("%zu %zu %zu\n", offsetof(moe_config_t, renorm), offsetof(moe_saved_t, y),
         offsetof(moe_grads_t, dx_perm));
  return 0;
}
''')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    a, b = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")[:2]
    sizes = [int(v) for v in a.split()]
    offs = [int(v) for v in b.split()]
    assert sizes == [ctypes.sizeof(L.Config), ctypes.sizeof(L.Weights), ctypes.sizeof(L.Saved),
                     ctypes.sizeof(L.Grads)]
    assert offs == [L.Config.renorm.offset, L.Saved.y.offset, L.Grads.dx_perm.offset]


def test_version_and_sizes(L):
    assert "sm_100a" in L.version()
    cfg = L.make_config(8192, 2048, 1024, 128, 4)
    assert L.max_rows(cfg) == 8192 * 4 + 31 * 128
    assert L.workspace_size(cfg) > 256


@pytest.mark.parametrize("T,d,F,E,k,dtype,renorm,code", [
    (0, 64, 128, 8, 2, 1, 1, -1),      # no tokens
    (16, 64, 128, 8, 9, 1, 1, -1),     # k > E
    (16, 64, 128, 8, 2, 7, 1, -1),     # bad dtype
    (16, 64, 128, 8, 2, 1, 2, -1),     # bad renorm flag
    (16, 96, 128, 8, 2, 1, 1, -2),     # d not a multiple of 64
    (16, 64, 192, 8, 2, 1, 1, -2),     # F not a multiple of 128
    (16, 64, 128, 300, 2, 1, 1, -2),   # E > 256
    (16, 64, 128, 16, 9, 1, 1, -2),    # k > 8
])
def test_bad_configs_rejected(L, T, d, F, E, k, dtype, renorm, code):
    cfg = L.make_config(T, d, F, E, k, dtype, renorm)
    n = ctypes.c_size_t(0)
    assert L.lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == code
    assert L.max_rows(cfg) == 0


def test_host_validation_before_any_launch(L):
    """Each call below must be refused on the host: no CUDA call happens (this box has no GPU)."""
    cfg = L.make_config(64, 64, 128, 8, 2)
    c = ctypes.byref(cfg)
    fake = 1 << 20  # a 16-byte aligned non-null "device" address, never dereferenced
    assert L.lib.moe_dispatch(c, None, fake, fake, fake, fake, None) == -1
    assert L.lib.moe_dispatch(c, fake + 8, fake, fake, fake, fake, None) == -1  # misaligned
    assert L.lib.moe_combine(c, fake, None, fake, fake, None) == -1
    assert L.lib.moe_route_metadata(c, fake, fake, fake, fake, fake, fake, fake, None, 0, None) == -3
    assert L.lib.moe_route_topk(c, fake, None, fake, fake, fake, 8, None) == -3  # workspace too small
    assert L.lib.moe_grouped_gemm(c, 99, fake, fake, fake, None, None, fake, fake, fake,
                                  10 ** 9, None) == -1  # unknown op
    assert L.lib.moe_grouped_gemm(c, 0, fake, fake, fake, None, None, fake, fake, fake,
                                  10 ** 9, None) == -1  # SwiGLU forward needs its second output
    assert L.lib.moe_grouped_gemm(c, 1, fake, fake, None, None, None, fake, fake, fake,
                                  10 ** 9, None) == -1  # only the SwiGLU forward may omit C
    rc = L.lib.moe_quantize_mxfp8_rowcol
    assert rc(fake, 96, 128, fake, fake, fake, fake, None) == -1    # rows % 128
    assert rc(fake, 128, 96, fake, fake, fake, fake, None) == -1    # cols % 128
    assert rc(fake, 128, 128, fake, fake, fake + 8, fake, None) == -1  # column codes 16-byte aligned
    assert rc(fake, 128, 128, fake + 4, fake, fake, fake, None) == -1  # row codes 8-byte aligned
    assert rc(fake, 128, 128, None, fake, fake, fake, None) == -1
    assert L.lib.moe_get_error(None, None, None) == -1
    mx = L.make_config(64, 64, 128, 8, 2, L.DTYPE_MXFP8)
    # the router GEMM and the bf16/fp32 grouped GEMM entry points do not take MXFP8 configs
    assert L.lib.moe_router_logits(ctypes.byref(mx), fake, fake, None, fake, fake, 10 ** 9, None) == -2
    assert L.lib.moe_grouped_gemm(ctypes.byref(mx), 1, fake, fake, fake, None, None, fake, fake, fake,
                                  10 ** 9, None) == -2
    # and the MXFP8 grouped GEMM needs d % 128 == 0
    assert L.lib.moe_grouped_gemm_mxfp8(ctypes.byref(mx), 1, fake, fake, fake, fake, fake, None, None,
                                        fake, fake, fake, 10 ** 9, None) == -2
    assert L.lib.moe_layer_fwd(c, None, fake, None, fake, None, fake, 10 ** 9, None) == -1


def test_layer_output_buffers_checked_on_host():
    """MoELayer.forward(out=) / backward(dx=) reject a buffer of the wrong shape, dtype or layout
    before anything is enqueued (host buffers: no GPU needed)."""
    import torch
    from mixture_experts_layer_row_b200 import MoELayer
    T, d, F, E, k = 64, 128, 128, 8, 2
    layer = MoELayer(T, d, F, E, k, dtype="bf16", device="cpu", learned_router=False)
    layer.set_weights(torch.zeros((E, 2 * F, d), dtype=torch.bfloat16),
                      torch.zeros((E, d, F), dtype=torch.bfloat16))
    x = torch.zeros((T, d), dtype=torch.bfloat16)
    kw = {"idx": torch.zeros((T, k), dtype=torch.int32), "gates": torch.zeros((T, k))}
    bad = [torch.zeros((T, d // 2), dtype=torch.bfloat16), torch.zeros((T, d), dtype=torch.float32),
           torch.zeros((d, T), dtype=torch.bfloat16).t()]
    for b in bad:
        with pytest.raises(ValueError):
            layer.forward(x, out=b, **kw)
        with pytest.raises(ValueError):
            layer.backward(x, dx=b)
