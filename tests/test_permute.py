"""GPU parity of the row-movement kernels: dispatch (bit-exact, it is a copy), combine, combine
backward (dy, gate and score gradients) and the token reduce, against the oracle."""
import numpy as np
import pytest
import torch

from oracle import moe as O
from _util import assert_close_rel, dev, idx_from_counts, np64

pytestmark = pytest.mark.gpu


def _lib():
    from mixture_experts_layer_row_b200 import _lib as L
    return L


def _setup(T, d, E, k, dtype, seed, counts=None):
    L = _lib()
    rng = np.random.default_rng(seed)
    if counts is None:
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
    else:
        idx = idx_from_counts(counts, T, k, rng)
    code = L.DTYPE_FP32 if dtype == torch.float32 else L.DTYPE_BF16
    cfg = L.make_config(T, d, 128, E, k, code)
    R = L.max_rows(cfg)
    meta = O.route_metadata(idx.astype(np.int64), E)
    t32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((T, d), generator=g).to(dtype)
    gates = torch.softmax(torch.randn((T, k), generator=g, dtype=torch.float64), 1).float()
    return L, cfg, R, idx, meta, t32, x, gates


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k,counts", [(300, 128, 8, 2, None), (33, 256, 5, 3, None),
                                            (700, 64, 16, 2, [0, 1, 31, 32, 33, 127, 128, 129, 300,
                                                              300, 100, 50, 50, 50, 36, 33]),
                                            (2048, 2048, 128, 4, None)])
def test_dispatch_bitexact(dtype, T, d, E, k, counts):
    L, cfg, R, idx, meta, t32, x, _ = _setup(T, d, E, k, dtype, 1, counts)
    xp = torch.full((R, d), 7.0, dtype=dtype, device=dev())  # garbage where nothing is written
    L.dispatch(cfg, x.to(dev()), t32(meta["prow"]), t32(meta["counts"]), t32(meta["poff"]), xp)
    torch.cuda.synchronize()
    ref = O.dispatch(x.double().numpy(), meta, k)
    used = ref.shape[0]
    assert np.array_equal(np64(xp[:used]), ref)  # exact copy, pad rows exactly zero
    assert torch.all(xp[used:] == 7.0)           # rows past the last group untouched


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k", [(300, 128, 8, 2), (1000, 2048, 128, 4), (17, 64, 3, 3)])
def test_combine(dtype, T, d, E, k):
    L, cfg, R, idx, meta, t32, _, gates = _setup(T, d, E, k, dtype, 2)
    g = torch.Generator().manual_seed(3)
    y = torch.randn((R, d), generator=g).to(dtype)
    out = torch.zeros((T, d), dtype=dtype, device=dev())
    L.combine(cfg, y.to(dev()), gates.to(dev()), t32(meta["prow"]), out)
    torch.cuda.synchronize()
    ref = O.combine(y.double().numpy(), gates.double().numpy(), meta)
    assert_close_rel(np64(out), ref, 1e-2 if dtype == torch.bfloat16 else 1e-6, "combine")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("T,d,E,k", [(300, 128, 8, 2), (1000, 2048, 128, 4),
                                     # k = 8, a ragged last block of the bulk-staged kernel
                                     (37, 64, 5, 5), (45, 128, 8, 8),
                                     # one token per block (rows of 16-32 KB), and rows too wide to
                                     # stage (the register-staged kernel)
                                     (40, 8192, 8, 8), (24, 16384, 8, 8)])
def test_combine_bwd(dtype, T, d, E, k):
    L, cfg, R, idx, meta, t32, _, gates = _setup(T, d, E, k, dtype, 4)
    g = torch.Generator().manual_seed(5)
    y = torch.randn((R, d), generator=g).to(dtype)
    dout = torch.randn((T, d), generator=g).to(dtype)
    dy = torch.full((R, d), 3.0, dtype=dtype, device=dev())
    dg = torch.zeros((T, k), dtype=torch.float32, device=dev())
    dls = torch.zeros((T, k), dtype=torch.float32, device=dev())
    dlog = torch.full((T, E), 9.0, dtype=dtype, device=dev())
    L.combine_bwd(cfg, dout.to(dev()), y.to(dev()), gates.to(dev()), t32(meta["prow"]), t32(idx),
                  t32(meta["counts"]), t32(meta["poff"]), dy, dg, dls, dlog)
    torch.cuda.synchronize()
    G, D, Y = gates.double().numpy(), dout.double().numpy(), y.double().numpy()
    used = int(meta["poff"][E])
    ref_dy, ref_dg = O.combine_bwd(D, Y[:used], G, meta)
    assert_close_rel(np64(dy[:used]), ref_dy, 1e-2, "dy")
    assert np.all(np64(dy[:used])[meta["row_token"] < 0] == 0), "pad rows of dy must be zero"
    assert_close_rel(dg.cpu().numpy(), ref_dg, 1e-5 if dtype == torch.float32 else 1e-4, "dgates")
    dl_ref = O.router_bwd(ref_dg, G, idx.astype(np.int64), E)
    assert_close_rel(dls.cpu().numpy(), np.take_along_axis(dl_ref, idx.astype(np.int64), 1),
                     1e-4, "dlsel")
    assert_close_rel(np64(dlog), dl_ref, 1e-2, "dense score gradient")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("router", [False, True])
def test_token_reduce(dtype, router):
    T, d, E, k = 500, 256, 16, 4
    L, cfg, R, idx, meta, t32, _, gates = _setup(T, d, E, k, dtype, 6)
    g = torch.Generator().manual_seed(7)
    dxp = torch.randn((R, d), generator=g).to(dtype)
    Wr = (torch.randn((E, d), generator=g) * 0.02).to(dtype)
    dls = torch.randn((T, k), generator=g) * 0.1
    dx = torch.zeros((T, d), dtype=dtype, device=dev())
    L.token_reduce(cfg, dxp.to(dev()), t32(meta["prow"]), dx,
                   dls.to(dev()) if router else None, t32(idx) if router else None,
                   Wr.to(dev()) if router else None)
    torch.cuda.synchronize()
    dl = None
    if router:  # the kernel takes the chosen experts' score gradients; the oracle the dense matrix
        dl = np.zeros((T, E))
        np.put_along_axis(dl, idx.astype(np.int64), dls.double().numpy(), 1)
    ref = O.token_reduce(dxp.double().numpy(), meta, T, k, dl, Wr.double().numpy() if router else None)
    assert_close_rel(np64(dx), ref, 1e-2 if dtype == torch.bfloat16 else 1e-6, "token_reduce")
