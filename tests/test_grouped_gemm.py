"""GPU parity of the device-scheduled grouped GEMM (tcgen05) for every op, on ragged expert groups
(empty, 1, 31, 32, 33, 127..129 rows, one expert holding every row, partial N and M tiles), against
the oracle's per-expert GEMM steps in fp64."""
import numpy as np
import pytest
import torch

from oracle import moe as O
from _util import TOL_BF16, assert_close_rel, dev, idx_from_counts, np64

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: (T, d, F, E, k, counts or None for uniform routing)
    "ragged": (512, 128, 256, 8, 2, [0, 1, 31, 33, 129, 200, 300, 330]),
    # d, F >= 256: fwd2 and dgrad1 run on CTA pairs (256-row tiles) over uneven groups, so tiles
    # with an empty second half, single-row and empty experts all occur
    "ragged_pairs": (512, 256, 256, 8, 2, [0, 1, 31, 33, 129, 200, 300, 330]),
    "edges": (400, 192, 384, 6, 2, [32, 127, 128, 0, 400, 113]),
    # fwd2 / dgrad1 on CTA pairs with 256-column n-blocks: d = 768 gives three of them, d = 320 a
    # second one with 64 valid columns (an expert holding every token, one holding none)
    "pairs_n768": (512, 768, 256, 8, 2, [0, 1, 31, 33, 129, 200, 300, 330]),
    "pairs_n320": (384, 320, 128, 4, 2, [100, 0, 284, 384]),
    "one_expert": (300, 128, 128, 4, 1, [300, 0, 0, 0]),
    "wide": (2048, 2048, 1024, 16, 4, None),
}


def _lib():
    from mixture_experts_layer_row_b200 import _lib as L
    return L


class Problem:
    def __init__(self, shape, dtype, seed=0):
        L = _lib()
        self.L = L
        T, d, F, E, k, counts = SHAPES[shape]
        self.T, self.d, self.F, self.E, self.k = T, d, F, E, k
        rng = np.random.default_rng(seed)
        if counts is None:
            idx = np.argsort(rng.random((T, E)), axis=1)[:, :k]
        else:
            idx = idx_from_counts(counts, T, k, rng)
        self.meta = O.route_metadata(idx.astype(np.int64), E)
        self.dtype = dtype
        code = L.DTYPE_FP32 if dtype == torch.float32 else L.DTYPE_BF16
        self.cfg = L.make_config(T, d, F, E, k, code)
        self.R = L.max_rows(self.cfg)
        self.ws = torch.zeros(L.workspace_size(self.cfg), dtype=torch.uint8, device=dev())
        self.g = torch.Generator().manual_seed(seed + 1)
        t32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())
        self.counts, self.poff = t32(self.meta["counts"]), t32(self.meta["poff"])
        self.valid = self.meta["row_token"] >= 0  # [used rows]

    def rows(self, cols, scale=1.0):
        """A routed-row buffer [R, cols] with random valid rows and zero pad rows (as the kernels
        that write these buffers leave them)."""
        used = int(self.meta["poff"][-1])
        t = torch.zeros((self.R, cols), dtype=torch.float32)
        v = torch.randn((used, cols), generator=self.g) * scale
        v[torch.from_numpy(~self.valid)] = 0
        t[:used] = v
        return t.to(self.dtype)

    def weights(self, *shape):
        return (torch.randn(shape, generator=self.g) * 0.05).to(self.dtype)

    def groups(self):
        for e in range(self.E):
            r0, n = int(self.meta["poff"][e]), int(self.meta["counts"][e])
            yield e, r0, n, int(self.meta["poff"][e + 1])

    def run(self, op, A, B, C, C2=None, aux=None):
        d = lambda t: t.to(dev()) if t is not None else None
        Cd, C2d = d(C), d(C2)
        self.L.grouped_gemm(self.cfg, op, d(A), d(B), Cd, C2d, d(aux), self.counts, self.poff, self.ws)
        torch.cuda.synchronize()
        assert self.L.get_error(self.ws) == 0
        return Cd, C2d


DTYPES = [torch.bfloat16, torch.float32]
TOL = TOL_BF16 / 2  # per-GEMM bar, tighter than the layer's


def _sentinel(rows, cols, dtype):
    return torch.full((rows, cols), 5.0, dtype=dtype)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", list(SHAPES))
def test_fwd1_swiglu(shape, dtype):
    P = Problem(shape, dtype)
    X, W13 = P.rows(P.d), P.weights(P.E, 2 * P.F, P.d)
    h13, a = P.run(P.L.GEMM_FWD1_SWIGLU, X, W13, _sentinel(P.R, 2 * P.F, dtype),
                   _sentinel(P.R, P.F, dtype))
    Xn, Wn, H, A = np64(X), np64(W13), np64(h13), np64(a)
    for e, r0, n, r1 in P.groups():
        if n:
            rh, ra = O.gemm_fwd1_swiglu(Xn[r0:r0 + n], Wn[e])
            assert_close_rel(H[r0:r0 + n], rh, TOL, f"h13 e{e}")
            assert_close_rel(A[r0:r0 + n], ra, TOL, f"a e{e}")
        assert np.all(H[r0 + n:r1] == 0) and np.all(A[r0 + n:r1] == 0), "pad rows must be zero"
    used = int(P.meta["poff"][-1])
    assert np.all(H[used:] == 5.0) and np.all(A[used:] == 5.0), "rows past the groups untouched"


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", list(SHAPES))
def test_fwd2(shape, dtype):
    P = Problem(shape, dtype)
    A, W2 = P.rows(P.F), P.weights(P.E, P.d, P.F)
    y, _ = P.run(P.L.GEMM_FWD2, A, W2, _sentinel(P.R, P.d, dtype))
    An, Wn, Y = np64(A), np64(W2), np64(y)
    for e, r0, n, r1 in P.groups():
        if n:
            assert_close_rel(Y[r0:r0 + n], O.gemm_fwd2(An[r0:r0 + n], Wn[e]), TOL, f"y e{e}")
        assert np.all(Y[r0 + n:r1] == 0)
    assert np.all(Y[int(P.meta["poff"][-1]):] == 5.0)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", list(SHAPES))
def test_dgrad2_swiglu(shape, dtype):
    P = Problem(shape, dtype)
    dY, W2, H13 = P.rows(P.d), P.weights(P.E, P.d, P.F), P.rows(2 * P.F, 2.0)
    dh, _ = P.run(P.L.GEMM_DGRAD2_SWIGLU, dY, W2, _sentinel(P.R, 2 * P.F, dtype), aux=H13)
    dYn, Wn, Hn, D = np64(dY), np64(W2), np64(H13), np64(dh)
    for e, r0, n, r1 in P.groups():
        if n:
            ref = O.gemm_dgrad2_swiglu(dYn[r0:r0 + n], Wn[e], Hn[r0:r0 + n])
            assert_close_rel(D[r0:r0 + n], ref, TOL, f"dh13 e{e}")
        assert np.all(D[r0 + n:r1] == 0)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", list(SHAPES))
def test_dgrad1(shape, dtype):
    P = Problem(shape, dtype)
    dH, W13 = P.rows(2 * P.F), P.weights(P.E, 2 * P.F, P.d)
    dx, _ = P.run(P.L.GEMM_DGRAD1, dH, W13, _sentinel(P.R, P.d, dtype))
    dHn, Wn, DX = np64(dH), np64(W13), np64(dx)
    for e, r0, n, r1 in P.groups():
        if n:
            assert_close_rel(DX[r0:r0 + n], O.gemm_dgrad1(dHn[r0:r0 + n], Wn[e]), TOL, f"dx e{e}")
        assert np.all(DX[r0 + n:r1] == 0)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("which", ["w2", "w13"])
def test_wgrad(shape, dtype, which):
    P = Problem(shape, dtype)
    if which == "w2":
        G, X, M, N, op = P.rows(P.d), P.rows(P.F), P.d, P.F, P.L.GEMM_WGRAD2
    else:
        G, X, M, N, op = P.rows(2 * P.F), P.rows(P.d), 2 * P.F, P.d, P.L.GEMM_WGRAD1
    dW = torch.full((P.E, M, N), 5.0, dtype=dtype)
    dW, _ = P.run(op, G, X, dW)
    Gn, Xn, DW = np64(G), np64(X), np64(dW)
    for e, r0, n, r1 in P.groups():
        if n == 0:
            assert np.all(DW[e] == 0), "an expert with no rows has a zero gradient"
        else:
            assert_close_rel(DW[e], O.gemm_wgrad(Gn[r0:r0 + n], Xn[r0:r0 + n]), TOL, f"dW e{e}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", ["ragged", "ragged_pairs", "wide"])
def test_fwd1_without_h13_and_dgrad2_in_place(shape, dtype):
    """The two GEMMs activation recompute relies on: GEMM1 with no h13 output stores the same a as
    with it, and the SwiGLU-backward GEMM overwriting its h13 input in place gives the same dh13 as
    with separate buffers."""
    P = Problem(shape, dtype)
    X, W13 = P.rows(P.d), P.weights(P.E, 2 * P.F, P.d)
    h13, a = P.run(P.L.GEMM_FWD1_SWIGLU, X, W13, _sentinel(P.R, 2 * P.F, dtype), _sentinel(P.R, P.F, dtype))
    _, a_only = P.run(P.L.GEMM_FWD1_SWIGLU, X, W13, None, _sentinel(P.R, P.F, dtype))
    assert torch.equal(a_only, a)
    dY, W2 = P.rows(P.d), P.weights(P.E, P.d, P.F)
    dh, _ = P.run(P.L.GEMM_DGRAD2_SWIGLU, dY, W2, _sentinel(P.R, 2 * P.F, dtype), aux=h13)
    buf = h13.clone()
    P.L.grouped_gemm(P.cfg, P.L.GEMM_DGRAD2_SWIGLU, dY.to(dev()), W2.to(dev()), buf, None, buf,
                     P.counts, P.poff, P.ws)
    torch.cuda.synchronize()
    assert P.L.get_error(P.ws) == 0
    assert torch.equal(buf, dh)


@pytest.mark.parametrize("dtype", DTYPES)
def test_gemm_is_deterministic(dtype):
    P = Problem("wide", dtype)
    G, X = P.rows(P.d), P.rows(P.F)
    a, _ = P.run(P.L.GEMM_WGRAD2, G, X, torch.zeros((P.E, P.d, P.F), dtype=dtype))
    b, _ = P.run(P.L.GEMM_WGRAD2, G, X, torch.zeros((P.E, P.d, P.F), dtype=dtype))
    assert torch.equal(a, b)
