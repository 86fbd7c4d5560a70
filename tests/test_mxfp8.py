"""MXFP8 on the GPU: quantisation must be bit-exact with the oracle's OCP-MX quantiser (codes and
scales, in the plain and in the tiled scale layouts), and every block-scaled grouped GEMM op must
match the oracle's GEMM step applied to the oracle's own MXFP8 fake-quantised operands (exact products
of E4M3 codes and power-of-two scales, so only fp32 accumulation order and the bf16 output rounding
differ)."""
import numpy as np
import pytest
import torch

from oracle import moe as O
from oracle import mxfp8 as MX
from _util import assert_close_rel, dev, idx_from_counts, np64

pytestmark = pytest.mark.gpu


def _lib():
    from mixture_experts_layer_row_b200 import _lib as L
    return L


def _bf16_matrix(rows, cols, seed):
    """Values spanning many binades per block, with all-zero blocks, tiny and huge magnitudes."""
    g = torch.Generator().manual_seed(seed)
    v = torch.randn((rows, cols), generator=g) * torch.exp2(torch.randint(-20, 20, (rows, 1), generator=g).float())
    v[::7, :32] = 0.0                       # all-zero blocks
    v[1::11, 32:64] *= 2.0 ** -110          # near the bottom of the scale range
    v[2::13, :] = torch.round(v[2::13, :])  # exact small integers
    return v.to(torch.bfloat16)


@pytest.mark.parametrize("rows,cols", [(64, 32), (96, 256), (1024, 4096), (7, 96)])
def test_quantize_row_bitexact(rows, cols):
    L = _lib()
    x = _bf16_matrix(rows, cols, rows + cols)
    q = torch.zeros((rows, cols), dtype=torch.uint8, device=dev())
    s = torch.zeros((rows, cols // 32), dtype=torch.uint8, device=dev())
    L.quantize_mxfp8(x.to(dev()), q, s, L.QUANT_ROW)
    torch.cuda.synchronize()
    rq, rs = MX.quantize_rows(x.double().numpy())
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(q.cpu().numpy(), rq)


@pytest.mark.parametrize("rows,cols", [(32, 8), (256, 128), (2048, 1536)])
def test_quantize_col_bitexact(rows, cols):
    L = _lib()
    x = _bf16_matrix(rows, cols, 3 * rows + cols)
    x[:32, 4:8] = -0.0  # an all-zero column block of negative zeros: zero codes
    q = torch.zeros((rows, cols), dtype=torch.uint8, device=dev())
    s = torch.zeros((cols, rows // 32), dtype=torch.uint8, device=dev())
    L.quantize_mxfp8(x.to(dev()), q, s, L.QUANT_COL)
    torch.cuda.synchronize()
    rq, rs = MX.quantize_cols(x.double().numpy())
    assert np.array_equal(s.cpu().numpy(), rs.T)  # scales are stored [cols, rows/32]
    assert np.array_equal(q.cpu().numpy(), rq)


def tiled(plain, gateup_G=0):
    """Re-index plain scales [MN, KB] into the tiled layout the GEMM streams: chunk (i/128, b/4) of 512
    bytes, byte (i%32)*16 + ((i%128)/32)*4 + b%4 (rows of [gate; up] stacks remapped for GATEUP)."""
    MN, KB = plain.shape
    out = np.zeros(MN * KB, dtype=np.uint8)
    i = np.arange(MN)[:, None]
    b = np.arange(KB)[None, :]
    if gateup_G:
        G = gateup_G
        e, rr = i // (2 * G), i % (2 * G)
        f, up = rr % G, rr // G
        i = e * 2 * G + (f // 64) * 128 + up * 64 + f % 64
    off = ((i // 128) * (KB // 4) + b // 4) * 512 + (i % 32) * 16 + ((i % 128) // 32) * 4 + b % 4
    out[off.reshape(-1)] = plain.reshape(-1)
    return out


@pytest.mark.parametrize("rows,cols,mode", [(128, 128, "row"), (256, 384, "col"), (1024, 2048, "row"),
                                            (2048, 1536, "col"), (1536, 256, "gateup")])
def test_quantize_tiled_bitexact(rows, cols, mode):
    L = _lib()
    x = _bf16_matrix(rows, cols, 5 * rows + cols)
    q = torch.zeros((rows, cols), dtype=torch.uint8, device=dev())
    s = torch.zeros(rows * cols // 32, dtype=torch.uint8, device=dev())
    m = {"row": L.QUANT_ROW_TILED, "col": L.QUANT_COL_TILED, "gateup": L.QUANT_ROW_TILED_GATEUP}[mode]
    G = 384 if mode == "gateup" else 0   # two [384 gate; 384 up] stacks
    L.quantize_mxfp8(x.to(dev()), q, s, m, G)
    torch.cuda.synchronize()
    if mode == "col":
        rq, rs = MX.quantize_cols(x.double().numpy())
        ref_s = tiled(rs.T)
    else:
        rq, rs = MX.quantize_rows(x.double().numpy())
        ref_s = tiled(rs, G)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy(), ref_s)


@pytest.mark.parametrize("rows,cols", [(128, 128), (384, 256), (1024, 2048), (2048, 1536)])
def test_quantize_rowcol_bitexact(rows, cols):
    """One pass writing both tiled orientations equals the oracle's row and column quantisers (and
    so the two single-orientation launches)."""
    L = _lib()
    x = _bf16_matrix(rows, cols, 7 * rows + cols)
    x[5::17, :] = -0.0                                   # negative zeros: all-zero row blocks
    x[32:64, :4] = -0.0                                  # and all-zero column blocks
    z = lambda *sh: torch.full(sh, 0xAB, dtype=torch.uint8, device=dev())
    qr, sr, qc, sc = z(rows, cols), z(rows * cols // 32), z(rows, cols), z(rows * cols // 32)
    L.quantize_mxfp8_rowcol(x.to(dev()), qr, sr, qc, sc)
    torch.cuda.synchronize()
    xn = x.double().numpy()
    rq, rs = MX.quantize_rows(xn)
    cq, cs = MX.quantize_cols(xn)
    assert np.array_equal(qr.cpu().numpy(), rq)
    assert np.array_equal(sr.cpu().numpy(), tiled(rs))
    assert np.array_equal(qc.cpu().numpy(), cq)
    assert np.array_equal(sc.cpu().numpy(), tiled(cs.T))
    # and the single-orientation kernels agree byte for byte (negative zeros included)
    q1, s1 = z(rows, cols), z(rows * cols // 32)
    L.quantize_mxfp8(x.to(dev()), q1, s1, L.QUANT_COL_TILED)
    q2, s2 = z(rows, cols), z(rows * cols // 32)
    L.quantize_mxfp8(x.to(dev()), q2, s2, L.QUANT_ROW_TILED)
    torch.cuda.synchronize()
    assert torch.equal(q1, qc) and torch.equal(s1, sc) and torch.equal(q2, qr) and torch.equal(s2, sr)


SHAPES = {
    "ragged": (512, 128, 256, 8, 2, [0, 1, 31, 33, 129, 200, 300, 330]),
    # d and F multiples of 256: the plain-store GEMMs take 256-column tiles with ragged groups
    "ragged_wide": (512, 256, 256, 8, 2, [0, 1, 31, 33, 129, 200, 300, 330]),
    "one_expert": (300, 128, 128, 4, 1, [300, 0, 0, 0]),
    "wide": (2048, 2048, 1024, 16, 4, None),
}


class MxProblem:
    def __init__(self, shape, seed=0):
        L = _lib()
        self.L = L
        T, d, F, E, k, counts = SHAPES[shape]
        self.T, self.d, self.F, self.E, self.k = T, d, F, E, k
        rng = np.random.default_rng(seed)
        idx = np.argsort(rng.random((T, E)), 1)[:, :k] if counts is None else idx_from_counts(counts, T, k, rng)
        self.meta = O.route_metadata(idx.astype(np.int64), E, 128)  # MXFP8 groups: 128 rows
        self.cfg = L.make_config(T, d, F, E, k, L.DTYPE_MXFP8)
        self.R32 = L.max_rows(self.cfg)
        self.ws = torch.zeros(L.workspace_size(self.cfg), dtype=torch.uint8, device=dev())
        self.g = torch.Generator().manual_seed(seed + 1)
        t32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())
        self.counts, self.poff = t32(self.meta["counts"]), t32(self.meta["poff"])
        self.valid = self.meta["row_token"] >= 0

    def rows(self, cols, scale=1.0):
        used = int(self.meta["poff"][-1])
        t = torch.zeros((self.R32, cols), dtype=torch.float32)
        v = torch.randn((used, cols), generator=self.g) * scale
        v[torch.from_numpy(~self.valid)] = 0
        t[:used] = v
        return t.to(torch.bfloat16)

    def weights(self, *shape):
        return (torch.randn(shape, generator=self.g) * 0.05).to(torch.bfloat16)

    def quant(self, x2d, mode, G=0):
        """mode 0: ROW (tiled scales), 1: COL (tiled), 2: ROW gate/up tiled (W13, G = F)."""
        rows, cols = x2d.shape
        q = torch.zeros((rows, cols), dtype=torch.uint8, device=dev())
        s = torch.zeros(rows * cols // 32, dtype=torch.uint8, device=dev())
        m = [self.L.QUANT_ROW_TILED, self.L.QUANT_COL_TILED, self.L.QUANT_ROW_TILED_GATEUP][mode]
        self.L.quantize_mxfp8(x2d.to(dev()).contiguous(), q, s, m, G)
        return q, s

    def groups(self):
        for e in range(self.E):
            yield e, int(self.meta["poff"][e]), int(self.meta["counts"][e]), int(self.meta["poff"][e + 1])

    def run(self, op, A, B, C, C2=None, aux=None):
        d = lambda t: t.to(dev()) if t is not None else None
        Cd, C2d = d(C), d(C2)
        self.L.grouped_gemm_mxfp8(self.cfg, op, A[0], A[1], B[0], B[1], Cd, C2d, d(aux), self.counts,
                                  self.poff, self.ws)
        torch.cuda.synchronize()
        assert self.L.get_error(self.ws) == 0
        return Cd, C2d


TOL = 1e-2
ROWQ, COLQ = O._mx_row, O._mx_col


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_fwd1(shape):
    P = MxProblem(shape)
    X, W13 = P.rows(P.d), P.weights(P.E, 2 * P.F, P.d)
    h13, a = P.run(P.L.GEMM_FWD1_SWIGLU, P.quant(X, 0), P.quant(W13.reshape(-1, P.d), 0),
                   torch.zeros((P.R32, 2 * P.F), dtype=torch.bfloat16),
                   torch.zeros((P.R32, P.F), dtype=torch.bfloat16))
    Xn, Wn, H, A = np64(X), np64(W13), np64(h13), np64(a)
    for e, r0, n, r1 in P.groups():
        if n:
            rh, ra = O.gemm_fwd1_swiglu(Xn[r0:r0 + n], Wn[e], ROWQ)
            assert_close_rel(H[r0:r0 + n], rh, TOL, f"h13 e{e}")
            assert_close_rel(A[r0:r0 + n], ra, TOL, f"a e{e}")
        assert np.all(H[r0 + n:r1] == 0) and np.all(A[r0 + n:r1] == 0)


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_fwd2(shape):
    P = MxProblem(shape)
    A, W2 = P.rows(P.F), P.weights(P.E, P.d, P.F)
    y, _ = P.run(P.L.GEMM_FWD2, P.quant(A, 0), P.quant(W2.reshape(-1, P.F), 0),
                 torch.zeros((P.R32, P.d), dtype=torch.bfloat16))
    An, Wn, Y = np64(A), np64(W2), np64(y)
    for e, r0, n, r1 in P.groups():
        if n:
            assert_close_rel(Y[r0:r0 + n], O.gemm_fwd2(An[r0:r0 + n], Wn[e], ROWQ), TOL, f"y e{e}")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_dgrad2(shape):
    P = MxProblem(shape)
    dY, W2, H13 = P.rows(P.d), P.weights(P.E, P.d, P.F), P.rows(2 * P.F, 2.0)
    dh, _ = P.run(P.L.GEMM_DGRAD2_SWIGLU, P.quant(dY, 0), P.quant(W2.reshape(-1, P.F), 1),
                  torch.zeros((P.R32, 2 * P.F), dtype=torch.bfloat16), aux=H13)
    dYn, Wn, Hn, D = np64(dY), np64(W2), np64(H13), np64(dh)
    for e, r0, n, r1 in P.groups():
        if n:
            ref = O.gemm_dgrad2_swiglu(dYn[r0:r0 + n], Wn[e], Hn[r0:r0 + n], ROWQ, COLQ)
            assert_close_rel(D[r0:r0 + n], ref, TOL, f"dh13 e{e}")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_dgrad1(shape):
    P = MxProblem(shape)
    dH, W13 = P.rows(2 * P.F), P.weights(P.E, 2 * P.F, P.d)
    dx, _ = P.run(P.L.GEMM_DGRAD1, P.quant(dH, 0), P.quant(W13.reshape(-1, P.d), 1),
                  torch.zeros((P.R32, P.d), dtype=torch.bfloat16))
    dHn, Wn, DX = np64(dH), np64(W13), np64(dx)
    for e, r0, n, r1 in P.groups():
        if n:
            assert_close_rel(DX[r0:r0 + n], O.gemm_dgrad1(dHn[r0:r0 + n], Wn[e], ROWQ, COLQ), TOL,
                             f"dx e{e}")


@pytest.mark.parametrize("shape", list(SHAPES))
@pytest.mark.parametrize("which", ["w2", "w13"])
def test_mx_wgrad(shape, which):
    P = MxProblem(shape)
    if which == "w2":
        G, X, M, N, op = P.rows(P.d), P.rows(P.F), P.d, P.F, P.L.GEMM_WGRAD2
    else:
        G, X, M, N, op = P.rows(2 * P.F), P.rows(P.d), 2 * P.F, P.d, P.L.GEMM_WGRAD1
    dW, _ = P.run(op, P.quant(G, 1), P.quant(X, 1), torch.full((P.E, M, N), 5.0, dtype=torch.bfloat16))
    Gn, Xn, DW = np64(G), np64(X), np64(dW)
    for e, r0, n, r1 in P.groups():
        if n == 0:
            assert np.all(DW[e] == 0)
        else:
            assert_close_rel(DW[e], O.gemm_wgrad(Gn[r0:r0 + n], Xn[r0:r0 + n], COLQ), TOL, f"dW e{e}")


# ------------------------------------------------------------------------------------------------
# Fused MXFP8 producers: the routed input, dy, a and dh13 leave their producing kernel only as their
# two quantised forms. Codes and scales must equal the oracle's quantisers applied to the values the
# unfused path holds in bf16 (bit for bit: the quantiser is exact given its input).
# ------------------------------------------------------------------------------------------------

def _operand(P, cols, fill=0xAB):
    z = lambda *sh: torch.full(sh, fill, dtype=torch.uint8, device=dev())
    t = dict(q_row=z(P.R32, cols), s_row=z(P.R32 * cols // 32), q_col=z(P.R32, cols),
             s_col=z(P.R32 * cols // 32))
    return t, P.L.mx_operand(t["q_row"], t["s_row"], t["q_col"], t["s_col"])


def _check_operand(t, vals, used, R32, what):
    """vals: [used, cols] fp64 values (exact bf16) of the routed operand's used rows; rows >= used are
    not written by the fused kernels and are not compared."""
    cols = vals.shape[1]
    rq, rs = MX.quantize_rows(vals)
    cq, cs = MX.quantize_cols(vals)
    assert np.array_equal(t["q_row"][:used].cpu().numpy(), rq), what + " row codes"
    assert np.array_equal(t["q_col"][:used].cpu().numpy(), cq), what + " column codes"
    assert np.array_equal(t["s_row"][:used * cols // 32].cpu().numpy(), tiled(rs)), what + " row scales"
    # column scales: tiled over (column, 32-row block) with R32/32 blocks per column
    full = np.zeros((cols, R32 // 32), dtype=np.uint8)
    full[:, :used // 32] = cs.T
    ref = tiled(full)
    mask = np.zeros((cols, R32 // 32), dtype=bool)
    mask[:, :used // 32] = True
    sel = tiled(mask.astype(np.uint8)).astype(bool)
    assert np.array_equal(t["s_col"].cpu().numpy()[sel], ref[sel]), what + " column scales"


@pytest.mark.parametrize("shape", list(SHAPES))
def test_dispatch_mxfp8_bitexact(shape):
    """Row-wise dispatch straight into the two MXFP8 forms = the oracle's dispatch (x_perm[prow] =
    x[t], zero pad rows) quantised by the oracle."""
    P = MxProblem(shape)
    L = P.L
    x = _bf16_matrix(P.T, P.d, 11 + P.T)
    t, op = _operand(P, P.d)
    row_token = torch.full((P.R32,), -1, dtype=torch.int32)
    row_token[:len(P.meta["row_token"])] = torch.from_numpy(P.meta["row_token"].astype(np.int32))
    L.dispatch_mxfp8(P.cfg, x.to(dev()), row_token.to(dev()), P.poff, op)
    torch.cuda.synchronize()
    used = int(P.meta["poff"][-1])
    xp = O.dispatch(x.double().numpy(), P.meta, P.k)
    _check_operand(t, xp[:used], used, P.R32, "x_perm")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_combine_bwd_mxfp8(shape):
    """Combine backward straight into dy's MXFP8 forms: dy = bf16(g * dout) quantised (bit-exact with
    the oracle's quantiser of the oracle's bf16-stored dy), and the gate gradients <dout_t, y_row>."""
    P = MxProblem(shape)
    L = P.L
    g = torch.Generator().manual_seed(3)
    dout = torch.randn((P.T, P.d), generator=g).to(torch.bfloat16)
    y = P.rows(P.d)
    gates = torch.rand((P.T, P.k), generator=g)
    t, op = _operand(P, P.d)
    dgates = torch.full((P.T, P.k), 9.0, device=dev())
    row_token = torch.full((P.R32,), -1, dtype=torch.int32)
    row_token[:len(P.meta["row_token"])] = torch.from_numpy(P.meta["row_token"].astype(np.int32))
    L.combine_bwd_mxfp8(P.cfg, dout.to(dev()), y.to(dev()), gates.to(dev()), row_token.to(dev()), P.poff,
                        dgates, op)
    torch.cuda.synchronize()
    used = int(P.meta["poff"][-1])
    dy, dg = O.combine_bwd(dout.double().numpy(), np64(y), gates.double().numpy(), P.meta)
    _check_operand(t, O.bf16_round(dy[:used]), used, P.R32, "dy")
    assert_close_rel(dgates.cpu().double().numpy(), dg, 1e-4, "dgates")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_fwd1_quantised_a(shape):
    """GEMM1 + SwiGLU with a quantised in the epilogue: h13 equals the unfused GEMM's bit for bit, and
    a's codes and scales equal the oracle's quantisers applied to the unfused GEMM's bf16 a (itself
    checked against the oracle in test_mx_fwd1)."""
    P = MxProblem(shape)
    L = P.L
    X, W13 = P.rows(P.d), P.weights(P.E, 2 * P.F, P.d)
    XA, WB = P.quant(X, 0), P.quant(W13.reshape(-1, P.d), 0)
    h13, a = P.run(L.GEMM_FWD1_SWIGLU, XA, WB, torch.zeros((P.R32, 2 * P.F), dtype=torch.bfloat16),
                   torch.zeros((P.R32, P.F), dtype=torch.bfloat16))
    h13q = torch.full((P.R32, 2 * P.F), 3.0, dtype=torch.bfloat16, device=dev())
    t, op = _operand(P, P.F)
    L.grouped_gemm_mxfp8_quant(P.cfg, L.GEMM_FWD1_SWIGLU, XA[0], XA[1], WB[0], WB[1], h13q, None, op,
                               P.counts, P.poff, P.ws)
    torch.cuda.synchronize()
    assert L.get_error(P.ws) == 0
    used = int(P.meta["poff"][-1])
    assert torch.equal(h13q[:used], h13[:used])
    _check_operand(t, np64(a)[:used], used, P.R32, "a")


@pytest.mark.parametrize("shape", list(SHAPES))
def test_mx_dgrad2_quantised_dh13(shape):
    """GEMM2 dgrad + SwiGLU backward with dh13 quantised in the epilogue: codes and scales equal the
    oracle's quantisers applied to the unfused GEMM's bf16 dh13 (checked in test_mx_dgrad2)."""
    P = MxProblem(shape)
    L = P.L
    dY, W2, H13 = P.rows(P.d), P.weights(P.E, P.d, P.F), P.rows(2 * P.F, 2.0)
    YA, WB = P.quant(dY, 0), P.quant(W2.reshape(-1, P.F), 1)
    dh, _ = P.run(L.GEMM_DGRAD2_SWIGLU, YA, WB, torch.zeros((P.R32, 2 * P.F), dtype=torch.bfloat16),
                  aux=H13)
    t, op = _operand(P, 2 * P.F)
    L.grouped_gemm_mxfp8_quant(P.cfg, L.GEMM_DGRAD2_SWIGLU, YA[0], YA[1], WB[0], WB[1], None,
                               H13.to(dev()), op, P.counts, P.poff, P.ws)
    torch.cuda.synchronize()
    assert L.get_error(P.ws) == 0
    used = int(P.meta["poff"][-1])
    _check_operand(t, np64(dh)[:used], used, P.R32, "dh13")
