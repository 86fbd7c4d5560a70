"""Pins of the CPU oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself: hand-worked fixtures in
tests/golden/, brute-force counting definitions, closed forms, finite differences, an independent
torch.autograd formulation, and the OCP MX specification's constants.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import moe as O
from oracle import mxfp8 as MX

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------------
# routing
# ------------------------------------------------------------------------------------------------

def test_topk_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "topk_worked.json")))
    logits = np.log(np.array(g["logits_ln"], dtype=np.float64))
    idx, gates = O.route(logits, g["k"])
    assert idx.tolist() == g["idx"]
    np.testing.assert_allclose(gates, np.array(g["gates"]), rtol=0, atol=1e-15)
    meta = O.route_metadata(idx, g["E"], align=4)
    assert meta["counts"].tolist() == g["counts"]
    assert meta["offsets"].tolist() == g["offsets"]
    assert meta["perm"].tolist() == g["perm"]
    assert meta["poff"].tolist() == g["poff_align4"]
    assert meta["prow"].tolist() == g["prow_align4"]


@pytest.mark.parametrize("seed", range(6))
def test_topk_matches_rank_count_definition(seed):
    """e is chosen iff fewer than k experts beat it (higher score, or equal score and lower id); its
    slot is exactly that count. No sort involved."""
    rng = np.random.default_rng(seed)
    T, E = 40, 9
    logits = rng.integers(-3, 4, size=(T, E)).astype(np.float64)  # many ties
    for k in range(1, E + 1):
        idx = O.topk_select(logits, k)
        for t in range(T):
            for e in range(E):
                beat = sum(1 for f in range(E) if logits[t, f] > logits[t, e]
                           or (logits[t, f] == logits[t, e] and f < e))
                if beat < k:
                    assert idx[t, beat] == e
                else:
                    assert e not in idx[t]


def test_topk_special_cases():
    rng = np.random.default_rng(1)
    l = rng.standard_normal((5, 6))
    idx = O.topk_select(l, 6)
    for t in range(5):
        assert list(idx[t]) == sorted(range(6), key=lambda e: (-l[t, e], e))
        assert np.all(np.diff(l[t, idx[t]]) <= 0)
    eq = np.zeros((3, 8))
    assert O.topk_select(eq, 3).tolist() == [[0, 1, 2]] * 3
    # -0.0 equals +0.0: tie goes to the lower id
    z = np.array([[0.0, -0.0, -1.0]])
    assert O.topk_select(z, 2).tolist() == [[0, 1]]
    z = np.array([[-0.0, 0.0, -1.0]])
    assert O.topk_select(z, 2).tolist() == [[0, 1]]


def test_gates_identities():
    rng = np.random.default_rng(2)
    l = rng.standard_normal((50, 16)) * 3
    idx, g = O.route(l, 4)
    np.testing.assert_allclose(g.sum(1), 1.0, atol=1e-15)
    sel = np.take_along_axis(l, idx, 1)
    direct = np.exp(sel) / np.exp(sel).sum(1, keepdims=True)  # softmax over the chosen scores
    np.testing.assert_allclose(g, direct, rtol=1e-13)
    idx2, g2 = O.route(l + 7.25, 4)  # shift invariance
    assert (idx2 == idx).all()
    np.testing.assert_allclose(g2, g, rtol=1e-13)
    # without renormalisation the gates are plain softmax probabilities
    _, gn = O.route(l, 4, renorm=False)
    p = np.exp(l) / np.exp(l).sum(1, keepdims=True)
    np.testing.assert_allclose(gn, np.take_along_axis(p, idx, 1), rtol=1e-13)


def _random_idx(rng, T, E, k):
    return np.stack([rng.permutation(E)[:k] for _ in range(T)])


@pytest.mark.parametrize("T,E,k,align", [(1, 1, 1, 32), (7, 5, 2, 4), (64, 8, 2, 32), (300, 16, 4, 32),
                                         (33, 40, 3, 8)])
def test_metadata_invariants(T, E, k, align):
    rng = np.random.default_rng(T * 1000 + E)
    idx = _random_idx(rng, T, E, k)
    m = O.route_metadata(idx, E, align)
    assert m["counts"].sum() == T * k
    loop = [0] * E
    for t in range(T):
        for j in range(k):
            loop[idx[t, j]] += 1
    assert m["counts"].tolist() == loop
    assert m["offsets"][0] == 0 and m["offsets"][E] == T * k
    assert np.all(m["poff"][:-1] % align == 0)
    assert np.all(np.diff(m["poff"]) >= m["counts"])
    assert sorted(m["perm"].tolist()) == list(range(T * k))  # bijection
    # brute force: rank of (t,j) inside its expert = number of earlier tokens that chose it
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            earlier = sum(1 for u in range(t) if e in idx[u])
            assert m["perm"][t * k + j] == m["offsets"][e] + earlier
            assert m["prow"][t * k + j] == m["poff"][e] + earlier
    rt = m["row_token"]
    assert (rt >= 0).sum() == T * k
    for n in range(T * k):
        assert rt[m["prow"][n]] == n
    for e in range(E):  # pad rows are exactly the tail of each group
        lo, hi = m["poff"][e], m["poff"][e + 1]
        assert np.all(rt[lo:lo + m["counts"][e]] >= 0) and np.all(rt[lo + m["counts"][e]:hi] == -1)
        toks = rt[lo:lo + m["counts"][e]] // k
        assert np.all(np.diff(toks) > 0)  # ascending token order within each expert


def test_unpermute_of_permute_is_identity():
    rng = np.random.default_rng(3)
    T, E, k, d = 50, 7, 3, 5
    idx = _random_idx(rng, T, E, k)
    x = rng.standard_normal((T, d))
    m = O.route_metadata(idx, E)
    xp = O.dispatch(x, m, k)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(xp[m["prow"][t * k + j]], x[t])
    assert np.all(xp[m["row_token"] < 0] == 0)
    ones = np.full((T, k), 1.0 / k)
    np.testing.assert_allclose(O.combine(xp, ones, m), x, rtol=1e-15)


# ------------------------------------------------------------------------------------------------
# layer forward: closed forms and the per-token definition
# ------------------------------------------------------------------------------------------------

def test_identity_experts_return_input():
    rng = np.random.default_rng(4)
    T, E, k, d = 64, 8, 3, 12
    x = rng.standard_normal((T, d))
    l = rng.standard_normal((T, E))
    idx, g = O.route(l, k)
    out, _ = O.layer_fwd(x, None, None, idx, g, expert=lambda e, X: X.copy())
    np.testing.assert_allclose(out, x, rtol=0, atol=1e-14)


def _square_experts(d, c):
    """SwiGLU weights whose expert e computes c_e * x**2 exactly: silu(z) - silu(-z) = z, so with
    gate rows [I; -I], up rows [I; I] and W2 = c_e [I, -I] the output is c_e x (silu(x) - silu(-x))."""
    E = len(c)
    I = np.eye(d)
    W13 = np.stack([np.concatenate([I, -I, I, I], 0)] * E)          # [E, 2F, d], F = 2d
    W2 = np.stack([ce * np.concatenate([I, -I], 1) for ce in c])     # [E, d, F]
    return W13, W2


def test_swiglu_closed_form_square():
    rng = np.random.default_rng(5)
    T, E, k, d = 40, 5, 2, 6
    c = rng.uniform(0.5, 2.0, E)
    W13, W2 = _square_experts(d, c)
    x = rng.standard_normal((T, d))
    idx, g = O.route(rng.standard_normal((T, E)), k)
    out, _ = O.layer_fwd(x, W13, W2, idx, g)
    ref = np.stack([sum(g[t, j] * c[idx[t, j]] for j in range(k)) * x[t] ** 2 for t in range(T)])
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    for t in range(0, T, 7):
        np.testing.assert_allclose(O.token_out(t, x, W13, W2, idx, g), ref[t], rtol=1e-12, atol=1e-12)


def _small_problem(seed, T=24, d=8, F=8, E=5, k=2, router=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    W_r = rng.standard_normal((E, d)) * 0.3
    W13 = rng.standard_normal((E, 2 * F, d)) * 0.3
    W2 = rng.standard_normal((E, d, F)) * 0.3
    dout = rng.standard_normal((T, d))
    return x, W_r, W13, W2, dout


def test_grouped_equals_per_token_definition():
    x, W_r, W13, W2, _ = _small_problem(6, T=60, E=7, k=3)
    l = O.router_logits(x, W_r)
    idx, g = O.route(l, 3)
    out, _ = O.layer_fwd(x, W13, W2, idx, g)
    direct = np.stack([O.token_out(t, x, W13, W2, idx, g) for t in range(60)])
    np.testing.assert_allclose(out, direct, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------------------
# backward: finite differences and torch.autograd
# ------------------------------------------------------------------------------------------------

def _loss(x, W_r, W13, W2, dout, idx, k):
    """Scalar <dout, out> with the selection held at idx (gates recomputed from the logits)."""
    l = O.router_logits(x, W_r)
    g = O.gates_for(l, idx)
    out, _ = O.layer_fwd(x, W13, W2, idx, g)
    return float(np.sum(out * dout))


def test_backward_finite_differences():
    k = 2
    x, W_r, W13, W2, dout = _small_problem(7, T=10, d=6, F=4, E=4, k=k)
    l = O.router_logits(x, W_r)
    idx, g = O.route(l, k)
    srt = -np.sort(-l, axis=1)
    assert np.min(srt[:, k - 1] - srt[:, k]) > 1e-3  # selection margin: FD steps cannot flip it
    out, saved = O.layer_fwd(x, W13, W2, idx, g)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, saved, W_r=W_r)
    h = 1e-6
    for name, arr, grad in [("x", x, gr["dx"]), ("W_r", W_r, gr["dW_r"]),
                            ("W13", W13, gr["dW13"]), ("W2", W2, gr["dW2"])]:
        rng = np.random.default_rng(hash(name) % 1000)
        for _ in range(12):
            pos = tuple(rng.integers(0, s) for s in arr.shape)
            old = arr[pos]
            arr[pos] = old + h
            lp = _loss(x, W_r, W13, W2, dout, idx, k)
            arr[pos] = old - h
            lm = _loss(x, W_r, W13, W2, dout, idx, k)
            arr[pos] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[pos]) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, grad[pos])


def test_backward_matches_torch_autograd():
    k = 3
    x, W_r, W13, W2, dout = _small_problem(8, T=30, d=8, F=6, E=6, k=k)
    l = O.router_logits(x, W_r)
    idx, g = O.route(l, k)
    out, saved = O.layer_fwd(x, W13, W2, idx, g)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, saved, W_r=W_r)

    tx, tWr, tW13, tW2 = (torch.tensor(a, dtype=torch.float64, requires_grad=True)
                          for a in (x, W_r, W13, W2))
    F = W13.shape[1] // 2
    ti = torch.tensor(idx)
    logits = tx @ tWr.T
    sel = torch.gather(logits, 1, ti)
    gates = torch.softmax(sel, dim=1)
    h13 = torch.einsum("tjfd,td->tjf", tW13[ti], tx)
    a = torch.nn.functional.silu(h13[..., :F]) * h13[..., F:]
    y = torch.einsum("tjdf,tjf->tjd", tW2[ti], a)
    tout = (gates[..., None] * y).sum(1)
    np.testing.assert_allclose(tout.detach().numpy(), out, rtol=1e-12, atol=1e-12)
    (tout * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(tx.grad.numpy(), gr["dx"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tWr.grad.numpy(), gr["dW_r"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tW13.grad.numpy(), gr["dW13"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tW2.grad.numpy(), gr["dW2"], rtol=1e-10, atol=1e-12)


def test_per_token_and_per_expert_gradients_match_grouped():
    k = 2
    x, W_r, W13, W2, dout = _small_problem(9, T=40, d=8, F=8, E=6, k=k)
    l = O.router_logits(x, W_r)
    idx, g = O.route(l, k)
    out, saved = O.layer_fwd(x, W13, W2, idx, g)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, saved, W_r=W_r)
    for t in range(0, 40, 5):
        np.testing.assert_allclose(O.token_dx(t, x, W13, W2, idx, g, dout, W_r), gr["dx"][t],
                                   rtol=1e-11, atol=1e-12)
    for e in range(6):
        dW13, dW2 = O.expert_grads(e, x, W13, W2, idx, g, dout)
        np.testing.assert_allclose(dW13, gr["dW13"][e], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(dW2, gr["dW2"][e], rtol=1e-11, atol=1e-12)


def test_square_experts_input_gradient_closed_form():
    """With the square experts and fixed gates, d/dx sum(dout * sum_j g_j c_j x^2) = 2 x dout sum_j g_j c_j."""
    rng = np.random.default_rng(10)
    T, E, k, d = 20, 4, 2, 5
    c = rng.uniform(0.5, 2.0, E)
    W13, W2 = _square_experts(d, c)
    x = rng.standard_normal((T, d))
    dout = rng.standard_normal((T, d))
    idx, g = O.route(rng.standard_normal((T, E)), k)
    _, saved = O.layer_fwd(x, W13, W2, idx, g)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, saved)
    s = np.array([sum(g[t, j] * c[idx[t, j]] for j in range(k)) for t in range(T)])
    np.testing.assert_allclose(gr["dx"], 2 * x * dout * s[:, None], rtol=1e-11, atol=1e-12)
    # gate gradient: <dout, c_e x^2>
    for t in range(T):
        for j in range(k):
            np.testing.assert_allclose(gr["dgates"][t, j], c[idx[t, j]] * np.dot(dout[t], x[t] ** 2),
                                       rtol=1e-11)


# ------------------------------------------------------------------------------------------------
# MXFP8
# ------------------------------------------------------------------------------------------------

def _parse_num(s):
    s = s.strip()
    if "*" in s:
        a, b = s.split("*")
        return _parse_num(a) * _parse_num(b)
    if s.startswith("-"):
        return -_parse_num(s[1:])
    if s.startswith("2^"):
        return 2.0 ** int(s[2:])
    return float(s)


def _expand(items, conv):
    out = []
    for it in items:
        parts = it.split(" x")
        out += [conv(parts[0])] * (int(parts[1]) if len(parts) > 1 else 1)
    return out


def test_mxfp8_worked_blocks():
    g = json.load(open(os.path.join(GOLDEN, "mxfp8_blocks.json")))
    for case in g["cases"]:
        vals = np.array(_expand(case["values"], _parse_num))
        codes = _expand(case["codes"], lambda s: int(s, 16))
        assert len(vals) == 32 and len(codes) == 32
        # the fixture values are exact in bf16
        assert np.array_equal(torch.tensor(vals).to(torch.bfloat16).double().numpy(), vals)
        c, s = MX.quantize_rows(vals[None, :])
        assert int(s[0, 0]) == case["scale"], case["name"]
        assert c[0].tolist() == codes, case["name"]


def test_e4m3_spec_constants():
    assert MX.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert MX.e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6
    assert MX.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9
    assert np.isnan(MX.e4m3_decode(np.array([0x7F, 0xFF]))).all()
    assert MX.e4m3_decode(np.array([0xFE]))[0] == -448.0
    assert MX.ue8m0_decode(np.array([127]))[0] == 1.0 and MX.ue8m0_decode(np.array([0]))[0] == 2.0 ** -127
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    dec = MX.e4m3_decode(np.array(finite))
    back = MX.e4m3_encode(dec)
    # every finite code round-trips (including -0.0 = 0x80)
    assert back.tolist() == finite


def test_e4m3_encode_matches_torch_cast():
    """torch's float8_e4m3fn cast is an independent round-to-nearest-even implementation; compared
    after clamping to the saturation bound."""
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.05, 1, 30, 300)])
    v = torch.tensor(v, dtype=torch.float32).to(torch.bfloat16).double().numpy()  # bf16 inputs
    ours = MX.e4m3_encode(v)
    t = torch.tensor(np.clip(v, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, t)


def test_mxfp8_roundtrip_error_bound():
    rng = np.random.default_rng(12)
    a = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-8, 8, (64, 1)))
    a = torch.tensor(a, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    c, s = MX.quantize_rows(a)
    deq = MX.dequantize_rows(c, s)
    X = MX.ue8m0_decode(s)
    scaled = np.abs(a).reshape(64, 8, 32) / X[..., None]
    normal = (scaled >= 2.0 ** -6) & (scaled <= 448)
    rel = np.abs(deq - a).reshape(64, 8, 32) / np.abs(a).reshape(64, 8, 32)
    assert np.all(rel[normal] <= 2.0 ** -4 + 1e-15)
    # every block's amax lands in [256, 512) before saturation
    amax = np.abs(a).reshape(64, 8, 32).max(-1)
    r = amax / X
    assert np.all((r >= 256) & (r < 512))
    # column quantisation is row quantisation of the transpose
    cc, sc = MX.quantize_cols(a.T)
    assert np.array_equal(cc, c.T) and np.array_equal(sc, s.T)


def test_mxfp8_layer_error_is_the_formats_own():
    """The emulated MXFP8 layer differs from the exact layer by what E4M3 rounding predicts: each
    quantised operand carries about 2-3% rms relative error, so a two-GEMM SwiGLU path lands near
    5-8% rms relative error -- nonzero, and well under 12%."""
    k = 2
    rng = np.random.default_rng(13)
    T, d, F, E = 64, 256, 128, 4
    x = rng.standard_normal((T, d))
    W13 = rng.standard_normal((E, 2 * F, d)) * 0.02
    W2 = rng.standard_normal((E, d, F)) * 0.02
    dout = rng.standard_normal((T, d))
    idx, g = O.route(rng.standard_normal((T, E)), k)
    out, sv = O.layer_fwd(x, W13, W2, idx, g)
    outq, svq = O.layer_fwd(x, W13, W2, idx, g, mx=True)
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    assert 0.01 < rel(outq, out) < 0.12
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, sv)
    grq = O.layer_bwd(dout, x, W13, W2, idx, g, svq, mx=True)
    for key in ("dx", "dW13", "dW2"):
        assert 0.01 < rel(grq[key], gr[key]) < 0.12, key


def test_mxfp8_quantisation_axes():
    """Operands whose blocks are exactly representable along the contraction axis pass through the
    emulated GEMMs unchanged; the same matrices blocked along the other axis do not."""
    rng = np.random.default_rng(14)
    # rows with very different power-of-two scales, entries small integers: exact along rows
    W = rng.integers(-7, 8, size=(64, 64)).astype(np.float64) * (2.0 ** rng.integers(-20, 20, (64, 1)))
    assert np.array_equal(O._mx_row(W), W)
    assert not np.array_equal(O._mx_col(W), W)
    assert np.array_equal(O._mx_col(W.T), W.T)
    # forward GEMM1 of a representable problem is exact
    T, d, F, E, k = 32, 64, 32, 2, 1
    x = rng.integers(-4, 5, size=(T, d)).astype(np.float64)
    W13 = rng.integers(-4, 5, size=(E, 2 * F, d)).astype(np.float64) / 16
    W2 = rng.standard_normal((E, d, F))
    idx, g = O.route(rng.standard_normal((T, E)), k)
    _, sv = O.layer_fwd(x, W13, W2, idx, g)
    _, svq = O.layer_fwd(x, W13, W2, idx, g, mx=True)
    np.testing.assert_array_equal(svq["h13"], sv["h13"])


def test_mxfp8_per_token_forms_match_grouped():
    """Row-wise quantisation is per row, so the per-token MXFP8 output and input gradient equal the
    grouped MXFP8 layer's (the wgrads, whose blocks span tokens, are not per-token)."""
    rng = np.random.default_rng(15)
    T, d, F, E, k = 40, 64, 64, 4, 2
    x = rng.standard_normal((T, d))
    W13 = rng.standard_normal((E, 2 * F, d)) * 0.1
    W2 = rng.standard_normal((E, d, F)) * 0.1
    dout = rng.standard_normal((T, d))
    idx, g = O.route(rng.standard_normal((T, E)), k)
    out, sv = O.layer_fwd(x, W13, W2, idx, g, mx=True)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, sv, mx=True)
    qw = {e: O.quantised_expert_weights(W13[e], W2[e]) for e in range(E)}
    for t in range(0, T, 3):
        np.testing.assert_allclose(O.token_out_mx(t, x, qw, idx, g), out[t], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(O.token_dx_mx(t, x, qw, idx, g, dout), gr["dx"][t], rtol=1e-10,
                                   atol=1e-12)


# ------------------------------------------------------------------------------------------------
# bf16 rounding, MXFP8 backward quantisation axes, router backward without renormalisation
# ------------------------------------------------------------------------------------------------

def test_bf16_round_matches_torch_cast():
    """The oracle's bf16 rounding (round to nearest, ties to even, through fp32) against torch's
    float32 -> bfloat16 cast, an independent implementation, on exact ties of both parities,
    subnormals, the largest finite values, signed zeros and random values over many binades."""
    rng = np.random.default_rng(21)
    # exact ties: the 16 discarded bits are 0x8000; the kept lsb is 0 (round down) or 1 (round up)
    hi = rng.integers(0, 1 << 15, 400, dtype=np.uint64) << 17  # bit 16 (kept lsb) = 0
    hi = hi[((hi >> 23) & 0xFF) < 0xFE]  # finite, and rounding up stays finite
    ties_even = (hi | 0x8000).astype(np.uint32).view(np.float32)
    ties_odd = (hi | 0x10000 | 0x8000).astype(np.uint32).view(np.float32)
    just_below = (hi | 0x7FFF).astype(np.uint32).view(np.float32)
    just_above = (hi | 0x8001).astype(np.uint32).view(np.float32)
    sub = (rng.integers(1, 1 << 23, 400, dtype=np.uint64)).astype(np.uint32).view(np.float32)
    big = np.array([3.3895313892515355e38, -3.3895313892515355e38, 3.389531e38, 1e38, -2e38],
                   dtype=np.float32)
    zeros = np.array([0.0, -0.0], dtype=np.float32)
    rnd = (rng.standard_normal(5000) * np.exp(rng.uniform(-60, 60, 5000))).astype(np.float32)
    vals = np.concatenate([ties_even, ties_odd, -ties_odd, just_below, just_above, sub, -sub, big,
                           zeros, rnd]).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    ours = O.bf16_round(vals.astype(np.float64))
    ref = torch.from_numpy(vals.copy()).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, ref)
    assert np.array_equal(np.signbit(ours), np.signbit(ref))  # -0.0 stays -0.0
    # the tie cases really are ties and really go both ways
    t_even = O.bf16_round(ties_even.astype(np.float64))
    assert np.array_equal(t_even.astype(np.float32).view(np.uint32), (hi.astype(np.uint32)))
    t_odd = O.bf16_round(ties_odd.astype(np.float64))
    assert np.array_equal(t_odd.astype(np.float32).view(np.uint32),
                          (hi + 0x20000).astype(np.uint32))


def _pow2_cols(rng, n, m, lo=-18, hi=18, vals=(-3, -2, -1, 1, 2, 3)):
    """[n, m] matrix exact in MXFP8 blocks of 32 rows (each column one power-of-two scale, small
    integer mantissas) whose 32-element row blocks mix scales far apart (so rounding along rows
    loses values)."""
    sc = 2.0 ** rng.integers(lo, hi, size=(1, m))
    return rng.choice(np.array(vals, dtype=np.float64), size=(n, m)) * sc


def _one_hot_rows(rng, n, m, scales):
    """[n, m] with one nonzero per row, row i holding scales[i] in a random column."""
    Y = np.zeros((n, m))
    Y[np.arange(n), rng.integers(0, m, n)] = scales
    return Y


def _swiglu_gate0(n, F):
    """Saved h13 with gate = 0 and up = 2: the SwiGLU backward then gives dgate = dA, dup = 0."""
    return np.concatenate([np.zeros((n, F)), np.full((n, F), 2.0)], axis=1)


@pytest.mark.parametrize("gemm", ["dgrad2", "wgrad2", "dgrad1", "wgrad1"])
def test_mxfp8_backward_quantisation_axes(gemm):
    """Each backward GEMM of the emulated MXFP8 expert quantises each operand along that GEMM's
    contraction axis: rows of dY and dH13 for the dgrads (blocks along d and 2F), 32-row blocks of
    the weight for the dgrads, 32-row blocks of both operands for the wgrads (contraction over the
    expert's tokens). Operands exact in blocks along the contraction axis -- and not along the
    other -- pass through unchanged, so that GEMM's emulated result equals the unquantised one bit
    for bit; quantising either operand along the other axis changes it."""
    rng = np.random.default_rng({"dgrad2": 31, "wgrad2": 32, "dgrad1": 33, "wgrad1": 34}[gemm])
    n, d, F = 64, 64, 64
    X = rng.standard_normal((n, d))
    W13 = rng.standard_normal((2 * F, d))
    W2 = rng.standard_normal((d, F))
    h13 = rng.standard_normal((n, 2 * F))
    a = rng.standard_normal((n, F))
    dY = rng.standard_normal((n, d))
    row_scales = 2.0 ** rng.integers(-18, 18, n)
    R, C = O._mx_row, O._mx_col
    if gemm == "dgrad2":
        # dA = R(dY) @ C(W2): dY exact along rows only, W2 exact along 32-row blocks only
        dY = _one_hot_rows(rng, n, d, row_scales)
        W2 = _pow2_cols(rng, d, F)
        h13 = _swiglu_gate0(n, F)
        operands = (dY, W2)
    elif gemm == "wgrad2":
        # dW2 = C(dY)^T C(a): both exact along 32-row blocks only
        dY = _pow2_cols(rng, n, d)
        a = _pow2_cols(rng, n, F)
        operands = (dY, a)
    elif gemm == "dgrad1":
        # dX = R(dH13) @ C(W13); dH13 = [dA, 0] with dA = one-hot(s_i) @ (+-1): exact along rows only
        dY = _one_hot_rows(rng, n, d, row_scales)
        W2 = rng.choice(np.array([-1.0, 1.0]), size=(d, F))
        h13 = _swiglu_gate0(n, F)
        W13 = _pow2_cols(rng, 2 * F, d)
        operands = (W13,)
    else:
        # dW13 = C(dH13)^T C(X); dH13 = [dA, 0] with dA = one-hot(1) @ W2, W2 column-scaled: exact
        # along 32-row blocks only
        dY = _one_hot_rows(rng, n, d, np.ones(n))
        W2 = _pow2_cols(rng, d, F, vals=(-1, 1))
        h13 = _swiglu_gate0(n, F)
        X = _pow2_cols(rng, n, d)
        operands = (X,)
    for M in operands:  # exact along the contraction axis, not along the other
        exact_rows = np.array_equal(R(M), M)
        exact_cols = np.array_equal(C(M), M)
        assert exact_rows != exact_cols
    dX, dW13, dW2, dH13 = O.expert_bwd(X, W13, W2, h13, a, dY, mx=True)
    eX, edW13, edW2, edH13 = O.expert_bwd(X, W13, W2, h13, a, dY, mx=False)
    ident = lambda m: m
    if gemm == "dgrad2":
        assert np.array_equal(dH13, O.bf16_round(edH13))  # bf16 storage of dH13 in the MXFP8 layer
        for qr, qc in ((C, C), (R, R), (C, R)):
            assert not np.array_equal(O.gemm_dgrad2_swiglu(dY, W2, h13, qr, qc),
                                      O.gemm_dgrad2_swiglu(dY, W2, h13, ident, ident))
    elif gemm == "wgrad2":
        assert np.array_equal(dW2, edW2)
        assert not np.array_equal(R(dY).T @ C(a), edW2)
        assert not np.array_equal(C(dY).T @ R(a), edW2)
    elif gemm == "dgrad1":
        assert np.array_equal(dH13, edH13) and not np.array_equal(C(dH13), dH13)
        assert np.array_equal(dX, eX)
        assert not np.array_equal(O.gemm_dgrad1(dH13, W13, C, C), eX)
        assert not np.array_equal(O.gemm_dgrad1(dH13, W13, R, R), eX)
    else:
        assert np.array_equal(dH13, edH13) and not np.array_equal(R(dH13[:, :F]), dH13[:, :F])
        assert np.array_equal(dW13, edW13)
        assert not np.array_equal(O.gemm_wgrad(dH13, X, R), edW13)
        assert not np.array_equal(C(dH13).T @ R(X), edW13)
        assert not np.array_equal(R(dH13).T @ C(X), edW13)


def test_router_backward_without_renormalisation_finite_differences():
    """router_bwd(renorm=False): the gates are plain softmax probabilities of the chosen experts,
    g_t,j = softmax(l_t)[S_j]. The dense score gradient it returns must match central finite
    differences of L(l) = sum_tj dg_tj g_tj(l), with the selection held fixed."""
    rng = np.random.default_rng(41)
    T, E, k = 9, 7, 3
    l = rng.standard_normal((T, E))
    idx = O.topk_select(l, k)
    dg = rng.standard_normal((T, k))
    g = O.gates_for(l, idx, renorm=False)
    dl = O.router_bwd(dg, g, idx, E, renorm=False, logits=l)

    def L(lv):
        return float(np.sum(dg * O.gates_for(lv, idx, renorm=False)))

    h = 1e-6
    fd = np.zeros_like(l)
    for t in range(T):
        for e in range(E):
            lp, lm = l.copy(), l.copy()
            lp[t, e] += h
            lm[t, e] -= h
            fd[t, e] = (L(lp) - L(lm)) / (2 * h)
    np.testing.assert_allclose(dl, fd, rtol=1e-7, atol=1e-9)
    # experts outside the selection get a gradient too (through the softmax denominator)
    outside = np.ones((T, E), bool)
    np.put_along_axis(outside, idx, False, axis=1)
    assert np.all(np.abs(dl[outside]) > 0)
    # and the renormalised branch is a different function: it matches its own finite differences
    gr = O.gates_for(l, idx, renorm=True)
    dlr = O.router_bwd(dg, gr, idx, E, renorm=True)
    assert np.all(dlr[outside] == 0)


def test_mxfp8_max_error_against_unquantised_is_the_formats_own():
    """How far an exact MXFP8 layer sits from the unquantised fp64 layer in the max-norm
    (max|err| / max|ref|), on the small MXFP8 test shapes (T=512 d=256 F=256 E=16 k=4, uniform
    routing, 128-row groups). This is the emulated oracle itself -- no kernel involved -- so it is the
    format's own error: out and dx stay near 8e-2, the weight gradients (whose contraction runs over
    32-token blocks of unrelated tokens) go above it. A GPU result can only be as close to the
    unquantised layer as this."""
    from moe_workloads import Workload, make_inputs
    w = Workload("mx_uniform", 512, 256, 256, 16, 4, "mxfp8", "uniform")
    inp = make_inputs(w, seed=0, device="cpu")
    f = lambda t: t.to(torch.float64).numpy()
    x, W13, W2, dout = f(inp["x"]), f(inp["W13"]), f(inp["W2"]), f(inp["dout"])
    idx, g = inp["idx"].numpy().astype(np.int64), f(inp["gates"])
    out, sv = O.layer_fwd(x, W13, W2, idx, g, align=128)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, sv)
    outq, svq = O.layer_fwd(x, W13, W2, idx, g, align=128, mx=True)
    grq = O.layer_bwd(dout, x, W13, W2, idx, g, svq, mx=True)
    rel = lambda a, b: float(np.max(np.abs(a - b)) / np.max(np.abs(b)))
    err = {"out": rel(outq, out), **{k: rel(grq[k], gr[k]) for k in ("dx", "dW13", "dW2", "dgates")}}
    assert all(0.02 < v < 0.2 for v in err.values()), err
    assert err["dW13"] > 0.08 and err["dW2"] > 0.08, err  # above the 8e-2 bar: the format, not a kernel


def test_token_expert_outputs_sum_to_the_output_and_give_the_gate_gradients():
    """Per-slot expert outputs of one token: their gate-weighted sum is the layer output, and their
    inner products with dout are the grouped backward's gate gradients."""
    k = 3
    x, W_r, W13, W2, dout = _small_problem(9, T=20, d=8, F=6, E=5, k=k)
    idx, g = O.route(O.router_logits(x, W_r), k)
    out, saved = O.layer_fwd(x, W13, W2, idx, g)
    gr = O.layer_bwd(dout, x, W13, W2, idx, g, saved)
    for t in range(20):
        ys = O.token_expert_outputs(t, x, W13, W2, idx)
        np.testing.assert_allclose(g[t] @ ys, out[t], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(ys @ dout[t], gr["dgates"][t], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------------------------------------
# expert parallelism layout
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("world,E,T,k", [(1, 8, 50, 2), (2, 8, 40, 3), (4, 16, 33, 4), (8, 32, 20, 2)])
def test_ep_layout_is_a_source_major_stable_placement(world, E, T, k):
    """Brute force: building each owner's buffer by appending, expert by expert, every source's entries
    in token order (then padding the group to 32 rows) gives exactly the rows the layout assigns; every
    owner row below its end is used once or is a pad row; with one rank it is the single-GPU
    metadata."""
    rng = np.random.default_rng(world * 100 + E)
    idx = [np.stack([rng.permutation(E)[:k] for _ in range(T)]) for _ in range(world)]
    all_counts = np.stack([np.bincount(i.reshape(-1), minlength=E) for i in idx])
    L = O.ep_layout(all_counts, world)
    EL = E // world
    for h in range(world):
        buf = []  # (source, entry) per row, None for pad rows
        for el in range(EL):
            e = h * EL + el
            assert len(buf) == L["poff_loc"][h, el]
            for g in range(world):
                buf += [(g, n) for n, ee in enumerate(idx[g].reshape(-1)) if ee == e]
            while len(buf) % 32:
                buf.append(None)
        assert len(buf) == L["poff_loc"][h, EL]
        for g in range(world):
            rows = O.ep_dst_rows(idx[g], L["base"][g], E)
            for n, ee in enumerate(idx[g].reshape(-1)):
                if ee // EL == h:
                    assert buf[rows[n]] == (g, n)
    if world == 1:
        meta = O.route_metadata(idx[0], E)
        assert np.array_equal(O.ep_dst_rows(idx[0], L["base"][0], E), meta["prow"])
        assert np.array_equal(L["poff_loc"][0], meta["poff"])
