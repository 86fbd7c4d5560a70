"""Plain fp64 CPU oracle of the MoE expert layer, forward and backward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module: only the tests,
`__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` use it. It shares no code with the
CUDA library (no kernels, headers, tables or helpers); the only thing both sides use is the seeded
input generator in `moe_workloads`.

What it computes (per token t, "Olmo-core 3", all three pages: k of E experts are active per token --
noticiarioia.com, "Mudanca de arquitetura e ganhos de desempenho"; routed rows land directly in the
experts' input buffers and one grouped GEMM runs the experts -- bytechap.com, "Como funciona" and
unite.ai, "Parallelismo, precisione e tecniche di memoria"):

    l_t    = W_r x_t (+ b)                         router scores ("routing scores", bytechap.com,
                                                   "Detalles clave")
    S_t    = the k experts with largest l_t,e; equal scores go to the lower expert id; slots in
             descending score order
    g_t,j  = softmax(l_t)[S_j] / sum_{i in S_t} softmax(l_t)[i]      (renormalised gates)
    out_t  = sum_j g_t,j * W2_e (silu(W1_e x_t) * W3_e x_t),  e = S_t,j  (SwiGLU expert, no biases;
             W13_e stacks W1_e (rows 0..F-1, "gate") over W3_e (rows F..2F-1, "up"))

The backward pass is the exact derivative of this with respect to x, W_r, W13 and W2 for a given
upstream gradient dout, with the selection S held fixed.

The pages fix none of the formulas above; the readings taken where they are silent (selection on
logits, renormalisation, tie-break, slot order, row order inside an expert, 32-row aligned group
starts, gate applied after W2, silu(z) = z*sigmoid(z)) are named constants or arguments here.

Everything is float64 numpy; library routines used as single steps: np.lexsort / np.argsort (stable
sorts), matrix products (BLAS) and np.exp.
"""
from __future__ import annotations

import numpy as np

ALIGN = 32  # row alignment of each expert's group start in the padded routed buffer (a reading)


def f64(a) -> np.ndarray:
    """Convert a torch tensor / array to a float64 numpy array (exact for fp32 and bf16 values)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------------------------
# Routing
# ----------------------------------------------------------------------------------------------

def router_logits(x: np.ndarray, W_r: np.ndarray, bias: np.ndarray | None = None) -> np.ndarray:
    """l = x W_r^T (+ bias), [T,E] float64. The bias is a constant input (no gradient)."""
    l = x @ W_r.T
    if bias is not None:
        l = l + bias[None, :]
    return l


def topk_select(logits: np.ndarray, k: int) -> np.ndarray:
    """Per token, the k experts with the largest score; ties to the lower expert id; slots in
    descending score order (then ascending id). Returns int64 [T,k]."""
    T, E = logits.shape
    ids = np.arange(E)
    idx = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        # lexsort: last key is primary -> sort by -score, then by expert id
        order = np.lexsort((ids, -logits[t]))
        idx[t] = order[:k]
    return idx


def softmax(v: np.ndarray, axis: int = -1) -> np.ndarray:
    m = np.max(v, axis=axis, keepdims=True)
    e = np.exp(v - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def gates_for(logits: np.ndarray, idx: np.ndarray, renorm: bool = True) -> np.ndarray:
    """Gate of each selected slot: softmax probability of the chosen expert, renormalised over the
    k chosen experts when `renorm` (the reading taken for every workload)."""
    p = softmax(logits, axis=1)
    sel = np.take_along_axis(p, idx, axis=1)
    if renorm:
        sel = sel / np.sum(sel, axis=1, keepdims=True)
    return sel


def route(logits: np.ndarray, k: int, renorm: bool = True):
    idx = topk_select(logits, k)
    return idx, gates_for(logits, idx, renorm)


def route_metadata(idx: np.ndarray, E: int, align: int = ALIGN) -> dict:
    """GPU-resident routing metadata, by its plain definitions.

    counts[e]    number of (t,j) with idx[t,j] = e                       (a bincount)
    offsets      exclusive prefix sum of counts, length E+1, offsets[E] = T*k
    poff         exclusive prefix sum of counts rounded up to `align`, length E+1
    perm[t*k+j]  position of (t,j) in the expert-sorted order, stable in t (a counting sort)
    prow[t*k+j]  its row in the padded buffer: poff[e] + perm - offsets[e]
    row_token[r] for each padded row r < poff[E]: the (t*k+j) it holds, or -1 for a pad row
    """
    T, k = idx.shape
    flat = idx.reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    padded = -(-counts // align) * align
    poff = np.concatenate([[0], np.cumsum(padded)])
    order = np.argsort(flat, kind="stable")  # entries are in (t, j) order, so stable => ascending t
    perm = np.empty(T * k, dtype=np.int64)
    perm[order] = np.arange(T * k)
    prow = poff[flat] + perm - offsets[flat]
    row_token = np.full(int(poff[E]), -1, dtype=np.int64)
    row_token[prow] = np.arange(T * k)
    return dict(counts=counts, offsets=offsets, poff=poff, perm=perm, prow=prow, row_token=row_token)


# ----------------------------------------------------------------------------------------------
# Permutation
# ----------------------------------------------------------------------------------------------

def dispatch(x: np.ndarray, meta: dict, k: int) -> np.ndarray:
    """x_perm[prow[t*k+j]] = x[t]; pad rows are zero."""
    rows = int(meta["poff"][-1])
    xp = np.zeros((rows,) + x.shape[1:], dtype=np.float64)
    for n, r in enumerate(meta["prow"]):
        xp[r] = x[n // k]
    return xp


def combine(y: np.ndarray, gates: np.ndarray, meta: dict) -> np.ndarray:
    """out[t] = sum_j gates[t,j] * y[prow[t*k+j]]."""
    T, k = gates.shape
    out = np.zeros((T,) + y.shape[1:], dtype=np.float64)
    for t in range(T):
        for j in range(k):
            out[t] += gates[t, j] * y[meta["prow"][t * k + j]]
    return out


def combine_bwd(dout: np.ndarray, y: np.ndarray, gates: np.ndarray, meta: dict):
    """Exact derivative of the combine: dy[prow[t*k+j]] = g[t,j] dout[t] (pad rows 0) and
    dgates[t,j] = <dout[t], y[prow[t*k+j]]>."""
    T, k = gates.shape
    dy = np.zeros((y.shape[0],) + dout.shape[1:])
    dgates = np.zeros((T, k))
    for t in range(T):
        for j in range(k):
            r = meta["prow"][t * k + j]
            dy[r] = gates[t, j] * dout[t]
            dgates[t, j] = float(np.dot(dout[t], y[r]))
    return dy, dgates


def token_reduce(dx_perm: np.ndarray, meta: dict, T: int, k: int, dlogits=None, W_r=None):
    """Gradient back to tokens: dx[t] = sum_j dx_perm[prow[t*k+j]] (+ dlogits[t] W_r, the router's
    input gradient, when given)."""
    dx = np.zeros((T,) + dx_perm.shape[1:])
    for t in range(T):
        for j in range(k):
            dx[t] += dx_perm[meta["prow"][t * k + j]]
    if dlogits is not None:
        dx = dx + dlogits @ W_r
    return dx


# ----------------------------------------------------------------------------------------------
# Expert MLP (SwiGLU)
# ----------------------------------------------------------------------------------------------

def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def silu(z):
    return z * sigmoid(z)


def silu_grad(z):
    s = sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def _ident(a):
    return a


def bf16_round(a):
    """Round to bfloat16 (nearest, ties to even) through fp32, the precision the MXFP8 workload stores
    every GEMM output and activation in ("bf16 outputs"). Returned as float64."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    b = f.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _mx_row(a):
    """MXFP8 fake-quantisation with blocks of 32 along the last (contraction) axis."""
    from . import mxfp8
    return mxfp8.fake_quant_rows(a)


def _mx_col(a):
    """MXFP8 fake-quantisation with blocks of 32 consecutive rows (contraction along rows); the
    rows are zero-padded to a multiple of 32 first, as the padded group buffers are."""
    from . import mxfp8
    n = a.shape[0]
    pad = (-n) % mxfp8.BLOCK
    ap = np.concatenate([a, np.zeros((pad,) + a.shape[1:])], axis=0) if pad else a
    return mxfp8.fake_quant_cols(ap)[:n]


def gemm_fwd1_swiglu(X, W13_e, qr=_ident):
    """First expert GEMM and SwiGLU: h13 = X W13_e^T = [gate | up]; a = silu(gate) * up."""
    F = W13_e.shape[0] // 2
    h13 = qr(X) @ qr(W13_e).T
    return h13, silu(h13[:, :F]) * h13[:, F:]


def gemm_fwd2(A, W2_e, qr=_ident):
    """Second expert GEMM: y = a W2_e^T."""
    return qr(A) @ qr(W2_e).T


def gemm_dgrad2_swiglu(dY, W2_e, h13, qr=_ident, qc=_ident):
    """dA = dY W2_e (contraction over d), then the SwiGLU backward with the saved h13:
    dgate = dA * up * silu'(gate), dup = dA * silu(gate); returns dH13 = [dgate | dup]."""
    F = h13.shape[1] // 2
    gate, up = h13[:, :F], h13[:, F:]
    dA = qr(dY) @ qc(W2_e)
    return np.concatenate([dA * up * silu_grad(gate), dA * silu(gate)], axis=1)


def gemm_dgrad1(dH13, W13_e, qr=_ident, qc=_ident):
    """dX = dH13 W13_e (contraction over 2F)."""
    return qr(dH13) @ qc(W13_e)


def gemm_wgrad(G, X, qc=_ident):
    """Weight gradient over one expert's rows: G^T X (contraction over the rows)."""
    return qc(G).T @ qc(X)


def expert_fwd(X: np.ndarray, W13_e: np.ndarray, W2_e: np.ndarray, mx: bool = False):
    """One expert on its rows X [n,d]: h13 = X W13_e^T = [gate | up], a = silu(gate)*up, y = a W2_e^T.
    With `mx`, every GEMM operand is MXFP8-quantised along that GEMM's contraction axis first."""
    qr = _mx_row if mx else _ident
    if not mx:
        h13, a = gemm_fwd1_swiglu(X, W13_e, qr)
        return h13, a, gemm_fwd2(a, W2_e, qr)
    # MXFP8 workload: GEMM outputs and activations are stored in bf16; SwiGLU reads the stored h13
    F = W13_e.shape[0] // 2
    h13 = bf16_round(qr(X) @ qr(W13_e).T)
    a = bf16_round(silu(h13[:, :F]) * h13[:, F:])
    return h13, a, bf16_round(gemm_fwd2(a, W2_e, qr))


def expert_bwd(X, W13_e, W2_e, h13, a, dY, mx: bool = False):
    """Exact gradients of y = W2 (silu(W1 x) * W3 x) for one expert, rows batched. With `mx`, each
    GEMM's operands are MXFP8-quantised along that GEMM's contraction axis (rows for the weight
    operand of a dgrad GEMM and for both operands of a wgrad GEMM)."""
    qr = _mx_row if mx else _ident
    qc = _mx_col if mx else _ident
    st = bf16_round if mx else _ident                  # MXFP8 workload: bf16 storage
    dH13 = st(gemm_dgrad2_swiglu(dY, W2_e, h13, qr, qc))   # [n,2F]
    dW2 = gemm_wgrad(dY, a, qc)                        # [d,F]
    dW13 = gemm_wgrad(dH13, X, qc)                     # [2F,d]
    dX = gemm_dgrad1(dH13, W13_e, qr, qc)              # [n,d]
    return dX, dW13, dW2, dH13


# ----------------------------------------------------------------------------------------------
# Layer, grouped form (what the GPU path computes)
# ----------------------------------------------------------------------------------------------

def layer_fwd(x, W13, W2, idx, gates, align: int = ALIGN, expert=None, mx: bool = False):
    """Grouped forward: route metadata -> dispatch -> per-expert MLP on its contiguous rows ->
    gate-weighted combine. `expert(e, X_e)` may replace the SwiGLU expert (used by closed-form
    checks); it must return y_e."""
    T, k = idx.shape
    E = W13.shape[0] if W13 is not None else int(idx.max()) + 1
    meta = route_metadata(idx, E, align)
    xp = dispatch(x, meta, k)
    d = x.shape[1]
    rows = xp.shape[0]
    y = np.zeros((rows, d))
    h13 = a = None
    if expert is None:
        F = W13.shape[1] // 2
        h13 = np.zeros((rows, 2 * F))
        a = np.zeros((rows, F))
    for e in range(E):
        r0, n = int(meta["poff"][e]), int(meta["counts"][e])
        if n == 0:
            continue
        X = xp[r0:r0 + n]
        if expert is None:
            h13[r0:r0 + n], a[r0:r0 + n], y[r0:r0 + n] = expert_fwd(X, W13[e], W2[e], mx)
        else:
            y[r0:r0 + n] = expert(e, X)
    out = combine(y, gates, meta)
    return out, dict(meta=meta, x_perm=xp, h13=h13, a=a, y=y)


def router_bwd(dgates, gates, idx, E: int, renorm: bool = True, logits=None):
    """d(loss)/d(logits), dense [T,E], from d(loss)/d(gates).

    renorm: g_j = exp(l_Sj) / sum_i exp(l_Si)  ->  dl_Sj = g_j (dg_j - sum_i g_i dg_i), zero elsewhere.
    no renorm: g_j = softmax(l)[S_j]           ->  dl_e = p_e ([e in S] dg_e - sum_j g_j dg_j).
    """
    T, k = idx.shape
    dl = np.zeros((T, E))
    s = np.sum(gates * dgates, axis=1)
    if renorm:
        for t in range(T):
            for j in range(k):
                dl[t, idx[t, j]] = gates[t, j] * (dgates[t, j] - s[t])
    else:
        p = softmax(logits, axis=1)
        for t in range(T):
            dsel = np.zeros(E)
            dsel[idx[t]] = dgates[t]
            dl[t] = p[t] * (dsel - s[t])
    return dl


def layer_bwd(dout, x, W13, W2, idx, gates, saved, W_r=None, renorm=True, logits=None,
              mx: bool = False):
    """Grouped backward. Returns dx, dW13, dW2, dgates, dlogits (or None), dW_r (or None), plus the
    routed intermediates dy (rows), dh13 (rows) and dx_perm (rows)."""
    meta = saved["meta"]
    T, k = idx.shape
    E, F2, d = W13.shape
    rows = saved["x_perm"].shape[0]
    dy, dgates = combine_bwd(dout, saved["y"], gates, meta)
    if mx:
        dy = bf16_round(dy)
    dW13 = np.zeros_like(W13, dtype=np.float64)
    dW2 = np.zeros_like(W2, dtype=np.float64)
    dxp = np.zeros((rows, d))
    dh13 = np.zeros((rows, F2))
    for e in range(E):
        r0, n = int(meta["poff"][e]), int(meta["counts"][e])
        if n == 0:
            continue
        sl = slice(r0, r0 + n)
        dX, dW13[e], dW2[e], dh13[sl] = expert_bwd(saved["x_perm"][sl], W13[e], W2[e],
                                                   saved["h13"][sl], saved["a"][sl], dy[sl], mx)
        dxp[sl] = dX
    dlogits = dW_r = None
    if W_r is not None:
        dlogits = router_bwd(dgates, gates, idx, E, renorm, logits)
        dW_r = dlogits.T @ x
    dx = token_reduce(dxp, meta, T, k, dlogits, W_r)
    return dict(dx=dx, dW13=dW13, dW2=dW2, dgates=dgates, dlogits=dlogits, dW_r=dW_r,
                dy=dy, dh13=dh13, dx_perm=dxp)


# ----------------------------------------------------------------------------------------------
# Expert parallelism across G ranks (row-wise: each routed row lands in the buffer of the rank that
# owns its expert -- unite.ai, "Parallelismo, precisione e tecniche di memoria"). Rank h owns experts
# [h*E/G, (h+1)*E/G). Inside an owner's group for expert e the rows come source rank by source rank,
# each source's rows in its own token order; groups start on ALIGN-row boundaries of the owner's
# buffer, experts in ascending order.
# ----------------------------------------------------------------------------------------------

def ep_layout(all_counts: np.ndarray, world: int, align: int = ALIGN) -> dict:
    """From every rank's per-expert counts all_counts [G, E]: per owner h its local counts and padded
    group starts, and base[g, e] = row in the owner's buffer of source g's first entry for expert e."""
    G, E = all_counts.shape
    EL = E // world
    total = all_counts.sum(axis=0)
    base = np.zeros((G, E), dtype=np.int64)
    counts_loc = np.zeros((world, EL), dtype=np.int64)
    poff_loc = np.zeros((world, EL + 1), dtype=np.int64)
    for h in range(world):
        start = 0
        for el in range(EL):
            e = h * EL + el
            counts_loc[h, el] = total[e]
            poff_loc[h, el] = start
            before = 0
            for g in range(G):
                base[g, e] = start + before
                before += all_counts[g, e]
            start += -(-int(total[e]) // align) * align
        poff_loc[h, EL] = start
    return dict(base=base, counts_loc=counts_loc, poff_loc=poff_loc)


def ep_dst_rows(idx_g: np.ndarray, base_g: np.ndarray, E: int) -> np.ndarray:
    """Row in the owner's buffer of each entry (t, j) of one source rank: the source's base for the
    expert plus the entry's rank among the source's own entries for that expert (token order)."""
    flat = idx_g.reshape(-1)
    seen = np.zeros(E, dtype=np.int64)
    rows = np.empty(flat.size, dtype=np.int64)
    for n, e in enumerate(flat):
        rows[n] = base_g[e] + seen[e]
        seen[e] += 1
    return rows


# ----------------------------------------------------------------------------------------------
# Layer, per-token direct form (no grouping; used to pin the grouped form and for sampled checks)
# ----------------------------------------------------------------------------------------------

def token_out(t, x, W13, W2, idx, gates) -> np.ndarray:
    """out_t = sum_j g_t,j W2_e(silu(W1_e x_t) * W3_e x_t), straight from the definition."""
    F = W13.shape[1] // 2
    acc = np.zeros(x.shape[1])
    for j in range(idx.shape[1]):
        e = int(idx[t, j])
        gate = W13[e, :F] @ x[t]
        up = W13[e, F:] @ x[t]
        acc += gates[t, j] * (W2[e] @ (silu(gate) * up))
    return acc


def token_expert_outputs(t, x, W13, W2, idx) -> np.ndarray:
    """The k expert outputs of token t before gating, y_{S_t,j}(x_t) = W2_e (silu(W1_e x_t) * W3_e
    x_t), one row per slot [k, d]; out_t is their gate-weighted sum and the gate gradient of slot j
    is <dout_t, row j>."""
    F = W13.shape[1] // 2
    ys = np.zeros((idx.shape[1], x.shape[1]))
    for j in range(idx.shape[1]):
        e = int(idx[t, j])
        ys[j] = W2[e] @ (silu(W13[e, :F] @ x[t]) * (W13[e, F:] @ x[t]))
    return ys


def token_dx(t, x, W13, W2, idx, gates, dout, W_r=None, renorm=True) -> np.ndarray:
    """d(loss)/d(x_t) for one token, straight from the definition (router term included when W_r
    is given, renormalised gates assumed)."""
    F = W13.shape[1] // 2
    k = idx.shape[1]
    dx = np.zeros(x.shape[1])
    dg = np.zeros(k)
    for j in range(k):
        e = int(idx[t, j])
        gate = W13[e, :F] @ x[t]
        up = W13[e, F:] @ x[t]
        yj = W2[e] @ (silu(gate) * up)
        dg[j] = dout[t] @ yj
        da = W2[e].T @ (gates[t, j] * dout[t])
        dx += W13[e, :F].T @ (da * up * silu_grad(gate)) + W13[e, F:].T @ (da * silu(gate))
    if W_r is not None:
        assert renorm
        s = float(np.dot(gates[t], dg))
        for j in range(k):
            dx += gates[t, j] * (dg[j] - s) * W_r[int(idx[t, j])]
    return dx


def expert_grads(e, x, W13, W2, idx, gates, dout):
    """dW13_e and dW2_e for one expert from the definition: sum over the (t,j) routed to e."""
    F = W13.shape[1] // 2
    tj = np.argwhere(idx == e)
    dW13 = np.zeros(W13.shape[1:])
    dW2 = np.zeros(W2.shape[1:])
    for t, j in tj:
        gate = W13[e, :F] @ x[t]
        up = W13[e, F:] @ x[t]
        a = silu(gate) * up
        dyv = gates[t, j] * dout[t]
        dW2 += np.outer(dyv, a)
        da = W2[e].T @ dyv
        dW13[:F] += np.outer(da * up * silu_grad(gate), x[t])
        dW13[F:] += np.outer(da * silu(gate), x[t])
    return dW13, dW2


# ----------------------------------------------------------------------------------------------
# MXFP8 per-token forms (sampled checks at full size). Row-wise quantisation of an activation row
# depends on that row only, so the forward and the input gradient of one token follow from the
# token's own rows plus the quantised expert weights:
#   qw[e] = (W13 fake-quantised along d, W2 along F, W13 along 2F, W2 along d)
# ----------------------------------------------------------------------------------------------

def quantised_expert_weights(W13_e, W2_e):
    """The four MXFP8 forms of one expert's weights used by its forward and dgrad GEMMs."""
    return (_mx_row(W13_e), _mx_row(W2_e), _mx_col(W13_e), _mx_col(W2_e))


def token_out_mx(t, x, qw, idx, gates) -> np.ndarray:
    """out_t with every expert GEMM operand MXFP8-quantised along its contraction axis."""
    acc = np.zeros(x.shape[1])
    for j in range(idx.shape[1]):
        e = int(idx[t, j])
        W13r, W2r, _, _ = qw[e]
        h13, a = _token_fwd1_mx(x[t], W13r)
        acc += gates[t, j] * bf16_round(gemm_fwd2(a, W2r, _mx_row))[0]
    return acc


def _token_fwd1_mx(xt, W13r):
    """GEMM1 + SwiGLU of one token with bf16 storage (W13r already quantised along d)."""
    F = W13r.shape[0] // 2
    h13 = bf16_round(_mx_row(xt[None, :]) @ W13r.T)
    return h13, bf16_round(silu(h13[:, :F]) * h13[:, F:])


def token_dx_mx(t, x, qw, idx, gates, dout, W_r=None) -> np.ndarray:
    """d(loss)/d(x_t) for the MXFP8 layer (renormalised gates; router term when W_r is given)."""
    k = idx.shape[1]
    dx = np.zeros(x.shape[1])
    dg = np.zeros(k)
    for j in range(k):
        e = int(idx[t, j])
        W13r, W2r, W13c, W2c = qw[e]
        h13, a = _token_fwd1_mx(x[t], W13r)
        dg[j] = float(dout[t] @ bf16_round(gemm_fwd2(a, W2r, _mx_row))[0])
        dy = bf16_round(gates[t, j] * dout[t][None, :])
        dH13 = bf16_round(gemm_dgrad2_swiglu(dy, W2c, h13, _mx_row, _ident))
        dx += gemm_dgrad1(dH13, W13c, _mx_row, _ident)[0]
    if W_r is not None:
        s = float(np.dot(gates[t], dg))
        for j in range(k):
            dx += gates[t, j] * (dg[j] - s) * W_r[int(idx[t, j])]
    return dx
