"""Whole-layer parity (moe_layer_fwd + moe_layer_bwd through the C ABI) against the fp64 oracle.

Small cases: every output compared element by element with the full grouped oracle.
Full-size workloads (the shapes the benchmark times, in the same launch configuration): routing and
metadata compared in full (bit-exact), outputs and gradients on sampled tokens and experts, each
computed by the oracle from its definition.
"""
import numpy as np
import pytest
import torch

from moe_workloads import WORKLOADS, Workload, make_inputs
from oracle import moe as O
from _util import TOL_BF16, assert_close_rel, dev, np64

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": WORKLOADS["tiny"],
    "e8_learned_small": Workload("e8_learned_small", 512, 256, 256, 8, 4, "bf16", "learned"),
    "e32_uniform_small": Workload("e32_uniform_small", 1024, 256, 256, 32, 4, "bf16", "uniform"),
    "e32_skew_small": Workload("e32_skew_small", 1024, 256, 384, 32, 4, "bf16", "learned", skew=1.2),
    "e128_uniform_ragged": Workload("e128_uniform_ragged", 333, 128, 128, 128, 4, "bf16", "uniform"),
}


def run_layer(w: Workload, inp: dict):
    from mixture_experts_layer_row_b200 import MoELayer
    learned = w.routing == "learned"
    layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=learned)
    layer.set_weights(inp["W13"], inp["W2"], inp["W_r"] if learned else None)
    out = layer.forward(inp["x"], bias=inp["bias"], idx=inp["idx"], gates=inp["gates"])
    layer.backward(inp["dout"])
    torch.cuda.synchronize()
    assert layer.error_flags() == 0
    return layer, out


def _routing_checks(w, layer, inp, x64, Wr64):
    """Bit-exact routing on the GPU's own fp32 scores, scores close to fp64, metadata bit-exact.
    Returns (idx, gates_ref) for the output checks."""
    if w.routing == "learned":
        lg = layer.logits.cpu()  # bias already included
        ref_l = O.router_logits(x64, Wr64, None if inp["bias"] is None else np64(inp["bias"]))
        assert_close_rel(lg.double().numpy(), ref_l, 1e-2, "router scores")
        idx = layer.idx.cpu().numpy().astype(np.int64)
        assert np.array_equal(idx, O.topk_select(lg.double().numpy(), w.k)), "top-k not bit-exact"
        np.testing.assert_allclose(layer.gates.cpu().numpy(),
                                   O.gates_for(lg.double().numpy(), idx, w.renorm), rtol=2e-6,
                                   atol=1e-7)
        gates_ref = O.gates_for(ref_l, idx, w.renorm)  # the oracle's gates on the chosen experts
    else:
        idx = inp["idx"].cpu().numpy().astype(np.int64)
        gates_ref = np64(inp["gates"])
    meta = O.route_metadata(idx, w.E, 128 if w.dtype == "mxfp8" else 32)  # MXFP8 groups: 128 rows
    for key in ("counts", "offsets", "poff", "perm", "prow"):
        assert np.array_equal(getattr(layer, key).cpu().numpy(), meta[key]), key
    used = int(meta["poff"][-1])
    assert np.array_equal(layer.row_token[:used].cpu().numpy(), meta["row_token"])
    return idx, gates_ref


@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small_full_oracle(name):
    w = SMALL[name]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    x64, W13, W2, Wr, dout = (np64(inp[n]) for n in ("x", "W13", "W2", "W_r", "dout"))
    learned = w.routing == "learned"
    idx, gates_ref = _routing_checks(w, layer, inp, x64, Wr)
    ref_out, saved = O.layer_fwd(x64, W13, W2, idx, gates_ref)
    assert_close_rel(np64(out), ref_out, TOL_BF16, "out")
    gr = O.layer_bwd(dout, x64, W13, W2, idx, gates_ref, saved, W_r=Wr if learned else None)
    assert_close_rel(np64(layer.dx), gr["dx"], TOL_BF16, "dx")
    assert_close_rel(np64(layer.dW13), gr["dW13"], TOL_BF16, "dW13")
    assert_close_rel(np64(layer.dW2), gr["dW2"], TOL_BF16, "dW2")
    assert_close_rel(layer.dgates.cpu().numpy(), gr["dgates"], TOL_BF16, "dgates")
    if learned:
        assert_close_rel(np64(layer.dW_r), gr["dW_r"], TOL_BF16, "dW_r")


def _sampled_full_size(w: Workload, n_tok=24, n_exp=2):
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    learned = w.routing == "learned"
    x64 = np64(inp["x"])
    Wr = np64(inp["W_r"])
    idx, gates_ref = _routing_checks(w, layer, inp, x64, Wr)
    dout = np64(inp["dout"])
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([[0, w.T - 1], rng.integers(0, w.T, n_tok)]))
    counts = np.bincount(idx.reshape(-1), minlength=w.E)
    exps = sorted({int(np.argmax(counts)), int(rng.integers(0, w.E))} |
                  ({int(np.argmin(counts))} if n_exp > 2 else set()))
    need = sorted(set(idx[toks].reshape(-1).tolist()) | set(exps))
    W13 = {e: np64(inp["W13"][e]) for e in need}
    W2 = {e: np64(inp["W2"][e]) for e in need}

    class _Stack:  # index W13[e] / W2[e] for the experts fetched
        def __init__(self, d, shape):
            self.d, self.shape = d, shape

        def __getitem__(self, key):
            if isinstance(key, tuple):
                return self.d[int(key[0])][key[1:]]
            return self.d[int(key)]

    F2, d = 2 * w.F, w.d
    W13s, W2s = _Stack(W13, (w.E, F2, d)), _Stack(W2, (w.E, d, w.F))
    got_out, got_dx = np64(out[toks]), np64(layer.dx[toks])
    ref_out = np.stack([O.token_out(t, x64, W13s, W2s, idx, gates_ref) for t in toks])
    assert_close_rel(got_out, ref_out, TOL_BF16, "sampled out")
    ref_dx = np.stack([O.token_dx(t, x64, W13s, W2s, idx, gates_ref, dout,
                                  Wr if learned else None) for t in toks])
    assert_close_rel(got_dx, ref_dx, TOL_BF16, "sampled dx")
    for e in exps:
        tj = np.argwhere(idx == e)
        X = x64[tj[:, 0]]
        dY = gates_ref[tj[:, 0], tj[:, 1]][:, None] * dout[tj[:, 0]]
        if len(tj):
            h13, a, _ = O.expert_fwd(X, W13[e], W2[e])
            _, dW13, dW2, _ = O.expert_bwd(X, W13[e], W2[e], h13, a, dY)
        else:
            dW13, dW2 = np.zeros((F2, d)), np.zeros((d, w.F))
        g13, g2 = np64(layer.dW13[e]), np64(layer.dW2[e])
        if len(tj):
            assert_close_rel(g13, dW13, TOL_BF16, f"dW13[{e}]")
            assert_close_rel(g2, dW2, TOL_BF16, f"dW2[{e}]")
        else:
            assert np.all(g13 == 0) and np.all(g2 == 0)
    if learned:
        # the router weight gradient at full size (its contraction over T is split into token
        # chunks on the GPU): dW_r = dlogits^T x, with dlogits from the GPU's gate gradients by the
        # oracle's router backward
        dl = O.router_bwd(layer.dgates.cpu().double().numpy(), gates_ref, idx, w.E)
        assert_close_rel(np64(layer.dW_r), dl.T @ x64, TOL_BF16, "dW_r")
    return layer


@pytest.mark.parametrize("name", ["e8_bf16", "e128_bf16", "e128_skew"])
def test_layer_full_size_sampled(name):
    _sampled_full_size(WORKLOADS[name], n_exp=3 if name == "e128_skew" else 2)


def test_layer_back_to_back_matches_isolated_runs():
    """Kernels are launched with programmatic dependent launch (each may start while its predecessor
    finishes and waits for it before touching memory). Many layer steps issued back to back, with
    two alternating inputs and no host synchronisation, must give bit-identical results to steps run
    one at a time."""
    from mixture_experts_layer_row_b200 import MoELayer
    w = SMALL["e8_learned_small"]
    inA = make_inputs(w, seed=5, device="cuda")
    inB = make_inputs(w, seed=6, device="cuda")
    layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=True)
    layer.set_weights(inA["W13"], inA["W2"], inA["W_r"])

    def step(inp):
        layer.forward(inp["x"], bias=inp["bias"])
        layer.backward(inp["dout"])

    def snap():
        return [t.clone() for t in (layer.out, layer.dx, layer.dW13, layer.dW2, layer.dW_r, layer.dgates)]

    step(inA); torch.cuda.synchronize(); refA = snap()
    step(inB); torch.cuda.synchronize(); refB = snap()
    for _ in range(8):
        step(inA)
        step(inB)
    torch.cuda.synchronize()
    for got, ref in zip(snap(), refB):
        assert torch.equal(got, ref)
    step(inA)
    torch.cuda.synchronize()
    for got, ref in zip(snap(), refA):
        assert torch.equal(got, ref)
    assert layer.error_flags() == 0


@pytest.mark.parametrize("name", ["e8_learned_small", "e128_uniform_ragged", "e32_skew_small"])
@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_layer_recompute_matches_stored_activations(name, dtype):
    """With activation recompute the forward keeps no h13 and the backward regenerates it with the
    same GEMM1 kernel; every output and gradient must equal the stored-activation layer's bit for
    bit."""
    from mixture_experts_layer_row_b200 import MoELayer
    w = SMALL[name]
    w = Workload(w.name, w.T, w.d, w.F, w.E, w.k, dtype, w.routing, skew=w.skew)
    inp = make_inputs(w, seed=11, device="cuda")
    learned = w.routing == "learned"
    res = []
    for rc in (False, True):
        layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=dtype, learned_router=learned, recompute=rc)
        assert (layer.h13 is None) == rc
        layer.set_weights(inp["W13"], inp["W2"], inp["W_r"] if learned else None)
        layer.forward(inp["x"], bias=inp["bias"], idx=inp["idx"], gates=inp["gates"])
        if rc:
            layer.a.fill_(7.0)  # the forward's a is not needed by the backward's recompute path
        layer.backward(inp["dout"])
        torch.cuda.synchronize()
        assert layer.error_flags() == 0
        ts = [layer.out, layer.dx, layer.dW13, layer.dW2, layer.dgates]
        if learned:
            ts.append(layer.dW_r)
        res.append([t.clone() for t in ts])
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_layer_twice_is_deterministic():
    w = SMALL["e32_uniform_small"]
    inp = make_inputs(w, seed=3, device="cuda")
    l1, o1 = run_layer(w, inp)
    o1, dx1, dw1 = o1.clone(), l1.dx.clone(), l1.dW13.clone()
    l2, o2 = run_layer(w, inp)
    assert torch.equal(o1, o2) and torch.equal(dx1, l2.dx) and torch.equal(dw1, l2.dW13)


# ------------------------------------------------------------------------------------------------
# MXFP8 layer: against the oracle with the same quantisation (OCP MX along every GEMM's contraction
# axis); the tolerance is the MXFP8 bar, 8e-2 * max|ref|. The distance to the unquantised fp64 layer
# is printed for the record (E4M3 itself carries several percent).
# ------------------------------------------------------------------------------------------------

TOL_MX = 8e-2
MX_SMALL = {
    "mx_uniform": Workload("mx_uniform", 512, 256, 256, 16, 4, "mxfp8", "uniform"),
    "mx_learned": Workload("mx_learned", 384, 256, 384, 8, 2, "mxfp8", "learned"),
}


@pytest.mark.parametrize("name", list(MX_SMALL))
def test_layer_mxfp8_small_full_oracle(name):
    w = MX_SMALL[name]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    x64, W13, W2, Wr, dout = (np64(inp[n]) for n in ("x", "W13", "W2", "W_r", "dout"))
    learned = w.routing == "learned"
    idx, gates_ref = _routing_checks(w, layer, inp, x64, Wr)
    ref_out, saved = O.layer_fwd(x64, W13, W2, idx, gates_ref, mx=True)
    gr = O.layer_bwd(dout, x64, W13, W2, idx, gates_ref, saved, W_r=Wr if learned else None, mx=True)
    errs = {"out": assert_close_rel(np64(out), ref_out, TOL_MX, "out"),
            "dx": assert_close_rel(np64(layer.dx), gr["dx"], TOL_MX, "dx"),
            "dW13": assert_close_rel(np64(layer.dW13), gr["dW13"], TOL_MX, "dW13"),
            "dW2": assert_close_rel(np64(layer.dW2), gr["dW2"], TOL_MX, "dW2")}
    if learned:
        errs["dW_r"] = assert_close_rel(np64(layer.dW_r), gr["dW_r"], TOL_MX, "dW_r")
    plain_out, _ = O.layer_fwd(x64, W13, W2, idx, gates_ref)
    print(name, "rel err vs MXFP8 oracle", {k: round(v, 5) for k, v in errs.items()},
          "| out vs unquantised fp64:",
          round(float(np.max(np.abs(np64(out) - plain_out)) / np.max(np.abs(plain_out))), 4))


def test_layer_mxfp8_full_size_sampled():
    w = WORKLOADS["e128_mxfp8"]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    x64 = np64(inp["x"])
    idx, gates_ref = _routing_checks(w, layer, inp, x64, None)
    dout = np64(inp["dout"])
    rng = np.random.default_rng(2)
    toks = [0, w.T - 1] + [int(t) for t in rng.integers(0, w.T, 4)]
    got_out, got_dx, ref_out, ref_dx = [], [], [], []
    for t in toks:  # quantised weights of the token's experts only, built per token
        qw = {int(e): O.quantised_expert_weights(np64(inp["W13"][int(e)]), np64(inp["W2"][int(e)]))
              for e in idx[t]}
        ref_out.append(O.token_out_mx(t, x64, qw, idx, gates_ref))
        ref_dx.append(O.token_dx_mx(t, x64, qw, idx, gates_ref, dout))
        got_out.append(np64(out[t]))
        got_dx.append(np64(layer.dx[t]))
    assert_close_rel(np.stack(got_out), np.stack(ref_out), TOL_MX, "sampled out")
    assert_close_rel(np.stack(got_dx), np.stack(ref_dx), TOL_MX, "sampled dx")
    counts = np.bincount(idx.reshape(-1), minlength=w.E)
    for e in sorted({int(np.argmax(counts)), int(rng.integers(0, w.E))}):
        tj = np.argwhere(idx == e)
        X = x64[tj[:, 0]]
        dY = O.bf16_round(gates_ref[tj[:, 0], tj[:, 1]][:, None] * dout[tj[:, 0]])  # stored bf16
        W13e, W2e = np64(inp["W13"][e]), np64(inp["W2"][e])
        h13, a, _ = O.expert_fwd(X, W13e, W2e, mx=True)
        _, dW13, dW2, _ = O.expert_bwd(X, W13e, W2e, h13, a, dY, mx=True)
        assert_close_rel(np64(layer.dW13[e]), dW13, TOL_MX, f"dW13[{e}]")
        assert_close_rel(np64(layer.dW2[e]), dW2, TOL_MX, f"dW2[{e}]")
