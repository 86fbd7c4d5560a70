"""Whole-layer parity (moe_layer_fwd + moe_layer_bwd through the C ABI) against the fp64 oracle.

Small cases: every output compared element by element with the full grouped oracle.
Full-size workloads (the shapes the benchmark times, in the same launch configuration): routing and
metadata compared in full (bit-exact), outputs and gradients on sampled tokens and experts, each
computed by the oracle from its definition.
"""
import os

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


def run_layer(w: Workload, inp: dict, recompute: bool = False):
    from mixture_experts_layer_row_b200 import MoELayer
    learned = w.routing == "learned"
    layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=learned,
                     recompute=recompute)
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


@pytest.mark.parametrize("recompute", [False, True], ids=["stored", "recompute"])
@pytest.mark.parametrize("name", list(SMALL))
def test_layer_small_full_oracle(name, recompute):
    """Every output and gradient against the fp64 oracle. With recompute the forward keeps no h13 and
    the backward regenerates it (activation recompute); the oracle is the same exact layer."""
    w = SMALL[name]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp, recompute=recompute)
    assert (layer.h13 is None) == recompute
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
    # gate gradients of the sampled tokens: <dout_t, y_e(x_t)> for each chosen expert
    ref_dg = np.stack([O.token_expert_outputs(t, x64, W13s, W2s, idx) @ dout[t] for t in toks])
    assert_close_rel(layer.dgates.cpu().double().numpy()[toks], ref_dg, TOL_BF16, "sampled dgates")
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
        # chunks on the GPU), entirely from the oracle: the grouped fp64 forward gives every token's
        # expert outputs, its combine backward the gate gradients, its router backward the score
        # gradients, and dW_r = dlogits^T x
        W13a, W2a = np64(inp["W13"]), np64(inp["W2"])
        _, saved = O.layer_fwd(x64, W13a, W2a, idx, gates_ref)
        _, dg_all = O.combine_bwd(dout, saved["y"], gates_ref, saved["meta"])
        del saved, W13a, W2a
        assert_close_rel(layer.dgates.cpu().double().numpy(), dg_all, TOL_BF16, "dgates (all tokens)")
        dl = O.router_bwd(dg_all, gates_ref, idx, w.E)
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


def test_layer_caller_output_buffers():
    """forward(out=...) / backward(dx=...) write the same bits into the caller's buffers as into the
    layer's own, and leave the layer's own untouched."""
    from mixture_experts_layer_row_b200 import MoELayer
    w = SMALL["e32_uniform_small"]
    inp = make_inputs(w, seed=5, device="cuda")
    layer = MoELayer(w.T, w.d, w.F, w.E, w.k, dtype=w.dtype, learned_router=w.routing == "learned")
    layer.set_weights(inp["W13"], inp["W2"], inp["W_r"] if w.routing == "learned" else None)
    kw = {} if w.routing == "learned" else {"idx": inp["idx"], "gates": inp["gates"]}
    o_ref = layer.forward(inp["x"], bias=inp["bias"], **kw).clone()
    dx_ref = layer.backward(inp["dout"]).clone()
    layer.out.zero_()
    layer.dx.zero_()
    out, dx = torch.full_like(o_ref, 7.0), torch.full_like(dx_ref, 7.0)
    assert layer.forward(inp["x"], bias=inp["bias"], out=out, **kw) is out
    assert layer.backward(inp["dout"], dx=dx) is dx
    torch.cuda.synchronize()
    assert torch.equal(out, o_ref) and torch.equal(dx, dx_ref)
    assert not layer.out.any() and not layer.dx.any()
    assert layer.error_flags() == 0


# ------------------------------------------------------------------------------------------------
# MXFP8 layer. Three comparisons:
#  - against the oracle with the same quantisation (OCP MX along every GEMM's contraction axis, bf16
#    storage of every GEMM output): what the kernels compute, to bf16-output rounding (2e-2);
#  - against the unquantised fp64 layer, at the MXFP8 bar of 8e-2 * max|ref| wherever an exact MXFP8
#    layer meets it. Where the format itself is further away (the emulated oracle's own distance is
#    above the bar: the weight gradients, whose blocks span 32 unrelated tokens), the GPU result must
#    be no further than that distance plus bf16 rounding, and the distance is printed;
#  - against the bf16 layer run on the same inputs, with the bf16 layer's own 2e-2 added.
# ------------------------------------------------------------------------------------------------

TOL_MX_EMU = 2e-2  # vs the emulated MXFP8 oracle
TOL_MX = 8e-2      # vs the unquantised fp64 layer
MX_SMALL = {
    "mx_uniform": Workload("mx_uniform", 512, 256, 256, 16, 4, "mxfp8", "uniform"),
    "mx_learned": Workload("mx_learned", 384, 256, 384, 8, 2, "mxfp8", "learned"),
}


def _rel(got, ref):
    return float(np.max(np.abs(np.asarray(got) - np.asarray(ref))) / np.max(np.abs(ref)))


def _unquantised_bar(name, got, emu, plain, extra=0.0):
    """The 8e-2 bar against the unquantised layer where the format meets it, else the format's own
    distance (the emulated oracle's) plus bf16 rounding. `extra` widens it for a reference that itself
    carries error (the bf16 layer). Returns (GPU distance, format distance)."""
    gap_fmt, gap_gpu = _rel(emu, plain), _rel(got, plain)
    bar = (TOL_MX if gap_fmt <= TOL_MX else gap_fmt + TOL_MX_EMU) + extra
    assert gap_gpu <= bar, f"{name}: {gap_gpu:.4f} from the unquantised reference > {bar:.4f} (format: {gap_fmt:.4f})"
    return gap_gpu, gap_fmt


@pytest.mark.parametrize("name", list(MX_SMALL))
def test_layer_mxfp8_small_full_oracle(name):
    w = MX_SMALL[name]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    x64, W13, W2, Wr, dout = (np64(inp[n]) for n in ("x", "W13", "W2", "W_r", "dout"))
    learned = w.routing == "learned"
    idx, gates_ref = _routing_checks(w, layer, inp, x64, Wr)
    ref_out, saved = O.layer_fwd(x64, W13, W2, idx, gates_ref, align=128, mx=True)
    gr = O.layer_bwd(dout, x64, W13, W2, idx, gates_ref, saved, W_r=Wr if learned else None, mx=True)
    plain_out, sv_plain = O.layer_fwd(x64, W13, W2, idx, gates_ref, align=128)
    gp = O.layer_bwd(dout, x64, W13, W2, idx, gates_ref, sv_plain, W_r=Wr if learned else None)
    got = {"out": np64(out), "dx": np64(layer.dx), "dW13": np64(layer.dW13), "dW2": np64(layer.dW2),
           "dgates": layer.dgates.cpu().double().numpy()}
    emu = {"out": ref_out, **{k: gr[k] for k in ("dx", "dW13", "dW2", "dgates")}}
    plain = {"out": plain_out, **{k: gp[k] for k in ("dx", "dW13", "dW2", "dgates")}}
    if learned:
        got["dW_r"], emu["dW_r"], plain["dW_r"] = np64(layer.dW_r), gr["dW_r"], gp["dW_r"]
    # the same layer in bf16 on the same inputs (same routing: the MXFP8 layer's router is bf16)
    wb = Workload(w.name + "_bf16", w.T, w.d, w.F, w.E, w.k, "bf16", w.routing, skew=w.skew)
    lb, outb = run_layer(wb, inp)
    assert torch.equal(lb.idx, layer.idx)
    bf = {"out": np64(outb), "dx": np64(lb.dx), "dW13": np64(lb.dW13), "dW2": np64(lb.dW2),
          "dgates": lb.dgates.cpu().double().numpy()}
    if learned:
        bf["dW_r"] = np64(lb.dW_r)
    rec = {}
    for key in got:
        e_emu = assert_close_rel(got[key], emu[key], TOL_MX_EMU, key)
        g_unq, g_fmt = _unquantised_bar(key, got[key], emu[key], plain[key])
        g_bf, _ = _unquantised_bar(key + " vs bf16 layer", got[key], emu[key], bf[key], TOL_BF16)
        rec[key] = (round(e_emu, 4), round(g_unq, 4), round(g_fmt, 4), round(g_bf, 4))
    print(name, "max-rel distance: (emulated oracle, unquantised, format's own, bf16 layer)", rec)


def _tokens_within_few_experts(idx, need, seed_experts):
    """Greedy: `need` tokens whose experts add as few new experts as possible to the set (so the
    per-token MXFP8 checks quantise few expert weight sets)."""
    S, chosen = set(seed_experts), []
    sets = [frozenset(r) for r in idx.tolist()]
    while len(chosen) < need:
        best, bn = None, 99
        for t, st in enumerate(sets):
            if t in chosen:
                continue
            n = len(st - S)
            if n < bn:
                best, bn = t, n
                if n == 0:
                    break
        chosen.append(best)
        S |= sets[best]
    return sorted(chosen), sorted(S)


def test_layer_mxfp8_full_size_sampled():
    """e128_mxfp8 at full size: 24+ tokens (output and input gradient, and their gate gradients)
    against the emulated oracle's per-token forms, and the weight gradients of three experts (the
    largest group, the smallest, and one more) against the emulated per-expert oracle; the
    unquantised fp64 forms with the bar as for the small cases."""
    import multiprocessing as mp
    w = WORKLOADS["e128_mxfp8"]
    inp = make_inputs(w, seed=0, device="cuda")
    layer, out = run_layer(w, inp)
    x64 = np64(inp["x"])
    idx, gates_ref = _routing_checks(w, layer, inp, x64, None)
    dout = np64(inp["dout"])
    rng = np.random.default_rng(2)
    counts = np.bincount(idx.reshape(-1), minlength=w.E)
    exps = sorted({int(np.argmax(counts)), int(np.argmin(counts)), int(rng.integers(0, w.E))})
    toks, need = _tokens_within_few_experts(idx, 24, exps)
    toks = sorted(set(toks) | {0} | {w.T - 1})
    need = sorted(set(need) | set(idx[0].tolist()) | set(idx[w.T - 1].tolist()))
    W13 = {e: np64(inp["W13"][e]) for e in need}
    W2 = {e: np64(inp["W2"][e]) for e in need}
    # the four MXFP8 forms of each needed expert's weights, one oracle call per expert in worker
    # processes (spawned: this process already holds a CUDA context)
    with mp.get_context("spawn").Pool(min(len(need), os.cpu_count() or 1)) as pool:
        forms = pool.starmap(O.quantised_expert_weights, [(W13[e], W2[e]) for e in need])
    qw = dict(zip(need, forms))

    class _Stack:  # index W13[e] / W2[e] for the experts fetched
        def __init__(self, d, shape):
            self.d, self.shape = d, shape

        def __getitem__(self, key):
            if isinstance(key, tuple):
                return self.d[int(key[0])][key[1:]]
            return self.d[int(key)]

    W13s, W2s = _Stack(W13, (w.E, 2 * w.F, w.d)), _Stack(W2, (w.E, w.d, w.F))
    got_out, got_dx = np64(out[toks]), np64(layer.dx[toks])
    ref_out = np.stack([O.token_out_mx(t, x64, qw, idx, gates_ref) for t in toks])
    ref_dx = np.stack([O.token_dx_mx(t, x64, qw, idx, gates_ref, dout) for t in toks])
    plain_out = np.stack([O.token_out(t, x64, W13s, W2s, idx, gates_ref) for t in toks])
    plain_dx = np.stack([O.token_dx(t, x64, W13s, W2s, idx, gates_ref, dout) for t in toks])
    rec = {"out": assert_close_rel(got_out, ref_out, TOL_MX_EMU, "sampled out"),
           "dx": assert_close_rel(got_dx, ref_dx, TOL_MX_EMU, "sampled dx")}
    unq = {"out": _unquantised_bar("sampled out", got_out, ref_out, plain_out),
           "dx": _unquantised_bar("sampled dx", got_dx, ref_dx, plain_dx)}
    for e in exps:
        tj = np.argwhere(idx == e)
        X = x64[tj[:, 0]]
        dY = O.bf16_round(gates_ref[tj[:, 0], tj[:, 1]][:, None] * dout[tj[:, 0]])  # stored bf16
        h13, a, _ = O.expert_fwd(X, W13[e], W2[e], mx=True)
        _, dW13, dW2, _ = O.expert_bwd(X, W13[e], W2[e], h13, a, dY, mx=True)
        ph13, pa, _ = O.expert_fwd(X, W13[e], W2[e])
        _, pW13, pW2, _ = O.expert_bwd(X, W13[e], W2[e], ph13, pa, dY)
        g13, g2 = np64(layer.dW13[e]), np64(layer.dW2[e])
        rec[f"dW13[{e}]"] = assert_close_rel(g13, dW13, TOL_MX_EMU, f"dW13[{e}]")
        rec[f"dW2[{e}]"] = assert_close_rel(g2, dW2, TOL_MX_EMU, f"dW2[{e}]")
        unq[f"dW13[{e}]"] = _unquantised_bar(f"dW13[{e}]", g13, dW13, pW13)
        unq[f"dW2[{e}]"] = _unquantised_bar(f"dW2[{e}]", g2, dW2, pW2)
    print(f"{len(toks)} tokens, experts {exps} (rows {[int(counts[e]) for e in exps]});",
          "vs emulated:", {k: round(v, 4) for k, v in rec.items()},
          "| vs unquantised (GPU, format):", {k: tuple(round(x, 4) for x in v) for k, v in unq.items()})
