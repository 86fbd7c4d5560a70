"""GPU routing parity: top-k indices, counts, offsets, padded offsets and the stable permutation must
be bit-exact with the oracle; gates within fp32 rounding."""
import numpy as np
import pytest
import torch

from oracle import moe as O
from _util import assert_close_rel, dev, idx_from_counts, np64

pytestmark = pytest.mark.gpu


def _lib():
    from mixture_experts_layer_row_b200 import _lib as L
    return L


def _run_topk(logits, k, bias=None, renorm=True):
    L = _lib()
    T, E = logits.shape
    cfg = L.make_config(T, 64, 128, E, k, L.DTYPE_BF16, 1 if renorm else 0)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev())
    idx = torch.full((T, k), -7, dtype=torch.int32, device=dev())
    gates = torch.zeros((T, k), dtype=torch.float32, device=dev())
    L.route_topk(cfg, logits, bias, idx, gates, ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), gates.cpu().numpy(), L.get_error(ws)


def _check_topk(logits_cpu, k, bias=None, renorm=True):
    lg = logits_cpu.to(dev())
    b = bias.to(dev()) if bias is not None else None
    idx, gates, err = _run_topk(lg, k, b, renorm)
    assert err == 0
    eff = (logits_cpu + bias) if bias is not None else logits_cpu  # the fp32 scores the GPU compares
    ref = eff.double().numpy()
    ridx = O.topk_select(ref, k)
    assert np.array_equal(idx, ridx)
    rg = O.gates_for(ref, ridx, renorm)
    np.testing.assert_allclose(gates, rg, rtol=2e-6, atol=1e-7)


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (1000, 8, 2), (777, 128, 4), (513, 256, 8), (300, 5, 3),
                                   (129, 33, 4), (64, 8, 8), (256, 40, 1)])
def test_topk_random(T, E, k):
    g = torch.Generator().manual_seed(T * 31 + E)
    _check_topk(torch.randn((T, E), generator=g), k)


@pytest.mark.parametrize("E,k", [(8, 2), (128, 4), (37, 5)])
def test_topk_ties(E, k):
    g = torch.Generator().manual_seed(E)
    lg = torch.randint(-2, 3, (500, E), generator=g).float()  # heavy ties
    lg[0] = 0.0
    lg[1, ::2] = -0.0  # signed zeros compare equal
    _check_topk(lg, k)


def test_topk_bias_and_no_renorm():
    g = torch.Generator().manual_seed(5)
    lg = torch.randn((400, 128), generator=g)
    bias = (1.2 * torch.log(1.0 / torch.arange(1, 129, dtype=torch.float64))).float()
    _check_topk(lg, 4, bias)
    _check_topk(lg, 4, None, renorm=False)


def test_topk_nonfinite_flag():
    lg = torch.randn((64, 16))
    lg[3, 5] = float("nan")
    lg[7, 2] = float("inf")
    _, _, err = _run_topk(lg.to(dev()), 2)
    assert err & _lib().DEVERR_NONFINITE


def _run_metadata(idx_np, E):
    L = _lib()
    T, k = idx_np.shape
    cfg = L.make_config(T, 64, 128, E, k)
    R = L.max_rows(cfg)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev())
    z = lambda n: torch.full((n,), -99, dtype=torch.int32, device=dev())
    counts, offsets, poff = z(E), z(E + 1), z(E + 1)
    perm, prow, row_token = z(T * k), z(T * k), z(R)
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).to(dev())
    L.route_metadata(cfg, idx, counts, offsets, poff, perm, prow, row_token, ws)
    torch.cuda.synchronize()
    out = {n: t.cpu().numpy().astype(np.int64) for n, t in
           dict(counts=counts, offsets=offsets, poff=poff, perm=perm, prow=prow,
                row_token=row_token).items()}
    return out, R, L.get_error(ws)


def _check_metadata(idx_np, E):
    got, R, err = _run_metadata(idx_np, E)
    assert err == 0
    ref = O.route_metadata(idx_np.astype(np.int64), E)
    for key in ("counts", "offsets", "poff", "perm", "prow"):
        assert np.array_equal(got[key], ref[key]), key
    used = int(ref["poff"][E])
    assert np.array_equal(got["row_token"][:used], ref["row_token"])
    assert np.all(got["row_token"][used:] == -1)


def _uniform_idx(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.argsort(rng.random((T, E)), axis=1)[:, :k]


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (1, 8, 8), (7, 5, 2), (255, 8, 2), (256, 8, 2),
                                   (257, 16, 3), (1000, 128, 4), (8192, 128, 4), (16384, 128, 4),
                                   (3000, 256, 8), (8192, 8, 4)])
def test_metadata_uniform(T, E, k):
    _check_metadata(_uniform_idx(T, E, k, T + E), E)


@pytest.mark.parametrize("counts_kind", ["one_hot", "ragged", "empty_experts"])
def test_metadata_skewed(counts_kind):
    rng = np.random.default_rng(11)
    T, k = 700, 2
    if counts_kind == "one_hot":
        E = 8
        idx = np.stack([np.zeros(T, np.int32), rng.integers(1, E, T).astype(np.int32)], 1)
    elif counts_kind == "ragged":
        E = 16
        counts = [0, 1, 31, 32, 33, 127, 128, 129, 300, 300, 100, 50, 50, 50, 36, 33]
        assert sum(counts) == T * k
        idx = idx_from_counts(counts, T, k, rng)
    else:
        E = 64
        idx = _uniform_idx(T, 10, k, 3) * 6  # experts 0, 6, 12, ... only
    _check_metadata(idx.astype(np.int32), E)


def test_metadata_zipf_like_router():
    """The skewed workload's routing: learned-router scores plus a 1.2*ln(1/rank) bias."""
    from moe_workloads import skew_bias
    g = torch.Generator().manual_seed(0)
    T, E, k, d = 4096, 128, 4, 256
    x = torch.randn((T, d), generator=g).bfloat16().double()
    Wr = (torch.randn((E, d), generator=g) * 0.02).bfloat16().double()
    lg = (x @ Wr.T).float() + skew_bias(E, 1.2)
    idx = O.topk_select(lg.double().numpy(), k)
    _check_metadata(idx.astype(np.int32), E)


def test_metadata_invalid_ids_flagged():
    L = _lib()
    idx = _uniform_idx(300, 8, 2, 1).astype(np.int32)
    idx[5, 0] = 8
    idx[9, 1] = -3
    got, R, err = _run_metadata(idx, 8)
    assert err & L.DEVERR_ROUTING
    # the valid entries still form a stable, in-range permutation of their own
    valid = (idx >= 0) & (idx < 8)
    pr = got["prow"].reshape(idx.shape)[valid]
    assert np.all((pr >= 0) & (pr < R)) and len(np.unique(pr)) == pr.size
    # the invalid entries have no row: perm and prow are -1 there (not a stale value)
    assert np.all(got["prow"].reshape(idx.shape)[~valid] == -1)
    assert np.all(got["perm"].reshape(idx.shape)[~valid] == -1)
    assert np.array_equal(got["counts"], np.bincount(idx[valid], minlength=8))


def test_row_kernels_skip_entries_without_a_row():
    """An entry with an invalid expert id gets prow = -1; dispatch, combine, combine_bwd and the token
    reduce skip it (no read or write through it) and treat the rest of the token as usual."""
    L = _lib()
    T, d, E, k = 64, 64, 8, 2
    idx = _uniform_idx(T, E, k, 3).astype(np.int32)
    idx[4, 1] = E + 3
    idx[17, 0] = -1
    valid = (idx >= 0) & (idx < E)
    cfg = L.make_config(T, d, 128, E, k)
    R = L.max_rows(cfg)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev())
    z = lambda n: torch.full((n,), -99, dtype=torch.int32, device=dev())
    counts, offsets, poff = z(E), z(E + 1), z(E + 1)
    perm, prow, row_token = z(T * k), z(T * k), z(R)
    tidx = torch.from_numpy(idx).to(dev())
    L.route_metadata(cfg, tidx, counts, offsets, poff, perm, prow, row_token, ws)
    g = torch.Generator(device=dev()).manual_seed(5)
    x = torch.randn((T, d), generator=g, device=dev()).to(torch.bfloat16)
    gates = torch.rand((T, k), generator=g, device=dev())
    xp = torch.full((R, d), 7.0, dtype=torch.bfloat16, device=dev())
    L.dispatch(cfg, x, prow, counts, poff, xp)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=dev())
    L.combine(cfg, xp, gates, prow, out)
    dy = torch.full((R, d), 7.0, dtype=torch.bfloat16, device=dev())
    dg = torch.full((T, k), 5.0, device=dev())
    L.combine_bwd(cfg, x, xp, gates, prow, tidx, counts, poff, dy, dg)
    dx = torch.empty((T, d), dtype=torch.bfloat16, device=dev())
    L.token_reduce(cfg, xp, prow, dx)
    torch.cuda.synchronize()
    assert L.get_error(ws) & L.DEVERR_ROUTING
    pr = prow.cpu().numpy().reshape(T, k)
    assert np.all(pr[~valid] == -1)
    x64, g64 = np64(x), gates.cpu().double().numpy()
    w = np.where(valid, g64, 0.0)
    assert_close_rel(np64(out), w.sum(1)[:, None] * x64, 1e-2, "combine")
    assert_close_rel(np64(dx), valid.sum(1)[:, None] * x64, 1e-2, "token reduce")
    dgn = dg.cpu().numpy()
    assert np.all(dgn[~valid] == 0.0)  # no row: nothing to contract with
    used = int(poff[E])
    xpn = np64(xp)
    assert np.all(xpn[used:] == 7.0)  # rows past the groups untouched
