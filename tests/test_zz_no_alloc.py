"""The allocation-free routing-metadata entry point (for callers that cannot allocate device memory
and so cannot pass a workspace) must produce exactly what moe_route_metadata produces, call after call,
although every call reuses the library's one static scratch array. Runs last: it touches state that
lives as long as the process."""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _outputs(L, cfg, dev):
    T, k, E = cfg.T, cfg.k, cfg.E
    z = lambda n: torch.full((n,), -5, dtype=torch.int32, device=dev)
    return dict(counts=z(E), offsets=z(E + 1), poff=z(E + 1), perm=z(T * k), prow=z(T * k),
                row_token=z(L.max_rows(cfg)))


def _idx(T, E, k, seed, skew=False):
    rng = np.random.default_rng(seed)
    u = rng.random((T, E))
    if skew:  # uneven loads, some experts empty
        u = u * np.exp(-np.arange(E) / 8.0)[None, :] ** -1
    return np.ascontiguousarray(np.argsort(u, axis=1)[:, :k].astype(np.int32))


@pytest.mark.parametrize("T,E,k", [(8192, 128, 4), (333, 8, 2)])
def test_noalloc_matches_workspace_entry_point_twice(T, E, k):
    from mixture_experts_layer_row_b200 import _lib as L
    dev = torch.device("cuda", 0)
    cfg = L.make_config(T, 64, 128, E, k)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev)
    for call, skew in enumerate((False, True)):  # two calls in a row, different routings
        idx = torch.from_numpy(_idx(T, E, k, 100 + call, skew)).to(dev)
        ref = _outputs(L, cfg, dev)
        L.route_metadata(cfg, idx, ref["counts"], ref["offsets"], ref["poff"], ref["perm"],
                         ref["prow"], ref["row_token"], ws)
        got = _outputs(L, cfg, dev)
        L.route_metadata_noalloc(cfg, idx, got["counts"], got["offsets"], got["poff"], got["perm"],
                                 got["prow"], got["row_token"])
        torch.cuda.synchronize()
        for name in ref:
            assert torch.equal(got[name], ref[name]), (call, name)  # integer outputs: bit-exact
        assert int(got["offsets"][E]) == T * k


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from mixture_experts_layer_row_b200 import _lib as L
    cfg = L.make_config(256 * 513, 64, 128, 128, 1)  # ceil(T/256) * E = 65664 > 65536
    fake = 1 << 20
    rc = L.lib.moe_route_metadata_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake,
                                          fake, None)
    assert rc == -3  # MOE_ERR_WORKSPACE, nothing enqueued


def test_noalloc_invalid_ids_get_no_row():
    """An expert id outside [0,E) is skipped by the allocation-free variant as by the workspace one:
    perm and prow are -1 for that entry (this variant has no error flag to raise)."""
    from mixture_experts_layer_row_b200 import _lib as L
    dev = torch.device("cuda", 0)
    T, E, k = 300, 8, 2
    cfg = L.make_config(T, 64, 128, E, k)
    idx_np = _idx(T, E, k, 7)
    idx_np[5, 0] = E
    idx_np[9, 1] = -3
    idx = torch.from_numpy(idx_np).to(dev)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev)
    ref, got = _outputs(L, cfg, dev), _outputs(L, cfg, dev)
    L.route_metadata(cfg, idx, ref["counts"], ref["offsets"], ref["poff"], ref["perm"], ref["prow"],
                     ref["row_token"], ws)
    L.route_metadata_noalloc(cfg, idx, got["counts"], got["offsets"], got["poff"], got["perm"],
                             got["prow"], got["row_token"])
    torch.cuda.synchronize()
    for name in ref:
        assert torch.equal(got[name], ref[name]), name
    bad = ~((idx_np >= 0) & (idx_np < E))
    assert np.all(got["prow"].cpu().numpy().reshape(T, k)[bad] == -1)
    assert np.all(got["perm"].cpu().numpy().reshape(T, k)[bad] == -1)
