"""Failure detection without faulting a GPU: a bounded pipeline wait that runs out reports
MOE_DEVERR_TIMEOUT through the workspace flag and returns; the context stays usable."""
import numpy as np
import pytest
import torch

from _util import dev

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    from mixture_experts_layer_row_b200 import _lib as L
    cfg = L.make_config(64, 64, 128, 8, 2)
    ws = torch.zeros(L.workspace_size(cfg), dtype=torch.uint8, device=dev())
    L.clear_error(ws)
    L.test_bounded_wait(ws, 2_000_000)  # 2 ms: nothing ever arrives on the barrier
    torch.cuda.synchronize()
    assert L.get_error(ws) & L.DEVERR_TIMEOUT
    L.clear_error(ws)
    assert L.get_error(ws) == 0
    # the context still runs work correctly afterwards
    idx = torch.from_numpy(np.argsort(np.random.default_rng(0).random((64, 8)), 1)[:, :2]
                           .astype(np.int32)).to(dev())
    z = lambda n: torch.zeros(n, dtype=torch.int32, device=dev())
    counts = z(8)
    L.route_metadata(cfg, idx, counts, z(9), z(9), z(128), z(128), z(L.max_rows(cfg)), ws)
    torch.cuda.synchronize()
    assert int(counts.sum()) == 128 and L.get_error(ws) == 0
