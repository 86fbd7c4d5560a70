"""Row-wise expert parallelism across G ranks.

CPU (gloo, two processes): the count exchange of `TorchComm`, and that every rank derives the same
layout of every owner's buffers from the gathered counts, with the sources' rows filling each owner's
groups exactly once (the oracle's layout definition, run on each rank). Host-side argument checks of
the C ABI. GPU (`-m gpu`): G ranks emulated on one GPU (`EmulatedNode`: every rank's buffers local,
the ranks' kernels one after another, so no kernel waits on another); the device layout is compared
bit for bit with the oracle's, and the whole layer -- forward and backward -- with the single-GPU fp64
oracle run on the concatenation of all ranks' tokens (rows only move between GPUs; the arithmetic is
the layer's)."""
import ctypes
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import moe as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, E, T, k, q):
    import sys
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    from mixture_experts_layer_row_b200.ep import TorchComm
    from oracle import moe as Oc
    comm = TorchComm()
    rng = np.random.default_rng(100 + rank)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    if rank == 1:
        idx[:, 0] = 0  # uneven load: every token of rank 1 also uses expert 0
        idx[:, 1:] = np.stack([rng.permutation(np.arange(1, E))[:k - 1] for _ in range(T)])
    counts = torch.from_numpy(np.bincount(idx.reshape(-1), minlength=E).astype(np.int32))
    all_counts = torch.zeros((world, E), dtype=torch.int32)
    comm.all_gather_counts(counts, all_counts)
    comm.order()
    L = Oc.ep_layout(all_counts.numpy().astype(np.int64), world)
    rows = Oc.ep_dst_rows(idx, L["base"][rank], E)
    # every rank's view of every owner's layout, and every rank's rows, gathered on every rank
    lay = torch.from_numpy(np.concatenate([L["poff_loc"].reshape(-1), L["counts_loc"].reshape(-1)]))
    lays = [torch.zeros_like(lay) for _ in range(world)]
    dist.all_gather(lays, lay)
    rws = [torch.zeros(T * k, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(rws, torch.from_numpy(rows))
    ids = [torch.zeros(T * k, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(ids, torch.from_numpy(idx.reshape(-1).astype(np.int64)))
    q.put((rank, all_counts.numpy(), [l.numpy() for l in lays], [r.numpy() for r in rws],
           [i.numpy() for i in ids]))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("E,T,k", [(8, 48, 2), (16, 40, 4)])
def test_ep_count_exchange_and_layout_agree_across_ranks_gloo(E, T, k):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, E, T, k, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict((r[0], r[1:]) for r in (q.get(timeout=120) for _ in range(world)))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    ac0, lays0, rows, ids = res[0]
    ac1, lays1, _, _ = res[1]
    # the gathered counts are rank-major and identical on both ranks; every rank derives the same
    # layout of every owner
    assert np.array_equal(ac0, ac1)
    for a, b in zip(lays0, lays1):
        assert np.array_equal(a, b)
    assert np.array_equal(lays0[0], lays0[1])
    EL = E // world
    L = O.ep_layout(ac0.astype(np.int64), world)
    for h in range(world):
        used = {}
        for g in range(world):
            for n, (e, r) in enumerate(zip(ids[g], rows[g])):
                if e // EL == h:
                    assert r not in used, "two entries on one owner row"
                    used[r] = (g, n)
        # the non-pad rows of each local group are exactly the entries routed there, source-major
        for el in range(EL):
            e = h * EL + el
            start, cnt = int(L["poff_loc"][h, el]), int(L["counts_loc"][h, el])
            got = [used[r] for r in range(start, start + cnt)]
            want = [(g, n) for g in range(world) for n, ee in enumerate(ids[g]) if ee == e]
            assert got == want


def test_ep_host_argument_checks():
    """moe_ep_* validate on the host before anything is enqueued (no GPU needed)."""
    from mixture_experts_layer_row_b200 import _lib as L
    c = L.make_config(256, 128, 256, 8, 2, L.DTYPE_BF16)
    assert L.ep_max_rows(c, 2) == (2 * 256 * 2 + 31 * 4 + 31) // 32 * 32
    assert L.ep_max_rows(c, 3) == 0          # E not a multiple of world
    assert L.ep_max_rows(c, 16) == 0         # more than 8 ranks
    mx = L.make_config(256, 128, 256, 8, 2, L.DTYPE_MXFP8)
    assert L.ep_max_rows(mx, 2) == 0         # bf16 only
    fake = ctypes.c_void_p(1 << 20)
    assert L.lib.moe_ep_layout(ctypes.byref(c), 2, 2, fake, fake, fake, fake, fake, fake, fake, fake,
                               None) == -1  # rank out of range
    assert L.lib.moe_ep_dispatch(ctypes.byref(c), 2, fake, fake, fake, None, None) == -1  # no peers


# ------------------------------------------------------------------------------------------------
# GPU: G ranks emulated on one GPU
# ------------------------------------------------------------------------------------------------

def _ep_inputs(world, T, d, F, E, k, seed, skew=False):
    g = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    xs = [torch.randn((T, d), generator=g).to(torch.bfloat16) for _ in range(world)]
    douts = [torch.randn((T, d), generator=g).to(torch.bfloat16) for _ in range(world)]
    W13 = (torch.randn((E, 2 * F, d), generator=g) * 0.05).to(torch.bfloat16)
    W2 = (torch.randn((E, d, F), generator=g) * 0.05).to(torch.bfloat16)
    idxs, gates = [], []
    for r in range(world):
        w = np.exp(-np.arange(E) / 2.0) if skew else np.ones(E)
        idx = np.stack([rng.choice(E, size=k, replace=False, p=w / w.sum()) for _ in range(T)])
        s = rng.standard_normal((T, k))
        gt = np.exp(s - s.max(1, keepdims=True))
        idxs.append(torch.from_numpy(idx.astype(np.int32)))
        gates.append(torch.from_numpy((gt / gt.sum(1, keepdims=True)).astype(np.float32)))
    return xs, douts, W13, W2, idxs, gates


@pytest.mark.gpu
@pytest.mark.parametrize("world,E,skew", [(2, 8, False), (4, 16, False), (4, 16, True), (8, 32, False)])
def test_ep_emulated_layout_bitexact(world, E, skew):
    from mixture_experts_layer_row_b200.ep import EmulatedNode
    T, d, F, k = 96, 128, 128, 2
    xs, douts, W13, W2, idxs, gates = _ep_inputs(world, T, d, F, E, k, 7, skew)
    node = EmulatedNode(world, T, d, F, E, k)
    node.set_weights(W13.cuda(), W2.cuda())
    node.step([x.cuda() for x in xs], [i.cuda() for i in idxs], [g.cuda() for g in gates])
    torch.cuda.synchronize()
    all_counts = np.stack([np.bincount(i.numpy().reshape(-1), minlength=E) for i in idxs])
    L = O.ep_layout(all_counts, world)
    for r, l in enumerate(node.layers):
        assert np.array_equal(l.all_counts.cpu().numpy(), all_counts)
        assert np.array_equal(l.src_base.cpu().numpy(), L["base"][r])
        assert np.array_equal(l.counts_loc.cpu().numpy(), L["counts_loc"][r])
        assert np.array_equal(l.poff_loc.cpu().numpy(), L["poff_loc"][r])
        assert np.array_equal(l.dst_row.cpu().numpy(), O.ep_dst_rows(idxs[r].numpy(), L["base"][r], E))
        assert l.error_flags() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("world,T,d,F,E,k,skew", [(2, 256, 256, 256, 8, 2, False),
                                                  (4, 192, 256, 384, 16, 4, True),
                                                  (8, 128, 128, 256, 32, 4, False)])
def test_ep_emulated_layer_matches_oracle(world, T, d, F, E, k, skew):
    from mixture_experts_layer_row_b200.ep import EmulatedNode
    from _util import TOL_BF16, assert_close_rel, np64
    xs, douts, W13, W2, idxs, gates = _ep_inputs(world, T, d, F, E, k, 11, skew)
    node = EmulatedNode(world, T, d, F, E, k)
    node.set_weights(W13.cuda(), W2.cuda())
    outs = node.step([x.cuda() for x in xs], [i.cuda() for i in idxs], [g.cuda() for g in gates],
                     [o.cuda() for o in douts])
    torch.cuda.synchronize()
    # the oracle: one layer over every rank's tokens (rank-major)
    x64 = np.concatenate([np64(x) for x in xs])
    dout = np.concatenate([np64(o) for o in douts])
    idx = np.concatenate([i.numpy() for i in idxs]).astype(np.int64)
    g64 = np.concatenate([np64(gt) for gt in gates])
    W13n, W2n = np64(W13), np64(W2)
    ref, saved = O.layer_fwd(x64, W13n, W2n, idx, g64)
    gr = O.layer_bwd(dout, x64, W13n, W2n, idx, g64, saved)
    got_out = np.concatenate([np64(o) for o in outs])
    got_dx = np.concatenate([np64(l.dx) for l in node.layers])
    got_dg = np.concatenate([l.dgates.cpu().double().numpy() for l in node.layers])
    assert_close_rel(got_out, ref, TOL_BF16, "out")
    assert_close_rel(got_dx, gr["dx"], TOL_BF16, "dx")
    assert_close_rel(got_dg, gr["dgates"], TOL_BF16, "dgates")
    got_dW13 = np.concatenate([np64(l.dW13) for l in node.layers])
    got_dW2 = np.concatenate([np64(l.dW2) for l in node.layers])
    assert_close_rel(got_dW13, gr["dW13"], TOL_BF16, "dW13")
    assert_close_rel(got_dW2, gr["dW2"], TOL_BF16, "dW2")
    for l in node.layers:
        assert l.error_flags() == 0
