"""Row-wise expert parallelism across the GPUs of one node, around the moe_ep_* calls of the C ABI.

Rank h of G owns experts [h*E/G, (h+1)*E/G). One step, on every rank, in this order:

    route (own tokens, all E experts) -> all-gather the per-expert counts -> layout
    -> [ranks ordered] dispatch (peer stores into the owners' x_perm) + zero the own pad rows
    -> [ranks ordered] own experts: GEMM1 + SwiGLU, GEMM2
    -> [ranks ordered] combine (peer loads of the owners' y)
    backward: combine backward (peer stores into the owners' dy) + zero the own dy pad rows
    -> [ranks ordered] own experts: GEMM2 dgrad + SwiGLU bwd, GEMM2 wgrad, GEMM1 dgrad, GEMM1 wgrad
    -> [ranks ordered] token reduce (peer loads of the owners' dx_perm)

"[ranks ordered]" is a collective that every rank enters after the previous phase's kernels: the
kernels themselves never wait on another GPU. PyTorch only allocates memory and runs the collectives;
every row movement and every GEMM runs in libmoe_b200's kernels.

Two ways to connect the ranks:
  - `TorchComm`: one process per GPU under torch.distributed (NCCL): an all-gather of the counts, a
    one-element all-reduce as the ordering point, and peer pointers from PyTorch's symmetric memory.
  - `EmulatedNode`: every rank's buffers on one GPU, the ranks' kernels issued one after another on
    one stream (the layout and the arithmetic are the multi-GPU ones; only the pointers are local).
"""
from __future__ import annotations

import torch

from . import _lib as L


class EPMoELayer:
    """One rank's share of an expert-parallel bf16 MoE layer (learned routing is done by the caller:
    idx / gates are inputs, as for the uniform-routing workloads)."""

    def __init__(self, rank, world, T, d, F, E, k, device="cuda", alloc=None):
        """alloc(shape, dtype) allocates the four peer-visible routed-row buffers (default: plain
        device memory, which is enough when all ranks share one GPU)."""
        if E % world or not 1 <= world <= 8:
            raise ValueError("E must be a multiple of world, 1 <= world <= 8")
        self.rank, self.world, self.T, self.d, self.F, self.E, self.k = rank, world, T, d, F, E, k
        self.EL = E // world
        self.cfg = L.make_config(T, d, F, E, k, L.DTYPE_BF16)
        self.R = L.ep_max_rows(self.cfg, world)
        # the owner's GEMMs see its E/G experts and up to G*T*k routed rows
        self.cfg_loc = L.make_config(world * T * k, d, F, self.EL, 1, L.DTYPE_BF16)
        if self.R <= 0 or L.max_rows(self.cfg_loc) != self.R:
            raise L.MoEError("invalid expert-parallel configuration")
        dev = torch.device(device)
        z = lambda shape, dt=torch.bfloat16: torch.zeros(shape, dtype=dt, device=dev)
        peer = alloc or z
        i32, f32 = torch.int32, torch.float32
        R, EL = self.R, self.EL
        # token side (this rank's tokens)
        self.idx, self.gates = z((T, k), i32), z((T, k), f32)
        R1 = L.max_rows(self.cfg)
        self.counts, self.offsets, self.poff = z(E, i32), z(E + 1, i32), z(E + 1, i32)
        self.perm, self.prow, self.row_token = z(T * k, i32), z(T * k, i32), z(R1, i32)
        self.all_counts = z((world, E), i32)
        self.src_base, self.dst_row = z(E, i32), z(T * k, i32)
        self.out, self.dx, self.dgates = z((T, d)), z((T, d)), z((T, k), f32)
        # owner side (this rank's experts); x_perm, y, dy, dx_perm are read or written by every rank
        self.counts_loc, self.poff_loc = z(EL, i32), z(EL + 1, i32)
        self.x_perm, self.y, self.dy, self.dx_perm = (peer((R, d), torch.bfloat16) for _ in range(4))
        self.h13, self.a, self.dh13 = z((R, 2 * F)), z((R, F)), z((R, 2 * F))
        self.dW13, self.dW2 = z((EL, 2 * F, d)), z((EL, d, F))
        self.ws = z(L.workspace_size(self.cfg), torch.uint8)
        self.ws_loc = z(L.workspace_size(self.cfg_loc), torch.uint8)
        self.W13 = self.W2 = None
        self.peers = None

    def set_weights(self, W13_loc, W2_loc):
        """This rank's experts: W13 [E/G, 2F, d], W2 [E/G, d, F] (bf16)."""
        if tuple(W13_loc.shape) != (self.EL, 2 * self.F, self.d) or tuple(W2_loc.shape) != (self.EL, self.d, self.F):
            raise ValueError("expert weight shape mismatch")
        self.W13, self.W2 = W13_loc.contiguous(), W2_loc.contiguous()

    def set_peers(self, x_perm, y, dy, dx_perm):
        """Device pointers of the four routed-row buffers on every rank (lists of G ints)."""
        self.peers = {n: L.peer_array(p) for n, p in
                      (("x_perm", x_perm), ("y", y), ("dy", dy), ("dx_perm", dx_perm))}

    # ---- phases ---------------------------------------------------------------------------------
    def route(self, idx, gates, stream=None):
        self.idx.copy_(idx)
        self.gates.copy_(gates)
        L.route_metadata(self.cfg, self.idx, self.counts, self.offsets, self.poff, self.perm, self.prow,
                         self.row_token, self.ws, stream)
        return self.counts

    def layout(self, stream=None):
        L.ep_layout(self.cfg, self.rank, self.world, self.all_counts, self.idx, self.perm, self.offsets,
                    self.src_base, self.counts_loc, self.poff_loc, self.dst_row, stream)

    def dispatch(self, x, stream=None):
        self._x = x
        L.ep_dispatch(self.cfg, self.world, x, self.idx, self.dst_row, self.peers["x_perm"], stream)
        L.ep_zero_pad(self.cfg, self.world, self.x_perm, self.counts_loc, self.poff_loc, stream)

    def experts_forward(self, stream=None):
        c, cl, po, ws = self.cfg_loc, self.counts_loc, self.poff_loc, self.ws_loc
        L.grouped_gemm(c, L.GEMM_FWD1_SWIGLU, self.x_perm, self.W13, self.h13, self.a, None, cl, po, ws, stream)
        L.grouped_gemm(c, L.GEMM_FWD2, self.a, self.W2, self.y, None, None, cl, po, ws, stream)

    def combine(self, stream=None):
        L.ep_combine(self.cfg, self.world, self.peers["y"], self.gates, self.idx, self.dst_row, self.out, stream)
        return self.out

    def combine_bwd(self, dout, stream=None):
        L.ep_combine_bwd(self.cfg, self.world, dout, self.peers["y"], self.gates, self.idx, self.dst_row,
                         self.peers["dy"], self.dgates, stream)
        L.ep_zero_pad(self.cfg, self.world, self.dy, self.counts_loc, self.poff_loc, stream)

    def experts_backward(self, stream=None):
        c, cl, po, ws = self.cfg_loc, self.counts_loc, self.poff_loc, self.ws_loc
        L.grouped_gemm(c, L.GEMM_DGRAD2_SWIGLU, self.dy, self.W2, self.dh13, None, self.h13, cl, po, ws, stream)
        L.grouped_gemm(c, L.GEMM_WGRAD2, self.dy, self.a, self.dW2, None, None, cl, po, ws, stream)
        L.grouped_gemm(c, L.GEMM_DGRAD1, self.dh13, self.W13, self.dx_perm, None, None, cl, po, ws, stream)
        L.grouped_gemm(c, L.GEMM_WGRAD1, self.dh13, self.x_perm, self.dW13, None, None, cl, po, ws, stream)

    def token_reduce(self, stream=None):
        L.ep_token_reduce(self.cfg, self.world, self.peers["dx_perm"], self.idx, self.dst_row, self.dx, stream)
        return self.dx

    def error_flags(self) -> int:
        return L.get_error(self.ws) | L.get_error(self.ws_loc)


def ep_step(layer: EPMoELayer, comm, x, idx, gates, dout=None):
    """One forward (+ backward when dout is given) of this rank, with the collectives between the
    phases. Every rank calls it with the same sequence of collectives."""
    counts = layer.route(idx, gates)
    comm.all_gather_counts(counts, layer.all_counts)
    layer.layout()
    comm.order()  # every owner's buffers are free
    layer.dispatch(x)
    comm.order()  # every row has arrived
    layer.experts_forward()
    comm.order()  # every owner's y is written
    out = layer.combine()
    if dout is None:
        return out
    comm.order()  # nobody reads y any more; the owners' dy may be written
    layer.combine_bwd(dout)
    comm.order()
    layer.experts_backward()
    comm.order()
    return layer.token_reduce()


class TorchComm:
    """The collectives of one rank under torch.distributed (NCCL between GPUs; gloo works for the
    count exchange on CPU). Stream-ordered: no host synchronisation."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self._flag = None

    def all_gather_counts(self, counts, out):
        self.dist.all_gather_into_tensor(out.view(-1), counts, group=self.group)

    def order(self):
        if self._flag is None:
            dev = "cuda" if self.dist.get_backend(self.group) == "nccl" else "cpu"
            self._flag = torch.zeros(1, dtype=torch.int32, device=dev)
        self.dist.all_reduce(self._flag, group=self.group)

    @staticmethod
    def symmetric_alloc(group_name):
        """Allocator for the peer-visible buffers: PyTorch symmetric memory, whose rendezvous gives
        every rank the other ranks' pointers (see `exchange_peers`)."""
        import torch.distributed._symmetric_memory as symm

        def alloc(shape, dtype):
            t = symm.empty(shape, dtype=dtype, device=torch.device("cuda", torch.cuda.current_device()))
            symm.rendezvous(t, group_name)
            return t
        return alloc

    @staticmethod
    def exchange_peers(layer: EPMoELayer, group_name):
        import torch.distributed._symmetric_memory as symm
        ptrs = []
        for t in (layer.x_perm, layer.y, layer.dy, layer.dx_perm):
            h = symm.rendezvous(t, group_name)
            ptrs.append([int(p) for p in h.buffer_ptrs])
        layer.set_peers(*ptrs)


class EmulatedNode:
    """G ranks on one GPU: every rank's buffers local, the ranks' kernels issued one after another on
    one stream, so nothing ever waits on another kernel. Used to run the expert-parallel path where
    only one GPU is available; the layout and arithmetic are those of G GPUs."""

    def __init__(self, world, T, d, F, E, k, device="cuda"):
        self.layers = [EPMoELayer(r, world, T, d, F, E, k, device) for r in range(world)]
        ptrs = [[int(getattr(l, n).data_ptr()) for l in self.layers] for n in ("x_perm", "y", "dy", "dx_perm")]
        for l in self.layers:
            l.set_peers(*ptrs)

    def set_weights(self, W13, W2):
        """Full expert weights [E, 2F, d], [E, d, F]: rank h takes its E/G experts."""
        for l in self.layers:
            sl = slice(l.rank * l.EL, (l.rank + 1) * l.EL)
            l.set_weights(W13[sl], W2[sl])

    def step(self, xs, idxs, gates, douts=None):
        """xs, idxs, gates, douts: one tensor per rank. Returns the ranks' outputs (and fills dx,
        dgates, dW13, dW2 on each rank when douts is given)."""
        ls = self.layers
        counts = [l.route(i, g) for l, i, g in zip(ls, idxs, gates)]
        gathered = torch.stack(counts)  # the all-gather
        for l in ls:
            l.all_counts.copy_(gathered)
            l.layout()
        for l, x in zip(ls, xs):
            l.dispatch(x)
        for l in ls:
            l.experts_forward()
        outs = [l.combine() for l in ls]
        if douts is not None:
            for l, dout in zip(ls, douts):
                l.combine_bwd(dout)
            for l in ls:
                l.experts_backward()
            for l in ls:
                l.token_reduce()
        return outs
