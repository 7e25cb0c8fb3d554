"""Expert-parallel MoE layer with device-initiated peer stores.

The same layer as CapAndSpillEP (each rank's output equals the single-GPU
layer on its tokens), with the all-to-all carried by two kernels that store
rows straight into the other ranks' buffers: the source puts each routed
token row into the x_loc of its expert's rank, the destination puts each
result row into the y of the token's rank.  Only the routed rows cross the
links -- the Cap-and-Spill second pass moves a slot sized for the worst case
whatever the routing (the point the "Cap-and-Spill" critique page, juhe.plus,
makes about that method) -- and neither side copies rows into or out of
exchange buffers.  The only collectives are an all-gather of the per-expert
counts (E int32 per rank) and two barriers, all stream-ordered: no host
synchronisation.

Peer addresses come from symmetric memory (on_process_group) or, for several
ranks held by one process on one device, from the ranks' own buffers
(connect_in_process); the kernels take them as device arrays of G addresses.
"""
from __future__ import annotations

import grouped_expert_gemm_router_b200 as moe


class DirectEP:
    """One rank of the expert-parallel layer (peer-store form).

    shape: this rank's batch (T tokens over all E experts), uncapped layout.
    G, rank: ranks and this one's index; rank d owns experts
             [d*E/G, (d+1)*E/G), whose weights are passed as [E/G, ...] slices.
    x_loc, y: optional caller-given buffers (symmetric memory, so that peers
             can store into them); allocated here otherwise.
    """

    def __init__(self, shape, G: int, rank: int, device="cuda", x_loc=None, y=None, fp8=False, x_loc_q=None,
                 scale_loc=None):
        import torch
        if shape.flags & moe.MOE_FLAG_CAPACITY:
            raise moe.MoeError("the peer-store layer uses the uncapped layout")
        self.shape, self.G, self.rank = shape, int(G), int(rank)
        self.Tloc = moe.moe_ep_direct_local_rows(shape, G)
        if self.Tloc < 0 or not 0 <= self.rank < self.G:
            raise moe.MoeError("unsupported expert-parallel shape %r for G=%d, rank %d" % (shape, G, rank))
        self.local = moe.moe_ep_direct_local_shape(shape, G)
        T, H, E, k = shape.T, shape.H, shape.E, shape.k
        P = moe.moe_permuted_rows(shape)
        dev = torch.device(device)
        bf16, i32, f32 = torch.bfloat16, torch.int32, torch.float32
        e = torch.empty
        self.b = dict(
            logits=e((T, E), dtype=f32, device=dev), topk_idx=e((T, k), dtype=i32, device=dev),
            topk_w=e((T, k), dtype=f32, device=dev), expert_counts=e((E,), dtype=i32, device=dev),
            expert_offsets=e((E + 1,), dtype=i32, device=dev), src_token=e((P,), dtype=i32, device=dev),
            dest_row=e((T * k,), dtype=i32, device=dev), out=e((T, H), dtype=bf16, device=dev))
        self.b["y"] = y if y is not None else e((P, H), dtype=bf16, device=dev)
        self.x_loc = x_loc if x_loc is not None else e((self.Tloc, H), dtype=bf16, device=dev)
        if tuple(self.b["y"].shape) != (P, H) or tuple(self.x_loc.shape) != (self.Tloc, H):
            raise moe.MoeError("x_loc must be [%d, %d] and y [%d, %d]" % (self.Tloc, H, P, H))
        self.h_loc = e((self.Tloc, shape.F), dtype=bf16, device=dev)
        self.y_loc = e((self.Tloc, H), dtype=bf16, device=dev)
        self.fp8 = bool(fp8)
        if self.fp8:  # e4m3 rows on the links: token codes + scales, received codes + scales, h codes
            u8 = torch.uint8
            self.x_q = e((T, H), dtype=u8, device=dev)
            self.x_scale = e((T,), dtype=f32, device=dev)
            self.x_loc_q = x_loc_q if x_loc_q is not None else e((self.Tloc, H), dtype=u8, device=dev)
            self.scale_loc = scale_loc if scale_loc is not None else e((self.Tloc,), dtype=f32, device=dev)
            self.h_q = e((self.Tloc, shape.F), dtype=u8, device=dev)
            self.h_scale = e((self.Tloc,), dtype=f32, device=dev)
            self.peer_x_loc_q = torch.zeros((G,), dtype=torch.int64, device=dev)
            self.peer_scale_loc = torch.zeros((G,), dtype=torch.int64, device=dev)
        self.cnt_all = e((G, E), dtype=i32, device=dev)
        self.peer_x_loc = torch.zeros((G,), dtype=torch.int64, device=dev)
        self.peer_y = torch.zeros((G,), dtype=torch.int64, device=dev)
        self.ws = e(((moe.moe_workspace_bytes(shape) + 255) // 256 * 256,), dtype=torch.uint8, device=dev)
        self.ws_loc = e(((moe.moe_workspace_bytes(self.local) + 255) // 256 * 256,), dtype=torch.uint8, device=dev)
        self.ep_ws = e(((moe.moe_ep_direct_workspace_bytes(shape, G) + 255) // 256 * 256,), dtype=torch.uint8,
                       device=dev)
        if dev.type == "cuda":
            moe.moe_workspace_init(shape, self.ws)
            moe.moe_workspace_init(self.local, self.ws_loc)

    def set_peers(self, x_loc_addrs, y_addrs, x_loc_q_addrs=None, scale_loc_addrs=None):
        """Rank d's x_loc and y (and, fp8, x_loc_q and scale_loc) addresses as
        this rank's kernels reach them."""
        import torch

        def put(table, addrs):
            table.copy_(torch.tensor([int(a) for a in addrs], dtype=torch.int64))

        put(self.peer_x_loc, x_loc_addrs)
        put(self.peer_y, y_addrs)
        if self.fp8:
            put(self.peer_x_loc_q, x_loc_q_addrs)
            put(self.peer_scale_loc, scale_loc_addrs)

    # ---- phases -------------------------------------------------------------
    def route(self, x, w_router, bias, stream=None):
        """Routing and the uncapped dispatch of this rank's tokens (no row copy)."""
        s, b = self.shape, self.b
        moe.moe_route_dispatch(s, x, w_router, bias, b["logits"], b["topk_idx"], b["topk_w"], b["expert_counts"],
                               b["expert_offsets"], b["src_token"], b["dest_row"], self.ws, stream)

    def gather_counts(self, all_gather):
        """cnt_all[s] = rank s's expert_counts; all_gather(out [G, E], inp [E])
        with the semantics of torch.distributed.all_gather_into_tensor."""
        all_gather(self.cnt_all, self.b["expert_counts"])

    def plan(self, stream=None):
        """Send positions, the local layout and schedule, the return segments."""
        moe.moe_ep_direct_plan(self.shape, self.G, self.rank, self.cnt_all, self.peer_y, self.ws_loc, self.ep_ws,
                               stream)

    def dispatch(self, x, stream=None):
        """Each routed token row into its expert's rank's x_loc (peer stores)."""
        b = self.b
        moe.moe_ep_direct_dispatch(self.shape, self.G, x, b["topk_idx"], b["dest_row"], b["expert_offsets"],
                                   self.peer_x_loc, self.ws, self.ep_ws, stream)

    # ---- fp8: e4m3 rows on the links, fp8 GEMMs on the local experts -------------
    def quantize_tokens(self, x, stream=None):
        """This rank's token rows as e4m3 codes with one scale per row."""
        moe.moe_quantize_rows_fp8(self.shape, moe.MOE_ROWS_TOKENS, x, None, self.x_q, self.x_scale, self.ws, stream)

    def dispatch_fp8(self, stream=None):
        """Each routed token's code row and scale into its expert's rank's
        x_loc_q and scale_loc (peer stores)."""
        b = self.b
        moe.moe_ep_direct_dispatch_fp8(self.shape, self.G, self.x_q, self.x_scale, b["topk_idx"], b["dest_row"],
                                       b["expert_offsets"], self.peer_x_loc_q, self.peer_scale_loc, self.ws,
                                       self.ep_ws, stream)

    def experts_fp8_and_return(self, wg_q, wg_scale, wu_q, wu_scale, wd_q, wd_scale, stream=None):
        """The fp8 SwiGLU GEMM on the received code rows, h quantized per row,
        then the fp8 down projection storing each result row straight into
        its token's rank's y (weights: the rank's slices of the codes and
        scales moe_quantize_weights_fp8 leaves)."""
        L = self.local
        moe.moe_grouped_swiglu_fp8(L, self.x_loc_q, self.scale_loc, None, wg_q, wg_scale, wu_q, wu_scale, self.h_loc,
                                   self.ws_loc, stream)
        moe.moe_ep_direct_quantize_h(self.shape, self.G, self.h_loc, self.h_q, self.h_scale, self.ep_ws, stream)
        moe.moe_ep_direct_down_return_fp8(self.shape, self.G, self.h_q, self.h_scale, wd_q, wd_scale, self.ws_loc,
                                          self.ep_ws, stream)

    def plan_and_dispatch(self, x, stream=None):
        """plan() and dispatch() in one launch.  fp8: x None sends the code
        rows quantize_tokens() left (dispatch_fp8()); x given (bf16 token
        rows) is quantized on the way, by the warps that send its rows."""
        b = self.b
        if self.fp8 and x is None:
            moe.moe_ep_direct_plan_dispatch(self.shape, self.G, self.rank, self.cnt_all, self.peer_y, self.x_q,
                                            self.x_scale, b["topk_idx"], b["dest_row"], b["expert_offsets"],
                                            self.peer_x_loc_q, self.peer_scale_loc, self.ws, self.ws_loc, self.ep_ws,
                                            stream)
        elif self.fp8:
            moe.moe_ep_direct_plan_dispatch_quantize(self.shape, self.G, self.rank, self.cnt_all, self.peer_y, x,
                                                     b["topk_idx"], b["dest_row"], b["expert_offsets"],
                                                     self.peer_x_loc_q, self.peer_scale_loc, self.ws, self.ws_loc,
                                                     self.ep_ws, stream)
        else:
            moe.moe_ep_direct_plan_dispatch(self.shape, self.G, self.rank, self.cnt_all, self.peer_y, x, None,
                                            b["topk_idx"], b["dest_row"], b["expert_offsets"], self.peer_x_loc,
                                            None, self.ws, self.ws_loc, self.ep_ws, stream)

    def experts(self, w_gate, w_up, w_down, stream=None):
        """The grouped GEMMs of this rank's experts on the rows it received."""
        L = self.local
        moe.moe_grouped_swiglu(L, self.x_loc, w_gate, w_up, self.h_loc, self.ws_loc, stream)
        moe.moe_grouped_down(L, self.h_loc, w_down, self.y_loc, self.ws_loc, stream)

    def experts_and_return(self, w_gate, w_up, w_down, stream=None):
        """The grouped SwiGLU GEMM, then the down projection whose epilogue
        stores each result row straight into its token's rank's y (one
        kernel for the down GEMM and the return)."""
        L = self.local
        moe.moe_grouped_swiglu(L, self.x_loc, w_gate, w_up, self.h_loc, self.ws_loc, stream)
        moe.moe_ep_direct_down_return(self.shape, self.G, self.h_loc, w_down, self.ws_loc, self.ep_ws, stream)

    def send_back(self, stream=None):
        """Each result row into its token's rank's y (peer stores)."""
        moe.moe_ep_direct_return(self.shape, self.G, self.y_loc, self.peer_y, self.ep_ws, stream)

    def finish(self, stream=None):
        """The weighted combine of this rank's tokens."""
        b = self.b
        moe.moe_combine(self.shape, b["y"], b["dest_row"], b["topk_w"], b["out"], stream)
        return b["out"]

    # ---- the layer on a process group ------------------------------------------
    @classmethod
    def on_process_group(cls, shape, group=None, device=None, fp8=False):
        """One rank per process of `group` (NCCL), x_loc and y (fp8: also
        x_loc_q and scale_loc) in symmetric memory so that every rank can store
        into every other rank's."""
        import torch
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        G, rank = dist.get_world_size(group), dist.get_rank(group)
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        Tloc, P = moe.moe_ep_direct_local_rows(shape, G), moe.moe_permuted_rows(shape)
        if Tloc < 0:
            raise moe.MoeError("unsupported expert-parallel shape %r for G=%d" % (shape, G))
        x_loc = symm_mem.empty((Tloc, shape.H), dtype=torch.bfloat16, device=dev)
        y = symm_mem.empty((P, shape.H), dtype=torch.bfloat16, device=dev)
        gname = (group if group is not None else dist.group.WORLD).group_name
        if hasattr(symm_mem, "enable_symm_mem_for_group"):  # required before rendezvous by some versions
            symm_mem.enable_symm_mem_for_group(gname)
        hx, hy = symm_mem.rendezvous(x_loc, gname), symm_mem.rendezvous(y, gname)
        handles, xq, sc = [hx, hy], None, None
        if fp8:
            xq = symm_mem.empty((Tloc, shape.H), dtype=torch.uint8, device=dev)
            sc = symm_mem.empty((Tloc,), dtype=torch.float32, device=dev)
            handles += [symm_mem.rendezvous(xq, gname), symm_mem.rendezvous(sc, gname)]
        ep = cls(shape, G, rank, dev, x_loc=x_loc, y=y, fp8=fp8, x_loc_q=xq, scale_loc=sc)
        ep.set_peers(hx.buffer_ptrs, hy.buffer_ptrs, handles[2].buffer_ptrs if fp8 else None,
                     handles[3].buffer_ptrs if fp8 else None)
        ep._handles = handles  # keep the mappings alive
        ep._flag = torch.zeros((1,), dtype=torch.int32, device=dev)
        ep._group = group
        return ep

    def forward(self, x, w_router, bias, w_gate, w_up, w_down, fused_return=True):
        """One layer on this rank (every rank of the group calls it);
        fused_return: the down GEMM stores the results into the owners' y
        itself (else a separate return kernel)."""
        import torch.distributed as dist
        group = self._group

        def barrier():  # stream-ordered: a one-element all-reduce
            dist.all_reduce(self._flag, group=group)

        self.route(x, w_router, bias)
        self.gather_counts(lambda out, inp: dist.all_gather_into_tensor(out, inp, group=group))
        self.plan_and_dispatch(x)
        barrier()
        if fused_return:
            self.experts_and_return(w_gate, w_up, w_down)
        else:
            self.experts(w_gate, w_up, w_down)
            self.send_back()
        barrier()
        return self.finish()


    def forward_fp8(self, x, w_router, bias, wg_q, wg_scale, wu_q, wu_scale, wd_q, wd_scale):
        """One layer of the fp8 form on this rank (e4m3 rows on the links;
        every rank of the group calls it)."""
        import torch.distributed as dist
        group = self._group

        def barrier():
            dist.all_reduce(self._flag, group=group)

        self.route(x, w_router, bias)
        self.gather_counts(lambda out, inp: dist.all_gather_into_tensor(out, inp, group=group))
        self.plan_and_dispatch(x)  # quantizes the rows it sends
        barrier()
        self.experts_fp8_and_return(wg_q, wg_scale, wu_q, wu_scale, wd_q, wd_scale)
        barrier()
        return self.finish()

def connect_in_process(ranks) -> None:
    """Several ranks held by one process on one device: each rank's peer
    tables point at the other ranks' own x_loc and y (and x_loc_q, scale_loc)."""
    xs = [r.x_loc.data_ptr() for r in ranks]
    ys = [r.b["y"].data_ptr() for r in ranks]
    xq = [r.x_loc_q.data_ptr() for r in ranks] if ranks[0].fp8 else None
    sc = [r.scale_loc.data_ptr() for r in ranks] if ranks[0].fp8 else None
    for r in ranks:
        r.set_peers(xs, ys, xq, sc)


def gather_counts_in_process(ranks) -> None:
    """The counts all-gather of ranks held by one process: every rank's
    cnt_all row s = rank s's expert_counts (stream-ordered copies)."""
    for d in ranks:
        for s, src in enumerate(ranks):
            d.cnt_all[s].copy_(src.b["expert_counts"])
