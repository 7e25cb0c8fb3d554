"""Expert-parallel Cap-and-Spill MoE layer over torch.distributed.

The "Cap-and-Spill" critique page (juhe.plus, section "Cap-and-Spill")
describes expert-parallel dispatch in two passes: a capacity pass with C slots
per expert, then a pass for the compacted overflow, whose buffer is sized for
the largest possible overflow so that it can be allocated before the routing
is known and no token is dropped.  Here both passes are equal-split
all-to-alls (NCCL over NVLink when the process group is NCCL), so no host
synchronisation sits between them:

  pass 1  the capacity region of x_perm [E*C rows] is destination-major, so it
          goes as it is; the per-expert capacity and overflow counts go with it;
  pass 2  each destination's overflow rows (contiguous in x_perm's compacted
          overflow region) go in a slot of S rows, S = min(k, E/G) max(0, T-C).

Everything that touches rows runs in the library's kernels (include/moe.h,
moe_ep_*): routing, the capacity layout, packing, the receiver's local layout
and GEMM schedule, the grouped GEMMs on the local experts, the return copies
and the combine.  This module allocates the buffers and calls the entry points
and the collectives in order.

The layer's steps are exposed as phases (route_and_pack, exchange_in,
local_experts = receive + experts + send_back, exchange_out, finish) so that the exchange can be any function
with the semantics of torch.distributed.all_to_all_single(out, inp): forward()
uses the process group's; one process can drive several ranks' phases with an
exchange that copies between their buffers.
"""
from __future__ import annotations

import grouped_expert_gemm_router_b200 as moe


class CapAndSpillEP:
    """One rank of the expert-parallel layer.

    shape: the global shape of this rank's batch (T tokens over all E experts),
           with the capacity layout (make_shape(..., C=C, capacity=True)).
    G:     ranks; rank d owns experts [d*E/G, (d+1)*E/G), whose weights are
           passed to local_experts / forward as [E/G, ...] slices.
    """

    def __init__(self, shape, G: int, device="cuda"):
        import torch
        if not (shape.flags & moe.MOE_FLAG_CAPACITY):
            raise moe.MoeError("the expert-parallel layer needs the capacity layout (MOE_FLAG_CAPACITY)")
        self.shape, self.G = shape, int(G)
        self.S = moe.moe_ep_overflow_rows(shape, G)
        if self.S < 0:
            raise moe.MoeError("unsupported expert-parallel shape %r for G=%d" % (shape, G))
        self.local = moe.moe_ep_local_shape(shape, G)
        T, H, E, k, C = shape.T, shape.H, shape.E, shape.k, shape.C
        Eg = E // G
        self.Eg, self.cap_rows = Eg, E * C
        P = moe.moe_permuted_rows(shape)
        dev = torch.device(device)
        bf16, i32, f32 = torch.bfloat16, torch.int32, torch.float32
        e = torch.empty
        self.b = dict(
            logits=e((T, E), dtype=f32, device=dev), topk_idx=e((T, k), dtype=i32, device=dev),
            topk_w=e((T, k), dtype=f32, device=dev), expert_counts=e((E,), dtype=i32, device=dev),
            expert_offsets=e((E + 1,), dtype=i32, device=dev), src_token=e((P,), dtype=i32, device=dev),
            dest_row=e((T * k,), dtype=i32, device=dev), x_perm=e((P, H), dtype=bf16, device=dev),
            y=e((P, H), dtype=bf16, device=dev), out=e((T, H), dtype=bf16, device=dev))
        self.ws = e(((moe.moe_workspace_bytes(shape) + 255) // 256 * 256,), dtype=torch.uint8, device=dev)
        slot = max(self.S, 1)
        self.send_meta = e((G * 2 * Eg,), dtype=i32, device=dev)
        self.recv_meta = e((G * 2 * Eg,), dtype=i32, device=dev)
        self.recv_cap = e((G * Eg * C, H), dtype=bf16, device=dev)
        self.back_cap = e((G * Eg * C, H), dtype=bf16, device=dev)
        self.send_ovf = e((G * slot, H), dtype=bf16, device=dev)
        self.recv_ovf = e((G * slot, H), dtype=bf16, device=dev)
        self.back_ovf = e((G * slot, H), dtype=bf16, device=dev)
        self.recv_back_ovf = e((G * slot, H), dtype=bf16, device=dev)
        L = self.local
        self.x_loc = e((L.T, H), dtype=bf16, device=dev)
        self.h_loc = e((L.T, L.F), dtype=bf16, device=dev)
        self.y_loc = e((L.T, H), dtype=bf16, device=dev)
        self.ws_loc = e(((moe.moe_workspace_bytes(L) + 255) // 256 * 256,), dtype=torch.uint8, device=dev)
        self.ep_ws = e(((moe.moe_ep_workspace_bytes(shape, G) + 255) // 256 * 256,), dtype=torch.uint8, device=dev)
        if dev.type == "cuda":
            moe.moe_workspace_init(shape, self.ws)
            moe.moe_workspace_init(L, self.ws_loc)

    # ---- phases -------------------------------------------------------------
    def route_and_pack(self, x, w_router, bias, stream=None, fused=True):
        """Routing and the capacity layout of this rank's tokens, then the
        per-destination counts and overflow slots (fused: the row copy writes
        the overflow rows straight into the slots; else the row copy of every
        permuted row, then the pack)."""
        s, b = self.shape, self.b
        moe.moe_route_dispatch(s, x, w_router, bias, b["logits"], b["topk_idx"], b["topk_w"], b["expert_counts"],
                               b["expert_offsets"], b["src_token"], b["dest_row"], self.ws, stream)
        if fused:
            moe.moe_ep_gather_pack(s, self.G, x, b["src_token"], b["x_perm"], self.ws, self.send_ovf, self.send_meta,
                                   self.ep_ws, stream)
        else:
            moe.moe_gather(s, x, b["src_token"], b["x_perm"], self.ws, stream)
            moe.moe_ep_pack(s, self.G, b["x_perm"], self.ws, self.send_ovf, self.send_meta, self.ep_ws, stream)

    def exchange_in(self, all_to_all):
        """Pass 1 (capacity rows and counts), pass 2 (overflow slots)."""
        all_to_all(self.recv_cap, self.b["x_perm"][:self.cap_rows])
        all_to_all(self.recv_meta, self.send_meta)
        all_to_all(self.recv_ovf, self.send_ovf)

    def receive(self, stream=None):
        """The received rows in the local expert-contiguous layout, and the
        local GEMM schedule."""
        moe.moe_ep_local_dispatch(self.shape, self.G, self.recv_meta, self.recv_cap, self.recv_ovf, self.x_loc,
                                  self.ws_loc, self.ep_ws, stream)

    def experts(self, w_gate, w_up, w_down, stream=None):
        """The grouped GEMMs of this rank's experts (weights: its [E/G, ...]
        slices) on the received rows."""
        L = self.local
        moe.moe_grouped_swiglu(L, self.x_loc, w_gate, w_up, self.h_loc, self.ws_loc, stream)
        moe.moe_grouped_down(L, self.h_loc, w_down, self.y_loc, self.ws_loc, stream)

    def send_back(self, stream=None):
        """Each result row to the position its input arrived at in the
        return buffers."""
        moe.moe_ep_local_return(self.shape, self.G, self.y_loc, self.back_cap, self.back_ovf, self.ep_ws, stream)

    def local_experts(self, w_gate, w_up, w_down, stream=None):
        """receive, experts, send_back."""
        self.receive(stream)
        self.experts(w_gate, w_up, w_down, stream)
        self.send_back(stream)

    def exchange_out(self, all_to_all):
        """The two passes back: results of the capacity rows straight into y,
        results of the overflow rows into their slots."""
        all_to_all(self.b["y"][:self.cap_rows], self.back_cap)
        all_to_all(self.recv_back_ovf, self.back_ovf)

    def finish(self, stream=None, fused=True):
        """The weighted combine into out, the overflow results read from the
        return slots (fused=False: copied into y first, then combined)."""
        s, b = self.shape, self.b
        if fused:
            moe.moe_ep_unpack_combine(s, self.G, self.recv_back_ovf, b["y"], b["dest_row"], b["topk_w"], b["out"],
                                      self.ep_ws, stream)
        else:
            moe.moe_ep_unpack(s, self.G, self.recv_back_ovf, b["y"], self.ep_ws, stream)
            moe.moe_combine(s, b["y"], b["dest_row"], b["topk_w"], b["out"], stream)
        return b["out"]

    # ---- the layer on a process group ------------------------------------------
    def forward(self, x, w_router, bias, w_gate, w_up, w_down, group=None):
        """One layer on this rank (every rank of `group` calls it; G must be
        the group's size).  Returns this rank's out [T, H]."""
        import torch
        import torch.distributed as dist

        def a2a(out, inp):
            # bf16 rows as their bytes (same splits; any backend moves bytes)
            if out.dtype == torch.bfloat16:
                out, inp = out.view(torch.uint8), inp.view(torch.uint8)
            dist.all_to_all_single(out, inp, group=group)

        self.route_and_pack(x, w_router, bias)
        self.exchange_in(a2a)
        self.local_experts(w_gate, w_up, w_down)
        self.exchange_out(a2a)
        return self.finish()


def exchange_in_process(ranks, phase: str) -> None:
    """Run one exchange phase ("exchange_in" or "exchange_out") of several
    ranks held by one process: every all_to_all the ranks issue, in order, is
    carried out as row-block copies (block d of rank s's input into block s
    of rank d's output), the semantics of all_to_all_single with equal
    splits.  The copies are stream-ordered after each rank's earlier work."""
    G = len(ranks)
    calls = []
    for r in ranks:
        rec = []
        getattr(r, phase)(lambda out, inp, rec=rec: rec.append((out, inp)))
        calls.append(rec)
    for i in range(len(calls[0])):
        ins = [c[i][1].tensor_split(G) for c in calls]
        for d in range(G):
            outs = calls[d][i][0].tensor_split(G)
            for s in range(G):
                outs[s].copy_(ins[s][d])
