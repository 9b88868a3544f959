"""Expert parallelism for the MoE layer over torch.distributed.

The pages name expert parallelism as future work of the method (page
"DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing paragraph): the experts
are split over ranks, and each token's routed rows travel to the ranks that
own their experts (an all-to-all before the up-projection) and back (an
all-to-all after the down-projection).  Here:

  * rank r of G owns experts [r E/G, (r+1) E/G) (E % G == 0) and holds only
    their W1, W2; the router Wr is replicated;
  * forward: route the rank's own tokens over all E experts; send each routed
    row (X of its token) and its gate to the expert's rank, in expert-major
    order so that each destination's rows are one block; the expert rank runs
    its experts on the rows it received (each row one "token" with K = 1 and
    the sender's gate, so it returns gate * Y); the rows come back in the
    order they were sent and are summed per token;
  * backward: dO rows travel like X; the expert rank runs the expert backward
    (dX~ rows, dW1 and dW2 of its experts: complete, since every token that
    used them sent its rows there, so no all-reduce) and returns dX~ rows and
    the router score gradient dS of each row; the sender sums dX~ per token,
    forms dz = s (dS - sum s dS) and adds the router path (dX += dz Wr^T,
    dWr = X^T dz); dWr is all-reduced, as in data parallelism.

The engine does the arithmetic (`CudaEngine`: the library's kernels); this
module holds the host-side plan and the exchanges.  The exchanges are NCCL
all-to-alls issued by torch.distributed (gloo in the CPU tests).
"""
from __future__ import annotations

import numpy as np


def exchange_plan(send_counts: np.ndarray, recv_counts: np.ndarray):
    """Split sizes of the two all-to-alls and the local expert of every
    received row.

    send_counts[g, l]: rows this rank sends for local expert l of rank g
    (this rank's per-expert row counts, reshaped [G, E/G]);
    recv_counts[g, l]: rows rank g sends here for this rank's local expert l.
    Received rows come source by source, and within a source expert by
    expert (the send order is expert-major)."""
    send_counts = np.asarray(send_counts, np.int64)
    recv_counts = np.asarray(recv_counts, np.int64)
    G, E_loc = recv_counts.shape
    send_splits = send_counts.sum(axis=1).tolist()
    recv_splits = recv_counts.sum(axis=1).tolist()
    local_expert = np.repeat(np.tile(np.arange(E_loc, dtype=np.int32), G), recv_counts.reshape(-1))
    return send_splits, recv_splits, local_expert


class ExpertParallelMoE:
    """One layer under expert parallelism on the ranks of `group`."""

    def __init__(self, T, d, E, n, K, engine, group=None):
        import torch.distributed as dist
        self.group = group
        self.G = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.G:
            raise ValueError(f"E = {E} experts do not split evenly over {self.G} ranks")
        self.T, self.d, self.E, self.n, self.K = T, d, E, n, K
        self.E_loc = E // self.G
        self.engine = engine
        self._saved = None

    # ------------------------------------------------------------------ helpers
    def _a2a(self, send, send_splits, recv_splits):
        import torch
        import torch.distributed as dist
        out = torch.empty((int(sum(recv_splits)),) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
        dist.all_to_all_single(out, send.contiguous(), output_split_sizes=list(recv_splits),
                               input_split_sizes=list(send_splits), group=self.group)
        return out

    # ------------------------------------------------------------------ forward
    def forward(self, X, Wr, bias, W1_loc, W2_loc):
        import torch
        import torch.distributed as dist
        eng = self.engine
        eng.route(X, Wr, bias)
        counts = eng.counts().to(torch.int64)
        recv_counts = torch.empty_like(counts)
        dist.all_to_all_single(recv_counts, counts.contiguous(), group=self.group)
        # The one host synchronisation of the step: the all-to-alls take their
        # split sizes as host integers.  Both count vectors come back in one
        # copy; everything else stays on the device.
        both = torch.stack([counts, recv_counts]).cpu().numpy()
        sc = both[0].reshape(self.G, self.E_loc)
        rc = both[1].reshape(self.G, self.E_loc)
        send_splits, recv_splits, _ = exchange_plan(sc, rc)
        # local expert of every received row, built on the device from the
        # received counts (rows arrive source by source, expert-major)
        R = int(sum(recv_splits))
        ids = torch.arange(self.E_loc, dtype=torch.int32, device=recv_counts.device).repeat(self.G)
        local_expert = torch.repeat_interleave(ids, recv_counts, output_size=R)
        rows, gate, pair_pos = eng.pack(X, with_gate=True, n=int(sum(send_splits)))
        recv_rows = self._a2a(rows, send_splits, recv_splits)
        recv_gate = self._a2a(gate, send_splits, recv_splits)
        out_loc = eng.local_forward(recv_rows, local_expert, recv_gate, W1_loc, W2_loc)
        back = self._a2a(out_loc, recv_splits, send_splits)
        O = eng.combine(back, pair_pos, "O")
        self._saved = (send_splits, recv_splits, pair_pos)
        return O

    # ------------------------------------------------------------------ backward
    def backward(self, dO, X, Wr, W1_loc, W2_loc):
        """Returns dX (router path included), dW1 and dW2 of this rank's
        experts, and dWr summed over the group."""
        import torch.distributed as dist
        if self._saved is None:
            raise RuntimeError("backward before forward")
        eng = self.engine
        send_splits, recv_splits, pair_pos = self._saved
        rows, _, _ = eng.pack(dO, with_gate=False, n=int(sum(send_splits)))
        recv_rows = self._a2a(rows, send_splits, recv_splits)
        dXt_loc, dS_loc, dW1_loc, dW2_loc = eng.local_backward(recv_rows, W1_loc, W2_loc)
        dXt = self._a2a(dXt_loc, recv_splits, send_splits)
        dS = self._a2a(dS_loc, recv_splits, send_splits)
        dX = eng.combine(dXt, pair_pos, "dX")
        dWr = eng.router_backward(X, Wr, dS, pair_pos, dX)
        dist.all_reduce(dWr, group=self.group)
        return dX, dW1_loc, dW2_loc, dWr


class CudaEngine:
    """The arithmetic of an expert-parallel rank on the library's kernels.

    Source side (this rank's tokens, all E experts): moe_route, moe_ep_pack,
    moe_ep_combine, moe_router_backward.  Expert side (the rows received,
    E/G experts, K = 1): moe_route_given, moe_forward, moe_backward with the
    per-row dS written to the routing's pair_dS.  Buffers are allocated once
    for T tokens per rank; the expert side is sized for the most rows it can
    receive, G times this rank's pair capacity.  round_mode: token rounding
    of this rank's routing before the exchange."""

    def __init__(self, T, d, E, n, K, G, device="cuda", seed=0, round_mode=0):
        import torch
        from . import moe
        self.moe = moe
        self.T, self.d, self.E, self.n, self.K, self.G = T, d, E, n, K, G
        self.E_loc = E // G
        self.dims = moe.dims_of(T, d, E, n, K)
        self.opts = moe.opts_of(round_mode, 1, seed)
        self.sizes = moe.query_sizes(self.dims, self.opts)
        self.routing = moe.Routing.allocate(self.dims, self.sizes, device)
        u8, bf, f32, i32 = torch.uint8, torch.bfloat16, torch.float32, torch.int32
        self.ws_route = torch.empty(self.sizes.route_ws, dtype=u8, device=device)
        self.ws_bwd = torch.empty(self.sizes.bwd_ws, dtype=u8, device=device)
        P = self.sizes.P_max
        self.send_rows = torch.empty(P, d, dtype=bf, device=device)
        self.send_gate = torch.empty(P, dtype=f32, device=device)
        self.pair_pos = torch.empty(P, dtype=i32, device=device)
        self.O = torch.empty(T, d, dtype=bf, device=device)
        self.dX = torch.empty(T, d, dtype=bf, device=device)
        self.dWr = torch.empty(d, E, dtype=f32, device=device)
        cap = G * self.sizes.P_max  # every rank may send all its routed rows here
        self.loc_opts = moe.opts_of(0, 0, 0)
        self.loc_sizes = moe.query_sizes(moe.dims_of(cap, d, self.E_loc, n, 1), self.loc_opts)
        self.loc_routing = moe.Routing.allocate(moe.dims_of(cap, d, self.E_loc, n, 1), self.loc_sizes, device,
                                                with_logits=False, with_pair_ds=True)
        self.loc_ws_route = torch.empty(self.loc_sizes.route_ws, dtype=u8, device=device)
        self.loc_ws_fwd = torch.empty(self.loc_sizes.fwd_ws, dtype=u8, device=device)
        self.loc_ws_bwd = torch.empty(self.loc_sizes.bwd_ws, dtype=u8, device=device)
        self.H_loc = torch.empty(self.loc_sizes.R_max, 2 * n, dtype=bf, device=device)
        self.out_loc = torch.empty(cap, d, dtype=bf, device=device)
        self.dXt_loc = torch.empty(cap, d, dtype=bf, device=device)
        self.dW1_loc = torch.empty(self.E_loc, d, 2 * n, dtype=bf, device=device)
        self.dW2_loc = torch.empty(self.E_loc, n, d, dtype=bf, device=device)
        self._rows = None
        self._R = 0

    def route(self, X, Wr, bias):
        self.moe.moe_route(self.dims, self.opts, X, Wr, bias, self.routing, self.ws_route)
        if self.opts.round_mode:
            self.moe.moe_token_round(self.dims, self.opts, self.routing, self.ws_route)

    def counts(self):
        return self.routing["counts"]

    def pack(self, src, with_gate, n):
        """Routed rows of `src` in expert-major send order (n of them: the
        routing's total count, known on the host from the exchange plan)."""
        m = self.moe
        m.moe_ep_pack(self.dims, self.opts, self.routing, src, self.send_rows,
                      self.send_gate if with_gate else None, self.pair_pos if with_gate else None, self.ws_route)
        return self.send_rows[:n], (self.send_gate[:n] if with_gate else None), self.pair_pos

    def _loc_dims(self, R):
        return self.moe.dims_of(R, self.d, self.E_loc, self.n, 1)

    def local_forward(self, rows, local_expert, gate, W1_loc, W2_loc):
        import torch
        m = self.moe
        R = rows.shape[0]
        self._rows, self._R = rows, R
        if R == 0:
            return self.out_loc[:0]
        rt = self.loc_routing
        rt["topk_idx"][:R, 0].copy_(local_expert)
        rt["topk_gate"][:R, 0].copy_(gate)
        dims = self._loc_dims(R)
        m.moe_route_given(dims, self.loc_opts, rt, self.loc_ws_route)
        m.moe_forward(dims, self.loc_opts, rows, W1_loc, W2_loc, rt, self.out_loc[:R], self.H_loc, self.loc_ws_fwd)
        return self.out_loc[:R]

    def local_backward(self, dO_rows, W1_loc, W2_loc):
        m = self.moe
        R = self._R
        if R == 0:
            self.dW1_loc.zero_()
            self.dW2_loc.zero_()
            return self.dXt_loc[:0], self.loc_routing["pair_dS"][:0], self.dW1_loc, self.dW2_loc
        dims = self._loc_dims(R)
        m.moe_backward(dims, self.loc_opts, dO_rows, self._rows, None, W1_loc, W2_loc, self.loc_routing, self.H_loc,
                       self.dXt_loc[:R], self.dW1_loc, self.dW2_loc, None, self.loc_ws_bwd)
        return self.dXt_loc[:R], self.loc_routing["pair_dS"][:R], self.dW1_loc, self.dW2_loc

    def combine(self, rows, pair_pos, which):
        """Sum of each token's returned rows into the layer output ("O") or
        the input gradient ("dX")."""
        out = self.O if which == "O" else self.dX
        self.moe.moe_ep_combine(self.dims, self.opts, self.routing, pair_pos, rows, out)
        return out

    def router_backward(self, X, Wr, dS, pair_pos, dX):
        self.moe.moe_router_backward(self.dims, self.opts, X, Wr, self.routing, dS, pair_pos, dX, self.dWr,
                                     self.ws_bwd)
        return self.dWr
