"""Expert-parallel engine on the fp64 oracle, for CPU ranks (gloo).

It has the interface of fine_grained_mixture_top_b200.ep.CudaEngine, with
every step computed by oracle/moe_oracle.py, so that the expert-parallel
plan and exchanges (ep.ExpertParallelMoE) can be checked on CPU against the
single-process full-batch oracle.  Test infrastructure only."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as orc


class OracleEngine:
    def __init__(self, E, K, G, round_mode=0, seed=0, tile=128):
        self.E, self.K, self.G = E, K, G
        self.E_loc = E // G
        self.round_mode, self.seed, self.tile = round_mode, seed, tile

    # ---- source side (this rank's tokens, all E experts)
    def route(self, X, Wr, bias):
        b = None if bias is None else bias.numpy()
        self.rt = orc.route(X.numpy(), Wr.numpy(), b, self.K)
        if self.round_mode:  # this rank's batch rounded on its own
            tr = orc.token_round(self.rt["probs"], self.rt["tok_ptr"], self.rt["pair_expert"], self.round_mode,
                                 self.seed, self.tile)
            self.rt.update({k: tr[k] for k in ("tok_ptr", "pair_expert", "pair_gate")})
        self.perm = orc.permute(self.rt["tok_ptr"], self.rt["pair_expert"], self.E)

    def counts(self):
        return torch.from_numpy(self.perm["counts"].astype(np.int64))

    def pack(self, src, with_gate, n):
        # expert-major rows without padding: the oracle's permutation order
        assert n == len(self.perm["row_tok"])
        rows = torch.from_numpy(np.ascontiguousarray(src.numpy()[self.perm["row_tok"]]))
        if not with_gate:
            return rows, None, None
        gate = torch.from_numpy(self.rt["pair_gate"][self.perm["row_pair"]].copy())
        pos = torch.from_numpy(self.perm["pair_row"].astype(np.int64))
        return rows, gate, pos

    def combine(self, rows, pair_pos, which):
        r = rows.numpy()
        tp = self.rt["tok_ptr"]
        out = np.zeros((len(tp) - 1, r.shape[1]))
        for t in range(len(tp) - 1):
            for p in range(tp[t], tp[t + 1]):
                out[t] += r[int(pair_pos[p])]
        return torch.from_numpy(out)

    def router_backward(self, X, Wr, dS, pair_pos, dX):
        dS_pair = dS.numpy()[pair_pos.numpy()]
        dz = orc.router_dz(dS_pair, self.rt["pair_gate"], self.rt["pair_expert"], self.rt["tok_ptr"], self.E)
        dX += torch.from_numpy(dz @ Wr.numpy().T)
        return torch.from_numpy(X.numpy().T @ dz)

    # ---- expert side (received rows, this rank's experts, K = 1)
    def local_forward(self, rows, local_expert, gate, W1_loc, W2_loc):
        R = rows.shape[0]
        self.loc_X = rows.numpy()
        rt = {"tok_ptr": np.arange(R + 1), "pair_expert": np.asarray(local_expert.numpy(), np.int64),
              "pair_gate": gate.numpy()}
        self.loc_fw = orc.forward(self.loc_X, None, None, W1_loc.numpy(), W2_loc.numpy(), 1, routing=rt)
        return torch.from_numpy(self.loc_fw["O"])

    def local_backward(self, dO_rows, W1_loc, W2_loc):
        bw = orc.backward(self.loc_fw, dO_rows.numpy(), self.loc_X, None, W1_loc.numpy(), W2_loc.numpy(),
                          router_grad=False)
        return (torch.from_numpy(bw["dX"]), torch.from_numpy(bw["dS_pair"]), torch.from_numpy(bw["dW1"]),
                torch.from_numpy(bw["dW2"]))
