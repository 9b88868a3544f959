"""Helpers of the GPU parity tests: run the layer through the C ABI and compare
with the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as orc

# Tolerances: the benchmark spec's bounds.  bf16-path outputs and gradients: max
# |gpu - ref| / max |ref| per tensor; fp32 router probabilities: absolute.
TOL_BF16 = 2e-2
TOL_PROBS = 1e-5
NEAR_TIE = 1e-4


def f64(t):
    return t.detach().to("cpu").double().numpy()


def i64(t):
    return t.detach().to("cpu").long().numpy()


def normwise(gpu, ref):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.abs(ref).max()
    if scale == 0:
        return float(np.abs(gpu).max())
    return float(np.abs(gpu - ref).max() / scale)


def elementwise(gpu, ref, floor=1e-2):
    """Largest elementwise relative error |gpu - ref| / |ref| over the entries
    with |ref| above `floor` times max |ref| (reported beside the normwise
    error; bf16 storage alone puts it near 2^-9)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    big = np.abs(ref) > floor * np.abs(ref).max()
    if not big.any():
        return 0.0
    return float((np.abs(gpu - ref)[big] / np.abs(ref)[big]).max())


def run_layer(inp, T, d, E, n, K, round_mode=0, router_grad=1, seed=0):
    import torch
    from fine_grained_mixture_top_b200 import moe
    layer = moe.MoELayer(T, d, E, n, K, round_mode=round_mode, router_grad=router_grad, seed=seed)
    layer.route(inp["X"], inp["Wr"], inp["bias"])
    layer.forward(inp["X"], inp["W1"], inp["W2"])
    layer.backward(inp["dO"], inp["X"], inp["Wr"], inp["W1"], inp["W2"])
    torch.cuda.synchronize()
    code, where = moe.moe_get_status()
    assert code == 0, (code, where)
    return layer


def gpu_routing(layer, T):
    r = layer.routing.tensors
    tok_ptr = i64(r["tok_ptr"])
    P = int(tok_ptr[T])
    return {
        "logits": f64(r["logits"]), "probs": f64(r["probs"]), "topk_idx": i64(r["topk_idx"]),
        "topk_gate": f64(r["topk_gate"]), "tok_ptr": tok_ptr, "pair_expert": i64(r["pair_expert"])[:P],
        "pair_gate": f64(r["pair_gate"])[:P], "pair_row": i64(r["pair_row"])[:P], "counts": i64(r["counts"]),
        "offsets": i64(r["offsets"]), "row_tok": i64(r["row_tok"]), "row_gate": f64(r["row_gate"]),
        "tile_expert": i64(r["tile_expert"]),
    }


def check_permutation(g, E):
    """Bit-exact check of the GPU's expert-major rows against the oracle's
    permutation of the GPU's own pairs."""
    perm = orc.permute(g["tok_ptr"], g["pair_expert"], E)
    np.testing.assert_array_equal(g["counts"], perm["counts"])
    off = g["offsets"]
    assert off[0] == 0
    for e in range(E):
        c = perm["counts"][e]
        assert off[e + 1] - off[e] == -(-c // 128) * 128
        seg = g["row_tok"][off[e]:off[e] + c]
        np.testing.assert_array_equal(seg, perm["row_tok"][perm["seg"][e]:perm["seg"][e + 1]])
        assert np.all(g["row_tok"][off[e] + c:off[e + 1]] == -1)
        assert np.all(g["row_gate"][off[e] + c:off[e + 1]] == 0.0)
        assert np.all(g["tile_expert"][off[e] // 128:off[e + 1] // 128] == e)
    # each pair's row: same position inside its segment as in the oracle
    pe = g["pair_expert"]
    np.testing.assert_array_equal(g["pair_row"] - off[pe], perm["pair_row"] - perm["seg"][pe])
    np.testing.assert_array_equal(g["row_gate"][g["pair_row"]], g["pair_gate"])
    return perm


def check_router(g, ref_z, ref_p, K):
    """probs within 1e-5; top-K exactly the oracle's on the GPU's own fp32
    logits; equal to the fp64 selection wherever the K-th/(K+1)-th gap is
    above the near-tie threshold."""
    perr = float(np.abs(g["probs"] - ref_p).max())
    zerr = float(np.abs(g["logits"] - ref_z).max())
    assert perr <= TOL_PROBS, f"probs max abs err {perr:.3e} (logits {zerr:.3e})"
    own = orc.topk_select(g["logits"], K)
    np.testing.assert_array_equal(own, g["topk_idx"])
    ref_idx = orc.topk_select(ref_z, K)
    E = ref_z.shape[1]
    if K < E:
        zs = np.sort(ref_z, axis=1)[:, ::-1]
        margin = zs[:, K - 1] - zs[:, K]
        clear = margin > NEAR_TIE
    else:
        clear = np.ones(ref_z.shape[0], bool)
    # the selected set is the fp64 one wherever the K/(K+1) gap is clear ...
    np.testing.assert_array_equal(np.sort(g["topk_idx"][clear], 1), np.sort(ref_idx[clear], 1))
    # ... and the slot order is descending in fp64 up to near-ties between slots
    zsel = np.take_along_axis(ref_z, g["topk_idx"], 1)
    assert np.all(np.diff(zsel, axis=1) <= NEAR_TIE)
    return int((~clear).sum())


def expert_rows_to_oracle_order(gpu_rows, g, perm, E):
    """Gather GPU per-row data (padded segments) into the oracle's packed order."""
    out = np.zeros((len(perm["row_tok"]),) + gpu_rows.shape[1:], gpu_rows.dtype)
    for e in range(E):
        c = perm["counts"][e]
        out[perm["seg"][e]:perm["seg"][e] + c] = gpu_rows[g["offsets"][e]:g["offsets"][e] + c]
    return out


class LazyExperts:
    """Per-expert fp64 view of a device weight tensor [E, a, b], converted on
    first use (the whole tensor may not fit on the host in fp64)."""

    def __init__(self, t, budget_bytes=6 << 30):
        self.t = t
        self.shape = tuple(t.shape)
        self.cache = {}
        self.per = 8 * int(np.prod(self.shape[1:]))
        self.cap = max(1, budget_bytes // self.per)

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            if len(self.cache) >= self.cap:
                self.cache.pop(next(iter(self.cache)))
            self.cache[e] = self.t[e].detach().to("cpu").double().numpy()
        return self.cache[e]


def sub_routing(g, z, toks):
    """The GPU's routing restricted to the tokens `toks` (CSR), with gates
    recomputed by the oracle from fp64 logits over each token's experts."""
    toks = np.asarray(toks, np.int64)
    ptr = [0]
    pe = []
    for t in toks:
        a, b = g["tok_ptr"][t], g["tok_ptr"][t + 1]
        pe.extend(g["pair_expert"][a:b].tolist())
        ptr.append(len(pe))
    tok_ptr = np.asarray(ptr, np.int64)
    pair_expert = np.asarray(pe, np.int64)
    zs = z[toks]
    return {"z": zs, "probs": orc.softmax_rows(zs), "topk_idx": g["topk_idx"][toks], "tok_ptr": tok_ptr,
            "pair_expert": pair_expert, "pair_gate": orc.gates_for_sets(zs, tok_ptr, pair_expert)}


def tokens_of_expert(g, e):
    pe = g["pair_expert"]
    pair_tok = np.repeat(np.arange(len(g["tok_ptr"]) - 1), np.diff(g["tok_ptr"]))
    return np.unique(pair_tok[pe == e])


def expert_columns_problem(g, z, e, te, J, W1, W2, n):
    """The oracle's sub-problem for columns J of expert e's weight gradients.

    SwiGLU acts column by column (A_j depends on g_j and u_j only), and
    dW1[e][:, j], dW1[e][:, n + j] and dW2[e][j, :] depend only on column j of
    the gate and up projections, on row j of W2[e] and on each row's gate s_r.
    So a layer whose only expert has the weights W1[e][:, J | n + J] and
    W2[e][J, :], fed the tokens of e with their full-set gates, has exactly the
    weight gradients dW1[e][:, J | n + J] and dW2[e][J, :] of the full layer.
    Returns (routing, W1 sub [1, d, 2|J|], W2 sub [1, |J|, d])."""
    te = np.asarray(te, np.int64)
    full = sub_routing(g, z, te)
    sel = full["pair_expert"] == e
    assert sel.sum() == len(te)
    gate = full["pair_gate"][sel]
    tok_ptr = np.arange(len(te) + 1, dtype=np.int64)
    rt = {"z": None, "probs": None, "topk_idx": np.zeros((len(te), 1), np.int64), "tok_ptr": tok_ptr,
          "pair_expert": np.zeros(len(te), np.int64), "pair_gate": gate}
    J = np.asarray(J, np.int64)
    cols = np.concatenate([J, n + J])
    W1s = np.asarray(W1[e], np.float64)[:, cols][None]
    W2s = np.asarray(W2[e], np.float64)[J, :][None]
    return rt, W1s, W2s
