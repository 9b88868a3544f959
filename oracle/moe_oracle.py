"""Plain fp64 CPU reference ("the oracle") of the fine-grained MoE expert layer.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does, and this
module imports nothing from the product package.

Every step is written out in the order the pages describe it, with numpy fp64
matmuls as the only library primitive; there is no tiling, fusion or reordering
beyond what the layer's definition states.

Sources (scraped web pages on SonicMoE):
  [P1] "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE" -- news article on the
       SonicMoE Blackwell blog; sections "MoE 与它的隐患" (MoE and its hazards),
       "核心创新：一次算法级的重新设计" (core innovation), "实验结果" (results).
  [P2] "SonicMoE：突破细粒度MoE硬件效率瓶颈，实现高稀疏性下的极致训练加速" --
       summary of the SonicMoE paper; paragraphs on the algorithm level (router
       gradient without cached activations), the scheduling level (token
       rounding) and the implementation details (the eight kernels).

Readings where the pages are silent (each listed in the design notes):
  R1 SwiGLU layout: W1[e][:, :n] is the gate projection g, W1[e][:, n:] the up
     projection u; A = silu(g) * u with silu(x) = x * sigmoid(x).
  R2 Gates: p = softmax over all E logits, top-K taken, gates renormalised to
     sum 1 (equal to a softmax over the K selected logits).
  R3 Top-K ties go to the lower expert index; slots ordered by descending
     logit, then ascending expert index.
  R4 Inside an expert segment rows are in ascending token order.
  R5 The backward includes the router path: dX gets dz @ Wr^T, dWr = X^T dz.
  R6 The router bias b (skewed loads) is added to the logits before softmax.
  R7 Token rounding: see token_round().

Parity status: every function here is pinned by tests under tests/ (brute-force
per-token loops, the E=1,K=1 dense special case, central finite differences,
the naive cached-output router gradient, routing/permutation/rounding
invariants, published splitmix64 outputs). The pages print no numeric example,
so no value here is pinned to a number printed on the pages.
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
MASK64 = (1 << 64) - 1


# --------------------------------------------------------------------------
# Router.  [P1] "MoE 与它的隐患": each token is sent to a small subset of the
# experts chosen by a router; spec shapes X[T,d], Wr[d,E].
# --------------------------------------------------------------------------
def router_logits(X, Wr, bias=None):
    """z[t, e] = sum_i X[t, i] * Wr[i, e] (+ b[e])   (fp64)."""
    z = np.asarray(X, F64) @ np.asarray(Wr, F64)
    if bias is not None:
        z = z + np.asarray(bias, F64)[None, :]
    return z


def softmax_rows(z):
    """p[t, :] = exp(z[t, :] - max) / sum exp(z[t, :] - max)."""
    z = np.asarray(z, F64)
    m = z.max(axis=1, keepdims=True)
    ez = np.exp(z - m)
    return ez / ez.sum(axis=1, keepdims=True)


def topk_select(z, K):
    """Indices of the K largest logits per row (R3: ties to the lower index).

    A stable sort of -z keeps equal keys in ascending index order.
    """
    z = np.asarray(z, F64)
    order = np.argsort(-z, axis=1, kind="stable")
    return order[:, :K].astype(np.int64)


def gates_for_sets(z, tok_ptr, pair_expert):
    """Gate of every (token, expert) pair: softmax over that token's selected
    logits (R2), i.e. p[t,e] / sum_{e' in S_t} p[t,e']."""
    z = np.asarray(z, F64)
    T = z.shape[0]
    g = np.zeros(len(pair_expert), F64)
    for t in range(T):
        a, b = tok_ptr[t], tok_ptr[t + 1]
        if b == a:
            continue
        zs = z[t, pair_expert[a:b]]
        ez = np.exp(zs - zs.max())
        g[a:b] = ez / ez.sum()
    return g


def pairs_from_topk(topk_idx):
    """CSR over tokens of the K selected experts: tok_ptr[T+1], pair_expert[T*K]."""
    topk_idx = np.asarray(topk_idx, np.int64)
    T, K = topk_idx.shape
    tok_ptr = np.arange(T + 1, dtype=np.int64) * K
    return tok_ptr, topk_idx.reshape(-1).copy()


# --------------------------------------------------------------------------
# Permutation into per-expert segments.  [P1] "核心创新" (gather fusion: the
# GEMM reads the routed rows directly); [P1] "MoE 与它的隐患" figure caption:
# the standard implementation stores the routing metadata pi.
# --------------------------------------------------------------------------
def permute(tok_ptr, pair_expert, E):
    """Expert-major order of all (token, expert) pairs (R4).

    Returns counts[E], seg[E+1] (exclusive prefix sum of counts), row_tok[R]
    (token of each row), pair_row[P] (row of each pair) and row_pair[R].
    """
    tok_ptr = np.asarray(tok_ptr, np.int64)
    pair_expert = np.asarray(pair_expert, np.int64)
    T = len(tok_ptr) - 1
    P = len(pair_expert)
    pair_tok = np.repeat(np.arange(T, dtype=np.int64), np.diff(tok_ptr))
    counts = np.zeros(E, np.int64)
    for p in range(P):
        counts[pair_expert[p]] += 1
    seg = np.zeros(E + 1, np.int64)
    seg[1:] = np.cumsum(counts)
    fill = seg[:-1].copy()
    row_tok = np.empty(P, np.int64)
    row_pair = np.empty(P, np.int64)
    pair_row = np.empty(P, np.int64)
    # tokens in ascending order; each token holds an expert at most once
    for t in range(T):
        for p in range(tok_ptr[t], tok_ptr[t + 1]):
            e = pair_expert[p]
            r = fill[e]
            fill[e] += 1
            row_tok[r] = t
            row_pair[r] = p
            pair_row[p] = r
    return {"counts": counts, "seg": seg, "row_tok": row_tok,
            "pair_row": pair_row, "row_pair": row_pair, "pair_tok": pair_tok}


# --------------------------------------------------------------------------
# Expert MLP.  [P2] implementation paragraph: forward kernels up-proj (A),
# down-proj (Y), expert aggregation (O); [P1] "第二，IO 感知的算子融合":
# SwiGLU is applied to the up-projection output (R1).
# --------------------------------------------------------------------------
def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def silu(x):
    return x * sigmoid(x)


def swiglu(H, n):
    """A = silu(g) * u with g = H[:, :n], u = H[:, n:2n]."""
    return silu(H[:, :n]) * H[:, n:2 * n]


def expert_rows_forward(X, W1, W2, perm):
    """H_r = X[tok_r] @ W1[e_r];  A_r = SwiGLU(H_r);  Y_r = A_r @ W2[e_r]."""
    X = np.asarray(X, F64)
    E, d, n2 = W1.shape
    n = n2 // 2
    R = len(perm["row_tok"])
    H = np.zeros((R, 2 * n), F64)
    A = np.zeros((R, n), F64)
    Y = np.zeros((R, d), F64)
    seg = perm["seg"]
    for e in range(E):
        a, b = seg[e], seg[e + 1]
        if b == a:
            continue
        Xe = X[perm["row_tok"][a:b]]
        H[a:b] = Xe @ np.asarray(W1[e], F64)
        A[a:b] = swiglu(H[a:b], n)
        Y[a:b] = A[a:b] @ np.asarray(W2[e], F64)
    return H, A, Y


def aggregate(Y, pair_gate, pair_row, tok_ptr, T):
    """O_t = sum over the pairs p of token t of gate_p * Y[row(p)]."""
    O = np.zeros((T, Y.shape[1]), F64)
    for t in range(T):
        for p in range(tok_ptr[t], tok_ptr[t + 1]):
            O[t] += pair_gate[p] * Y[pair_row[p]]
    return O


# --------------------------------------------------------------------------
# Full layer.
# --------------------------------------------------------------------------
def route(X, Wr, bias, K, topk_idx=None):
    """Router stage: logits, probabilities, top-K (or the given selection),
    CSR pairs and gates."""
    z = router_logits(X, Wr, bias)
    p = softmax_rows(z)
    if topk_idx is None:
        topk_idx = topk_select(z, K)
    tok_ptr, pair_expert = pairs_from_topk(topk_idx)
    pair_gate = gates_for_sets(z, tok_ptr, pair_expert)
    return {"z": z, "probs": p, "topk_idx": np.asarray(topk_idx, np.int64),
            "tok_ptr": tok_ptr, "pair_expert": pair_expert, "pair_gate": pair_gate}


def forward(X, Wr, bias, W1, W2, K, topk_idx=None, routing=None):
    """Layer forward.  Returns a dict with O and every intermediate."""
    X = np.asarray(X, F64)
    T = X.shape[0]
    E = W1.shape[0]
    rt = routing if routing is not None else route(X, Wr, bias, K, topk_idx)
    perm = permute(rt["tok_ptr"], rt["pair_expert"], E)
    H, A, Y = expert_rows_forward(X, W1, W2, perm)
    O = aggregate(Y, rt["pair_gate"], perm["pair_row"], rt["tok_ptr"], T)
    out = dict(rt)
    out.update(perm)
    out.update({"H": H, "A": A, "Y": Y, "O": O})
    return out


def backward(fw, dO, X, Wr, W1, W2, router_grad=True, weight_grad_experts=None):
    """Layer backward as the method orders it ([P2] implementation paragraph:
    activation-gradient kernels dH (down-proj), the up-proj activation gradient,
    dX aggregation, and the two weight-gradient kernels dW1, dW2).

    The router-score gradient uses dS = <dA'_r, A_r> with dA'_r =
    dO[tok_r] @ W2[e]^T, so no per-expert output Y is needed ([P2] algorithm
    paragraph; [P1] "第一，激活内存与专家粒度解耦": the contraction order is
    rearranged so the down-projection output is not cached, and no extra
    matmul is recomputed).

    weight_grad_experts: None computes dW1/dW2 for every expert as [E, ...]
    arrays; a list computes them only for those experts and returns dicts
    {expert: array} (for layers whose full weight gradients do not fit in
    host memory).  The arithmetic is the same either way.
    """
    X = np.asarray(X, F64)
    dO = np.asarray(dO, F64)
    T, d = X.shape
    E, _, n2 = W1.shape
    n = n2 // 2
    seg, row_tok = fw["seg"], fw["row_tok"]
    R = len(row_tok)
    row_gate = fw["pair_gate"][fw["row_pair"]]
    H = fw["H"]
    dH = np.zeros((R, 2 * n), F64)
    Ahat = np.zeros((R, n), F64)
    dS_row = np.zeros(R, F64)
    dXt = np.zeros((R, d), F64)
    if weight_grad_experts is None:
        dW1 = np.zeros((E, d, 2 * n), F64)
        dW2 = np.zeros((E, n, d), F64)
        wanted = set(range(E))
    else:
        dW1, dW2 = {}, {}
        wanted = set(int(e) for e in weight_grad_experts)
        for e in wanted:
            dW1[e] = np.zeros((d, 2 * n), F64)
            dW2[e] = np.zeros((n, d), F64)
    for e in range(E):
        a, b = seg[e], seg[e + 1]
        if b == a:
            continue
        W1e = np.asarray(W1[e], F64)
        W2e = np.asarray(W2[e], F64)
        dOe = dO[row_tok[a:b]]
        s = row_gate[a:b][:, None]
        # dH kernel: dA' = dO[tok] W2^T; recompute A from H; dS; dSwiGLU
        dAp = dOe @ W2e.T
        g, u = H[a:b, :n], H[a:b, n:]
        sg = sigmoid(g)
        A = g * sg * u
        dS_row[a:b] = np.sum(dAp * A, axis=1)
        dA = s * dAp
        dg = dA * u * sg * (1.0 + g * (1.0 - sg))
        du = dA * g * sg
        dH[a:b, :n] = dg
        dH[a:b, n:] = du
        Ahat[a:b] = s * A
        # weight gradients and the up-proj activation gradient
        dXt[a:b] = dH[a:b] @ W1e.T
        if e in wanted:
            dW2[e] = Ahat[a:b].T @ dOe
            dW1[e] = X[row_tok[a:b]].T @ dH[a:b]
    # dX aggregation over each token's pairs
    tok_ptr, pair_row, pair_expert, pair_gate = (fw["tok_ptr"], fw["pair_row"],
                                                 fw["pair_expert"], fw["pair_gate"])
    dX = np.zeros((T, d), F64)
    for t in range(T):
        for p in range(tok_ptr[t], tok_ptr[t + 1]):
            dX[t] += dXt[pair_row[p]]
    out = {"dH": dH, "Ahat": Ahat, "dS_row": dS_row, "dXt": dXt,
           "dW1": dW1, "dW2": dW2, "dX_expert": dX.copy()}
    dS_pair = dS_row[pair_row]
    out["dS_pair"] = dS_pair
    if router_grad:
        dz = router_dz(dS_pair, pair_gate, pair_expert, tok_ptr, E)
        dWr = X.T @ dz
        dX = dX + dz @ np.asarray(Wr, F64).T
        out.update({"dz": dz, "dWr": dWr})
    out["dX"] = dX
    return out


def router_dz(dS_pair, pair_gate, pair_expert, tok_ptr, E):
    """Gradient of the loss w.r.t. the router logits.

    Gates are a softmax over each token's selected logits (R2), so for e in
    S_t: dz[t,e] = s_e * (dS_e - sum_{j in S_t} s_j dS_j); zero elsewhere.
    """
    T = len(tok_ptr) - 1
    dz = np.zeros((T, E), F64)
    for t in range(T):
        a, b = tok_ptr[t], tok_ptr[t + 1]
        if b == a:
            continue
        s = pair_gate[a:b]
        dS = dS_pair[a:b]
        inner = float(np.sum(s * dS))
        dz[t, pair_expert[a:b]] = s * (dS - inner)
    return dz


# --------------------------------------------------------------------------
# Plain-definition forms used to pin the method's form.
# --------------------------------------------------------------------------
def forward_bruteforce(X, Wr, bias, W1, W2, K, topk_idx=None):
    """Per-token loops over each token's experts: O_t = sum_k s_k MLP_e(X_t)."""
    X = np.asarray(X, F64)
    T, d = X.shape
    n = W1.shape[2] // 2
    z = router_logits(X, Wr, bias)
    O = np.zeros((T, d), F64)
    for t in range(T):
        if topk_idx is None:
            sel = sorted(range(z.shape[1]), key=lambda e: (-z[t, e], e))[:K]
        else:
            sel = [int(e) for e in topk_idx[t]]
        zs = np.array([z[t, e] for e in sel])
        w = np.exp(zs - zs.max())
        w = w / w.sum()
        for k, e in enumerate(sel):
            h = X[t] @ np.asarray(W1[e], F64)
            a = silu(h[:n]) * h[n:]
            O[t] += w[k] * (a @ np.asarray(W2[e], F64))
    return O


def router_dS_naive(fw, dO):
    """dS for each pair from the cached down-proj output: dS_p = <dO_t, Y_row(p)>."""
    dO = np.asarray(dO, F64)
    Y = fw["Y"]
    P = len(fw["pair_row"])
    out = np.zeros(P, F64)
    for t in range(dO.shape[0]):
        for p in range(fw["tok_ptr"][t], fw["tok_ptr"][t + 1]):
            out[p] = float(dO[t] @ Y[fw["pair_row"][p]])
    return out


def loss(O, dO):
    """Scalar loss whose gradient w.r.t. O is dO: L = sum(O * dO)."""
    return float(np.sum(np.asarray(O, F64) * np.asarray(dO, F64)))


# --------------------------------------------------------------------------
# Token rounding.  [P2] scheduling paragraph: the number of tokens sent to each
# expert is rounded to a multiple of the grouped-GEMM tile (e.g. 128), each
# expert deviates by at most one tile, the total is preserved in expectation.
# Readings (R7), where the pages are silent:
#   r = c_e mod tile; r == 0 leaves e unchanged.
#   mode 1 "nearest": round up iff r >= tile/2.
#   mode 2 "stochastic": round up iff splitmix64(seed XOR e) mod tile < r,
#     which rounds up with probability r/tile, so E[c'_e] = c_e.
#   Rounding up never exceeds T tokens (round down instead).
#   Down: drop the r routed tokens with the smallest p[t,e] (ties: larger t
#     dropped first).  Up: add the tile - r unrouted tokens with the largest
#     p[t,e] (ties: smaller t first).
#   Afterwards each token's gates are p[t,e] renormalised over its final set;
#   pairs of a token are listed in ascending expert order.  Probabilities are
#   compared in the precision they are given in.
# --------------------------------------------------------------------------
def splitmix64(x: int) -> int:
    """First output of Steele-Lea-Flood's SplitMix64 generator seeded with x
    (golden-gamma increment, then the variant-13 finaliser)."""
    z = (int(x) + 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def round_up_decision(c: int, e: int, T: int, mode: int, seed: int, tile: int = 128) -> bool:
    r = c % tile
    if r == 0:
        return False
    if mode == 1:
        up = r >= tile // 2
    elif mode == 2:
        up = (splitmix64((int(seed) ^ int(e)) & MASK64) % tile) < r
    else:
        raise ValueError("mode must be 1 or 2")
    if up and c - r + tile > T:
        up = False
    return up


def token_round(probs, tok_ptr, pair_expert, mode, seed, tile=128):
    """Rounded routing: returns tok_ptr', pair_expert', pair_gate' and the
    per-expert decisions."""
    probs = np.asarray(probs, F64)
    T, E = probs.shape
    member = np.zeros((T, E), bool)
    for t in range(T):
        for p in range(tok_ptr[t], tok_ptr[t + 1]):
            member[t, pair_expert[p]] = True
    new = member.copy()
    decisions = np.zeros(E, np.int64)   # +1 up, -1 down, 0 unchanged
    for e in range(E):
        c = int(member[:, e].sum())
        r = c % tile
        if r == 0:
            continue
        if round_up_decision(c, e, T, mode, seed, tile):
            decisions[e] = 1
            cand = np.nonzero(~member[:, e])[0]
            # primary key: p descending; secondary: t ascending
            order = np.lexsort((cand, -probs[cand, e]))
            new[cand[order[:tile - r]], e] = True
        else:
            decisions[e] = -1
            cand = np.nonzero(member[:, e])[0]
            # primary key: p ascending; secondary: t descending
            order = np.lexsort((-cand, probs[cand, e]))
            new[cand[order[:r]], e] = False
    counts = new.sum(axis=0)
    new_ptr = np.zeros(T + 1, np.int64)
    new_ptr[1:] = np.cumsum(new.sum(axis=1))
    new_exp = np.zeros(int(new_ptr[-1]), np.int64)
    new_gate = np.zeros(int(new_ptr[-1]), F64)
    for t in range(T):
        es = np.nonzero(new[t])[0]
        a = new_ptr[t]
        new_exp[a:a + len(es)] = es
        if len(es):
            ps = probs[t, es]
            new_gate[a:a + len(es)] = ps / ps.sum()
    return {"tok_ptr": new_ptr, "pair_expert": new_exp, "pair_gate": new_gate,
            "counts": counts, "decisions": decisions, "member": new}
