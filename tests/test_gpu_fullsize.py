"""Parity at the full sizes of every workload, in the launch configuration the
benchmark uses: routing, permutation and token rounding checked on every token
(bit-exact after the near-tie rule); O and dX on sampled tokens; dW1, dW2
and the dWr column of the least-loaded, median and most-loaded experts, each
computed by the oracle from only the rows it needs (on sampled columns where
an expert's tokens are too many for the whole layer in fp64).  Normwise errors
are asserted; elementwise relative errors are reported beside them."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from workloads import CONFIGS, make_inputs

import parity as P

torch = pytest.importorskip("torch")

FULL = ["7b", "qwen3", "dsv3", "olmoe"] + sorted(k for k in CONFIGS if k.startswith("sweep"))


# fp64 oracle work allowed for one expert's full check (its tokens through
# the whole layer, forward and backward): above it, the expert's weight
# gradients are checked on sampled columns instead (expert_columns_problem)
FULL_EXPERT_FLOPS = 2e12
SAMPLED_COLUMNS = 64


def _budget(cfg):
    """Sampled tokens for O and dX, scaled so the fp64 oracle finishes in
    seconds to a minute per layer."""
    big = cfg.d * cfg.n > 1536 * 768
    return 64 if big else 128


@pytest.mark.gpu
@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled(name):
    cfg = CONFIGS[name]
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=cfg.round_mode, seed=cfg.seed)
    g = P.gpu_routing(layer, cfg.T)
    X = P.f64(inp["X"])
    Wr = P.f64(inp["Wr"])
    b = None if inp["bias"] is None else P.f64(inp["bias"])
    dO = P.f64(inp["dO"])
    z = orc.router_logits(X, Wr, b)
    near = P.check_router(g, z, orc.softmax_rows(z), cfg.K)
    if cfg.round_mode:
        tok_ptr0, pe0 = orc.pairs_from_topk(g["topk_idx"])
        tr = orc.token_round(g["probs"], tok_ptr0, pe0, cfg.round_mode, cfg.seed)
        np.testing.assert_array_equal(g["tok_ptr"], tr["tok_ptr"])
        np.testing.assert_array_equal(g["pair_expert"], tr["pair_expert"])
        assert np.all(g["counts"] % 128 == 0)
        assert np.all(np.abs(g["counts"] - np.bincount(pe0, minlength=cfg.E)) < 128)
    P.check_permutation(g, cfg.E)
    np.testing.assert_allclose(g["pair_gate"], orc.gates_for_sets(z, g["tok_ptr"], g["pair_expert"]),
                               rtol=1e-5, atol=1e-7)

    W1 = P.LazyExperts(inp["W1"])
    W2 = P.LazyExperts(inp["W2"])
    ntok = _budget(cfg)
    rs = np.random.RandomState(cfg.seed + 7)
    toks = np.sort(rs.choice(cfg.T, ntok, replace=False))
    sub = P.sub_routing(g, z, toks)
    fw = orc.forward(X[toks], Wr, b, W1, W2, cfg.K, routing=sub)
    bw = orc.backward(fw, dO[toks], X[toks], Wr, W1, W2, weight_grad_experts=[])
    pairs = {"O": (P.f64(layer.O[toks]), fw["O"]), "dX": (P.f64(layer.dX[toks]), bw["dX"])}

    # the least-loaded, the median and the most-loaded expert: the last has
    # the longest K loop of the weight-gradient kernels and is the first tile
    # their largest-first queue hands out
    counts = g["counts"]
    nz = np.nonzero(counts > 0)[0]
    order = nz[np.argsort(counts[nz], kind="stable")]
    picks = sorted(set(int(x) for x in (order[0], order[len(order) // 2], order[-1])))
    for e in picks:
        te = P.tokens_of_expert(g, e)
        if 18.0 * len(te) * cfg.K * cfg.d * cfg.n <= FULL_EXPERT_FLOPS:
            sub = P.sub_routing(g, z, te)
            fw = orc.forward(X[te], Wr, b, W1, W2, cfg.K, routing=sub)
            bw = orc.backward(fw, dO[te], X[te], Wr, W1, W2, weight_grad_experts=[e])
            pairs[f"dW1[{e}]"] = (P.f64(layer.dW1[e]), bw["dW1"][e])
            pairs[f"dW2[{e}]"] = (P.f64(layer.dW2[e]), bw["dW2"][e])
            pairs[f"dWr[:,{e}]"] = (P.f64(layer.dWr[:, e]), bw["dWr"][:, e])
        else:
            # too many tokens for the whole layer in fp64: sampled columns of
            # this expert's weight gradients, from the exact sub-problem
            J = np.sort(rs.choice(cfg.n, SAMPLED_COLUMNS, replace=False))
            rt, W1s, W2s = P.expert_columns_problem(g, z, e, te, J, W1, W2, cfg.n)
            fw = orc.forward(X[te], Wr, None, W1s, W2s, 1, routing=rt)
            bw = orc.backward(fw, dO[te], X[te], Wr, W1s, W2s, router_grad=False, weight_grad_experts=[0])
            cols = np.concatenate([J, cfg.n + J])
            pairs[f"dW1[{e}][:,J]"] = (P.f64(layer.dW1[e][:, torch.as_tensor(cols, device=layer.dW1.device)]),
                                       bw["dW1"][0])
            pairs[f"dW2[{e}][J,:]"] = (P.f64(layer.dW2[e][torch.as_tensor(J, device=layer.dW2.device)]),
                                       bw["dW2"][0])
    errs = {k: P.normwise(gv, rv) for k, (gv, rv) in pairs.items()}
    elem = {k: P.elementwise(gv, rv) for k, (gv, rv) in pairs.items()}
    print(name, "near-ties:", near, "expert rows:", {e: int(counts[e]) for e in picks})
    print("  normwise:   ", {k: f"{v:.2e}" for k, v in errs.items()})
    print("  elementwise:", {k: f"{v:.2e}" for k, v in elem.items()})
    for k, v in errs.items():
        assert v <= P.TOL_BF16, (k, v)
