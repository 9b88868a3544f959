"""Parity at the full sizes of every workload, in the launch configuration the
benchmark uses: routing, permutation and token rounding checked on every token
(bit-exact after the near-tie rule); O and dX on sampled tokens and dW1, dW2
and the dWr columns of sampled experts, each computed by the oracle from only
the rows it needs."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from workloads import CONFIGS, make_inputs

import parity as P

torch = pytest.importorskip("torch")

FULL = ["7b", "qwen3", "dsv3", "olmoe"] + sorted(k for k in CONFIGS if k.startswith("sweep"))


def _budget(cfg):
    """(sampled tokens, sampled experts: the least loaded, then the median),
    scaled so the fp64 oracle finishes in seconds to a minute per layer."""
    big = cfg.d * cfg.n > 1536 * 768
    return (16, 1) if big else (128, 2)


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
    ntok, nexp = _budget(cfg)
    rs = np.random.RandomState(cfg.seed + 7)
    toks = np.sort(rs.choice(cfg.T, ntok, replace=False))
    sub = P.sub_routing(g, z, toks)
    fw = orc.forward(X[toks], Wr, b, W1, W2, cfg.K, routing=sub)
    bw = orc.backward(fw, dO[toks], X[toks], Wr, W1, W2, weight_grad_experts=[])
    errs = {"O": P.normwise(P.f64(layer.O[toks]), fw["O"]), "dX": P.normwise(P.f64(layer.dX[toks]), bw["dX"])}

    counts = g["counts"]
    nz = np.nonzero(counts > 0)[0]
    picks = [nz[np.argmin(counts[nz])], nz[np.argsort(counts[nz])[len(nz) // 2]]]
    for e in sorted(set(int(x) for x in picks[:nexp])):
        te = P.tokens_of_expert(g, e)
        sub = P.sub_routing(g, z, te)
        fw = orc.forward(X[te], Wr, b, W1, W2, cfg.K, routing=sub)
        bw = orc.backward(fw, dO[te], X[te], Wr, W1, W2, weight_grad_experts=[e])
        errs[f"dW1[{e}]"] = P.normwise(P.f64(layer.dW1[e]), bw["dW1"][e])
        errs[f"dW2[{e}]"] = P.normwise(P.f64(layer.dW2[e]), bw["dW2"][e])
        errs[f"dWr[:,{e}]"] = P.normwise(P.f64(layer.dWr[:, e]), bw["dWr"][:, e])
    print(name, "near-ties:", near, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= P.TOL_BF16, (k, v)
