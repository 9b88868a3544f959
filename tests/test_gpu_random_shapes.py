"""GPU parity over seeded random shapes: token counts from 1 to a few
thousand (a single token, fewer than a tile, ragged tails), one to 130
experts (one expert, E not a multiple of 64, K = E), the smallest d and n the
boundary accepts, with and without router bias, router gradient and token
rounding.  Each case runs the whole path through the C ABI and is compared
with the fp64 oracle like the fixed shapes of test_gpu_parity.py."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from workloads import MoEConfig, make_inputs

import parity as P

torch = pytest.importorskip("torch")


def _cases(n_cases=14, seed=2024):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n_cases):
        E = int(rng.choice([1, 2, 3, 5, 8, 16, 33, 64, 65, 130]))
        K = int(rng.integers(1, min(E, 8) + 1))
        T = int(rng.choice([1, 7, 100, 129, 256, 1000, 1500, 3000]))
        d = int(rng.choice([128, 256, 384, 512]))
        n = int(rng.choice([64, 128, 192, 256, 320]))
        bias = str(rng.choice(["none", "normal"]))
        rmode = int(rng.choice([0, 0, 1, 2])) if T * K >= 256 else 0
        rg = int(rng.choice([0, 1, 1]))
        out.append((MoEConfig(f"r{i}_T{T}_d{d}_E{E}_n{n}_K{K}_bias{int(bias != 'none')}_tr{rmode}_rg{rg}", T=T, d=d,
                              E=E, n=n, K=K, w_std=0.05, bias=bias, seed=100 + i, round_mode=rmode), rg))
    # two fixed corners: E = 130 (padded to 192 router columns) with K = 8 and
    # rounding; a wide d with an odd expert count
    out.append((MoEConfig("c0_T777_d128_E130_n64_K8_bias1_tr2_rg1", T=777, d=128, E=130, n=64, K=8, w_std=0.05,
                          bias="normal", seed=150, round_mode=2), 1))
    out.append((MoEConfig("c1_T2048_d640_E33_n128_K7_bias0_tr0_rg1", T=2048, d=640, E=33, n=128, K=7, w_std=0.05,
                          seed=151), 1))
    return out


CASES = _cases()


@pytest.mark.gpu
@pytest.mark.parametrize("cfg,rg", CASES, ids=[c.name for c, _ in CASES])
def test_random_shape_parity(cfg, rg):
    inp = make_inputs(cfg, "cuda")
    seed = 77
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=cfg.round_mode, router_grad=rg,
                        seed=seed)
    g = P.gpu_routing(layer, cfg.T)
    X, Wr = P.f64(inp["X"]), P.f64(inp["Wr"])
    b = None if inp["bias"] is None else P.f64(inp["bias"])
    W1, W2, dO = P.f64(inp["W1"]), P.f64(inp["W2"]), P.f64(inp["dO"])
    z = orc.router_logits(X, Wr, b)
    P.check_router(g, z, orc.softmax_rows(z), cfg.K)
    if cfg.round_mode:
        # rounding decisions in the GPU's fp32 probs, bit-exact
        tok_ptr0, pe0 = orc.pairs_from_topk(g["topk_idx"])
        tr = orc.token_round(g["probs"], tok_ptr0, pe0, cfg.round_mode, seed)
        np.testing.assert_array_equal(g["tok_ptr"], tr["tok_ptr"])
        np.testing.assert_array_equal(g["pair_expert"], tr["pair_expert"])
        routing = {"z": z, "probs": orc.softmax_rows(z), "topk_idx": g["topk_idx"], "tok_ptr": tr["tok_ptr"],
                   "pair_expert": tr["pair_expert"],
                   "pair_gate": orc.gates_for_sets(z, tr["tok_ptr"], tr["pair_expert"])}
        fw = orc.forward(X, Wr, b, W1, W2, cfg.K, routing=routing)
    else:
        fw = orc.forward(X, Wr, b, W1, W2, cfg.K, topk_idx=g["topk_idx"])
    np.testing.assert_allclose(g["pair_gate"], fw["pair_gate"], rtol=1e-5, atol=1e-7)
    perm = P.check_permutation(g, cfg.E)
    assert np.all(g["counts"] % 128 == 0) or not cfg.round_mode
    bw = orc.backward(fw, dO, X, Wr, W1, W2, router_grad=bool(rg))
    errs = {"O": P.normwise(P.f64(layer.O), fw["O"]),
            "H": P.normwise(P.expert_rows_to_oracle_order(P.f64(layer.H), g, perm, cfg.E), fw["H"]),
            "dX": P.normwise(P.f64(layer.dX), bw["dX"]),
            "dW1": P.normwise(P.f64(layer.dW1), bw["dW1"]),
            "dW2": P.normwise(P.f64(layer.dW2), bw["dW2"])}
    if rg:
        errs["dWr"] = P.normwise(P.f64(layer.dWr), bw["dWr"])
    print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= P.TOL_BF16, (k, v)
