"""CPU checks of the parity helpers the GPU tests rely on: the column-sampled
sub-problem for one expert's weight gradients must give exactly the full
layer's columns (oracle against oracle, fp64)."""
import numpy as np

from oracle import moe_oracle as orc

import parity as P


def test_expert_columns_problem_matches_the_full_layer():
    rng = np.random.default_rng(11)
    T, d, E, n, K = 96, 32, 6, 16, 2
    X = rng.standard_normal((T, d))
    Wr = rng.standard_normal((d, E)) * 0.3
    b = rng.standard_normal(E)
    W1 = rng.standard_normal((E, d, 2 * n)) * 0.2
    W2 = rng.standard_normal((E, n, d)) * 0.2
    dO = rng.standard_normal((T, d))
    fw = orc.forward(X, Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    g = {"tok_ptr": fw["tok_ptr"], "pair_expert": fw["pair_expert"], "topk_idx": fw["topk_idx"]}
    z = fw["z"]
    counts = np.bincount(fw["pair_expert"], minlength=E)
    for e in (int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30)))):
        te = P.tokens_of_expert(g, e)
        J = np.array([1, 4, 5, 11, 15])
        rt, W1s, W2s = P.expert_columns_problem(g, z, e, te, J, W1, W2, n)
        f2 = orc.forward(X[te], Wr, None, W1s, W2s, 1, routing=rt)
        b2 = orc.backward(f2, dO[te], X[te], Wr, W1s, W2s, router_grad=False, weight_grad_experts=[0])
        cols = np.concatenate([J, n + J])
        np.testing.assert_allclose(b2["dW1"][0], bw["dW1"][e][:, cols], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(b2["dW2"][0], bw["dW2"][e][J, :], rtol=1e-12, atol=1e-12)
    # a dropped gate (all gates 1) would not match: the check is sensitive to s_r
    rt["pair_gate"] = np.ones_like(rt["pair_gate"])
    f3 = orc.forward(X[te], Wr, None, W1s, W2s, 1, routing=rt)
    b3 = orc.backward(f3, dO[te], X[te], Wr, W1s, W2s, router_grad=False, weight_grad_experts=[0])
    assert not np.allclose(b3["dW1"][0], bw["dW1"][e][:, cols])


def test_elementwise_error_ignores_small_reference_entries():
    ref = np.array([1.0, -0.5, 1e-4, 0.0])
    gpu = np.array([1.01, -0.5, 2e-4, 1e-6])
    assert abs(P.elementwise(gpu, ref) - 0.01) < 1e-12
    assert abs(P.normwise(gpu, ref) - 0.01) < 1e-12


def test_input_subsets_hold_the_full_tensors_experts():
    import torch
    from workloads import CONFIGS, make_inputs
    cfg = CONFIGS["tiny"]
    full = make_inputs(cfg, "cpu")
    sub = make_inputs(cfg, "cpu", experts=[5, 0, 11])
    for i, e in enumerate([5, 0, 11]):
        assert torch.equal(full["W1"][e], sub["W1"][i])
        assert torch.equal(full["W2"][e], sub["W2"][i])
    assert torch.equal(full["X"], sub["X"]) and torch.equal(full["dO"], sub["dO"])
