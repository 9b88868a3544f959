"""Pins of the fp64 oracle against facts fixed by the pages and by mathematics:
brute-force per-token loops, the dense special case, central finite
differences, the naive cached-output router gradient, routing invariants and an
independent stable sort.  CPU only."""
import math

import numpy as np
import pytest

from oracle import moe_oracle as orc


def rand_layer(T, d, E, n, K, seed, xs=1.0, ws=0.3, wrs=0.5, bias=False):
    rs = np.random.RandomState(seed)
    X = rs.randn(T, d) * xs
    W1 = rs.randn(E, d, 2 * n) * ws
    W2 = rs.randn(E, n, d) * ws
    Wr = rs.randn(d, E) * wrs
    b = rs.randn(E) * 0.5 if bias else None
    dO = rs.randn(T, d)
    return X, W1, W2, Wr, b, dO


# ---------------------------------------------------------------- routing
def test_topk_matches_full_sort_with_ties():
    rs = np.random.RandomState(0)
    z = rs.randint(-3, 4, size=(200, 12)).astype(float)   # many exact ties
    K = 4
    idx = orc.topk_select(z, K)
    for t in range(z.shape[0]):
        brute = sorted(range(12), key=lambda e: (-z[t, e], e))[:K]
        assert list(idx[t]) == brute


def test_routing_invariants():
    X, W1, W2, Wr, b, _ = rand_layer(300, 16, 10, 4, 3, 1, bias=True)
    rt = orc.route(X, Wr, b, 3)
    idx = rt["topk_idx"]
    assert idx.shape == (300, 3)
    for t in range(300):
        assert len(set(idx[t])) == 3
        assert all(0 <= e < 10 for e in idx[t])
        s = rt["pair_gate"][3 * t:3 * t + 3]
        assert abs(s.sum() - 1.0) < 1e-12
        assert np.all(np.diff(s) <= 1e-15)          # sorted by descending logit
        # gate = p / sum(p) over the selected set
        p = rt["probs"][t, idx[t]]
        np.testing.assert_allclose(s, p / p.sum(), rtol=1e-12)
    np.testing.assert_allclose(rt["probs"].sum(axis=1), 1.0, rtol=1e-12)
    # bias enters before the softmax
    z0 = X @ Wr
    np.testing.assert_allclose(rt["z"], z0 + b[None, :], rtol=1e-13)


def test_permutation_matches_stable_argsort():
    rs = np.random.RandomState(2)
    T, E, K = 500, 9, 3
    idx = np.stack([rs.choice(E, K, replace=False) for _ in range(T)])
    tok_ptr, pe = orc.pairs_from_topk(idx)
    perm = orc.permute(tok_ptr, pe, E)
    order = np.argsort(pe, kind="stable")        # independent routine
    np.testing.assert_array_equal(perm["row_pair"], order)
    np.testing.assert_array_equal(perm["row_tok"], order // K)
    np.testing.assert_array_equal(perm["counts"], np.bincount(pe, minlength=E))
    assert perm["counts"].sum() == T * K
    # rows of each segment ascend in token order; pair_row inverts row_pair
    for e in range(E):
        a, b = perm["seg"][e], perm["seg"][e + 1]
        assert np.all(np.diff(perm["row_tok"][a:b]) > 0)
        assert np.all(pe[perm["row_pair"][a:b]] == e)
    np.testing.assert_array_equal(perm["row_pair"][perm["pair_row"]], np.arange(T * K))


# ---------------------------------------------------------------- forward
@pytest.mark.parametrize("bias", [False, True])
def test_forward_matches_bruteforce(bias):
    X, W1, W2, Wr, b, _ = rand_layer(96, 24, 7, 8, 3, 3, bias=bias)
    fw = orc.forward(X, Wr, b, W1, W2, 3)
    O_bf = orc.forward_bruteforce(X, Wr, b, W1, W2, 3)
    np.testing.assert_allclose(fw["O"], O_bf, rtol=1e-12, atol=1e-12)


def test_tiny_config_forward_matches_bruteforce():
    from workloads import CONFIGS, make_inputs
    cfg = CONFIGS["tiny"]
    inp = make_inputs(cfg, "cpu")
    X = inp["X"].double().numpy()
    W1 = inp["W1"].double().numpy()
    W2 = inp["W2"].double().numpy()
    Wr = inp["Wr"].double().numpy()
    fw = orc.forward(X, Wr, None, W1, W2, cfg.K)
    O_bf = orc.forward_bruteforce(X, Wr, None, W1, W2, cfg.K)
    scale = np.abs(O_bf).max()
    assert scale > 0
    assert np.abs(fw["O"] - O_bf).max() <= 1e-12 * scale


def test_dense_special_case_E1_K1():
    """One expert, top-1: the layer is a dense SwiGLU MLP with gate 1."""
    X, W1, W2, Wr, _, _ = rand_layer(40, 12, 1, 6, 1, 4)
    fw = orc.forward(X, Wr, None, W1, W2, 1)
    h = X @ W1[0]
    g, u = h[:, :6], h[:, 6:]
    dense = (g / (1.0 + np.exp(-g)) * u) @ W2[0]
    np.testing.assert_allclose(fw["O"], dense, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fw["pair_gate"], 1.0)


def test_hand_worked_single_token():
    """T=1, d=1, E=2, n=1, K=1 -- every quantity by hand.

    x=2, Wr=[[1, -1]] -> z=[2,-2], expert 0 picked with gate 1.
    W1[0]=[[1, 3]] -> g=2, u=6;  silu(2) = 2/(1+e^-2);  A = 6*silu(2).
    W2[0]=[[0.5]] -> Y = 3*silu(2) = O.
    """
    X = np.array([[2.0]])
    Wr = np.array([[1.0, -1.0]])
    W1 = np.array([[[1.0, 3.0]], [[7.0, 7.0]]])
    W2 = np.array([[[0.5]], [[9.0]]])
    fw = orc.forward(X, Wr, None, W1, W2, 1)
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    assert fw["topk_idx"][0, 0] == 0
    assert abs(fw["O"][0, 0] - 3.0 * silu2) < 1e-15
    # backward with dO = 1: dX = d/dx [0.5 * silu(x) * 3x] + router path (0 for K=1)
    dO = np.array([[1.0]])
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    sig = 1.0 / (1.0 + math.exp(-2.0))
    dsilu = sig * (1.0 + 2.0 * (1.0 - sig))
    # O(x) = 0.5 * silu(x) * 3x  ->  O'(x) = 1.5 * (dsilu(x) * x + silu(x))
    assert abs(bw["dX"][0, 0] - 1.5 * (dsilu * 2.0 + silu2)) < 1e-14
    # with one selected expert the gate is constant: no router gradient
    assert abs(bw["dWr"]).max() == 0.0


# ---------------------------------------------------------------- backward
def test_router_gradient_reformulation_equals_naive():
    """dS from <dA', A> equals dS from the cached output <dO, Y>."""
    X, W1, W2, Wr, b, dO = rand_layer(128, 32, 8, 16, 2, 5, bias=True)
    fw = orc.forward(X, Wr, b, W1, W2, 2)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    naive = orc.router_dS_naive(fw, dO)
    np.testing.assert_allclose(bw["dS_pair"], naive, rtol=1e-11, atol=1e-12)


def _loss_of(X, W1, W2, Wr, b, K, dO):
    fw = orc.forward(X, Wr, b, W1, W2, K)
    return orc.loss(fw["O"], dO), fw["topk_idx"]


@pytest.mark.parametrize("bias", [False, True])
def test_gradients_match_central_differences(bias):
    T, d, E, n, K = 24, 8, 6, 4, 2
    X, W1, W2, Wr, b, dO = rand_layer(T, d, E, n, K, 11 + int(bias), bias=bias)
    fw = orc.forward(X, Wr, b, W1, W2, K)
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    base_idx = fw["topk_idx"]
    rs = np.random.RandomState(7)
    h = 1e-6
    for name, arr, grad in (("X", X, bw["dX"]), ("W1", W1, bw["dW1"]),
                            ("W2", W2, bw["dW2"]), ("Wr", Wr, bw["dWr"])):
        flat = arr.reshape(-1)
        gflat = grad.reshape(-1)
        checked = 0
        for i in rs.choice(flat.size, min(flat.size, 60), replace=False):
            old = flat[i]
            flat[i] = old + h
            lp, ip = _loss_of(X, W1, W2, Wr, b, K, dO)
            flat[i] = old - h
            lm, im = _loss_of(X, W1, W2, Wr, b, K, dO)
            flat[i] = old
            if not (np.array_equal(ip, base_idx) and np.array_equal(im, base_idx)):
                continue            # the perturbation moved the top-K set
            fd = (lp - lm) / (2 * h)
            assert abs(fd - gflat[i]) <= 1e-6 * max(1.0, abs(fd)), (name, i, fd, gflat[i])
            checked += 1
        assert checked >= 20, name


def test_router_dz_is_softmax_jacobian():
    """dz = J^T dS for the softmax over the selected logits, built explicitly."""
    rs = np.random.RandomState(3)
    k = 5
    z = rs.randn(k)
    s = np.exp(z - z.max()); s /= s.sum()
    dS = rs.randn(k)
    J = np.diag(s) - np.outer(s, s)        # ds_i / dz_j
    expect = J.T @ dS
    dz = orc.router_dz(dS, s, np.arange(k), np.array([0, k]), k)
    np.testing.assert_allclose(dz[0], expect, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- token rounding
def _splitmix_golden():
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "splitmix64.txt")
    vals = []
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            vals.append(int(line, 16))
    return vals


def test_splitmix64_published_outputs():
    """Successive outputs of SplitMix64 from state 0 (published test vector).

    Output i of the generator started at state s is splitmix64(s + i*gamma)."""
    gamma = 0x9E3779B97F4A7C15
    for i, v in enumerate(_splitmix_golden()):
        assert orc.splitmix64((i * gamma) & orc.MASK64) == v


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("tile", [8, 16])
def test_token_round_invariants(mode, tile):
    rs = np.random.RandomState(20 + mode + tile)
    T, E, K = 200, 12, 3
    z = rs.randn(T, E) + rs.randn(E)[None, :]
    probs = orc.softmax_rows(z).astype(np.float32).astype(np.float64)
    idx = orc.topk_select(z, K)
    tok_ptr, pe = orc.pairs_from_topk(idx)
    c0 = np.bincount(pe, minlength=E)
    out = orc.token_round(probs, tok_ptr, pe, mode, seed=99, tile=tile)
    c1 = out["counts"]
    assert np.all(c1 % tile == 0)
    assert np.all(np.abs(c1 - c0) < tile)
    member0 = np.zeros((T, E), bool)
    member0[np.repeat(np.arange(T), K), pe] = True
    m1 = out["member"]
    for e in range(E):
        dropped = np.nonzero(member0[:, e] & ~m1[:, e])[0]
        added = np.nonzero(~member0[:, e] & m1[:, e])[0]
        assert len(dropped) == 0 or len(added) == 0
        if len(dropped):
            kept = np.nonzero(member0[:, e] & m1[:, e])[0]
            if len(kept):
                # every dropped pair ranks below every kept one (p asc, t desc)
                worst_kept = min(kept, key=lambda t: (probs[t, e], -t))
                for t in dropped:
                    assert (probs[t, e], -t) < (probs[worst_kept, e], -worst_kept)
            assert out["decisions"][e] == -1
        if len(added):
            rest = np.nonzero(~m1[:, e])[0]
            if len(rest):
                best_rest = min(rest, key=lambda t: (-probs[t, e], t))
                for t in added:
                    assert (-probs[t, e], t) < (-probs[best_rest, e], best_rest)
            assert out["decisions"][e] == 1
        r = c0[e] % tile
        if mode == 1 and r:
            assert out["decisions"][e] == (1 if (r >= tile // 2 and c0[e] - r + tile <= T) else -1)
    # gates renormalised over the final set
    for t in range(T):
        a, b = out["tok_ptr"][t], out["tok_ptr"][t + 1]
        es = out["pair_expert"][a:b]
        assert np.all(np.diff(es) > 0)
        if b > a:
            np.testing.assert_allclose(out["pair_gate"][a:b], probs[t, es] / probs[t, es].sum(),
                                       rtol=1e-13)
            assert abs(out["pair_gate"][a:b].sum() - 1) < 1e-12


def test_token_round_stochastic_preserves_total_in_expectation():
    rs = np.random.RandomState(5)
    T, E, K, tile = 300, 10, 2, 16
    z = rs.randn(T, E)
    probs = orc.softmax_rows(z)
    idx = orc.topk_select(z, K)
    tok_ptr, pe = orc.pairs_from_topk(idx)
    c0 = np.bincount(pe, minlength=E)
    r = c0 % tile
    totals = []
    for seed in range(1000):
        ups = [orc.round_up_decision(int(c0[e]), e, T, 2, seed, tile) for e in range(E)]
        totals.append(sum(int(c0[e] - r[e] + (tile if u else 0)) for e, u in enumerate(ups)))
    totals = np.array(totals, float)
    var = float(np.sum((r / tile) * (1 - r / tile))) * tile * tile
    assert abs(totals.mean() - T * K) <= 3 * math.sqrt(var / len(totals))


def test_token_round_never_exceeds_T():
    T, E, tile = 20, 3, 16
    probs = np.full((T, E), 1.0 / E)
    # expert 0 holds 19 of 20 tokens: 19 mod 16 = 3 -> nearest rounds down anyway,
    # expert 1 holds 15: nearest rounds up to 16 <= T
    member = np.zeros((T, E), bool)
    member[:19, 0] = True
    member[:15, 1] = True
    member[19, 2] = True
    tok_ptr = np.zeros(T + 1, np.int64)
    tok_ptr[1:] = np.cumsum(member.sum(1))
    pe = np.concatenate([np.nonzero(member[t])[0] for t in range(T)])
    out = orc.token_round(probs, tok_ptr, pe, 1, 0, tile)
    assert list(out["counts"]) == [16, 16, 0]
    # a count of 14 of T=20 with tile 16: nearest would round up to 16 (fine);
    # with T=15 the round-up would exceed T, so it rounds down
    assert orc.round_up_decision(14, 0, 15, 1, 0, 16) is False
    assert orc.round_up_decision(14, 0, 20, 1, 0, 16) is True


def test_token_round_tie_order():
    """Equal probabilities: rounding down drops the largest token ids first,
    rounding up adds the smallest unrouted token ids first."""
    T, E, tile = 40, 2, 8
    probs = np.full((T, E), 0.5)
    member = np.zeros((T, E), bool)
    member[:11, 0] = True          # 11 mod 8 = 3 -> nearest: down, drop 3
    member[11:17, 1] = True        # 6 mod 8 = 6 -> nearest: up, add 2
    tok_ptr = np.zeros(T + 1, np.int64)
    tok_ptr[1:] = np.cumsum(member.sum(1))
    pe = np.concatenate([np.nonzero(member[t])[0] for t in range(T)] + [np.zeros(0, np.int64)])
    out = orc.token_round(probs, tok_ptr, pe, 1, 0, tile)
    m = out["member"]
    assert list(np.nonzero(m[:, 0])[0]) == list(range(8))           # 8, 9, 10 dropped
    assert list(np.nonzero(m[:, 1])[0]) == [0, 1] + list(range(11, 17))  # 0, 1 added


def test_weight_grads_for_an_expert_subset_match_the_full_backward():
    X, W1, W2, Wr, b, dO = rand_layer(64, 12, 6, 4, 2, 9, bias=True)
    fw = orc.forward(X, Wr, b, W1, W2, 2)
    full = orc.backward(fw, dO, X, Wr, W1, W2)
    part = orc.backward(fw, dO, X, Wr, W1, W2, weight_grad_experts=[1, 4])
    for e in (1, 4):
        np.testing.assert_array_equal(part["dW1"][e], full["dW1"][e])
        np.testing.assert_array_equal(part["dW2"][e], full["dW2"][e])
    np.testing.assert_array_equal(part["dX"], full["dX"])
    assert set(part["dW1"]) == {1, 4}
