"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs.  Routing, permutation and token rounding bit-exact (after
the near-tie rule), floating-point outputs within the stated tolerances."""
import numpy as np
import pytest

from oracle import moe_oracle as orc
from workloads import CONFIGS, MoEConfig, make_inputs

import parity as P

torch = pytest.importorskip("torch")

SHAPES = [
    CONFIGS["tiny"],
    # BN 256 paths (n % 128 == 0, d % 256 == 0), skewed router
    MoEConfig("bn256", T=300, d=256, E=8, n=128, K=2, w_std=0.05, bias="normal", seed=11),
    # BN 128 / 64 paths (d % 256 != 0, n % 128 != 0), several dH N tiles
    MoEConfig("bn64", T=1000, d=384, E=12, n=192, K=3, w_std=0.05, seed=12),
    # one expert, top-1: a dense SwiGLU MLP
    MoEConfig("dense", T=200, d=128, E=1, n=64, K=1, w_std=0.05, seed=13),
    # fewer tokens than a tile, E not a multiple of 64, empty experts
    MoEConfig("sparse", T=64, d=128, E=70, n=64, K=4, w_std=0.05, seed=14),
    # several M tiles per expert, even and odd counts: down-proj and dX~ on CTA
    # pairs plus each expert's leftover tile on one CTA (dX~ with 8 epilogue warps)
    MoEConfig("pairs", T=1500, d=512, E=6, n=128, K=3, w_std=0.05, bias="normal", seed=15),
    # the same with a long dX~ main loop (2n = 1280: 4 epilogue warps)
    MoEConfig("pairs_n640", T=600, d=256, E=3, n=640, K=2, w_std=0.05, bias="normal", seed=16),
]


def _np_inputs(inp):
    return (P.f64(inp["X"]), P.f64(inp["Wr"]), None if inp["bias"] is None else P.f64(inp["bias"]),
            P.f64(inp["W1"]), P.f64(inp["W2"]), P.f64(inp["dO"]))


def _compare_layer(layer, cfg, inp, routing=None, router_grad=True):
    g = P.gpu_routing(layer, cfg.T)
    X, Wr, b, W1, W2, dO = _np_inputs(inp)
    if routing is None:
        fw = orc.forward(X, Wr, b, W1, W2, cfg.K, topk_idx=g["topk_idx"])
    else:
        fw = orc.forward(X, Wr, b, W1, W2, cfg.K, routing=routing)
    np.testing.assert_allclose(g["pair_gate"], fw["pair_gate"], rtol=1e-5, atol=1e-7)
    perm = P.check_permutation(g, cfg.E)
    errs = {"O": P.normwise(P.f64(layer.O), fw["O"])}
    H = P.expert_rows_to_oracle_order(P.f64(layer.H), g, perm, cfg.E)
    errs["H"] = P.normwise(H, fw["H"])
    bw = orc.backward(fw, dO, X, Wr, W1, W2, router_grad=router_grad)
    errs["dX"] = P.normwise(P.f64(layer.dX), bw["dX"])
    errs["dW1"] = P.normwise(P.f64(layer.dW1), bw["dW1"])
    errs["dW2"] = P.normwise(P.f64(layer.dW2), bw["dW2"])
    if router_grad:
        errs["dWr"] = P.normwise(P.f64(layer.dWr), bw["dWr"])
    print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= P.TOL_BF16, (k, v)
    return g, fw, bw


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", SHAPES, ids=[c.name for c in SHAPES])
def test_layer_parity(cfg):
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    g = P.gpu_routing(layer, cfg.T)
    X, Wr, b, *_ = _np_inputs(inp)
    z = orc.router_logits(X, Wr, b)
    P.check_router(g, z, orc.softmax_rows(z), cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["pairs", "pairs_n640"])
def test_layer_parity_pair_tiles(name, monkeypatch):
    """Down-proj and dX~ on CTA pairs (256-row tiles over two M tiles of one
    expert, leftover tiles on single CTAs), an opt-in path."""
    monkeypatch.setenv("MOE_GM_PAIR", "1")
    cfg = next(c for c in SHAPES if c.name == name)
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["pairs", "pairs_n640", "bn256"])
def test_layer_parity_wide_tiles(name, monkeypatch):
    """Down-proj and dX~ with 256 x 256 tiles on one CTA (two M tiles of one
    expert sharing B; an expert's odd last M tile as a half-filled tile),
    forced on small layers: even and odd tile counts per expert, experts of
    one tile only, the router path of dX~."""
    monkeypatch.setenv("MOE_GM_WIDE", "1")
    cfg = next(c for c in SHAPES if c.name == name)
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
@pytest.mark.parametrize("name,wide,order", [("pairs", "0", "0"), ("bn64", "0", "1"), ("pairs", "1", "1"),
                                             ("pairs_n640", "1", "0"), ("pairs_n640", "1", "1")])
def test_layer_parity_both_tile_orders(name, wide, order, monkeypatch):
    """The grouped-M GEMMs walk an expert's tiles M-tile-major or
    weight-stationary (its M tiles side by side within each N tile), as the
    plan picks from the shape; both orders, forced, on the 128-row and the
    256-row tiles."""
    monkeypatch.setenv("MOE_TILE_ORDER", order)
    monkeypatch.setenv("MOE_GM_WIDE", wide)
    cfg = next(c for c in SHAPES if c.name == name)
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", ["0", "1", "2"])
def test_weight_gradients_under_every_claim_order(mode, monkeypatch):
    """The weight-gradient tiles come from a dynamic queue: largest experts
    first (0), from both ends by CTA parity (1), or alternating ends in every
    CTA (2, the default).  Each order covers every tile exactly once."""
    monkeypatch.setenv("MOE_DW_DUAL", mode)
    cfg = next(c for c in SHAPES if c.name == "pairs")
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
@pytest.mark.parametrize("var,warps,name", [("MOE_EPI_DW", "8", "sparse"), ("MOE_EPI_DW", "8", "bn64"),
                                            ("MOE_EPI_DH", "4", "bn64"), ("MOE_EPI_DH", "4", "bn256"),
                                            ("MOE_EPI_DXT", "4", "bn256"), ("MOE_EPI_DXT", "8", "pairs_n640")])
def test_layer_parity_other_epilogue_widths(var, warps, name, monkeypatch):
    """The plan picks 4 or 8 epilogue warps per kernel from the shape; the
    other width of the weight-gradient (empty experts included), dH and dX~
    kernels, forced."""
    monkeypatch.setenv(var, warps)
    cfg = next(c for c in SHAPES if c.name == name)
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    _compare_layer(layer, cfg, inp)


@pytest.mark.gpu
def test_expert_only_gradient_without_router_path():
    cfg = SHAPES[1]
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, router_grad=0)
    _compare_layer(layer, cfg, inp, router_grad=False)


@pytest.mark.gpu
@pytest.mark.parametrize("mode,T,E,K,wr_std", [(1, 2048, 16, 2, 0.02), (2, 2048, 16, 2, 0.02), (2, 53248, 16, 2, 0.02),
                                                (2, 16384, 512, 8, 0.02), (1, 4096, 130, 4, 0.02),
                                                (2, 6000, 8, 2, 0.0)])
def test_token_rounding_parity(mode, T, E, K, wr_std):
    """E = 512 and 130: several groups of 32 experts per token in the pair
    writer.  wr_std = 0 (no bias): every p is exactly 1 / E, so each expert's
    candidates share one histogram bin, more than the sorted list holds, and
    the selection falls back to radix passes over all candidates; the ties
    are then broken by token index alone."""
    cfg = MoEConfig("tr", T=T, d=128, E=E, n=64, K=K, w_std=0.05, wr_std=wr_std,
                    bias="normal" if wr_std > 0 else "none", seed=21)
    _check_token_rounding(cfg, mode)


@pytest.mark.gpu
@pytest.mark.parametrize("wr_std", [0.02, 0.0])
def test_token_rounding_parity_unstaged(wr_std, monkeypatch):
    """The selection's path for expert rows too long to stage in shared
    memory (reading candidates and keys from global memory), forced on a
    small layer; with wr_std = 0 it also takes the radix fallback there."""
    monkeypatch.setenv("MOE_TR_UNSTAGED", "1")
    cfg = MoEConfig("tr", T=6000, d=128, E=8 if wr_std == 0 else 130, n=64, K=2 if wr_std == 0 else 4, w_std=0.05,
                    wr_std=wr_std, bias="normal" if wr_std > 0 else "none", seed=22)
    _check_token_rounding(cfg, 2)


def _check_token_rounding(cfg, mode):
    seed = 1234
    inp = make_inputs(cfg, "cuda")
    layer = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=mode, seed=seed)
    g = P.gpu_routing(layer, cfg.T)
    tok_ptr0, pe0 = orc.pairs_from_topk(g["topk_idx"])
    c0 = np.bincount(pe0, minlength=cfg.E)
    tr = orc.token_round(g["probs"], tok_ptr0, pe0, mode, seed)   # decisions in the GPU's fp32 probs
    np.testing.assert_array_equal(g["tok_ptr"], tr["tok_ptr"])
    np.testing.assert_array_equal(g["pair_expert"], tr["pair_expert"])
    np.testing.assert_allclose(g["pair_gate"], tr["pair_gate"], rtol=2e-6)
    assert np.all(g["counts"] % 128 == 0)
    assert np.all(np.abs(g["counts"] - c0) < 128)
    assert np.any(g["counts"] != c0)
    X, Wr, b, *_ = _np_inputs(inp)
    z = orc.router_logits(X, Wr, b)
    routing = {"z": z, "probs": orc.softmax_rows(z), "topk_idx": g["topk_idx"], "tok_ptr": tr["tok_ptr"],
               "pair_expert": tr["pair_expert"],
               "pair_gate": orc.gates_for_sets(z, tr["tok_ptr"], tr["pair_expert"])}
    _compare_layer(layer, cfg, inp, routing=routing)


@pytest.mark.gpu
def test_bounded_wait_reports_timeout():
    from fine_grained_mixture_top_b200 import moe
    assert moe.moe_get_status() == (0, 0)
    moe.moe_set_spin_limit(2_000_000)          # about a millisecond
    flag = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    try:
        moe.moe_selftest_wait_timeout(flag)
        code, where = moe.moe_get_status()
    finally:
        moe.moe_set_spin_limit(1 << 31)
    assert int(flag.item()) == 0
    assert (code, where) == (moe.MOE_ERR_TIMEOUT, 999)
    assert moe.moe_get_status() == (0, 0)      # cleared; the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum().item()) == 4.0


@pytest.mark.gpu
def test_argument_errors_are_synchronous():
    from fine_grained_mixture_top_b200 import moe
    layer = moe.MoELayer(512, 128, 16, 64, 2)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    X = torch.zeros(512, 128, dtype=torch.bfloat16, device="cuda")
    Wr = torch.zeros(128, 16, device="cuda")
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route(layer.dims, layer.opts, X, Wr, None, layer.routing, small)
    assert ei.value.code == moe.MOE_ERR_WORKSPACE
    with pytest.raises(moe.MoEError) as ei:
        moe.moe_route(layer.dims, layer.opts, X[:, 1:], Wr, None, layer.routing, layer.ws_route)
    assert ei.value.code == moe.MOE_ERR_INVALID_ARG


@pytest.mark.gpu
def test_host_fed_runner_matches_device_steps():
    """Steps fed from pinned host memory give the same outputs as steps on
    device-resident inputs."""
    from fine_grained_mixture_top_b200 import moe
    cfg = SHAPES[1]
    inp = make_inputs(cfg, "cuda")
    ref = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    runner = moe.HostFedRunner(layer)
    Xh = inp["X"].cpu().pin_memory()
    dOh = inp["dO"].cpu().pin_memory()
    outs = [torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    grads = [torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    for Oh, dXh in zip(outs, grads):   # three steps in a row, both buffer sets used
        runner.step(Xh, dOh, Oh, inp["Wr"], inp["bias"], inp["W1"], inp["W2"], dXh=dXh)
    runner.finish()
    torch.cuda.synchronize()
    assert moe.moe_get_status() == (0, 0)
    for Oh, dXh in zip(outs, grads):
        assert torch.equal(Oh, ref.O.cpu())
        assert torch.equal(dXh, ref.dX.cpu())
    for k in ("dW1", "dW2", "dWr"):
        assert torch.equal(getattr(layer, k), getattr(ref, k)), k


@pytest.mark.gpu
def test_sm_budget_does_not_change_results():
    """Persistent GEMMs on fewer CTAs (SMs left to a communication kernel)
    give bitwise the same outputs: every tile's arithmetic is independent of
    which CTA computes it."""
    from fine_grained_mixture_top_b200 import moe
    cfg = SHAPES[2]
    inp = make_inputs(cfg, "cuda")
    ref = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    try:
        moe.moe_set_sm_budget(37)
        lim = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    finally:
        moe.moe_set_sm_budget(0)
    rows = int(ref.routing["offsets"][cfg.E].item())  # H rows past the last segment are never written
    assert torch.equal(lim.H[:rows], ref.H[:rows])
    for k in ("O", "dX", "dW1", "dW2", "dWr"):
        assert torch.equal(getattr(lim, k), getattr(ref, k)), k


@pytest.mark.gpu
def test_grad_ready_events_mark_final_gradients():
    """A copy of dW2, dW1 and dWr taken on another stream right after their
    events equals the gradient at the end of the backward."""
    from fine_grained_mixture_top_b200 import moe
    cfg = SHAPES[1]
    inp = make_inputs(cfg, "cuda")
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    evs = [torch.cuda.Event() for _ in range(3)]
    side = torch.cuda.Stream()
    for _ in range(2):   # the second step overwrites the first step's gradients
        layer.step(inp["X"], inp["Wr"], inp["bias"], inp["W1"], inp["W2"], inp["dO"], grad_events=evs)
        with torch.cuda.stream(side):
            copies = []
            for ev, g in zip(evs, (layer.dW2, layer.dW1, layer.dWr)):
                side.wait_event(ev)
                copies.append(g.clone())
        torch.cuda.synchronize()
        for c, g in zip(copies, (layer.dW2, layer.dW1, layer.dWr)):
            assert torch.equal(c, g)
    assert moe.moe_get_status() == (0, 0)


@pytest.mark.gpu
def test_overlapped_reduce_on_one_rank_equals_plain_step():
    """The overlapped data-parallel step on a one-rank NCCL group (the sum over
    one rank is the identity) gives the plain step's outputs."""
    import os
    import socket
    import torch.distributed as dist
    from fine_grained_mixture_top_b200 import moe
    cfg = SHAPES[1]
    inp = make_inputs(cfg, "cuda")
    ref = P.run_layer(inp, cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
        red = moe.OverlappedGradReduce(layer)
        for _ in range(2):
            red.step(inp["X"], inp["Wr"], inp["bias"], inp["W1"], inp["W2"], inp["dO"])
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    for k in ("dX", "dW1", "dW2", "dWr"):
        assert torch.equal(getattr(layer, k), getattr(ref, k)), k
