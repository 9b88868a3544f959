"""GPU parity of caller-given routing, the expert-parallel pack/combine, the
per-pair dS output of the backward, the router backward from given dS, and
one expert-parallel layer on a single-rank NCCL group, against the fp64
oracle."""
import datetime
import os
import socket

import numpy as np
import pytest

from oracle import moe_oracle as orc
from workloads import MoEConfig, make_inputs

import parity as P

torch = pytest.importorskip("torch")

CFGS = [
    MoEConfig("ep_small", T=300, d=256, E=8, n=128, K=2, w_std=0.05, bias="normal", seed=31),
    MoEConfig("ep_ragged", T=1000, d=384, E=12, n=192, K=3, w_std=0.05, seed=32),
]


def _np(inp):
    return (P.f64(inp["X"]), P.f64(inp["Wr"]), None if inp["bias"] is None else P.f64(inp["bias"]),
            P.f64(inp["W1"]), P.f64(inp["W2"]), P.f64(inp["dO"]))


def _routed_layer(cfg, inp, pair_ds=False):
    from fine_grained_mixture_top_b200 import moe
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, seed=cfg.seed)
    if pair_ds:
        layer.routing = moe.Routing.allocate(layer.dims, layer.sizes, "cuda", with_pair_ds=True)
    layer.route(inp["X"], inp["Wr"], inp["bias"])
    return layer


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", CFGS, ids=[c.name for c in CFGS])
def test_route_given_reproduces_the_permutation(cfg):
    from fine_grained_mixture_top_b200 import moe
    inp = make_inputs(cfg, "cuda")
    ref = _routed_layer(cfg, inp)
    other = moe.Routing.allocate(ref.dims, ref.sizes, "cuda")
    other["topk_idx"].copy_(ref.routing["topk_idx"])
    other["topk_gate"].copy_(ref.routing["topk_gate"])
    ws = torch.empty(ref.sizes.route_ws, dtype=torch.uint8, device="cuda")
    moe.moe_route_given(ref.dims, ref.opts, other, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    a, b = P.gpu_routing(ref, cfg.T), P.gpu_routing(type("L", (), {"routing": other})(), cfg.T)
    for k in ("tok_ptr", "pair_expert", "pair_gate", "pair_row", "counts", "offsets"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
    R = int(a["offsets"][-1])
    np.testing.assert_array_equal(a["tile_expert"][:R // 128], b["tile_expert"][:R // 128])  # tiles in use
    np.testing.assert_array_equal(a["row_tok"][:R], b["row_tok"][:R])
    np.testing.assert_array_equal(a["row_gate"][:R], b["row_gate"][:R])


@pytest.mark.gpu
def test_route_given_rejects_a_repeated_expert():
    from fine_grained_mixture_top_b200 import moe
    cfg = CFGS[0]
    layer = moe.MoELayer(64, cfg.d, cfg.E, cfg.n, 2)
    idx = torch.tensor([[0, 1]] * 64, dtype=torch.int32, device="cuda")
    idx[5] = torch.tensor([3, 3], dtype=torch.int32)
    layer.routing["topk_idx"].copy_(idx)
    layer.routing["topk_gate"].fill_(0.5)
    moe.moe_route_given(layer.dims, layer.opts, layer.routing, layer.ws_route)
    code, where = moe.moe_get_status()
    assert code == moe.MOE_ERR_DEVICE_CHECK
    # the offending token was replaced by experts 0, 1 with gate 0; the rest stands
    g = P.gpu_routing(layer, 64)
    np.testing.assert_array_equal(g["pair_expert"][10:12], [0, 1])
    assert g["pair_gate"][10] == 0.0 and g["pair_gate"][11] == 0.0
    assert g["counts"].sum() == 128


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", CFGS, ids=[c.name for c in CFGS])
def test_ep_pack_and_combine(cfg):
    from fine_grained_mixture_top_b200 import moe
    inp = make_inputs(cfg, "cuda")
    layer = _routed_layer(cfg, inp)
    g = P.gpu_routing(layer, cfg.T)
    Ptot = int(g["tok_ptr"][-1])
    rows = torch.empty(Ptot, cfg.d, dtype=torch.bfloat16, device="cuda")
    gate = torch.empty(Ptot, dtype=torch.float32, device="cuda")
    pos = torch.empty(Ptot, dtype=torch.int32, device="cuda")
    moe.moe_ep_pack(layer.dims, layer.opts, layer.routing, inp["X"], rows, gate, pos, layer.ws_route)
    torch.cuda.synchronize()
    perm = P.check_permutation(g, cfg.E)
    # expert-major rows without padding, bit-exact; each pair's position
    X = inp["X"].cpu()
    np.testing.assert_array_equal(rows.cpu().view(torch.int16).numpy(),
                                  X[torch.from_numpy(perm["row_tok"])].view(torch.int16).numpy())
    np.testing.assert_array_equal(P.i64(pos), perm["pair_row"])
    np.testing.assert_array_equal(P.f64(gate), g["pair_gate"][perm["row_pair"]])
    # combine: the rows' per-token sums (fp32, pair order), against fp64
    out = torch.empty(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    moe.moe_ep_combine(layer.dims, layer.opts, layer.routing, pos, rows, out)
    torch.cuda.synchronize()
    ref = np.zeros((cfg.T, cfg.d))
    Xf = P.f64(X)
    for t in range(cfg.T):
        ref[t] = (g["tok_ptr"][t + 1] - g["tok_ptr"][t]) * Xf[t]
    assert P.normwise(P.f64(out), ref) <= 2.0 ** -8


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", CFGS, ids=[c.name for c in CFGS])
def test_pair_ds_and_router_backward(cfg):
    from fine_grained_mixture_top_b200 import moe
    inp = make_inputs(cfg, "cuda")
    layer = _routed_layer(cfg, inp, pair_ds=True)
    layer.forward(inp["X"], inp["W1"], inp["W2"])
    layer.backward(inp["dO"], inp["X"], inp["Wr"], inp["W1"], inp["W2"])
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    g = P.gpu_routing(layer, cfg.T)
    X, Wr, b, W1, W2, dO = _np(inp)
    fw = orc.forward(X, Wr, b, W1, W2, cfg.K, topk_idx=g["topk_idx"])
    bw = orc.backward(fw, dO, X, Wr, W1, W2)
    dS = layer.routing["pair_dS"][:len(g["pair_gate"])]
    assert P.normwise(P.f64(dS), bw["dS_pair"]) <= P.TOL_BF16
    # router backward from the oracle's dS (fp32), onto a zero dX
    dS_in = torch.from_numpy(bw["dS_pair"].astype(np.float32)).cuda()
    dX = torch.zeros(cfg.T, cfg.d, dtype=torch.bfloat16, device="cuda")
    dWr = torch.empty(cfg.d, cfg.E, dtype=torch.float32, device="cuda")
    moe.moe_router_backward(layer.dims, layer.opts, inp["X"], inp["Wr"], layer.routing, dS_in, None, dX, dWr,
                            layer.ws_bwd)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    assert P.normwise(P.f64(dWr), bw["dWr"]) <= P.TOL_BF16
    assert P.normwise(P.f64(dX), bw["dX"] - bw["dX_expert"]) <= P.TOL_BF16


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", CFGS, ids=[c.name for c in CFGS])
def test_expert_parallel_layer_on_one_rank(cfg):
    """The expert-parallel layer through NCCL with one rank: routing, pack,
    all-to-all, the expert side on K = 1 given routing, combine and the
    router backward from the returned dS, against the oracle."""
    import torch.distributed as dist
    from fine_grained_mixture_top_b200.ep import CudaEngine, ExpertParallelMoE
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        inp = make_inputs(cfg, "cuda")
        eng = CudaEngine(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, 1, seed=cfg.seed)
        ep = ExpertParallelMoE(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, eng)
        O = ep.forward(inp["X"], inp["Wr"], inp["bias"], inp["W1"], inp["W2"])
        dX, dW1, dW2, dWr = ep.backward(inp["dO"], inp["X"], inp["Wr"], inp["W1"], inp["W2"])
        torch.cuda.synchronize()
        from fine_grained_mixture_top_b200 import moe
        assert moe.moe_get_status()[0] == 0
        topk = P.i64(eng.routing["topk_idx"])
        X, Wr, b, W1, W2, dO = _np(inp)
        fw = orc.forward(X, Wr, b, W1, W2, cfg.K, topk_idx=topk)
        bw = orc.backward(fw, dO, X, Wr, W1, W2)
        errs = {"O": P.normwise(P.f64(O), fw["O"]), "dX": P.normwise(P.f64(dX), bw["dX"]),
                "dW1": P.normwise(P.f64(dW1), bw["dW1"]), "dW2": P.normwise(P.f64(dW2), bw["dW2"]),
                "dWr": P.normwise(P.f64(dWr), bw["dWr"])}
        print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()})
        for k, v in errs.items():
            assert v <= P.TOL_BF16, (k, v)
    finally:
        dist.destroy_process_group()
