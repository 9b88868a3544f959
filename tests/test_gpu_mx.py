"""GPU MXFP8 quantization and the MXFP8 forward against the MX oracle.
Codes and scales are integer results: bit-exact."""
import numpy as np
import pytest

from oracle import mx_oracle as mx

torch = pytest.importorskip("torch")


def _bf16(shape, seed, spread=0):
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn(*shape, generator=g)
    if spread:   # blocks whose magnitudes differ by many binades
        x = x * torch.exp2(torch.randint(-spread, spread + 1, shape[:-1] + (1,), generator=g).float())
    return x.to(torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("rows,K,spread", [(1, 32, 0), (37, 256, 0), (300, 1536, 20), (64, 128, 60)])
def test_quantize_rows_bit_exact(rows, K, spread):
    from fine_grained_mixture_top_b200 import moe
    x = _bf16((rows, K), 7 + rows, spread)
    x[0, :4] = torch.tensor([0.0, -0.0, 1e-30, -1e-30]).to(torch.bfloat16)   # zeros and underflow keep their sign
    codes, scales = moe.mx_quantize_rows(x.cuda())
    ref_c, ref_s = mx.mx_quantize(x.float().numpy().astype(np.float64))
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


@pytest.mark.gpu
@pytest.mark.parametrize("E,K,N", [(1, 32, 1), (3, 128, 70), (4, 256, 512)])
def test_quantize_cols_bit_exact(E, K, N):
    from fine_grained_mixture_top_b200 import moe
    w = _bf16((E, K, N), 11 + N, 8)
    codes, scales = moe.mx_quantize_cols(w.cuda())
    ref_c, ref_s = mx.mx_quantize(np.swapaxes(w.float().numpy().astype(np.float64), 1, 2))
    np.testing.assert_array_equal(scales.cpu().numpy(), ref_s)
    np.testing.assert_array_equal(codes.cpu().numpy(), ref_c)


# ----------------------------------------------------------------------------
# The MXFP8 forward against mx_oracle.forward_mxfp8 on the GPU's own routing.
# ----------------------------------------------------------------------------
from oracle import moe_oracle as orc        # noqa: E402
from workloads import CONFIGS, MoEConfig, make_inputs   # noqa: E402

import parity as P                          # noqa: E402

MX_SHAPES = [
    MoEConfig("mx_small", T=512, d=256, E=8, n=128, K=2, w_std=0.05, seed=21),
    # ragged expert tails, several N tiles of both GEMMs, skewed router
    MoEConfig("mx_ragged", T=1000, d=384, E=12, n=256, K=3, w_std=0.05, bias="normal", seed=22),
    # one expert, top-1: a dense MLP on quantized operands
    MoEConfig("mx_dense", T=200, d=128, E=1, n=128, K=1, w_std=0.05, seed=23),
    # fewer tokens than a tile, many empty experts
    MoEConfig("mx_sparse", T=64, d=128, E=70, n=128, K=4, w_std=0.05, seed=24),
]


def _mx_layer(cfg, inp):
    from fine_grained_mixture_top_b200 import moe
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, seed=cfg.seed)
    layer.route(inp["X"], inp["Wr"], inp["bias"])
    layer.forward(inp["X"], inp["W1"], inp["W2"], mxfp8=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    return layer


def _check_h_elementwise(Hg, fq, X, W1, rows_tok, perm):
    """Each H element is the bf16 rounding of the product of the quantized
    operands, up to the tensor core's accumulation error:
    |err| <= 2^-8 |H| + 2^-9 (|Xq| |W1q|) for the element's row and column.
    The block-scaled MMA accumulates far less precisely than fp32 (errors
    near 2^-10 |Xq| |W1q| were seen on B200), but a misplaced block scale
    moves a 32-term partial sum by a power of two, an error of 2^-7
    (|Xq| |W1q|) or more for d up to 1536.  Returns log2 of the largest
    accumulation error seen, relative to |Xq| |W1q|."""
    Xq = mx.mx_round(X)
    seg = perm["seg"]
    worst = -np.inf
    for e in range(len(seg) - 1):
        a, b = seg[e], seg[e + 1]
        if a == b:
            continue
        W1q = mx.mx_round(np.asarray(W1[e], np.float64).T).T
        mag = np.abs(Xq[rows_tok[a:b]]) @ np.abs(W1q)
        ref = fq["H"][a:b]
        err = np.abs(Hg[a:b] - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2.0 ** -9 * mag), e
        acc = np.maximum(err - 2.0 ** -9 * np.abs(ref) * (1 + 2.0 ** -8), 0) / np.maximum(mag, 1e-300)
        worst = max(worst, float(np.log2(max(acc.max(), 2.0 ** -60))))
    return worst


@pytest.mark.gpu
@pytest.mark.parametrize("cfg", MX_SHAPES, ids=[c.name for c in MX_SHAPES])
def test_mxfp8_forward_parity(cfg):
    inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
    layer = _mx_layer(cfg, inp)
    g = P.gpu_routing(layer, cfg.T)
    X, Wr, W1, W2 = (P.f64(inp[k]) for k in ("X", "Wr", "W1", "W2"))
    b = None if inp["bias"] is None else P.f64(inp["bias"])
    fq = mx.forward_mxfp8(X, Wr, b, W1, W2, cfg.K, topk_idx=g["topk_idx"])
    perm = P.check_permutation(g, cfg.E)
    H = P.expert_rows_to_oracle_order(P.f64(layer.H), g, perm, cfg.E)
    acc = _check_h_elementwise(H, fq, X, W1, fq["row_tok"], perm)
    errs = {"O": P.normwise(P.f64(layer.O), fq["O"]), "H": P.normwise(H, fq["H"])}
    # the quantized layer is a different function from the bf16 one: its
    # distance to the exact forward is the quantization error, well above
    # the kernel's distance to the quantized oracle
    fw = orc.forward(X, Wr, b, W1, W2, cfg.K, topk_idx=g["topk_idx"])
    errs["O_vs_exact"] = P.normwise(fq["O"], fw["O"])
    print(cfg.name, {k: f"{v:.2e}" for k, v in errs.items()}, f"H accumulation error <= 2^{acc:.1f} |Xq||W1q|")
    assert errs["O"] <= P.TOL_BF16 and errs["H"] <= P.TOL_BF16, errs
    assert errs["O"] < errs["O_vs_exact"], errs


@pytest.mark.gpu
def test_mxfp8_forward_full_size_sampled():
    """7B-class layer (T 16384, d 1536, E 128, n 256, K 8) in the benchmark's
    launch configuration; O on sampled tokens, H of the least loaded expert."""
    cfg = CONFIGS["7b"]
    inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
    layer = _mx_layer(cfg, inp)
    g = P.gpu_routing(layer, cfg.T)
    X = P.f64(inp["X"])
    Wr = P.f64(inp["Wr"])
    b = None if inp["bias"] is None else P.f64(inp["bias"])
    z = orc.router_logits(X, Wr, b)
    P.check_permutation(g, cfg.E)
    W1 = P.LazyExperts(inp["W1"])
    W2 = P.LazyExperts(inp["W2"])
    rs = np.random.RandomState(cfg.seed + 9)
    toks = np.sort(rs.choice(cfg.T, 128, replace=False))
    fq = mx.forward_mxfp8(X[toks], Wr, b, W1, W2, cfg.K, routing=P.sub_routing(g, z, toks))
    err = P.normwise(P.f64(layer.O[toks]), fq["O"])
    counts = g["counts"]
    nz = np.nonzero(counts > 0)[0]
    e = int(nz[np.argmin(counts[nz])])
    te = P.tokens_of_expert(g, e)
    fe = mx.forward_mxfp8(X[te], Wr, b, W1, W2, cfg.K, routing=P.sub_routing(g, z, te))
    # rows of expert e in the oracle's order: its tokens ascending, as on the GPU
    a, c = g["offsets"][e], g["offsets"][e] + counts[e]
    Hg = P.f64(layer.H[a:c])
    sel = fe["seg"][e], fe["seg"][e + 1]
    errH = P.normwise(Hg, fe["H"][sel[0]:sel[1]])
    print("7b mxfp8", f"O {err:.2e}", f"H[{e}] {errH:.2e}")
    assert err <= P.TOL_BF16 and errH <= P.TOL_BF16


@pytest.mark.gpu
def test_mxfp8_forward_rejects_unsupported_n():
    from fine_grained_mixture_top_b200 import moe
    cfg = MoEConfig("mx_n64", T=64, d=128, E=4, n=64, K=2, seed=25)
    inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K)
    assert layer.sizes.fwd_mx_ws == 0
    layer.route(inp["X"], inp["Wr"], inp["bias"])
    with pytest.raises(moe.MoEError):
        layer.forward(inp["X"], inp["W1"], inp["W2"], mxfp8=True)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", [1, 2])
def test_mxfp8_forward_after_token_rounding(mode):
    """Token-rounded routing (every expert a multiple of 128 rows, tokens
    with a varying number of experts) feeds the MXFP8 forward unchanged."""
    from fine_grained_mixture_top_b200 import moe
    cfg = MoEConfig("mx_tr", T=1500, d=256, E=16, n=128, K=2, w_std=0.05, bias="normal", seed=26,
                    round_mode=mode)
    inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
    layer = moe.MoELayer(cfg.T, cfg.d, cfg.E, cfg.n, cfg.K, round_mode=mode, seed=cfg.seed)
    layer.route(inp["X"], inp["Wr"], inp["bias"])
    layer.forward(inp["X"], inp["W1"], inp["W2"], mxfp8=True)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    g = P.gpu_routing(layer, cfg.T)
    assert np.all(g["counts"] % 128 == 0)
    X, Wr, W1, W2 = (P.f64(inp[k]) for k in ("X", "Wr", "W1", "W2"))
    rt = {"tok_ptr": g["tok_ptr"], "pair_expert": g["pair_expert"], "pair_gate": g["pair_gate"]}
    fq = mx.forward_mxfp8(X, Wr, None, W1, W2, cfg.K, routing=rt)
    err = P.normwise(P.f64(layer.O), fq["O"])
    print("mx_tr", mode, f"O {err:.2e}")
    assert err <= P.TOL_BF16


@pytest.mark.gpu
def test_prequantized_weights_give_the_same_forward():
    """Weights quantized once (moe_mx_quantize_weights) then
    moe_forward_mxfp8_q: bit for bit the forward that quantizes them itself."""
    from fine_grained_mixture_top_b200 import moe
    cfg = MX_SHAPES[1]
    inp = make_inputs(cfg, "cuda", need_grad_inputs=False)
    layer = _mx_layer(cfg, inp)
    O1, H1 = layer.O.clone(), layer.H.clone()
    wq = layer.quantize_weights_mxfp8(inp["W1"], inp["W2"])
    layer.O.zero_()
    layer.H.zero_()
    layer.forward_mxfp8_q(inp["X"], wq)
    torch.cuda.synchronize()
    assert moe.moe_get_status()[0] == 0
    assert torch.equal(layer.O.view(torch.int16), O1.view(torch.int16))
    R = int(layer.routing["offsets"][cfg.E].item())
    assert torch.equal(layer.H[:R].view(torch.int16), H1[:R].view(torch.int16))
