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
