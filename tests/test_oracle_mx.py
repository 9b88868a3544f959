"""Pins of the MXFP8 oracle against the format's definition (OCP Microscaling
formats: E4M3 elements, E8M0 block scales of 32) and plain mathematics --
nothing here re-derives a value through the function under test.

The scale rule is reading M1 (the smallest non-saturating power of two), a
stated departure from OCP MX v1.0 section 6.3; both rules are pinned below,
each by brute force, together with the blocks on which they differ."""
import numpy as np

from oracle import moe_oracle as mo
from oracle import mx_oracle as mx


def test_e4m3_table_matches_the_closed_form():
    # hand-computed values from the bit layout S.EEEE.MMM, bias 7
    known = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5, 0x38: 1.0,
             0x39: 1.125, 0x40: 2.0, 0x4E: 4 * 1.75, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0, 0xFE: -448.0}
    for c, v in known.items():
        assert mx.e4m3_decode(c) == v, hex(c)
    assert np.isnan(mx.e4m3_decode(0x7F)) and np.isnan(mx.e4m3_decode(0xFF))
    mags = mx.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(mags) > 0)                      # strictly increasing magnitudes
    # normals: consecutive codes inside a binade differ by 2^(e-7)/8
    for ex in range(1, 16):
        codes = np.arange(ex * 8, min(ex * 8 + 8, 0x7F))
        assert np.allclose(np.diff(mx.e4m3_decode(codes)), 2.0 ** (ex - 7) / 8)


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F])
    np.testing.assert_array_equal(mx.e4m3_encode(mx.e4m3_decode(codes)), codes)


def test_rounding_is_to_nearest_with_ties_to_even():
    mags = mx.e4m3_decode(np.arange(0x7F))
    mid = (mags[:-1] + mags[1:]) / 2                      # exact midpoints
    got = mx.e4m3_encode(mid)
    even = np.where(np.arange(1, 0x7F) % 2 == 0, np.arange(1, 0x7F), np.arange(0, 0x7E))
    np.testing.assert_array_equal(got, even)
    # a hair off the midpoint goes to the nearer neighbour
    np.testing.assert_array_equal(mx.e4m3_encode(mid * (1 + 1e-9)), np.arange(1, 0x7F))
    np.testing.assert_array_equal(mx.e4m3_encode(mid[1:] * (1 - 1e-9)), np.arange(1, 0x7E))
    # saturation and signed zero
    np.testing.assert_array_equal(mx.e4m3_encode([449.0, 1e30, -1e30]), [0x7E, 0x7E, 0xFE])
    np.testing.assert_array_equal(mx.e4m3_encode([-(2.0 ** -11), 0.0, -0.0]), [0x80, 0x00, 0x80])


def test_scale_rule_is_the_smallest_non_saturating_exponent():
    # reading M1, the rule the quantizers and the oracle use
    rng = np.random.default_rng(1)
    amax = np.concatenate([rng.lognormal(0, 6, 2000), [448.0, 449.0, 1.0, 1.75, 1.7500001, 2.0 ** -120]])
    e = mx.scale_exponent(amax)
    # brute force over exponents: amax <= 448 2^e and not amax <= 448 2^(e-1)
    assert np.all(amax <= 448.0 * np.exp2(e.astype(float)))
    assert np.all(amax > 448.0 * np.exp2(e.astype(float) - 1))
    assert mx.scale_exponent(0.0) == -127 and mx.scale_code(0.0) == 0


def _floor_log2_brute(a):
    """Largest integer k with 2^k <= a, by walking k (no frexp, no log)."""
    k = 0
    while 2.0 ** k > a:
        k -= 1
    while 2.0 ** (k + 1) <= a:
        k += 1
    return k


def test_ocp_rule_is_floor_log2_minus_8():
    # OCP MX v1.0 section 6.3: shared exponent = floor(log2 amax) - emax_elem,
    # emax_elem = 8 for E4M3 (448 = 1.75 * 2^8)
    rng = np.random.default_rng(1)
    amax = np.concatenate([rng.lognormal(0, 6, 2000), [448.0, 449.0, 1.0, 1.75, 1.7500001, 2.0 ** -120]])
    brute = np.array([_floor_log2_brute(a) - 8 for a in amax])
    np.testing.assert_array_equal(mx.scale_exponent_ocp(amax), brute)
    assert mx.scale_exponent_ocp(0.0) == -127


def test_m1_departs_from_ocp_exactly_where_ocp_clamps():
    rng = np.random.default_rng(4)
    amax = np.concatenate([rng.lognormal(0, 6, 2000), [1.75, 1.7500001, 1.999, 448.0, 449.0, 511.0]])
    f = amax / np.exp2([_floor_log2_brute(a) for a in amax])      # significand in [1, 2)
    e_m1 = mx.scale_exponent(amax)
    e_ocp = mx.scale_exponent_ocp(amax)
    np.testing.assert_array_equal(e_m1 - e_ocp, (f > 1.75).astype(int))
    # under OCP's exponent the block maximum lands above 448 exactly on those
    # blocks, and E4M3 encoding clamps it to 448; under M1 it never does
    over = amax / np.exp2(e_ocp.astype(float)) > 448.0
    np.testing.assert_array_equal(over, f > 1.75)
    assert np.all(mx.e4m3_decode(mx.e4m3_encode(amax[over] / np.exp2(e_ocp[over].astype(float)))) == 448.0)
    assert np.all(amax / np.exp2(e_m1.astype(float)) <= 448.0)
    # about one block in eight for Gaussian blocks of 32
    g = np.abs(rng.standard_normal((20000, 32))).max(axis=1)
    frac = np.mean(mx.scale_exponent(g) != mx.scale_exponent_ocp(g))
    assert 0.05 < frac < 0.25


def test_block_quantization_error_bound():
    rng = np.random.default_rng(2)
    M = rng.standard_normal((64, 256)) * np.exp2(rng.integers(-20, 20, (64, 1)))
    codes, sc = mx.mx_quantize(M)
    D = mx.mx_dequantize(codes, sc)
    X = np.repeat(mx.scale_value(sc), mx.BLOCK, axis=-1)
    # half a unit in the last place: 2^-4 relative for normals, 2^-10 X below 2^-6 X
    bound = np.maximum(np.abs(M) * 2.0 ** -4, X * 2.0 ** -10)
    assert np.all(np.abs(D - M) <= bound)
    assert np.all(np.abs(M) <= 448.0 * X)                 # nothing saturates


def test_power_of_two_scaling_moves_only_the_scales():
    rng = np.random.default_rng(3)
    M = rng.standard_normal((8, 128))
    c0, s0 = mx.mx_quantize(M)
    for k in (-5, 3, 17):
        c1, s1 = mx.mx_quantize(M * 2.0 ** k)
        np.testing.assert_array_equal(c1, c0)
        np.testing.assert_array_equal(s1.astype(int), s0.astype(int) + k)


def _bf16_torch(x):
    import torch
    return torch.from_numpy(np.asarray(x, np.float64)).float().to(torch.bfloat16).double().numpy()


def test_bf16_rounding_matches_the_format():
    # ties to even at 1: spacing 2^-7 above 1, 2^-8 below
    v = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 - 2.0 ** -9, 1 - 3 * 2.0 ** -9, -(1 + 2.0 ** -8),
                  3 * 2.0 ** -134, 2.0 ** -134, 0.0])
    np.testing.assert_array_equal(mx.bf16_round(v), [1.0, 1 + 2.0 ** -6, 1.0, 1 - 2.0 ** -7, -1.0,
                                                     2.0 ** -132, 0.0, 0.0])
    # fp32 inputs (no double rounding through fp32): the library conversion
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(20000) * np.exp2(rng.integers(-60, 60, 20000))).astype(np.float32).astype(np.float64)
    np.testing.assert_array_equal(mx.bf16_round(x), _bf16_torch(x))


def _layer(T, d, E, n, K, seed, integer=False):
    rng = np.random.default_rng(seed)
    if integer:   # every 32-block holds +-15 and integers: quantization is exact
        X = rng.integers(-15, 16, (T, d)).astype(float)
        X[:, ::32] = 15
        W1 = rng.integers(-15, 16, (E, d, 2 * n)).astype(float)
        W1[:, ::32, :] = -15
    else:
        X = rng.standard_normal((T, d))
        W1 = rng.standard_normal((E, d, 2 * n)) * 0.05
    W2 = rng.standard_normal((E, n, d)) * 0.05
    Wr = rng.standard_normal((d, E)) * 0.05
    return X, Wr, W1, W2


def test_representable_inputs_give_the_exact_up_projection():
    X, Wr, W1, W2 = _layer(40, 64, 4, 32, 2, 4, integer=True)
    np.testing.assert_array_equal(mx.mx_round(X), X)
    fw = mo.forward(X, Wr, None, W1, W2, 2)
    fq = mx.forward_mxfp8(X, Wr, None, W1, W2, 2)
    np.testing.assert_array_equal(fq["H"], fw["H"])
    # A from the stored (bf16) H
    np.testing.assert_array_equal(fq["A"], mo.swiglu(_bf16_torch(fw["H"]), 32))


def test_dense_case_matches_plain_matmuls():
    # E = 1, K = 1: one expert with gate 1, so the layer is a dense MLP on the
    # quantized operands, written out here with numpy alone
    X, Wr, W1, W2 = _layer(33, 64, 1, 64, 1, 5)
    fq = mx.forward_mxfp8(X, Wr, None, W1, W2, 1)

    def q(M, axis):   # quantize along `axis` in blocks of 32, then back
        Mt = np.moveaxis(M, axis, -1)
        B = Mt.reshape(Mt.shape[:-1] + (-1, 32))
        am = np.abs(B).max(-1)
        f, Ex = np.frexp(am)
        e = (Ex - 1) - 8 + (2 * f > 1.75)
        S = np.exp2(e)[..., None]
        return np.moveaxis((mx.e4m3_decode(mx.e4m3_encode(B / S)) * S).reshape(Mt.shape), -1, axis)

    H = q(X, 1) @ q(W1[0], 0)
    np.testing.assert_allclose(fq["H"], H, rtol=1e-12, atol=1e-12)
    Hb = _bf16_torch(H)
    g, u = Hb[:, :64], Hb[:, 64:]
    A = g / (1 + np.exp(-g)) * u
    O = q(A, 1) @ q(W2[0], 0)
    np.testing.assert_allclose(fq["O"], O, rtol=1e-12, atol=1e-12)


def test_quantized_forward_stays_near_the_exact_forward():
    X, Wr, W1, W2 = _layer(64, 128, 8, 64, 2, 6)
    fw = mo.forward(X, Wr, None, W1, W2, 2)
    fq = mx.forward_mxfp8(X, Wr, None, W1, W2, 2)
    rel = np.abs(fq["O"] - fw["O"]).max() / np.abs(fw["O"]).max()
    # three 3-bit-mantissa roundings on the path to O: a few percent, not more
    assert 1e-4 < rel < 0.1, rel


def test_quantized_forward_equals_per_token_loops():
    """Several experts, K = 2, skewed router: every token's output written out
    as a loop over its experts (quantize X_t and the expert's weight columns,
    SwiGLU of the bf16-rounded H, quantize A, multiply, gate), with numpy
    alone for the arithmetic and the format's codec for the rounding."""
    rng = np.random.default_rng(8)
    T, d, E, n, K = 24, 64, 5, 32, 2
    X = rng.standard_normal((T, d))
    W1 = rng.standard_normal((E, d, 2 * n)) * 0.1
    W2 = rng.standard_normal((E, n, d)) * 0.1
    Wr = rng.standard_normal((d, E))
    b = rng.standard_normal(E)
    fq = mx.forward_mxfp8(X, Wr, b, W1, W2, K)

    def q(v):   # blocks of 32 along the last axis
        B = v.reshape(v.shape[:-1] + (-1, 32))
        am = np.abs(B).max(-1)
        f, Ex = np.frexp(am)
        e = np.where(am > 0, (Ex - 1) - 8 + (2 * f > 1.75), -127)
        S = np.exp2(e.astype(float))[..., None]
        return (mx.e4m3_decode(mx.e4m3_encode(B / S)) * S).reshape(v.shape)

    z = X @ Wr + b
    O = np.zeros((T, d))
    for t in range(T):
        top = sorted(range(E), key=lambda e: (-z[t, e], e))[:K]
        g = np.exp(z[t, top] - z[t, top].max())
        g /= g.sum()
        for s, e in zip(g, top):
            h = q(X[t]) @ q(W1[e].T).T
            hb = _bf16_torch(h)
            a = hb[:n] / (1 + np.exp(-hb[:n])) * hb[n:]
            O[t] += s * (q(a) @ q(W2[e].T).T)
    np.testing.assert_allclose(fq["O"], O, rtol=1e-12, atol=1e-12)
