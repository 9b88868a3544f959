"""MXFP8 reference ("the oracle") for the layer's forward with block-scaled
8-bit GEMM operands.

TEST INFRASTRUCTURE ONLY, like moe_oracle: only the tests, the smoke check
and the benchmark's CPU-baseline leg may use it, and it imports nothing from
the product package.

The pages name "MXFP8/FP4 precision support" as the method's future work
(page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing paragraph) and
give nothing more.  The format is therefore taken from its public
definition, the OCP Microscaling (MX) formats: blocks of 32 consecutive
elements along the GEMM's K dimension share one power-of-two scale stored as
E8M0 (an 8-bit biased exponent, bias 127), and each element is an FP8 E4M3
value (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; subnormals; no
infinities; the one NaN pattern S.1111.111; largest finite 448).

Readings (each listed in the design notes):
  M1 Shared exponent: the smallest e with amax <= 448 * 2^e, so no element
     of a block saturates.  With amax = f * 2^E, 1 <= f < 2, that is
     e = E - 8, plus 1 when f > 1.75.  An all-zero block gets scale code 0.
     This DEPARTS from the OCP MX v1.0 specification (section 6.3), whose
     shared exponent is floor(log2 amax) - 8 (8 = the exponent of E4M3's
     largest normal, 448 = 1.75 * 2^8) with the elements that then exceed 448
     clamped to 448.  The two rules agree when f <= 1.75 and differ by one
     when f > 1.75 (about one block in eight for Gaussian data): OCP's rule
     clamps that block's largest element(s), by up to 12.5 %; M1 instead
     doubles the block's scale, so no element is clamped and every element
     keeps the half-ulp error bound, at the cost of one bit of resolution
     for the block's smallest elements.  `scale_exponent_ocp` states OCP's
     rule for comparison; the tests pin both and the cases where they
     differ.
  M2 Elements: v / 2^e rounded to the nearest E4M3 value, ties to the even
     code; magnitudes above 448 (none, given M1) saturate to 448.  A value
     that rounds to zero keeps its sign (code 0x80 for negative).
  M3 What is quantized: X along d per row, W1[e] along d per output column,
     A along n per row, W2[e] along n per output column -- the K dimension
     of each forward GEMM.  H and Y stay bf16 outputs of fp32 accumulation;
     the backward is unchanged (bf16).
  M4 The quantized forward computes A = SwiGLU(H) from H rounded to bf16 --
     the activation the layer stores for its backward -- then quantizes A per
     row in blocks of 32 along n.  The A codes are integer decisions taken
     from floating-point values, so both sides take them from the same bf16
     H (H itself is returned unrounded, the exact product of the quantized
     operands).

Parity status: pinned by tests/test_oracle_mx.py (the E4M3 table against the
format's closed form, round trips of every code, ties to even, the scale
rule against brute force, the element error bound, power-of-two
equivariance, exactness on representable inputs, the E=1, K=1 dense case
against plain numpy matmuls, and several experts against per-token loops).
"""
from __future__ import annotations

import numpy as np

from . import moe_oracle as mo

F64 = np.float64
BLOCK = 32
E4M3_MAX = 448.0


# --------------------------------------------------------------------------
# E4M3 elements.
# --------------------------------------------------------------------------
def e4m3_decode(code):
    """Value of E4M3 codes (uint8 array or int); NaN for S.1111.111."""
    c = np.asarray(code, np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    m = c & 0x7
    sub = s * (m / 8.0) * 2.0 ** -6
    nrm = s * (1.0 + m / 8.0) * np.exp2(ex.astype(F64) - 7.0)
    v = np.where(ex == 0, sub, nrm)
    return np.where((c & 0x7F) == 0x7F, np.nan, v)


# the 127 non-negative finite magnitudes, codes 0x00 .. 0x7E (increasing)
_MAG = e4m3_decode(np.arange(0x7F))


def e4m3_encode(x):
    """Nearest E4M3 code of each value (M2): ties to the even code, saturate
    to +-448, the sign of a value that rounds to zero is kept."""
    x = np.asarray(x, F64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.searchsorted(_MAG, a, side="left")          # first magnitude >= a
    hi = np.minimum(hi, 0x7E)
    lo = np.maximum(hi - 1, 0)
    dlo = a - _MAG[lo]
    dhi = _MAG[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a == _MAG[hi], hi, mag)
    neg = np.signbit(x)
    return (mag | np.where(neg, 0x80, 0)).astype(np.uint8)


# --------------------------------------------------------------------------
# E8M0 block scales.
# --------------------------------------------------------------------------
def scale_exponent(amax):
    """Shared exponent e of M1 for block maxima amax (>= 0); -127 for 0."""
    amax = np.asarray(amax, F64)
    f, E = np.frexp(amax)          # amax = f * 2^E with 0.5 <= f < 1
    f = 2.0 * f                    # 1 <= f < 2
    E = E.astype(np.int64) - 1
    e = E - 8 + (f > 1.75)
    return np.where(amax > 0, e, -127)


def scale_exponent_ocp(amax):
    """Shared exponent of the OCP MX v1.0 rule (section 6.3), for comparison
    with M1: floor(log2 amax) - 8 for E4M3; -127 for 0.  Not used by the
    quantized forward."""
    amax = np.asarray(amax, F64)
    _, E = np.frexp(amax)          # amax = f * 2^E with 0.5 <= f < 1
    e = E.astype(np.int64) - 1 - 8
    return np.where(amax > 0, e, -127)


def scale_code(amax):
    """E8M0 code (biased exponent, clamped to 0 .. 254)."""
    return np.clip(scale_exponent(amax) + 127, 0, 254).astype(np.uint8)


def scale_value(code):
    return np.exp2(np.asarray(code, F64) - 127.0)


# --------------------------------------------------------------------------
# Quantization along the last axis.
# --------------------------------------------------------------------------
def mx_quantize(M):
    """Quantize along the last axis in blocks of 32: returns (codes, scale
    codes) with codes.shape == M.shape and scales [..., K/32]."""
    M = np.asarray(M, F64)
    K = M.shape[-1]
    assert K % BLOCK == 0
    B = M.reshape(M.shape[:-1] + (K // BLOCK, BLOCK))
    sc = scale_code(np.abs(B).max(axis=-1))
    codes = e4m3_encode(B / scale_value(sc)[..., None])
    return codes.reshape(M.shape), sc


def mx_dequantize(codes, scales):
    c = np.asarray(codes)
    K = c.shape[-1]
    B = e4m3_decode(c).reshape(c.shape[:-1] + (K // BLOCK, BLOCK))
    return (B * scale_value(scales)[..., None]).reshape(c.shape)


def bf16_round(x):
    """Nearest bfloat16 value of each fp64 value (8 significant bits, ties to
    even; below 2^-126 the spacing stays 2^-133)."""
    x = np.asarray(x, F64)
    _, E = np.frexp(x)                                   # |x| in [2^(E-1), 2^E)
    ulp = np.exp2(np.maximum(E.astype(F64) - 8.0, -133.0))
    return np.round(x / ulp) * ulp                       # np.round: half to even


def mx_round(M):
    """M through quantization and back (the values the 8-bit GEMM multiplies)."""
    return mx_dequantize(*mx_quantize(M))


# --------------------------------------------------------------------------
# The quantized forward (M3, M4).
# --------------------------------------------------------------------------
def forward_mxfp8(X, Wr, bias, W1, W2, K, topk_idx=None, routing=None):
    """Layer forward with MXFP8 GEMM operands; same routing, permutation and
    aggregation as moe_oracle.forward.  Returns O and the intermediates."""
    X = np.asarray(X, F64)
    T = X.shape[0]
    E, d, n2 = W1.shape
    n = n2 // 2
    rt = routing if routing is not None else mo.route(X, Wr, bias, K, topk_idx)
    perm = mo.permute(rt["tok_ptr"], rt["pair_expert"], E)
    Xq = mx_round(X)                                     # X along d, per row
    R = len(perm["row_tok"])
    H = np.zeros((R, 2 * n), F64)
    A = np.zeros((R, n), F64)
    Aq = np.zeros((R, n), F64)
    Y = np.zeros((R, d), F64)
    seg = perm["seg"]
    for e in range(E):
        a, b = seg[e], seg[e + 1]
        if b == a:
            continue
        W1q = mx_round(np.asarray(W1[e], F64).T).T       # along d, per output column
        W2q = mx_round(np.asarray(W2[e], F64).T).T       # along n, per output column
        H[a:b] = Xq[perm["row_tok"][a:b]] @ W1q
        A[a:b] = mo.swiglu(bf16_round(H[a:b]), n)         # M4
        Aq[a:b] = mx_round(A[a:b])                       # A along n, per row
        Y[a:b] = Aq[a:b] @ W2q
    O = mo.aggregate(Y, rt["pair_gate"], perm["pair_row"], rt["tok_ptr"], T)
    out = dict(rt)
    out.update(perm)
    out.update({"H": H, "A": A, "Aq": Aq, "Y": Y, "O": O})
    return out
