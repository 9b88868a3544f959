// MXFP8 element and scale helpers: E4M3 elements with one power-of-two
// (E8M0) scale per 32 consecutive K elements.  The element and scale
// encodings are those of the public OCP Microscaling formats; the pages name
// "MXFP8/FP4 precision support" as future work of the method (page
// "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing paragraph)
// without further detail.  The scale rule departs from OCP MX v1.0 (section
// 6.3), see mx_scale_code.
#pragma once
#include <cuda_fp8.h>
#include <cstdint>

namespace moe {

constexpr int kMxBlock = 32;

// E8M0 code of a block maximum: the smallest exponent e with
// amax <= 448 * 2^e (no element saturates), biased by 127 and clamped to
// [0, 254].  With amax = f * 2^E (1 <= f < 2) that is e = E - 8, plus one when
// f > 1.75, decided on the bits of amax.  Zero and fp32-subnormal maxima
// (their e is far below -127) get code 0.  OCP MX v1.0 section 6.3 takes
// floor(log2 amax) - 8 instead and clamps the elements above 448; the two
// differ by one exactly when f > 1.75, where this rule keeps the block's
// maximum unclamped.
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ef = (int)((b >> 23) & 0xFFu);  // biased fp32 exponent = E + 127
  if (ef == 0) return 0u;
  int c = ef - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
  c = c < 0 ? 0 : (c > 254 ? 254 : c);
  return (uint32_t)c;
}

// 2^(127 - code): the exact factor that brings a block onto the element grid.
__device__ __forceinline__ float mx_inv_scale(uint32_t code) {
  return code == 254u ? __uint_as_float(0x00400000u)          // 2^-127, an fp32 subnormal
                      : __uint_as_float((254u - code) << 23);   // 2^(127 - code)
}

// Two fp32 values to two E4M3 codes (round to nearest even, saturating);
// the first value in the low byte, i.e. first in memory.
__device__ __forceinline__ uint32_t mx_e4m3x2(float lo, float hi) {
  return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
}

}  // namespace moe
