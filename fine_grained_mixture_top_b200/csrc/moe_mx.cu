// MXFP8 quantization kernels: rows (X, quantized along d), columns of expert
// weights (W1 along d, W2 along n, written transposed so that K is
// contiguous), and the rearrangement of weight scales into the 512-byte
// scale tiles the block-scaled MMA copies into tensor memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.h"
#include "mx.cuh"

namespace moe {

// Eight lanes per 32-element block, four elements per lane.
__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                                            int K, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int kblocks = K / kMxBlock;
  const int64_t blk = g >> 3;
  const int l = (int)(g & 7);
  const bool live = blk < rows * kblocks;
  const int64_t row = live ? blk / kblocks : 0;
  const int kb = live ? (int)(blk - row * kblocks) : 0;
  const size_t off = (size_t)row * K + (size_t)kb * kMxBlock + 4 * l;
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    const uint2 raw = *reinterpret_cast<const uint2*>(in + off);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    x[0] = fa.x; x[1] = fa.y; x[2] = fb.x; x[3] = fb.y;
  }
  float m = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  const uint32_t code = mx_scale_code(m);
  const float s = mx_inv_scale(code);
  if (!live) return;
  const uint32_t q = mx_e4m3x2(x[0] * s, x[1] * s) | (mx_e4m3x2(x[2] * s, x[3] * s) << 16);
  *reinterpret_cast<uint32_t*>(codes + off) = q;
  if (l == 0) scales[(size_t)row * kblocks + kb] = (uint8_t)code;
}

// One thread per (expert, column, 32-block of K): in[e][k][c] for the block's
// 32 k (consecutive threads take consecutive columns, so every load is
// coalesced) -> codes[e][c][k] (32 contiguous bytes) and its scale.
__global__ void __launch_bounds__(256) mx_quant_cols_kernel(const __nv_bfloat16* __restrict__ in, int E, int K,
                                                            int N, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int kblocks = K / kMxBlock;
  if (g >= (int64_t)E * kblocks * N) return;
  const int c = (int)(g % N);
  const int64_t ek = g / N;
  const int kb = (int)(ek % kblocks);
  const int e = (int)(ek / kblocks);
  const __nv_bfloat16* src = in + ((size_t)e * K + (size_t)kb * kMxBlock) * N + c;
  float x[kMxBlock];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < kMxBlock; ++i) {
    x[i] = __bfloat162float(src[(size_t)i * N]);
    m = fmaxf(m, fabsf(x[i]));
  }
  const uint32_t code = mx_scale_code(m);
  const float s = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = mx_e4m3x2(x[4 * i] * s, x[4 * i + 1] * s) | (mx_e4m3x2(x[4 * i + 2] * s, x[4 * i + 3] * s) << 16);
  uint4* dst = reinterpret_cast<uint4*>(codes + ((size_t)e * N + c) * K + (size_t)kb * kMxBlock);
  dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
  dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[((size_t)e * N + c) * kblocks + kb] = (uint8_t)code;
}

// Scale tiles of a weight operand: for expert e, N tile nt (128 columns) and
// K block kb (128 elements, 4 scales), 512 bytes with the scale of tile row m
// (0..127) and K sub-block j (0..3) at byte 16 (m % 32) + 4 (m / 32) + j.
// split_half: the tile's rows are 64 columns of the first half of N (gate)
// followed by the same 64 columns of the second half (up), the up-proj's
// N tile; otherwise 128 consecutive columns.
__global__ void __launch_bounds__(256) mx_scale_tiles_kernel(const uint8_t* __restrict__ scales, int E, int K,
                                                             int N, int split_half, uint8_t* __restrict__ tiles) {
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int ntiles = split_half ? N / 128 : N / 128;  // 128 tile rows either way
  const int kb128 = K / 128;
  if (g >= (int64_t)E * ntiles * kb128 * 512) return;
  const int byte = (int)(g & 511);
  const int64_t t = g >> 9;
  const int kb = (int)(t % kb128);
  const int nt = (int)((t / kb128) % ntiles);
  const int e = (int)(t / ((int64_t)kb128 * ntiles));
  const int r = byte >> 4, m1 = (byte >> 2) & 3, j = byte & 3;
  const int m = r + 32 * m1;
  int c;
  if (split_half) {
    const int half = N / 2;
    c = m < 64 ? nt * 64 + m : half + nt * 64 + (m - 64);
  } else {
    c = nt * 128 + m;
  }
  tiles[g] = scales[((size_t)e * N + c) * (K / kMxBlock) + kb * 4 + j];
}

cudaError_t launch_mx_quant_rows(const __nv_bfloat16* in, int64_t rows, int K, uint8_t* codes, uint8_t* scales,
                                 cudaStream_t s) {
  const int64_t threads = rows * (K / kMxBlock) * 8;
  if (threads == 0) return cudaSuccess;
  mx_quant_rows_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(in, rows, K, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const __nv_bfloat16* in, int E, int K, int N, uint8_t* codes, uint8_t* scales,
                                 cudaStream_t s) {
  const int64_t threads = (int64_t)E * (K / kMxBlock) * N;
  if (threads == 0) return cudaSuccess;
  mx_quant_cols_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(in, E, K, N, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_scale_tiles(const uint8_t* scales, int E, int K, int N, int split_half, uint8_t* tiles,
                                  cudaStream_t s) {
  const int64_t threads = (int64_t)E * (N / 128) * (K / 128) * 512;
  if (threads == 0) return cudaSuccess;
  mx_scale_tiles_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, s>>>(scales, E, K, N, split_half, tiles);
  return cudaGetLastError();
}

}  // namespace moe
