// MXFP8 quantization kernels: rows (X, quantized along d), columns of expert
// weights (W1 along d, W2 along n, written transposed so that K is
// contiguous), and the rearrangement of weight scales into the 512-byte
// scale tiles the block-scaled MMA copies into tensor memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.h"
#include "mx.cuh"

namespace moe {

// Four lanes per 32-element block, eight elements (16 bytes) per lane; each
// thread takes kRowIters blocks a grid apart and issues all their loads
// before any arithmetic, so that enough bytes are in flight per SM.
constexpr int kRowIters = 4;

__global__ void __launch_bounds__(256) mx_quant_rows_kernel(const __nv_bfloat16* __restrict__ in, int64_t rows,
                                                            int K, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  pdl_wait();
  const int kblocks = K / kMxBlock;
  const int64_t slots = rows * kblocks * 4;  // 4 lanes per block
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t g0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint4 raw[kRowIters];
#pragma unroll
  for (int it = 0; it < kRowIters; ++it) {
    const int64_t g = g0 + it * stride;
    raw[it] = make_uint4(0u, 0u, 0u, 0u);
    if (g < slots) raw[it] = __ldg(reinterpret_cast<const uint4*>(in) + g);  // slot g = elements [8g, 8g + 8)
  }
#pragma unroll
  for (int it = 0; it < kRowIters; ++it) {
    const int64_t g = g0 + it * stride;
    float x[8];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[it]);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    // the 4 lanes of a block are adjacent and share liveness (slots and the
    // grid stride are multiples of 4)
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    if (g >= slots) continue;
    const uint32_t code = mx_scale_code(m);
    const float s = mx_inv_scale(code);
    uint2 q;
    q.x = mx_e4m3x2(x[0] * s, x[1] * s) | (mx_e4m3x2(x[2] * s, x[3] * s) << 16);
    q.y = mx_e4m3x2(x[4] * s, x[5] * s) | (mx_e4m3x2(x[6] * s, x[7] * s) << 16);
    reinterpret_cast<uint2*>(codes)[g] = q;
    if ((g & 3) == 0) scales[g >> 2] = (uint8_t)code;  // block index = row * kblocks + kb
  }
}

// One thread per (expert, column, 32-block of K): in[e][k][c] for the block's
// 32 k (consecutive threads take consecutive columns, so every load is
// coalesced) -> codes[e][c][k] (32 contiguous bytes) and its scale.  Any
// shape with K % 32 == 0.
__global__ void __launch_bounds__(256) mx_quant_cols_kernel(const __nv_bfloat16* __restrict__ in, int E, int K,
                                                            int N, uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ scales) {
  pdl_wait();
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

// Tiled form for K % 128 == 0 and N % 64 == 0: a block takes one expert, 128
// K rows and 64 columns.  The 16 KB tile comes in with 16-byte coalesced
// loads into shared memory; each thread then quantizes one (column, 32-block)
// from there.  Scales go to the linear layout [E][N][K/32] and/or straight
// into the GEMM's scale tiles: for expert e, N tile nt (128 tile rows) and K
// block kb (128 elements, 4 scales), 512 bytes with the scale of tile row m
// and K sub-block j at byte 16 (m % 32) + 4 (m / 32) + j.  split_half: a tile's
// rows are 64 columns of the first half of N (gate) followed by the same 64
// columns of the second half (up), the up-projection's N tile; otherwise
// 128 consecutive columns.
__global__ void __launch_bounds__(256) mx_quant_cols_tiled_kernel(const __nv_bfloat16* __restrict__ in, int K,
                                                                  int N, int split_half, uint8_t* __restrict__ codes,
                                                                  uint8_t* __restrict__ scales,
                                                                  uint8_t* __restrict__ tiles) {
  pdl_wait();
  __shared__ __align__(16) __nv_bfloat16 tile[128][64];
  const int e = blockIdx.z;
  const int k0 = blockIdx.y * 128;
  const int c0 = blockIdx.x * 64;
  const int t = threadIdx.x;
  const __nv_bfloat16* src = in + ((size_t)e * K + k0) * N + c0;
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // 1024 16-byte pieces: row = piece / 8, 8 pieces per row
    const int piece = t + 256 * i;
    v[i] = __ldg(reinterpret_cast<const uint4*>(src + (size_t)(piece >> 3) * N) + (piece & 7));
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int piece = t + 256 * i;
    *reinterpret_cast<uint4*>(&tile[piece >> 3][(piece & 7) * 8]) = v[i];
  }
  __syncthreads();
  const int c = t & 63;   // column within the tile
  const int j = t >> 6;   // 32-block within the 128 K rows
  float x[kMxBlock];
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < kMxBlock; ++i) {
    x[i] = __bfloat162float(tile[32 * j + i][c]);
    m = fmaxf(m, fabsf(x[i]));
  }
  const uint32_t code = mx_scale_code(m);
  const float s = mx_inv_scale(code);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    w[i] = mx_e4m3x2(x[4 * i] * s, x[4 * i + 1] * s) | (mx_e4m3x2(x[4 * i + 2] * s, x[4 * i + 3] * s) << 16);
  // codes and scales through shared memory, so that each column's 128 code
  // bytes and 4 scale bytes leave as whole 16- and 4-byte pieces
  __shared__ __align__(16) uint8_t qs[64][128 + 16];   // padded rows: the 16-byte writes below spread over banks
  __shared__ __align__(4) uint8_t ss[64][4];
  __syncthreads();  // every thread has read its tile column
  *reinterpret_cast<uint4*>(&qs[c][32 * j]) = make_uint4(w[0], w[1], w[2], w[3]);
  *reinterpret_cast<uint4*>(&qs[c][32 * j + 16]) = make_uint4(w[4], w[5], w[6], w[7]);
  ss[c][j] = (uint8_t)code;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 2; ++i) {  // 512 16-byte pieces: column = piece / 8
    const int piece = t + 256 * i;
    const int cc = piece >> 3, q = piece & 7;
    *reinterpret_cast<uint4*>(codes + ((size_t)e * N + c0 + cc) * K + k0 + 16 * q) =
        *reinterpret_cast<const uint4*>(&qs[cc][16 * q]);
  }
  if (t < 64) {
    const int cg = c0 + t;
    const uint32_t sw = *reinterpret_cast<const uint32_t*>(&ss[t][0]);
    if (scales) {
      uint8_t* dst = scales + ((size_t)e * N + cg) * (K / kMxBlock) + k0 / kMxBlock;
#pragma unroll
      for (int b = 0; b < 4; ++b) dst[b] = (uint8_t)(sw >> (8 * b));
    }
    if (tiles) {
      int nt, mrow;
      if (split_half) {
        const int half = N / 2;
        const int h = cg >= half ? 1 : 0;
        const int cc = cg - h * half;
        nt = cc / 64;
        mrow = h * 64 + cc % 64;
      } else {
        nt = cg / 128;
        mrow = cg % 128;
      }
      const size_t tix = ((size_t)e * (N / 128) + nt) * (K / 128) + k0 / 128;
      *reinterpret_cast<uint32_t*>(tiles + tix * 512 + 16 * (mrow & 31) + 4 * (mrow >> 5)) = sw;
    }
  }
}

cudaError_t launch_mx_quant_rows(const __nv_bfloat16* in, int64_t rows, int K, uint8_t* codes, uint8_t* scales,
                                 cudaStream_t s) {
  const int64_t slots = rows * (K / kMxBlock) * 4;
  if (slots == 0) return cudaSuccess;
  const int64_t threads = (slots + kRowIters - 1) / kRowIters;
  const int64_t blocks = (threads + 255) / 256;  // grid stride = blocks * 256, a multiple of 4
  launch_pdl(mx_quant_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, s, in, rows, K, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_mx_quant_cols(const __nv_bfloat16* in, int E, int K, int N, uint8_t* codes, uint8_t* scales,
                                 uint8_t* tiles, int split_half, cudaStream_t s) {
  if ((int64_t)E * K * N == 0) return cudaSuccess;
  if (K % 128 == 0 && N % 64 == 0) {
    if (tiles && N % 128 != 0) return cudaErrorInvalidValue;
    dim3 grid((unsigned)(N / 64), (unsigned)(K / 128), (unsigned)E);
    launch_pdl(mx_quant_cols_tiled_kernel, dim3(grid), dim3(256), 0, s, in, K, N, split_half, codes, scales, tiles);
    return cudaGetLastError();
  }
  if (tiles) return cudaErrorInvalidValue;
  const int64_t threads = (int64_t)E * (K / kMxBlock) * N;
  launch_pdl(mx_quant_cols_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0, s, in, E, K, N, codes, scales);
  return cudaGetLastError();
}

}  // namespace moe
