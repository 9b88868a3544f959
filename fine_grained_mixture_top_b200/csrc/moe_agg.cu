// Bandwidth-bound kernels: expert aggregation (forward O and backward dX) and
// the router backward (dS reduction, softmax-over-selected-logits Jacobian).
//
// Sources: page "SonicMoE：突破细粒度MoE硬件效率瓶颈，实现高稀疏性下的极致训练加速",
// implementation paragraph (expert aggregation kernel O in the forward, dX
// aggregation in the backward; the layer is grouped GEMMs plus aggregation)
// and algorithm paragraph (router gradient without cached activations).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ void acc8(float (&acc)[8], uint4 v, float g) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    acc[2 * i] = fmaf(g, f.x, acc[2 * i]);
    acc[2 * i + 1] = fmaf(g, f.y, acc[2 * i + 1]);
  }
}
__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
  uint4 o;
  o.x = pack_bf16x2(acc[0], acc[1]);
  o.y = pack_bf16x2(acc[2], acc[3]);
  o.z = pack_bf16x2(acc[4], acc[5]);
  o.w = pack_bf16x2(acc[6], acc[7]);
  return o;
}

// O[t, 8c .. 8c+8) = sum_p gate_p * Y[row_p, 8c .. 8c+8)   (fp32 accumulate)
__global__ void __launch_bounds__(256) aggregate_fwd_kernel(int T, int d8, const int* __restrict__ tok_ptr,
                                                            const int* __restrict__ pair_row,
                                                            const float* __restrict__ pair_gate,
                                                            const uint4* __restrict__ Y, uint4* __restrict__ O) {
  pdl_wait();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)T * d8) return;
  const int t = (int)(idx / d8), c = (int)(idx - (int64_t)t * d8);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int p0 = __ldg(tok_ptr + t), p1 = __ldg(tok_ptr + t + 1);
  int p = p0;
  for (; p + 4 <= p1; p += 4) {
    uint4 v[4];
    float g[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[j] = __ldg(Y + (size_t)__ldg(pair_row + p + j) * d8 + c);
      g[j] = __ldg(pair_gate + p + j);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) acc8(acc, v[j], g[j]);
  }
  for (; p < p1; ++p) acc8(acc, __ldg(Y + (size_t)__ldg(pair_row + p) * d8 + c), __ldg(pair_gate + p));
  O[idx] = pack8(acc);
}

cudaError_t launch_aggregate_fwd(int T, int d, const int* tok_ptr, const int* pair_row, const float* pair_gate,
                                 const __nv_bfloat16* Y, __nv_bfloat16* O, cudaStream_t s) {
  const int d8 = d / 8;
  const int64_t n = (int64_t)T * d8;
  launch_pdl(aggregate_fwd_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, 
      T, d8, tok_ptr, pair_row, pair_gate, reinterpret_cast<const uint4*>(Y), reinterpret_cast<uint4*>(O));
  return cudaGetLastError();
}

// One warp per token.  dS_p = sum of the dH kernel's per-N-tile partials of
// row(p); dz_p = s_p (dS_p - sum_j s_j dS_j).  Writes dz per padded row
// (fp32, dz_row[row(p)]; padding rows are not written) for the dX~ epilogue,
// and the token's dense dz row split into bf16 hi + lo parts for the
// tensor-core dWr = X^T dz GEMM (layout: group g of 64 experts at columns
// [128 g, 128 g + 128): hi parts then lo parts).
__device__ __forceinline__ void router_bwd_token(const BwdPrepArgs& a, int t, int sub) {
  // a segment of a.lanes lanes (a power of two, aligned in the warp) per
  // token, so that one warp overlaps the dependent loads of several tokens;
  // every lane runs the shuffles, tokens past T do no memory work
  const int T = a.T, Epad = a.Epad, nts = a.nds, L = a.lanes;
  const int* __restrict__ tok_ptr = a.tok_ptr;
  const int* __restrict__ pair_row = a.pair_row;
  const int* __restrict__ pair_expert = a.pair_expert;
  const float* __restrict__ pair_gate = a.pair_gate;
  const float* __restrict__ dS_part = a.dS_part;
  float* __restrict__ dz_row = a.dz_row;
  __nv_bfloat16* __restrict__ dz_split = a.dz_split;
  const bool live = t < T;
  const int p0 = live ? tok_ptr[t] : 0, p1 = live ? tok_ptr[t + 1] : 0;
  float inner = 0.f;
  for (int p = p0 + sub; p < p1; p += L) {
    const float* part = dS_part + (size_t)pair_row[p] * nts;
    float ds = 0.f;
    for (int j = 0; j < nts; ++j) ds += part[j];
    if (a.pair_dS) a.pair_dS[p] = ds;
    if (!a.router) continue;
    dz_row[pair_row[p]] = ds;  // dS for now
    inner += pair_gate[p] * ds;
  }
  if (!a.router) return;
  for (int o = L >> 1; o > 0; o >>= 1) inner += __shfl_xor_sync(0xffffffffu, inner, o);
  if (live) {  // the dense dz row: zeros, then each pair's hi and lo parts
    uint4* row4 = reinterpret_cast<uint4*>(dz_split + (size_t)t * 2 * Epad);
    for (int c = sub; c < Epad / 4; c += L) row4[c] = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncwarp();
  __nv_bfloat16* row = dz_split + (size_t)t * 2 * Epad;
  for (int p = p0 + sub; p < p1; p += L) {
    const int r = pair_row[p];
    const float dz = pair_gate[p] * (dz_row[r] - inner);
    dz_row[r] = dz;
    const int e = pair_expert[p];
    const __nv_bfloat16 hi = __float2bfloat16_rn(dz);
    const __nv_bfloat16 lo = __float2bfloat16_rn(dz - __bfloat162float(hi));
    const int col = (e >> 6) * 128 + (e & 63);
    row[col] = hi;
    row[col + 64] = lo;
  }
}



// WrT[e, i] = Wr[i, e]
// 32 x 32 tile (bx, by) of the transpose, 256 threads (32 x 8)
__device__ __forceinline__ void transpose_tile(const float* __restrict__ in, float* __restrict__ out, int rows,
                                               int cols, int bx, int by) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c0 = bx * 32, r0 = by * 32;
  for (int i = ty; i < 32; i += 8) {
    const int r = r0 + i, c = c0 + tx;
    if (r < rows && c < cols) tile[i][tx] = in[(size_t)r * cols + c];
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int c = c0 + i, r = r0 + tx;
    if (r < rows && c < cols) out[(size_t)c * rows + r] = tile[tx][i];
  }
}



// Wr^T as a kernel of its own (the router backward from given dS).
__global__ void __launch_bounds__(256) wr_transpose_kernel(const float* __restrict__ Wr, float* __restrict__ WrT,
                                                           int d, int E) {
  pdl_wait();
  const int nbx = (E + 31) / 32;
  transpose_tile(Wr, WrT, d, E, blockIdx.x % nbx, blockIdx.x / nbx);
}

// Router backward from caller-given dS per pair (dS[pos[p]], or dS[p] without
// pos): one warp per token.  dz_p = s_p (dS_p - sum_q s_q dS_q) over the
// token's pairs; the dense dz row split into bf16 hi + lo parts for the
// dWr = X^T dz GEMM (layout as in router_bwd_token); dX_t += sum_p dz_p Wr[:, e_p]
// (bf16 in and out, fp32 sums).
__global__ void __launch_bounds__(256) router_bwd_given_kernel(int T, int d, int Epad, const int* __restrict__ tok_ptr,
                                                               const int* __restrict__ pair_expert,
                                                               const float* __restrict__ pair_gate,
                                                               const float* __restrict__ dS,
                                                               const int* __restrict__ pos,
                                                               const float* __restrict__ WrT,
                                                               __nv_bfloat16* __restrict__ dz_split,
                                                               __nv_bfloat16* __restrict__ dX) {
  pdl_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int p0 = tok_ptr[t], p1 = tok_ptr[t + 1];
  auto ds_of = [&](int p) { return dS[pos ? pos[p] : p]; };
  float inner = 0.f;
  for (int p = p0 + lane; p < p1; p += 32) inner += pair_gate[p] * ds_of(p);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) inner += __shfl_xor_sync(0xffffffffu, inner, o);
  __nv_bfloat16* row = dz_split + (size_t)t * 2 * Epad;
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  for (int c = lane; c < 2 * Epad; c += 32) row[c] = zero;
  __syncwarp();
  for (int p = p0 + lane; p < p1; p += 32) {
    const float dz = pair_gate[p] * (ds_of(p) - inner);
    const int e = pair_expert[p];
    const __nv_bfloat16 hi = __float2bfloat16_rn(dz);
    const __nv_bfloat16 lo = __float2bfloat16_rn(dz - __bfloat162float(hi));
    const int col = (e >> 6) * 128 + (e & 63);
    row[col] = hi;
    row[col + 64] = lo;
  }
  // dX row: 8 columns per lane per step
  uint4* xr = reinterpret_cast<uint4*>(dX + (size_t)t * d);
  for (int c8 = lane; c8 < d / 8; c8 += 32) {
    float acc[8];
    const uint4 v = xr[c8];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      acc[2 * i] = f.x;
      acc[2 * i + 1] = f.y;
    }
    for (int p = p0; p < p1; ++p) {
      const float dz = pair_gate[p] * (ds_of(p) - inner);
      const float4* w = reinterpret_cast<const float4*>(WrT + (size_t)pair_expert[p] * d) + 2 * c8;
      const float4 a = __ldg(w), b = __ldg(w + 1);
      acc[0] = fmaf(dz, a.x, acc[0]);
      acc[1] = fmaf(dz, a.y, acc[1]);
      acc[2] = fmaf(dz, a.z, acc[2]);
      acc[3] = fmaf(dz, a.w, acc[3]);
      acc[4] = fmaf(dz, b.x, acc[4]);
      acc[5] = fmaf(dz, b.y, acc[5]);
      acc[6] = fmaf(dz, b.z, acc[6]);
      acc[7] = fmaf(dz, b.w, acc[7]);
    }
    xr[c8] = pack8(acc);
  }
}

cudaError_t launch_router_bwd_given(int T, int d, int E, int Epad, const int* tok_ptr, const int* pair_expert,
                                    const float* pair_gate, const float* dS, const int* pos, const float* Wr,
                                    float* WrT, __nv_bfloat16* dz_split, __nv_bfloat16* dX, cudaStream_t s) {
  const int nb = ((E + 31) / 32) * ((d + 31) / 32);
  launch_pdl(wr_transpose_kernel, dim3(nb), dim3(256), 0, s, Wr, WrT, d, E);
  launch_pdl(router_bwd_given_kernel, dim3((unsigned)((T + 7) / 8)), dim3(256), 0, s, T, d, Epad, tok_ptr,
             pair_expert, pair_gate, dS, pos, (const float*)WrT, dz_split, dX);
  return cudaGetLastError();
}

// dWr[i, e] = sum over K splits of the split-K partials, in split order
__global__ void dwr_reduce_kernel(int d, int E, int Epad, int splits, const float* __restrict__ part,
                                  float* __restrict__ dWr) {
  pdl_wait();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)d * E) return;
  const int i = (int)(idx / E), e = (int)(idx - (int64_t)i * E);
  float s = 0.f;
  for (int k = 0; k < splits; ++k) s += part[((size_t)k * d + i) * Epad + e];
  dWr[idx] = s;
}

cudaError_t launch_dwr_reduce(int d, int E, int Epad, int splits, const float* part, float* dWr, cudaStream_t s) {
  const int64_t n = (int64_t)d * E;
  launch_pdl(dwr_reduce_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, d, E, Epad, splits, part, dWr);
  return cudaGetLastError();
}

// dX[t, 8c .. 8c+8) = sum_p dX~[row_p, ...]  (the router path's dz_p Wr[:, e_p]
// is already inside dX~, added by the dX~ GEMM's epilogue)
__global__ void __launch_bounds__(256) aggregate_bwd_kernel(int T, int d8, const int* __restrict__ tok_ptr,
                                                            const int* __restrict__ pair_row,
                                                            const uint4* __restrict__ dXt,
                                                            uint4* __restrict__ dX) {
  pdl_wait();
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)T * d8) return;
  const int t = (int)(idx / d8), c = (int)(idx - (int64_t)t * d8);
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const int p0 = __ldg(tok_ptr + t), p1 = __ldg(tok_ptr + t + 1);
  int p = p0;
  for (; p + 4 <= p1; p += 4) {
    uint4 v[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) v[j] = __ldg(dXt + (size_t)__ldg(pair_row + p + j) * d8 + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) acc8(acc, v[j], 1.0f);
  }
  for (; p < p1; ++p) acc8(acc, __ldg(dXt + (size_t)__ldg(pair_row + p) * d8 + c), 1.0f);
  dX[idx] = pack8(acc);
}

cudaError_t launch_aggregate_bwd(int T, int d, const int* tok_ptr, const int* pair_row, const __nv_bfloat16* dXt,
                                 __nv_bfloat16* dX, cudaStream_t s) {
  const int d8 = d / 8;
  const int64_t n = (int64_t)T * d8;
  launch_pdl(aggregate_bwd_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, 
      T, d8, tok_ptr, pair_row, reinterpret_cast<const uint4*>(dXt), reinterpret_cast<uint4*>(dX));
  return cudaGetLastError();
}

// Experts sorted by descending token count (ties: lower index first); the
// weight-gradient GEMMs take their tiles in this order so that the longest
// tiles start first.
__device__ __forceinline__ void expert_order_block(int E, const int* __restrict__ counts, int* __restrict__ order) {
  __shared__ int c[1024];
  for (int e = threadIdx.x; e < E; e += blockDim.x) c[e] = counts[e];
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int ce = c[e];
    int rank = 0;
    for (int j = 0; j < E; ++j) rank += (c[j] > ce) || (c[j] == ce && j < e);
    order[rank] = e;
  }
}

// One launch before the weight-gradient GEMMs (after the dH kernel):
//   blocks [0, tok_blocks)              router backward, one warp per token
//   next tr_blocks blocks               Wr^T for the dX~ epilogue's router path
//   last block                          expert order (largest first) for the
//                                       weight-gradient scheduler; zeroes its
//                                       tile counters
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdPrepArgs a) {
  pdl_wait();
  const int b = blockIdx.x;
  if (b < a.tok_blocks) {
    const int per_warp = 32 / a.lanes;
    const int lane = threadIdx.x & 31;
    router_bwd_token(a, (b * 8 + (threadIdx.x >> 5)) * per_warp + lane / a.lanes, lane & (a.lanes - 1));
    return;
  }
  if (b < a.tok_blocks + a.tr_blocks) {
    const int i = b - a.tok_blocks;
    const int nbx = (a.E + 31) / 32;
    transpose_tile(a.Wr, a.WrT, a.d, a.E, i % nbx, i / nbx);
    return;
  }
  if (threadIdx.x < 16) a.sched[threadIdx.x] = 0;
  expert_order_block(a.E, a.counts, a.expert_order);
}

cudaError_t launch_bwd_prep(const BwdPrepArgs& a0, cudaStream_t s) {
  BwdPrepArgs a = a0;
  // lanes per token: the power of two at or above K, at most 32 (tokens that
  // gained pairs in token rounding loop over them)
  a.lanes = 1;
  while (a.lanes < a.K && a.lanes < 32) a.lanes <<= 1;
  const int tok_per_block = 8 * (32 / a.lanes);
  a.tok_blocks = (a.router || a.pair_dS) ? (a.T + tok_per_block - 1) / tok_per_block : 0;
  a.tr_blocks = a.router ? ((a.E + 31) / 32) * ((a.d + 31) / 32) : 0;
  launch_pdl(bwd_prep_kernel, dim3(a.tok_blocks + a.tr_blocks + 1), dim3(256), 0, s, a);
  return cudaGetLastError();
}


// Failure-detection self test: one thread waits on an mbarrier that nothing
// will ever complete, through the same bounded wait the GEMM kernels use, and
// must come back with ST_TIMEOUT recorded in the status word.
__global__ void wait_selftest_kernel(int* out, DevStatus st) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(smem_u32(&bar), 0, &abort_flag, st, 999);
    out[0] = ok ? 1 : 0;
    mbar_arrive(smem_u32(&bar));  // complete the phase so the barrier is left consistent
  }
}

cudaError_t launch_wait_selftest(int* flag, DevStatus st, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(flag, st);
  return cudaGetLastError();
}

}  // namespace moe
