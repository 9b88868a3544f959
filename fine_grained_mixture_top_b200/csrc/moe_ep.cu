// Expert parallelism and caller-given routing.
//
// The pages name expert parallelism as future work of the method (page
// "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing paragraph) with a
// token all-to-all before the up-projection and after the down-projection.
// The exchange itself is the caller's (NCCL all-to-all); the kernels here lay
// the routed rows out for it and take them back:
//   given_pairs_kernel  routing pairs from a caller's [T, K] selection, with
//                       the range and distinctness checks the permutation
//                       relies on
//   ep_scan_kernel      exclusive prefix sum of the per-expert row counts
//   ep_pack_kernel      the routed rows of a [T, d] tensor in expert-major
//                       order without padding (the send buffer), their gates
//   ep_pos_kernel       each pair's position in that order (for the combine)
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "moe_internal.h"

namespace moe {

// One thread per token.  A token whose selection has an expert outside
// [0, E) or the same expert twice is replaced by experts 0 .. K-1 with gate 0
// (so that the permutation stays in bounds) and reported as a failed check.
__global__ void __launch_bounds__(256) given_pairs_kernel(int T, int K, int E, const int* __restrict__ topk_idx,
                                                          const float* __restrict__ topk_gate, int* __restrict__ tok_ptr,
                                                          int* __restrict__ pair_expert, float* __restrict__ pair_gate,
                                                          DevStatus st) {
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t > T) return;
  tok_ptr[t] = t * K;
  if (t == T) return;
  bool ok = true;
  for (int k = 0; k < K; ++k) {
    const int e = topk_idx[(size_t)t * K + k];
    ok = ok && e >= 0 && e < E;
    for (int j = 0; j < k; ++j) ok = ok && topk_idx[(size_t)t * K + j] != e;
  }
  if (!ok) raise_status(st, ST_DEVICE_CHECK, 100);
  for (int k = 0; k < K; ++k) {
    const size_t p = (size_t)t * K + k;
    pair_expert[p] = ok ? topk_idx[p] : k;
    pair_gate[p] = ok ? topk_gate[p] : 0.f;
  }
}

// cum[e] = rows of experts before e (unpadded); cum[E] = all rows.  One block.
__global__ void __launch_bounds__(1024) ep_scan_kernel(int E, const int* __restrict__ counts, int* __restrict__ cum) {
  pdl_wait();
  __shared__ int s[1024];
  const int i = threadIdx.x;
  s[i] = i < E ? counts[i] : 0;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {  // inclusive Hillis-Steele scan
    const int v = i >= o ? s[i - o] : 0;
    __syncthreads();
    s[i] += v;
    __syncthreads();
  }
  if (i < E) cum[i + 1] = s[i];
  if (i == 0) cum[0] = 0;
}

// One warp per padded row: the row's real position j in expert-major order
// (padding rows are skipped), send[j] = src[token] in 16-byte pieces, four
// loads in flight per lane, and lane 0 writes the gate.
__global__ void __launch_bounds__(256) ep_pack_kernel(int64_t R_max, int d8, const int* __restrict__ offsets, int E,
                                                      const int* __restrict__ counts, const int* __restrict__ cum,
                                                      const int* __restrict__ tile_expert,
                                                      const int* __restrict__ row_tok, const float* __restrict__ row_gate,
                                                      const uint4* __restrict__ src, uint4* __restrict__ send,
                                                      float* __restrict__ send_gate) {
  pdl_wait();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R_max || r >= __ldg(offsets + E)) return;
  const int e = __ldg(tile_expert + (r >> 7));
  const int i = (int)r - __ldg(offsets + e);
  if (i >= __ldg(counts + e)) return;  // padding row
  const int64_t j = (int64_t)__ldg(cum + e) + i;
  const uint4* s = src + (size_t)__ldg(row_tok + r) * d8;
  uint4* o = send + j * d8;
  for (int c = lane; c < d8; c += 128) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c + 32 * u < d8) v[u] = __ldg(s + c + 32 * u);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c + 32 * u < d8) o[c + 32 * u] = v[u];
  }
  if (lane == 0 && send_gate) send_gate[j] = __ldg(row_gate + r);
}

// pair_pos[p] = position of pair p's row in the send order.
__global__ void __launch_bounds__(256) ep_pos_kernel(int T, const int* __restrict__ tok_ptr,
                                                     const int* __restrict__ pair_expert,
                                                     const int* __restrict__ pair_row, const int* __restrict__ offsets,
                                                     const int* __restrict__ cum, int* __restrict__ pair_pos) {
  pdl_wait();
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= __ldg(tok_ptr + T)) return;
  const int e = __ldg(pair_expert + p);
  pair_pos[p] = __ldg(cum + e) + (__ldg(pair_row + p) - __ldg(offsets + e));
}

cudaError_t launch_given_pairs(int T, int K, int E, const int* topk_idx, const float* topk_gate, int* tok_ptr,
                               int* pair_expert, float* pair_gate, DevStatus st, cudaStream_t s) {
  launch_pdl(given_pairs_kernel, dim3((unsigned)((T + 1 + 255) / 256)), dim3(256), 0, s, T, K, E, topk_idx,
             topk_gate, tok_ptr, pair_expert, pair_gate, st);
  return cudaGetLastError();
}

cudaError_t launch_ep_pack(int T, int d, int E, int64_t R_max, int64_t P_max, const int* tok_ptr,
                           const int* pair_expert, const int* pair_row, const int* counts, const int* offsets,
                           const int* tile_expert, const int* row_tok, const float* row_gate,
                           const __nv_bfloat16* src, __nv_bfloat16* send, float* send_gate, int* pair_pos, int* cum,
                           cudaStream_t s) {
  launch_pdl(ep_scan_kernel, dim3(1), dim3(1024), 0, s, E, counts, cum);
  const int d8 = d / 8;
  if (send) {
    launch_pdl(ep_pack_kernel, dim3((unsigned)((R_max + 7) / 8)), dim3(256), 0, s, R_max, d8, offsets, E, counts,
               (const int*)cum, tile_expert, row_tok, row_gate, reinterpret_cast<const uint4*>(src),
               reinterpret_cast<uint4*>(send), send_gate);
  }
  if (pair_pos)
    launch_pdl(ep_pos_kernel, dim3((unsigned)((P_max + 255) / 256)), dim3(256), 0, s, T, tok_ptr, pair_expert,
               pair_row, offsets, (const int*)cum, pair_pos);
  return cudaGetLastError();
}

}  // namespace moe
