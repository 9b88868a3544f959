// Routing kernels: router-weight split for the tensor-core logits, softmax +
// top-K + gates, the stable counting-sort permutation into 128-padded expert
// segments, and token rounding.
//
// Sources: page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", section
// "MoE 与它的隐患" (each token is routed to a few experts; the standard
// implementation keeps the routing metadata as a mask) and section
// "第二，IO 感知的算子融合" (the GEMM gathers routed rows itself, so the
// permutation only has to produce row indices); page
// "SonicMoE：突破细粒度MoE硬件效率瓶颈，实现高稀疏性下的极致训练加速",
// scheduling paragraph (token rounding to multiples of the GEMM tile).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <climits>

#include "moe_internal.h"

namespace moe {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Exclusive scan over a 1024-thread block; *total receives the block sum.
__device__ int block_exclusive_scan_1024(int v, int* sh /*[33]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = sh[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    sh[lane] = w;
  }
  __syncthreads();
  const int prefix = warp > 0 ? sh[warp - 1] : 0;
  *total = sh[31];
  __syncthreads();
  return prefix + x - v;
}

// ---------------------------------------------------------------- Wr split
// Wr (fp32) = hi + mid + lo with each part a bf16; X is exactly bf16, so the
// three tensor-core products accumulated in fp32 give fp32-accurate logits.
// Layout: column group g (64 experts) occupies columns [192 g, 192 g + 192):
// hi, mid, lo parts of experts 64 g .. 64 g + 63 (zero beyond E).
__global__ void split_wr_kernel(const float* __restrict__ Wr, __nv_bfloat16* __restrict__ out, int d, int E,
                                int Epad) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)d * Epad) return;
  const int i = (int)(idx / Epad), e = (int)(idx % Epad);
  const float w = e < E ? Wr[(size_t)i * E + e] : 0.f;
  const __nv_bfloat16 hi = __float2bfloat16_rn(w);
  const float r1 = w - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
  __nv_bfloat16* row = out + (size_t)i * 3 * Epad + (e >> 6) * 192 + (e & 63);
  row[0] = hi;
  row[64] = mid;
  row[128] = lo;
}

cudaError_t launch_split_wr(const RouteArgs& a, cudaStream_t s) {
  const int64_t n = (int64_t)a.d * a.Epad;
  split_wr_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(a.Wr, a.Wr_split, a.d, a.E, a.Epad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- softmax + top-K
// One warp per token.  p = softmax(z) over all E; the K largest logits are
// selected (ties to the lower expert index, slots in descending order); the
// gates are a softmax over the selected logits (= p renormalised).
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(256) softmax_topk_kernel(RouteArgs a) {
  extern __shared__ float sh[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* z = sh + warp * a.E;
  uint32_t* sel = reinterpret_cast<uint32_t*>(sh + kTopkWarps * a.E) + warp * 32;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= a.T) return;  // warp-uniform
  const float* lg = a.logits + (size_t)t * a.E;
  float m = -FLT_MAX;
  for (int e = lane; e < a.E; e += 32) {
    const float v = lg[e];
    z[e] = v;
    m = fmaxf(m, v);
  }
  sel[lane] = 0u;
  m = warp_max(m);
  float sum = 0.f;
  for (int e = lane; e < a.E; e += 32) sum += expf(z[e] - m);
  sum = warp_sum(sum);
  const float inv = 1.0f / sum;
  float* pr = a.probs + (size_t)t * a.E;
  for (int e = lane; e < a.E; e += 32) pr[e] = expf(z[e] - m) * inv;
  __syncwarp();

  float my_v = 0.f;
  int my_e = 0;
  for (int k = 0; k < a.K; ++k) {
    float bv = -FLT_MAX;
    int be = INT_MAX;
    for (int e = lane; e < a.E; e += 32) {
      if ((sel[e >> 5] >> (e & 31)) & 1u) continue;
      const float v = z[e];
      if (be == INT_MAX || v > bv || (v == bv && e < be)) {
        bv = v;
        be = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oe = __shfl_xor_sync(0xffffffffu, be, o);
      if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
        bv = ov;
        be = oe;
      }
    }
    if (lane == 0) sel[be >> 5] |= 1u << (be & 31);
    if (lane == k) {
      my_v = bv;
      my_e = be;
    }
    __syncwarp();
  }
  const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
  const float ex = lane < a.K ? expf(my_v - vmax) : 0.f;
  const float den = warp_sum(ex);
  if (lane < a.K) {
    const float g = ex / den;
    const size_t o = (size_t)t * a.K + lane;
    a.topk_idx[o] = my_e;
    a.topk_gate[o] = g;
    a.pair_expert[o] = my_e;
    a.pair_gate[o] = g;
  }
  if (lane == 0) {
    a.tok_ptr[t] = t * a.K;
    if (t == a.T - 1) a.tok_ptr[a.T] = a.T * a.K;
  }
}

cudaError_t launch_softmax_topk(const RouteArgs& a, cudaStream_t s) {
  const int blocks = (a.T + kTopkWarps - 1) / kTopkWarps;
  const size_t smem = (size_t)kTopkWarps * a.E * sizeof(float) + kTopkWarps * 32 * sizeof(uint32_t);
  softmax_topk_kernel<<<blocks, 256, smem, s>>>(a);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- permutation
// Stable counting sort of all (token, expert) pairs by expert.  Tokens are cut
// into chunks of 256; inside a chunk the rank of token t among the chunk's
// tokens routed to e is a popcount over a per-expert bit mask, so the result
// does not depend on the order in which threads run.
__global__ void __launch_bounds__(kChunk) rank_kernel(RouteArgs a) {
  extern __shared__ uint32_t bits[];  // [E][8]
  const int words = kChunk / 32;
  for (int i = threadIdx.x; i < a.E * words; i += blockDim.x) bits[i] = 0u;
  __syncthreads();
  const int t = blockIdx.x * kChunk + threadIdx.x;
  const int w = threadIdx.x >> 5, b = threadIdx.x & 31;
  int p0 = 0, p1 = 0;
  if (t < a.T) {
    p0 = a.tok_ptr[t];
    p1 = a.tok_ptr[t + 1];
    for (int p = p0; p < p1; ++p) atomicOr(&bits[a.pair_expert[p] * words + w], 1u << b);
  }
  __syncthreads();
  for (int p = p0; p < p1; ++p) {
    const uint32_t* be = bits + a.pair_expert[p] * words;
    int r = __popc(be[w] & ((1u << b) - 1u));
    for (int j = 0; j < w; ++j) r += __popc(be[j]);
    a.local_rank[p] = r;
  }
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int c = 0;
    for (int j = 0; j < words; ++j) c += __popc(bits[e * words + j]);
    a.hist[(size_t)blockIdx.x * a.E + e] = c;
  }
}

// Per expert (one warp each, many blocks): exclusive scan over the chunks of
// its per-chunk counts (chunk bases relative to the expert's segment) and
// the expert's total count.
__global__ void __launch_bounds__(256) chunk_scan_kernel(RouteArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= a.E) return;
  int carry = 0;
  for (int c0 = 0; c0 < a.nchunks; c0 += 32) {
    const int c = c0 + lane;
    const int h = c < a.nchunks ? a.hist[(size_t)c * a.E + e] : 0;
    int x = h;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (c < a.nchunks) a.hist[(size_t)c * a.E + e] = carry + x - h;
    carry += __shfl_sync(0xffffffffu, x, 31);
  }
  if (lane == 0) a.counts[e] = carry;
}

// One block: 128-padded segment offsets (exclusive scan over experts).
__global__ void __launch_bounds__(1024) offsets_kernel(RouteArgs a) {
  __shared__ int sh[33];
  int carry = 0;
  for (int e0 = 0; e0 < a.E; e0 += 1024) {
    const int e = e0 + threadIdx.x;
    const int padded = e < a.E ? ((a.counts[e] + kTile - 1) / kTile) * kTile : 0;
    int total;
    const int ex = block_exclusive_scan_1024(padded, sh, &total);
    if (e < a.E) a.offsets[e] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) a.offsets[a.E] = carry;
}

// Per expert (one warp each): the tile -> expert list and the padding rows
// (token -1, gate 0) of its segment.
__global__ void __launch_bounds__(256) segment_fill_kernel(RouteArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= a.E) return;
  const int base = a.offsets[e];
  const int end = a.offsets[e + 1];
  for (int tt = base / kTile + lane; tt < end / kTile; tt += 32) a.tile_expert[tt] = e;
  for (int r = base + a.counts[e] + lane; r < end; r += 32) {
    a.row_tok[r] = -1;
    a.row_gate[r] = 0.f;
  }
}

__global__ void scatter_kernel(RouteArgs a) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= a.T) return;
  const int* base = a.hist + (size_t)(t / kChunk) * a.E;
  for (int p = a.tok_ptr[t]; p < a.tok_ptr[t + 1]; ++p) {
    const int e = a.pair_expert[p];
    const int row = a.offsets[e] + base[e] + a.local_rank[p];
    a.row_tok[row] = t;
    a.row_gate[row] = a.pair_gate[p];
    a.pair_row[p] = row;
  }
}

cudaError_t launch_permute(const RouteArgs& a, cudaStream_t s) {
  {
    ProfScope ps(s, "permute_rank");
    rank_kernel<<<a.nchunks, kChunk, (size_t)a.E * (kChunk / 32) * sizeof(uint32_t), s>>>(a);
  }
  const int eb = (a.E + 7) / 8;
  {
    ProfScope ps(s, "permute_chunk_scan");
    chunk_scan_kernel<<<eb, 256, 0, s>>>(a);
  }
  {
    ProfScope ps(s, "permute_offsets");
    offsets_kernel<<<1, 1024, 0, s>>>(a);
  }
  {
    ProfScope ps(s, "permute_segment_fill");
    segment_fill_kernel<<<eb, 256, 0, s>>>(a);
  }
  {
    ProfScope ps(s, "permute_scatter");
    scatter_kernel<<<(a.T + 255) / 256, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- token rounding
// Readings of the scheduling paragraph (the pages give only the goal: counts
// rounded to multiples of the tile, at most one tile of deviation, total kept
// in expectation):  r = c mod 128; "nearest" rounds up iff r >= 64;
// "stochastic" rounds up iff splitmix64(seed ^ e) mod 128 < r; never above T.
// Down drops the r routed tokens of least p (ties: larger t first); up adds
// the 128 - r unrouted tokens of largest p (ties: smaller t first).
__device__ __forceinline__ unsigned long long splitmix64_dev(unsigned long long x) {
  unsigned long long z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__global__ void tr_member_kernel(const int* tok_ptr, const int* pair_expert, int T, int Ew, uint32_t* member) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  for (int p = tok_ptr[t]; p < tok_ptr[t + 1]; ++p) {
    const int e = pair_expert[p];
    atomicOr(&member[(size_t)t * Ew + (e >> 5)], 1u << (e & 31));
  }
}

// One block per expert: radix select (8 passes of 8 bits) of the k extreme
// 64-bit keys (p bits << 32 | ~t) among the candidate tokens.
__global__ void __launch_bounds__(1024) tr_select_kernel(int T, int E, int Ew, int mode, unsigned long long seed,
                                                         const int* counts, const float* probs,
                                                         const uint32_t* member, uint32_t* final_) {
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_k;
  const int e = blockIdx.x;
  const int c = counts[e];
  const int rem = c % kTile;
  if (rem == 0) return;
  bool up;
  if (mode == 1) up = rem >= kTile / 2;
  else up = (int)(splitmix64_dev(seed ^ (unsigned long long)e) % (unsigned long long)kTile) < rem;
  if (up && c - rem + kTile > T) up = false;
  const int k = up ? kTile - rem : rem;
  const uint32_t wmask = 1u << (e & 31);
  const int wi = e >> 5;
  auto is_cand = [&](int t) -> bool {
    const bool m = (member[(size_t)t * Ew + wi] & wmask) != 0u;
    return up ? !m : m;
  };
  auto key_of = [&](int t) -> unsigned long long {
    const unsigned long long kk =
        ((unsigned long long)__float_as_uint(probs[(size_t)t * E + e]) << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)t);
    return up ? ~kk : kk;   // select the k smallest of this key
  };
  unsigned long long prefix = 0ull, mask = 0ull;
  int kk = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      if (!is_cand(t)) continue;
      const unsigned long long key = key_of(t);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255ull], 1u);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, dg = 0;
      for (; dg < 256; ++dg) {
        if (cum + (int)hist[dg] >= kk) break;
        cum += (int)hist[dg];
      }
      s_prefix = prefix | ((unsigned long long)dg << shift);
      s_k = kk - cum;
    }
    __syncthreads();
    prefix = s_prefix;
    kk = s_k;
    mask |= 255ull << shift;
    __syncthreads();
  }
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    if (!is_cand(t)) continue;
    if (key_of(t) <= prefix) {
      if (up) atomicOr(&final_[(size_t)t * Ew + wi], wmask);
      else atomicAnd(&final_[(size_t)t * Ew + wi], ~wmask);
    }
  }
}

__global__ void tr_count_kernel(const uint32_t* final_, int T, int Ew, int* cnt) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  int c = 0;
  for (int w = 0; w < Ew; ++w) c += __popc(final_[(size_t)t * Ew + w]);
  cnt[t] = c;
}

__global__ void __launch_bounds__(1024) tr_ptr_scan_kernel(const int* cnt, int T, int* tok_ptr) {
  __shared__ int sh[33];
  const int per = (T + 1023) / 1024;
  const int t0 = threadIdx.x * per;
  int local = 0;
  for (int t = t0; t < t0 + per && t < T; ++t) local += cnt[t];
  int total;
  int run = block_exclusive_scan_1024(local, sh, &total);
  for (int t = t0; t < t0 + per && t < T; ++t) {
    tok_ptr[t] = run;
    run += cnt[t];
  }
  if (threadIdx.x == 0) tok_ptr[T] = total;
}

__global__ void tr_write_kernel(const uint32_t* final_, const float* probs, int T, int E, int Ew,
                                const int* tok_ptr, int* pair_expert, float* pair_gate) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= T) return;
  const uint32_t* f = final_ + (size_t)t * Ew;
  const float* pr = probs + (size_t)t * E;
  float sum = 0.f;
  for (int w = 0; w < Ew; ++w)
    for (uint32_t m = f[w]; m; m &= m - 1u) sum += pr[w * 32 + __ffs(m) - 1];
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  int p = tok_ptr[t];
  for (int w = 0; w < Ew; ++w)
    for (uint32_t m = f[w]; m; m &= m - 1u) {
      const int e = w * 32 + __ffs(m) - 1;
      pair_expert[p] = e;
      pair_gate[p] = pr[e] * inv;
      ++p;
    }
}

cudaError_t launch_token_round(const RouteArgs& a, const RoundArgs& r, cudaStream_t s) {
  const size_t mbytes = (size_t)r.T * r.Ew * sizeof(uint32_t);
  cudaError_t err = cudaMemsetAsync(r.member, 0, mbytes, s);
  if (err != cudaSuccess) return err;
  const int tb = (r.T + 255) / 256;
  {
    ProfScope ps(s, "round_member");
    tr_member_kernel<<<tb, 256, 0, s>>>(a.tok_ptr, a.pair_expert, r.T, r.Ew, r.member);
  }
  err = cudaMemcpyAsync(r.final_, r.member, mbytes, cudaMemcpyDeviceToDevice, s);
  if (err != cudaSuccess) return err;
  {
    ProfScope ps(s, "round_select");
    tr_select_kernel<<<r.E, 1024, 0, s>>>(r.T, r.E, r.Ew, r.mode, r.seed, a.counts, r.probs, r.member, r.final_);
  }
  {
    ProfScope ps(s, "round_count");
    tr_count_kernel<<<tb, 256, 0, s>>>(r.final_, r.T, r.Ew, r.cnt);
  }
  {
    ProfScope ps(s, "round_scan");
    tr_ptr_scan_kernel<<<1, 1024, 0, s>>>(r.cnt, r.T, a.tok_ptr);
  }
  {
    ProfScope ps(s, "round_write");
    tr_write_kernel<<<tb, 256, 0, s>>>(r.final_, r.probs, r.T, r.E, r.Ew, a.tok_ptr, a.pair_expert, a.pair_gate);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_permute(a, s);
}

}  // namespace moe
