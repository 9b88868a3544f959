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
#include <cstdlib>

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

// ---------------------------------------------------------------- Wr split
// Wr (fp32) = hi + mid + lo with each part a bf16; X is exactly bf16, so the
// three tensor-core products accumulated in fp32 give fp32-accurate logits.
// Layout: column group g (64 experts) occupies columns [192 g, 192 g + 192):
// hi, mid, lo parts of experts 64 g .. 64 g + 63 (zero beyond E).
__global__ void split_wr_kernel(const float* __restrict__ Wr, __nv_bfloat16* __restrict__ out, int d, int E,
                                int Epad) {
  pdl_wait();
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
  launch_pdl(split_wr_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s, a.Wr, a.Wr_split, a.d, a.E, a.Epad);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- softmax + top-K
// One warp per token; lane l holds the logits of experts l, l + 32, ... in
// registers (PER of them).  p = softmax(z) over all E.  The K largest logits
// are selected in K rounds (ties to the lower expert index, slots in
// descending order): each lane keeps its best unselected logit as an
// order-preserving integer key; one warp-wide max finds the round's value and
// one warp-wide min the lowest expert holding it.  Only the lane that gave up
// its logit looks for its next best.  The gates are a softmax over the
// selected logits (= p renormalised).
constexpr int kTopkWarps = 8;

// Unsigned key with the order of the float (no NaNs among logits); 0 is
// below the key of every float.
__device__ __forceinline__ uint32_t order_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

template <int PER>
__global__ void __launch_bounds__(256) softmax_topk_kernel(RouteArgs a) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= a.T) return;  // warp-uniform
  const float* lg = a.logits + (size_t)t * a.E;
  float z[PER];
  float m = -FLT_MAX;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int e = lane + 32 * j;
    z[j] = e < a.E ? lg[e] : -FLT_MAX;
    if (e < a.E) m = fmaxf(m, z[j]);
  }
  m = warp_max(m);
  float ex[PER];
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    ex[j] = expf(z[j] - m);
    if (lane + 32 * j < a.E) sum += ex[j];
  }
  sum = warp_sum(sum);
  const float inv = 1.0f / sum;
  float* pr = a.probs + (size_t)t * a.E;
#pragma unroll
  for (int j = 0; j < PER; ++j)
    if (lane + 32 * j < a.E) pr[lane + 32 * j] = ex[j] * inv;

  // keys of this lane's unselected logits (0: none); -0 keys like +0
  uint32_t key[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) key[j] = (lane + 32 * j < a.E) ? order_key(z[j] == 0.f ? 0.f : z[j]) : 0u;
  uint32_t best = 0u;
  int bj = 0;
  auto local_best = [&]() {  // strict >: the lower expert of a lane wins a tie
    best = 0u;
    bj = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j)
      if (key[j] > best) {
        best = key[j];
        bj = j;
      }
  };
  local_best();
  uint32_t my_key = 0u;
  int my_e = 0;
  for (int k = 0; k < a.K; ++k) {
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, best);
    const uint32_t win = __reduce_min_sync(0xffffffffu, best == kmax ? (uint32_t)(lane + 32 * bj) : 0xFFFFFFFFu);
    if (lane == (int)(win & 31u)) {
#pragma unroll
      for (int j = 0; j < PER; ++j)
        if (j == bj) key[j] = 0u;
      local_best();
    }
    if (lane == k) {
      my_key = kmax;
      my_e = (int)win;
    }
  }
  const float my_v = key_value(my_key);
  const float vmax = __shfl_sync(0xffffffffu, my_v, 0);
  const float g_ex = lane < a.K ? expf(my_v - vmax) : 0.f;
  const float den = warp_sum(g_ex);
  if (lane < a.K) {
    const float g = g_ex / den;
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
  const int per = (a.E + 31) / 32;
  if (per <= 1) launch_pdl(softmax_topk_kernel<1>, dim3(blocks), dim3(256), 0, s, a);
  else if (per <= 2) launch_pdl(softmax_topk_kernel<2>, dim3(blocks), dim3(256), 0, s, a);
  else if (per <= 4) launch_pdl(softmax_topk_kernel<4>, dim3(blocks), dim3(256), 0, s, a);
  else if (per <= 8) launch_pdl(softmax_topk_kernel<8>, dim3(blocks), dim3(256), 0, s, a);
  else if (per <= 16) launch_pdl(softmax_topk_kernel<16>, dim3(blocks), dim3(256), 0, s, a);
  else if (per <= 32) launch_pdl(softmax_topk_kernel<32>, dim3(blocks), dim3(256), 0, s, a);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

// ---------------------------------------------------------------- permutation
// Stable counting sort of all (token, expert) pairs by expert, in two
// launches.  Tokens are cut into chunks of 256; inside a chunk the rank of
// token t among the chunk's tokens routed to e is a popcount over a
// per-expert bit mask, so the result does not depend on the order in which
// threads run.

// Exclusive scan over a block of kScanThreads threads; *total gets the sum.
constexpr int kScanThreads = 256;
__device__ int block_exclusive_scan_256(int v, int* sh /*[8]*/, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int kWarps = kScanThreads / 32;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  int prefix = 0, sum = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    const int wv = sh[i];
    if (i < warp) prefix += wv;
    sum += wv;
  }
  __syncthreads();
  *total = sum;
  return prefix + x - v;
}

// One block per chunk: each pair's rank inside its chunk and expert, and the
// chunk's per-expert counts.  The last block to finish then scans, per
// expert (a thread each), its chunk counts into chunk bases relative to the
// expert's segment and the expert's total count, and the 128-padded segment
// offsets over the experts (*a.sync zeroed before the launch).
static_assert(kChunk == kScanThreads, "the rank kernel's block scans with kScanThreads threads");
__global__ void __launch_bounds__(kChunk) rank_kernel(RouteArgs a) {
  pdl_wait();
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
  // The last block to arrive sees every block's counts: each block fences its
  // writes before it counts itself done, and the last one fences before reading.
  __shared__ int is_last;
  __shared__ int sh[kScanThreads / 32];
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(a.sync, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // a thread per expert: its chunk counts (coalesced over the experts) in
  // batches of 16 loads in flight, scanned in chunk order
  constexpr int kB = 16;
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) {
    int carry = 0;
    for (int c0 = 0; c0 < a.nchunks; c0 += kB) {
      int h[kB];
#pragma unroll
      for (int j = 0; j < kB; ++j) h[j] = c0 + j < a.nchunks ? __ldcg(a.hist + (size_t)(c0 + j) * a.E + e) : 0;
#pragma unroll
      for (int j = 0; j < kB; ++j)
        if (c0 + j < a.nchunks) {
          a.hist[(size_t)(c0 + j) * a.E + e] = carry;
          carry += h[j];
        }
    }
    a.counts[e] = carry;
  }
  __syncthreads();  // every count written (and visible to the block)
  int carry = 0;
  for (int e0 = 0; e0 < a.E; e0 += kScanThreads) {
    const int ee = e0 + threadIdx.x;
    const int padded = ee < a.E ? ((a.counts[ee] + kTile - 1) / kTile) * kTile : 0;
    int total;
    const int ex = block_exclusive_scan_256(padded, sh, &total);
    if (ee < a.E) a.offsets[ee] = carry + ex;
    carry += total;
  }
  if (threadIdx.x == 0) a.offsets[a.E] = carry;
}

// Blocks [0, token_blocks): one thread per token writes its pairs' rows.
// The blocks after those: one warp per expert writes the tile -> expert list
// and the padding rows (token -1, gate 0) of its segment.
__global__ void __launch_bounds__(256) scatter_kernel(RouteArgs a, int token_blocks) {
  pdl_wait();
  if ((int)blockIdx.x >= token_blocks) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = ((int)blockIdx.x - token_blocks) * 8 + warp;
    if (e >= a.E) return;
    const int base = a.offsets[e];
    const int end = a.offsets[e + 1];
    for (int tt = base / kTile + lane; tt < end / kTile; tt += 32) a.tile_expert[tt] = e;
    for (int r = base + a.counts[e] + lane; r < end; r += 32) {
      a.row_tok[r] = -1;
      a.row_gate[r] = 0.f;
    }
    return;
  }
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
  cudaError_t err = cudaMemsetAsync(a.sync, 0, sizeof(int), s);  // the rank kernel's last-block counter
  if (err != cudaSuccess) return err;
  {
    ProfScope ps(s, "permute_rank");
    launch_pdl(rank_kernel, dim3(a.nchunks), dim3(kChunk), (size_t)a.E * (kChunk / 32) * sizeof(uint32_t), s, a);
  }
  {
    ProfScope ps(s, "permute_scatter");
    const int token_blocks = (a.T + 255) / 256;
    launch_pdl(scatter_kernel, dim3(token_blocks + (a.E + 7) / 8), dim3(256), 0, s, a, token_blocks);
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

// Token rounding works on per-expert rows: memberT[e][w] holds bit t & 31 of
// word w = t / 32 for each token t routed to e, probsT[e][t] = p[t, e].  One
// block per expert then reads its row contiguously.  tr_member also records
// each token's pair count, which the selection adjusts token by token, and
// counts each expert's routed tokens (counts zeroed before the launch): per
// block in shared memory, then one global add per block and expert (a hot
// expert's count would otherwise take thousands of same-address atomics).
__global__ void __launch_bounds__(256) tr_member_kernel(const int* tok_ptr, const int* pair_expert, int T, int E,
                                                        int W, uint32_t* memberT, int* tok_count, int* counts,
                                                        int* sync) {
  pdl_wait();
  __shared__ int s_cnt[1024];  // E <= 1024
  for (int e = threadIdx.x; e < E; e += blockDim.x) s_cnt[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t == 0) *sync = 0;  // for tr_scan_kernel's last block
  if (t < T) {
    const int p0 = tok_ptr[t], p1 = tok_ptr[t + 1];
    tok_count[t] = p1 - p0;
    for (int p = p0; p < p1; ++p) {
      const int e = pair_expert[p];
      atomicOr(&memberT[(size_t)e * W + (t >> 5)], 1u << (t & 31));
      atomicAdd(&s_cnt[e], 1);
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (s_cnt[e]) atomicAdd(&counts[e], s_cnt[e]);
}

// probsT[e, t] = probs[t, e] through shared memory, 64 x 64 tiles (256
// threads; float4 loads and stores where E and T are multiples of 4, the
// rows then being 16-byte aligned).
constexpr int kTrTile = 64;
__global__ void __launch_bounds__(256) tr_transpose_kernel(const float* __restrict__ probs, float* __restrict__ probsT,
                                                          int T, int E) {
  pdl_wait();
  __shared__ float tile[kTrTile][kTrTile + 1];
  const int e0 = blockIdx.x * kTrTile, t0 = blockIdx.y * kTrTile;
  const int c4 = (threadIdx.x & 15) * 4;  // 4 consecutive columns of the tile
  const int r0 = threadIdx.x >> 4;        // rows r0, r0 + 16, r0 + 32, r0 + 48
  const bool vec = ((E | T) & 3) == 0;
  float v[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // tokens t0 + r, experts e0 + c4 .. + 3
    const int t = t0 + r0 + 16 * i, e = e0 + c4;
    if (vec && t < T && e + 3 < E) {
      const float4 f = *reinterpret_cast<const float4*>(probs + (size_t)t * E + e);
      v[i][0] = f.x;
      v[i][1] = f.y;
      v[i][2] = f.z;
      v[i][3] = f.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[i][j] = (t < T && e + j < E) ? probs[(size_t)t * E + e + j] : 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[r0 + 16 * i][c4 + j] = v[i][j];
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // experts e0 + r, tokens t0 + c4 .. + 3
    const int e = e0 + r0 + 16 * i, t = t0 + c4;
    float o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) o[j] = tile[c4 + j][r0 + 16 * i];
    if (vec && e < E && t + 3 < T) {
      *reinterpret_cast<float4*>(probsT + (size_t)e * T + t) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (e < E && t + j < T) probsT[(size_t)e * T + t + j] = o[j];
    }
  }
}

// Exclusive scan over the block (blockDim.x a multiple of 32, at most 1024);
// *total gets the sum.  sh: 32 ints of shared memory.
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < nw ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    sh[lane] = s;  // inclusive warp totals
  }
  __syncthreads();
  *total = sh[nw - 1];
  const int r = (warp > 0 ? sh[warp - 1] : 0) + x - v;
  __syncthreads();
  return r;
}

// The selection of one expert (one block): the k smallest 64-bit keys among
// the candidate tokens, key = (p bits << 32) | (~0 - t) when rounding down
// (least p first, ties: larger t first) and (~p bits << 32) | t when rounding
// up (largest p first, ties: smaller t first).  Keys are distinct, so "key <=
// the k-th smallest" selects exactly k tokens.
//
// The expert's candidate words are staged in shared memory (when they fit);
// its p row is read from L2 four tokens per load with several loads in
// flight per thread.  Each thread keeps the four smallest keys among its own
// candidates; the
// k-th smallest of these per-thread minima, tau, bounds the k-th smallest
// key from above (k threads each hold a candidate <= tau), so only the
// candidates <= tau -- about k of them when the candidates are spread over
// the threads -- are collected and sorted, which gives the k-th key.  If
// more than kTrListCap candidates are <= tau (fewer than k threads hold
// candidates, or many equal p), 8 radix passes of 8 bits over all
// candidates find it instead.
constexpr int kTrListCap = 2048;
constexpr int kTrSelThreads = 256;  // > the largest k (127)
constexpr size_t kTrSelFixed = (size_t)256 * 4 + (size_t)kTrListCap * 8;  // radix histogram + list
constexpr size_t kTrSelMax = 200 * 1024;  // dynamic shared memory of the staged selection, at most

// Candidates and keys of one expert's selection.  STAGED: the candidate
// words [W] are in shared memory; otherwise they are read from the expert's
// row in global memory, like the keys always are.
template <bool STAGED>
struct TrSelect {
  int T, W;
  bool up;
  const uint32_t* mrow;    // routed tokens of the expert (global)
  const float* prow;       // p of the expert (global)
  const uint32_t* s_cand;  // STAGED: candidate words [W]
  __device__ __forceinline__ uint32_t valid(int w) const {
    return (w == W - 1 && (T & 31)) ? ((1u << (T & 31)) - 1u) : 0xFFFFFFFFu;
  }
  __device__ __forceinline__ uint32_t cand_word(int w) const {
    if constexpr (STAGED) {
      return s_cand[w];
    } else {
      const uint32_t m = mrow[w];
      return (up ? ~m : m) & valid(w);
    }
  }
  __device__ __forceinline__ uint32_t mem_word(int w) const {  // the routed tokens
    if constexpr (STAGED) {
      const uint32_t c = s_cand[w];
      return up ? (~c & valid(w)) : c;
    } else {
      return mrow[w];
    }
  }
  __device__ __forceinline__ uint32_t key32(int t) const {
    const uint32_t pb = __float_as_uint(prow[t]);
    return up ? ~pb : pb;
  }
  __device__ __forceinline__ unsigned long long key64(int t) const {
    return ((unsigned long long)key32(t) << 32) | (up ? (unsigned)t : (0xFFFFFFFFu - (unsigned)t));
  }
};

// 8 passes of 8 bits over all candidates (warp-aggregated histogram
// updates): the k-th smallest key.
template <bool STAGED>
__device__ unsigned long long tr_radix_kth(const TrSelect<STAGED>& s, int k, unsigned* hist /*[256]*/) {
  __shared__ unsigned long long s_prefix;
  __shared__ int s_k;
  const int lane = threadIdx.x & 31;
  unsigned long long prefix = 0ull, mask = 0ull;
  int kk = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int t0 = 0; t0 < s.T; t0 += blockDim.x) {  // warp-uniform trip count
      const int t = t0 + threadIdx.x;
      bool hit = false;
      uint32_t digit = 0u;
      if (t < s.T && ((s.cand_word(t >> 5) >> (t & 31)) & 1u)) {
        const unsigned long long key = s.key64(t);
        hit = (key & mask) == prefix;
        digit = (uint32_t)((key >> shift) & 255ull);
      }
      const uint32_t active = __ballot_sync(0xffffffffu, hit);
      if (hit) {
        const uint32_t peers = __match_any_sync(active, digit);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {  // warp 0: first digit whose running count reaches kk
      int loc[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        loc[i] = (int)hist[8 * lane + i];
        sum += loc[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t reach = __ballot_sync(0xffffffffu, incl >= kk);
      const int owner = __ffs(reach) - 1;  // kk <= number of matching candidates
      if (lane == owner) {
        int cum = incl - sum, dg = 8 * lane;
#pragma unroll 1
        for (int i = 0; i < 8; ++i, ++dg) {
          if (cum + loc[i] >= kk) break;
          cum += loc[i];
        }
        s_prefix = prefix | ((unsigned long long)dg << shift);
        s_k = kk - cum;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    kk = s_k;
    mask |= 255ull << shift;
    __syncthreads();
  }
  return prefix;  // all 64 bits fixed: the k-th smallest key itself
}

// Ascending bitonic sort of n keys in shared memory, padded with ~0 to a
// power of two (the buffer holds it).
__device__ __forceinline__ void tr_sort(unsigned long long* a, int n) {
  int P = 2;
  while (P < n) P <<= 1;
  for (int i = n + threadIdx.x; i < P; i += blockDim.x) a[i] = ~0ull;
  __syncthreads();
  for (int kk = 2; kk <= P; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const unsigned long long x = a[i], y = a[ixj];
          if ((x > y) == ((i & kk) == 0)) {
            a[i] = y;
            a[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Ascending bitonic sort over the block, one key per thread (blockDim.x a
// power of two): returns the key of rank threadIdx.x.  Partners within a
// warp exchange by shuffles; wider strides go through shared memory
// (buf: blockDim.x keys).
__device__ __forceinline__ unsigned long long tr_block_sort1(unsigned long long v, unsigned long long* buf) {
  const int n = (int)blockDim.x, i = (int)threadIdx.x;
  for (int kk = 2; kk <= n; kk <<= 1) {
    for (int j = kk >> 1; j > 0; j >>= 1) {
      unsigned long long o;
      if (j >= 32) {
        buf[i] = v;
        __syncthreads();
        o = buf[i ^ j];
        __syncthreads();
      } else {
        o = __shfl_xor_sync(0xffffffffu, v, j);
      }
      const bool asc = (i & kk) == 0;
      const bool lower = (i & j) == 0;
      v = (lower == asc) ? (o < v ? o : v) : (o > v ? o : v);
    }
  }
  return v;
}

// One block per expert: the expert's final token row finalT[e] (memberT[e]
// with the selected tokens added when rounding up, removed when rounding
// down), its final count (counts[e], rewritten in place), each token's pair
// count adjusted (tok_count[t] += 1 or -= 1), and rowpre[e][w], the number of
// the expert's final tokens before word w (the rank of a token's row inside
// the expert's segment is rowpre plus a popcount within its word).
// STAGED: shared memory holds, after the radix histogram and the list, the
// expert's candidate words [W].  Tokens are visited four at a time (one
// vector load, one candidate nibble).
template <bool STAGED>
__global__ void __launch_bounds__(kTrSelThreads, 4) tr_select_kernel(int T, int W, int mode, unsigned long long seed,
                                                                 int* counts, const float* probsT,
                                                                 const uint32_t* memberT, uint32_t* finalT,
                                                                 int* rowpre, int* tok_count) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t tr_smem[];
  unsigned* hist = reinterpret_cast<unsigned*>(tr_smem);                                 // [256]
  unsigned long long* list = reinterpret_cast<unsigned long long*>(tr_smem + 256 * 4);  // [kTrListCap]
  const int T4 = (T + 3) & ~3;
  uint32_t* s_cand = reinterpret_cast<uint32_t*>(tr_smem + kTrSelFixed);  // STAGED: [W]
  __shared__ int sh[32];
  __shared__ int s_cnt;
  __shared__ unsigned long long s_thr;
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nthr = (int)blockDim.x;
  uint32_t* frow = finalT + (size_t)e * W;
  const int c = counts[e];
  const int rem = c % kTile;
  bool up = false;
  if (rem != 0) {
    if (mode == 1) up = rem >= kTile / 2;
    else up = (int)(splitmix64_dev(seed ^ (unsigned long long)e) % (unsigned long long)kTile) < rem;
    if (up && c - rem + kTile > T) up = false;
  }
  const int k = rem == 0 ? 0 : (up ? kTile - rem : rem);
  TrSelect<STAGED> s;
  s.T = T;
  s.W = W;
  s.up = up;
  s.mrow = memberT + (size_t)e * W;
  s.prow = probsT + (size_t)e * T;
  s.s_cand = s_cand;
  const bool vec = (T & 3) == 0;  // the row is 16-byte aligned: float4 loads
  auto tie = [&](int t) -> unsigned long long { return up ? (unsigned)t : (0xFFFFFFFFu - (unsigned)t); };
  // p keys of tokens 4q .. 4q+3 (past T: the largest key, never a candidate)
  auto load_quad = [&](int q, uint32_t (&kq)[4]) {
    const int t0 = 4 * q;
    float v[4];
    if (vec) {
      const float4 f = reinterpret_cast<const float4*>(s.prow)[q];
      v[0] = f.x;
      v[1] = f.y;
      v[2] = f.z;
      v[3] = f.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) v[j] = t0 + j < T ? s.prow[t0 + j] : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t pb = __float_as_uint(v[j]);
      kq[j] = t0 + j < T ? (up ? ~pb : pb) : 0xFFFFFFFFu;
    }
  };
  auto nibble = [&](int q) -> uint32_t { return (s.cand_word(q >> 3) >> ((4 * q) & 31)) & 0xFu; };
  const int Q = T4 / 4;
  // 1. the candidate words staged (STAGED); each thread's four smallest
  // candidate keys (m[0] <= .. <= m[3], ~0 past its count cnt)
  unsigned long long m[4] = {~0ull, ~0ull, ~0ull, ~0ull};
  uint32_t m3hi = 0xFFFFFFFFu;  // high word of m[3]: keys above it are rejected with one compare
  int cnt = 0;
  auto keep = [&](unsigned long long x) {
    if (x < m[3]) {
      if (x < m[2]) {
        m[3] = m[2];
        if (x < m[1]) {
          m[2] = m[1];
          if (x < m[0]) {
            m[1] = m[0];
            m[0] = x;
          } else {
            m[1] = x;
          }
        } else {
          m[2] = x;
        }
      } else {
        m[3] = x;
      }
      m3hi = (uint32_t)(m[3] >> 32);
    }
  };
  if constexpr (STAGED) {
    for (int w = threadIdx.x; w < W; w += nthr) {
      const uint32_t m = s.mrow[w];
      s_cand[w] = (up ? ~m : m) & s.valid(w);
    }
    __syncthreads();
  }
  if (k > 0) {
    constexpr int kBatch = 4;  // quads per thread whose loads are in flight together
    for (int q0 = threadIdx.x; q0 < Q; q0 += kBatch * nthr) {
      uint32_t kq[kBatch][4];
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (q0 + u * nthr < Q) load_quad(q0 + u * nthr, kq[u]);
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int q = q0 + u * nthr;
        if (q < Q) {
          const uint32_t nb = nibble(q);
          cnt += __popc(nb);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (((nb >> j) & 1u) && kq[u][j] <= m3hi) keep(((unsigned long long)kq[u][j] << 32) | tie(4 * q + j));
        }
      }
    }
  }
  unsigned long long thr = 0ull;
  bool listed = false;  // the selected tokens are the list entries <= thr
  int len = 0;
  if (k > 0) {
    // 2. tau: the k-th smallest thread minimum (k < 128 <= nthr)
    const unsigned long long r = tr_block_sort1(m[0], list);
    if (threadIdx.x == k - 1) s_thr = r;
    if (threadIdx.x == 0) s_cnt = 0;
    __syncthreads();
    const unsigned long long tau = s_thr;
    // 3. the candidates <= tau; the k-th smallest of them is the k-th key.
    // A thread's kept keys hold all of its candidates <= tau unless it saw
    // more than four and its fourth is <= tau; only then does it read its
    // tokens again.
    auto push = [&](unsigned long long x) {
      const int i = atomicAdd(&s_cnt, 1);
      if (i < kTrListCap) list[i] = x;
    };
    if (cnt > 4 && m[3] <= tau) {
      for (int q = threadIdx.x; q < Q; q += nthr) {
        const uint32_t nb = nibble(q);
        if (nb == 0u) continue;
        uint32_t kq[4];
        load_quad(q, kq);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if ((nb >> j) & 1u) {
            const unsigned long long x = ((unsigned long long)kq[j] << 32) | tie(4 * q + j);
            if (x <= tau) push(x);
          }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (i < cnt && m[i] <= tau) push(m[i]);
    }
    __syncthreads();
    len = s_cnt;
    if (len <= nthr) {
      const unsigned long long v = threadIdx.x < len ? list[threadIdx.x] : ~0ull;
      __syncthreads();  // list[] is reused as the sort's exchange buffer
      const unsigned long long r2 = tr_block_sort1(v, list);
      if (threadIdx.x == k - 1) s_thr = r2;
      __syncthreads();
      if (threadIdx.x < len) list[threadIdx.x] = r2;  // sorted: the first k are the selected
      __syncthreads();
      thr = s_thr;
      listed = true;
    } else if (len <= kTrListCap) {
      tr_sort(list, len);
      thr = list[k - 1];
      listed = true;
    } else {
      thr = tr_radix_kth<STAGED>(s, k, hist);
    }
  }
  if (STAGED && (listed || k == 0)) {
    // 4a. final row in shared memory: the routed words with the k selected
    // tokens (the first k sorted list entries) set or cleared
    for (int w = threadIdx.x; w < W; w += nthr) s_cand[w] = s.mem_word(w);
    __syncthreads();
    for (int i = threadIdx.x; i < k; i += nthr) {
      const unsigned lo = (unsigned)(list[i] & 0xFFFFFFFFull);
      const int t = up ? (int)lo : (int)(0xFFFFFFFFu - lo);
      if (up) atomicOr(&s_cand[t >> 5], 1u << (t & 31));
      else atomicAnd(&s_cand[t >> 5], ~(1u << (t & 31)));
      atomicAdd(&tok_count[t], up ? 1 : -1);
    }
    __syncthreads();
    for (int w = threadIdx.x; w < W; w += nthr) frow[w] = s_cand[w];
  } else {
    // 4b. final row: a warp per word of 32 tokens; the selected candidates
    // are the keys <= thr
    for (int w0 = 0; w0 < W; w0 += nthr / 32) {
      const int w = w0 + warp;
      if (w < W) {  // warp-uniform
        const int t = 32 * w + lane;
        const uint32_t mem = s.mem_word(w);
        uint32_t sel = 0u;
        if (k > 0) {
          const bool take = ((s.cand_word(w) >> lane) & 1u) && s.key64(t) <= thr;
          sel = __ballot_sync(0xffffffffu, take);
          if (take) atomicAdd(&tok_count[t], up ? 1 : -1);
        }
        const uint32_t fin = up ? (mem | sel) : (mem & ~sel);
        __syncwarp();
        if (lane == 0) {
          frow[w] = fin;
          if constexpr (STAGED) s_cand[w] = fin;  // only this warp reads word w here
        }
      }
    }
  }
  if (threadIdx.x == 0) counts[e] = rem == 0 ? c : (up ? c - rem + kTile : c - rem);
  __syncthreads();  // the row's words are written (visible to the block after the barrier)
  // 5. rowpre: exclusive prefix popcount of the row, contiguous chunks per thread
  const uint32_t* fin_row = STAGED ? s_cand : frow;
  const int per = (W + nthr - 1) / nthr;
  const int w_lo = threadIdx.x * per, w_hi = min(W, w_lo + per);
  int loc = 0;
  for (int w = w_lo; w < w_hi; ++w) loc += __popc(fin_row[w]);
  int tot;
  int run = block_exclusive_scan(loc, sh, &tot);
  int* rp = rowpre + (size_t)e * W;
  for (int w = w_lo; w < w_hi; ++w) {
    rp[w] = run;
    run += __popc(fin_row[w]);
  }
}

// Per token: exclusive scan of the final pair counts inside each block of
// 256 tokens (local[t]) and the block totals; the last block to finish scans
// the block totals (blk, total at [nblocks]), the experts' final counts into
// segment offsets (no padding: every count is a multiple of the tile) and
// writes the tile -> expert list.
__global__ void __launch_bounds__(256) tr_scan_kernel(int T, int E, int* local /* in: counts, out: offsets */,
                                                      int* blk, int* sync, const int* counts, int* offsets,
                                                      int* tile_expert) {
  pdl_wait();
  __shared__ int sh[32];
  __shared__ int is_last;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int c = t < T ? local[t] : 0;
  int total;
  const int ex = block_exclusive_scan(c, sh, &total);
  if (t < T) local[t] = ex;
  if (threadIdx.x == 0) blk[blockIdx.x] = total;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) is_last = (atomicAdd(sync, 1) == (int)gridDim.x - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  const int nb = gridDim.x;
  int carry = 0;
  for (int b0 = 0; b0 < nb; b0 += blockDim.x) {
    const int b = b0 + threadIdx.x;
    const int v = b < nb ? __ldcg(blk + b) : 0;
    int tot;
    const int bex = block_exclusive_scan(v, sh, &tot);
    if (b < nb) blk[b] = carry + bex;
    carry += tot;
  }
  if (threadIdx.x == 0) blk[nb] = carry;
  carry = 0;
  for (int e0 = 0; e0 < E; e0 += blockDim.x) {
    const int e = e0 + threadIdx.x;
    const int v = e < E ? __ldcg(counts + e) : 0;
    int tot;
    const int eex = block_exclusive_scan(v, sh, &tot);
    if (e < E) {
      const int o = carry + eex;
      offsets[e] = o;
      for (int tt = o / kTile; tt < (o + v) / kTile; ++tt) tile_expert[tt] = e;
    }
    carry += tot;
  }
  if (threadIdx.x == 0) offsets[E] = carry;
}

// Column `lane` of the 32 x 32 bit matrix whose row i is lane i's x (bit j
// of row i = entry (i, j)): five exchange steps of halving block size.
__device__ __forceinline__ uint32_t transpose32(uint32_t x, int lane) {
  uint32_t m = 0x0000FFFFu;
#pragma unroll
  for (int s = 16; s > 0; s >>= 1, m ^= (m << s)) {
    const uint32_t o = __shfl_xor_sync(0xffffffffu, x, s);
    x = (lane & s) ? ((x & ~m) | ((o >> s) & m)) : ((x & m) | ((o & m) << s));
  }
  return x;
}

// Per token (a warp holds the 32 tokens of one finalT word): the token's
// final experts from the expert rows (one 32 x 32 bit transpose per group of
// 32 experts), its gates (p renormalised over the final set, summed in
// ascending expert order), its pairs in ascending expert order, and each
// pair's row in the expert-major layout: the expert's offset + rowpre + the
// expert's tokens before it in the word.  Writes tok_ptr, pair_*, row_tok,
// row_gate.  Blocks of kTwThreads tokens (small, so that the T / 32 warps
// spread over every SM); the pair offsets come from tr_scan_kernel's blocks of
// 256 tokens.  Shared memory: the finalT words of each warp's column [E],
// each token's expert masks [groups][kTwThreads] and its first kTwList
// experts [kTwList][kTwThreads].
constexpr int kTwThreads = 64;
constexpr int kTwList = 16;
__global__ void __launch_bounds__(kTwThreads) tr_write_kernel(const uint32_t* finalT, const int* rowpre,
                                                              const float* probs, int T, int E, int W,
                                                              const int* local, const int* blk, int nblk,
                                                              const int* offsets, int* tok_ptr, int* pair_expert,
                                                              float* pair_gate, int* pair_row, int* row_tok,
                                                              float* row_gate) {
  pdl_wait();
  extern __shared__ uint32_t tw_smem[];
  const int groups = (E + 31) / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t* s_x = tw_smem + (size_t)warp * groups * 32;  // [groups * 32]: finalT[e][w] of this warp's word
  uint32_t* s_y = tw_smem + (size_t)(kTwThreads / 32) * groups * 32;  // [groups][kTwThreads]: token masks
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int w = t >> 5;
  const bool live = t < T;
  const float* pr = probs + (size_t)(live ? t : 0) * E;
  // the warp's word of every expert first (independent loads in flight),
  // then one transpose per group of 32 experts
  for (int g = 0; g < groups; ++g) {
    const int e = 32 * g + lane;
    s_x[32 * g + lane] = (e < E && w < W) ? finalT[(size_t)e * W + w] : 0u;
  }
  __syncwarp();
  for (int g = 0; g < groups; ++g) s_y[g * kTwThreads + threadIdx.x] = transpose32(s_x[32 * g + lane], lane);
  __syncwarp();
  if (!live) return;
  // the token's final experts in ascending order; the first kTwList of them
  // have their p, segment offset and row prefix loaded together
  uint32_t* s_e = s_y + (size_t)groups * kTwThreads;  // [kTwList][kTwThreads]
  int n = 0;
  for (int g = 0; g < groups; ++g)
    for (uint32_t r = s_y[g * kTwThreads + threadIdx.x]; r; r &= r - 1u) {
      if (n < kTwList) s_e[n * kTwThreads + threadIdx.x] = 32 * g + __ffs(r) - 1;
      ++n;
    }
  float pv[kTwList];
  int ro[kTwList];
#pragma unroll
  for (int j = 0; j < kTwList; ++j) {
    pv[j] = 0.f;
    ro[j] = 0;
    if (j < n) {
      const int e = s_e[j * kTwThreads + threadIdx.x];
      pv[j] = pr[e];
      ro[j] = offsets[e] + rowpre[(size_t)e * W + w];
    }
  }
  float sum = 0.f;  // in ascending expert order
#pragma unroll
  for (int j = 0; j < kTwList; ++j)
    if (j < n) sum += pv[j];
  if (n > kTwList) {  // the rest, one at a time
    int i = 0;
    for (int g = 0; g < groups; ++g)
      for (uint32_t r = s_y[g * kTwThreads + threadIdx.x]; r; r &= r - 1u, ++i)
        if (i >= kTwList) sum += pr[32 * g + __ffs(r) - 1];
  }
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  int p = blk[t >> 8] + local[t];
  tok_ptr[t] = p;
  if (t == T - 1) tok_ptr[T] = blk[nblk];
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int j = 0; j < kTwList; ++j) {
    if (j < n) {
      const int e = s_e[j * kTwThreads + threadIdx.x];
      const float gate = pv[j] * inv;
      const int row = ro[j] + __popc(s_x[e] & below);
      pair_expert[p] = e;
      pair_gate[p] = gate;
      pair_row[p] = row;
      row_tok[row] = t;
      row_gate[row] = gate;
      ++p;
    }
  }
  if (n > kTwList) {
    int i = 0;
    for (int g = 0; g < groups; ++g)
      for (uint32_t r = s_y[g * kTwThreads + threadIdx.x]; r; r &= r - 1u, ++i) {
        if (i < kTwList) continue;
        const int b = __ffs(r) - 1;
        const int e = 32 * g + b;
        const float gate = pr[e] * inv;
        const int row = offsets[e] + rowpre[(size_t)e * W + w] + __popc(s_x[e] & below);
        pair_expert[p] = e;
        pair_gate[p] = gate;
        pair_row[p] = row;
        row_tok[row] = t;
        row_gate[row] = gate;
        ++p;
      }
  }
}

cudaError_t launch_token_round(const RouteArgs& a, const RoundArgs& r, cudaStream_t s) {
  const int W = (r.T + 31) / 32;
  cudaError_t err = cudaMemsetAsync(r.memberT, 0, (size_t)r.E * W * sizeof(uint32_t), s);
  if (err == cudaSuccess) err = cudaMemsetAsync(a.counts, 0, (size_t)r.E * sizeof(int), s);
  if (err != cudaSuccess) return err;
  const int tb = (r.T + 255) / 256;
  {
    ProfScope ps(s, "round_member");
    launch_pdl(tr_member_kernel, dim3(tb), dim3(256), 0, s, a.tok_ptr, a.pair_expert, r.T, r.E, W, r.memberT,
               r.local, a.counts, r.sync);
  }
  {
    ProfScope ps(s, "round_transpose");
    dim3 grid((r.E + kTrTile - 1) / kTrTile, (r.T + kTrTile - 1) / kTrTile);
    launch_pdl(tr_transpose_kernel, dim3(grid), dim3(256), 0, s, r.probs, r.probsT, r.T, r.E);
  }
  {
    ProfScope ps(s, "round_select");
    // stage the expert's keys and routed-token words when they fit
    const size_t staged = kTrSelFixed + (size_t)W * sizeof(uint32_t);
    // MOE_TR_UNSTAGED=1 takes the path of rows too long to stage (for tests)
    const char* fu = std::getenv("MOE_TR_UNSTAGED");
    const bool force_unstaged = fu && std::atoi(fu) != 0;
    if (staged <= kTrSelMax && !force_unstaged) {
      err = set_max_dynamic_smem(reinterpret_cast<const void*>(tr_select_kernel<true>), (int)kTrSelMax);
      if (err != cudaSuccess) return err;
      launch_pdl(tr_select_kernel<true>, dim3(r.E), dim3(kTrSelThreads), staged, s, r.T, W, r.mode, r.seed, a.counts,
                 r.probsT, r.memberT, r.finalT, r.rowpre, r.local);
    } else {
      launch_pdl(tr_select_kernel<false>, dim3(r.E), dim3(kTrSelThreads), kTrSelFixed, s, r.T, W, r.mode, r.seed,
                 a.counts, r.probsT, r.memberT, r.finalT, r.rowpre, r.local);
    }
  }
  {
    ProfScope ps(s, "round_scan");
    launch_pdl(tr_scan_kernel, dim3(tb), dim3(256), 0, s, r.T, r.E, r.local, r.blk, r.sync, a.counts, a.offsets,
               a.tile_expert);
  }
  {
    ProfScope ps(s, "round_write");
    const int groups = (r.E + 31) / 32;
    const size_t smem = ((size_t)(kTwThreads + kTwThreads) * groups + (size_t)kTwList * kTwThreads) *
                        sizeof(uint32_t);  // at most 20 KB
    launch_pdl(tr_write_kernel, dim3((r.T + kTwThreads - 1) / kTwThreads), dim3(kTwThreads), smem, s, r.finalT,
               r.rowpre, r.probs, r.T, r.E, W, r.local, r.blk, tb, a.offsets, a.tok_ptr, a.pair_expert, a.pair_gate,
               a.pair_row, a.row_tok, a.row_gate);
  }
  return cudaGetLastError();
}

}  // namespace moe
