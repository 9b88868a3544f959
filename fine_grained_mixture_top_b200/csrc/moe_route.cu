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
// Stable counting sort of all (token, expert) pairs by expert, in three
// launches.  Tokens are cut into chunks of 256; inside a chunk the rank of
// token t among the chunk's tokens routed to e is a popcount over a
// per-expert bit mask, so the result does not depend on the order in which
// threads run.
__global__ void __launch_bounds__(kChunk) rank_kernel(RouteArgs a) {
  pdl_wait();
  extern __shared__ uint32_t bits[];  // [E][8]
  if (blockIdx.x == 0 && threadIdx.x == 0) *a.sync = 0;  // for chunk_scan_kernel's last block
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

// Per expert (one warp each, several blocks): exclusive scan over the chunks
// of its per-chunk counts (chunk bases relative to the expert's segment) and
// the expert's total count.  The last block to finish then computes the
// 128-padded segment offsets (exclusive scan over experts).
__global__ void __launch_bounds__(kScanThreads) chunk_scan_kernel(RouteArgs a) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * (kScanThreads / 32) + warp;
  if (e < a.E) {
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
  int carry = 0;
  for (int e0 = 0; e0 < a.E; e0 += kScanThreads) {
    const int ee = e0 + threadIdx.x;
    const int padded = ee < a.E ? ((__ldcg(a.counts + ee) + kTile - 1) / kTile) * kTile : 0;
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
  {
    ProfScope ps(s, "permute_rank");
    launch_pdl(rank_kernel, dim3(a.nchunks), dim3(kChunk), (size_t)a.E * (kChunk / 32) * sizeof(uint32_t), s, a);
  }
  {
    ProfScope ps(s, "permute_scan");
    launch_pdl(chunk_scan_kernel, dim3((a.E + 7) / 8), dim3(kScanThreads), 0, s, a);
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
// block per expert then reads its row contiguously.
__global__ void tr_member_kernel(const int* tok_ptr, const int* pair_expert, int T, int W, uint32_t* memberT,
                                 int* sync) {
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t == 0) *sync = 0;  // for tr_count_kernel's last block
  if (t >= T) return;
  for (int p = tok_ptr[t]; p < tok_ptr[t + 1]; ++p)
    atomicOr(&memberT[(size_t)pair_expert[p] * W + (t >> 5)], 1u << (t & 31));
}

// probsT[e, t] = probs[t, e], 32 x 32 tiles through shared memory
__global__ void tr_transpose_kernel(const float* __restrict__ probs, float* __restrict__ probsT, int T, int E) {
  pdl_wait();
  __shared__ float tile[32][33];
  const int e0 = blockIdx.x * 32, t0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int t = t0 + i, e = e0 + threadIdx.x;
    if (t < T && e < E) tile[i][threadIdx.x] = probs[(size_t)t * E + e];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int e = e0 + i, t = t0 + threadIdx.x;
    if (t < T && e < E) probsT[(size_t)e * T + t] = tile[threadIdx.x][i];
  }
}

// One block per expert: radix select (8 passes of 8 bits) of the k extreme
// 64-bit keys (p bits << 32 | ~t) among the candidate tokens, then the
// expert's final row finalT[e] = memberT[e] with the selected tokens added
// (rounding up) or removed (rounding down).  With STAGED the expert's p row
// and candidate mask are first copied into shared memory; histogram updates
// are aggregated per warp over lanes with the same digit.
template <bool STAGED>
__global__ void __launch_bounds__(1024) tr_select_kernel(int T, int W, int mode, unsigned long long seed,
                                                         const int* counts, const float* probsT,
                                                         const uint32_t* memberT, uint32_t* finalT) {
  pdl_wait();
  extern __shared__ uint32_t stage[];  // STAGED: p bits [T], then the candidate mask [W]
  __shared__ unsigned int hist[256];
  __shared__ unsigned long long s_prefix;
  __shared__ int s_k;
  const int e = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const uint32_t* mrow = memberT + (size_t)e * W;
  uint32_t* frow = finalT + (size_t)e * W;
  const float* prow = probsT + (size_t)e * T;
  const int c = counts[e];
  const int rem = c % kTile;
  if (rem == 0) {  // already a multiple of the tile: keep the routed set
    for (int w = threadIdx.x; w < W; w += blockDim.x) frow[w] = mrow[w];
    return;
  }
  bool up;
  if (mode == 1) up = rem >= kTile / 2;
  else up = (int)(splitmix64_dev(seed ^ (unsigned long long)e) % (unsigned long long)kTile) < rem;
  if (up && c - rem + kTile > T) up = false;
  const int k = up ? kTile - rem : rem;
  // candidates: unrouted tokens when rounding up, routed ones when rounding down
  const uint32_t tail = (T & 31) ? ((1u << (T & 31)) - 1u) : 0xFFFFFFFFu;
  auto cand_word = [&](int w) -> uint32_t {
    const uint32_t m = mrow[w];
    const uint32_t valid = (w == W - 1) ? tail : 0xFFFFFFFFu;
    return (up ? ~m : m) & valid;
  };
  uint32_t* s_p = stage;
  uint32_t* s_cand = stage + T;
  if constexpr (STAGED) {
    for (int t = threadIdx.x; t < T; t += blockDim.x) s_p[t] = __float_as_uint(prow[t]);
    for (int w = threadIdx.x; w < W; w += blockDim.x) s_cand[w] = cand_word(w);
    __syncthreads();
  }
  auto is_cand = [&](int t) -> bool {
    const uint32_t cw = STAGED ? s_cand[t >> 5] : cand_word(t >> 5);
    return (cw >> (t & 31)) & 1u;
  };
  auto key_of = [&](int t) -> unsigned long long {
    const uint32_t pb = STAGED ? s_p[t] : __float_as_uint(prow[t]);
    const unsigned long long kk = ((unsigned long long)pb << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)t);
    return up ? ~kk : kk;   // select the k smallest of this key
  };
  __shared__ int s_done;
  unsigned long long prefix = 0ull, mask = 0ull;
  int kk = k;
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0u;
    __syncthreads();
    for (int t0 = 0; t0 < T; t0 += blockDim.x) {  // warp-uniform trip count
      const int t = t0 + threadIdx.x;
      bool hit = false;
      uint32_t digit = 0u;
      if (t < T && is_cand(t)) {
        const unsigned long long key = key_of(t);
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
      const int owner = __ffs(reach) - 1;  // kk <= number of matching candidates, so some lane reaches it
      if (lane == owner) {
        int cum = incl - sum, dg = 8 * lane;
#pragma unroll 1
        for (int i = 0; i < 8; ++i, ++dg) {
          if (cum + loc[i] >= kk) break;
          cum += loc[i];
        }
        const int left = kk - cum;
        s_prefix = prefix | ((unsigned long long)dg << shift);
        s_k = left;
        // once the p bits are fixed (after 4 passes), stop if every candidate
        // with that p is selected: the token bits only break ties
        s_done = (shift == 32 && left == (int)hist[dg]) ? 1 : 0;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    kk = s_k;
    mask |= 255ull << shift;
    const bool done = s_done != 0 && shift == 32;
    __syncthreads();
    if (done) {
      prefix |= 0xFFFFFFFFull;  // select every candidate whose p bits are <= the k-th one's
      break;
    }
  }
  // the selected candidates are those with key <= prefix (exactly k of them)
  for (int w = threadIdx.x; w < W; w += blockDim.x) {
    uint32_t sel = 0u;
    const uint32_t cw = STAGED ? s_cand[w] : cand_word(w);
    for (uint32_t m = cw; m; m &= m - 1u) {
      const int b = __ffs(m) - 1;
      if (key_of(w * 32 + b) <= prefix) sel |= 1u << b;
    }
    const uint32_t mem = mrow[w];
    frow[w] = up ? (mem | sel) : (mem & ~sel);
  }
}

// A warp holds 32 consecutive tokens (one word column w of finalT).  For each
// group of 32 experts, lane j loads expert (32 c + j)'s word and 32 ballots
// transpose the 32 x 32 bit block, so that lane i ends with the group's
// expert mask of token 32 w + i.
__device__ __forceinline__ uint32_t tr_token_mask(const uint32_t* finalT, int E, int W, int w, int c, int lane) {
  const int e = 32 * c + lane;
  const uint32_t x = (e < E && w < W) ? finalT[(size_t)e * W + w] : 0u;
  uint32_t mine = 0u;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t b = __ballot_sync(0xffffffffu, (x >> i) & 1u);
    if (lane == i) mine = b;
  }
  return mine;
}

// Per token: its expert count after rounding; a block-wide exclusive scan
// gives its offset inside the block, and the last block to finish scans the
// block totals (exclusive, total at [nblocks]).
__global__ void __launch_bounds__(256) tr_count_kernel(const uint32_t* finalT, int T, int E, int W, int* local,
                                                       int* blk, int* sync) {
  pdl_wait();
  __shared__ int sh[8];
  __shared__ int is_last;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  int c = 0;
  for (int g = 0; g < (E + 31) / 32; ++g) c += __popc(tr_token_mask(finalT, E, W, t >> 5, g, lane));
  if (t >= T) c = 0;
  int total;
  const int ex = block_exclusive_scan_256(c, sh, &total);
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
    const int bex = block_exclusive_scan_256(v, sh, &tot);
    if (b < nb) blk[b] = carry + bex;
    carry += tot;
  }
  if (threadIdx.x == 0) blk[nb] = carry;
}

// Per token: tok_ptr and its pairs in ascending expert order, gates = p
// renormalised over the token's final expert set.
__global__ void __launch_bounds__(256) tr_write_kernel(const uint32_t* finalT, const float* probs, int T, int E,
                                                       int W, const int* local, const int* blk, int* tok_ptr,
                                                       int* pair_expert, float* pair_gate) {
  pdl_wait();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  const bool live = t < T;
  int p = live ? blk[blockIdx.x] + local[t] : 0;
  if (live) {
    tok_ptr[t] = p;
    if (t == T - 1) tok_ptr[T] = blk[gridDim.x];
  }
  const float* pr = probs + (size_t)(live ? t : 0) * E;
  const int groups = (E + 31) / 32;
  float sum = 0.f;
  for (int g = 0; g < groups; ++g) {
    const uint32_t m = tr_token_mask(finalT, E, W, t >> 5, g, lane);
    if (live)
      for (uint32_t r = m; r; r &= r - 1u) sum += pr[32 * g + __ffs(r) - 1];
  }
  const float inv = sum > 0.f ? 1.0f / sum : 0.f;
  for (int g = 0; g < groups; ++g) {
    const uint32_t m = tr_token_mask(finalT, E, W, t >> 5, g, lane);
    if (live)
      for (uint32_t r = m; r; r &= r - 1u) {
        const int e = 32 * g + __ffs(r) - 1;
        pair_expert[p] = e;
        pair_gate[p] = pr[e] * inv;
        ++p;
      }
  }
}

constexpr size_t kTrStageMax = 200 * 1024;  // dynamic shared memory of the staged select

cudaError_t launch_token_round(const RouteArgs& a, const RoundArgs& r, cudaStream_t s) {
  const int W = (r.T + 31) / 32;
  cudaError_t err = cudaMemsetAsync(r.memberT, 0, (size_t)r.E * W * sizeof(uint32_t), s);
  if (err != cudaSuccess) return err;
  const int tb = (r.T + 255) / 256;
  {
    ProfScope ps(s, "round_member");
    launch_pdl(tr_member_kernel, dim3(tb), dim3(256), 0, s, a.tok_ptr, a.pair_expert, r.T, W, r.memberT, r.sync);
  }
  {
    ProfScope ps(s, "round_transpose");
    dim3 grid((r.E + 31) / 32, (r.T + 31) / 32), block(32, 8);
    launch_pdl(tr_transpose_kernel, dim3(grid), dim3(block), 0, s, r.probs, r.probsT, r.T, r.E);
  }
  {
    ProfScope ps(s, "round_select");
    // stage the expert's p row and candidate mask when they fit in shared memory
    const size_t staged = ((size_t)r.T + (size_t)W) * sizeof(uint32_t);
    if (staged <= kTrStageMax) {
      err = set_max_dynamic_smem(reinterpret_cast<const void*>(tr_select_kernel<true>), (int)kTrStageMax);
      if (err != cudaSuccess) return err;
      launch_pdl(tr_select_kernel<true>, dim3(r.E), dim3(1024), staged, s, r.T, W, r.mode, r.seed, a.counts, r.probsT, r.memberT,
                                                        r.finalT);
    } else {
      launch_pdl(tr_select_kernel<false>, dim3(r.E), dim3(1024), 0, s, r.T, W, r.mode, r.seed, a.counts, r.probsT, r.memberT,
                                                    r.finalT);
    }
  }
  {
    ProfScope ps(s, "round_count");
    launch_pdl(tr_count_kernel, dim3(tb), dim3(256), 0, s, r.finalT, r.T, r.E, W, r.local, r.blk, r.sync);
  }
  {
    ProfScope ps(s, "round_write");
    launch_pdl(tr_write_kernel, dim3(tb), dim3(256), 0, s, r.finalT, r.probs, r.T, r.E, W, r.local, r.blk, a.tok_ptr, a.pair_expert,
                                       a.pair_gate);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  return launch_permute(a, s);
}

}  // namespace moe
