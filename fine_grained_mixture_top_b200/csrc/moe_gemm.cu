// Instantiations and launcher of the tcgen05 grouped GEMM (see gemm.cuh).
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <map>
#include <set>
#include <utility>

#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_pair_m.cuh"
#include "gemm_wide_m.cuh"
#include "moe_internal.h"

namespace moe {

thread_local char g_launch_diag[256] = "";

template <int KIND, int BN, int EPI>
static cudaError_t launch_one(const GemmParams& p, int grid, cudaStream_t stream) {
  using EC = EpiCfg<KIND, EPI>;
  constexpr int smem = GemmShape<KIND, BN, EC::kNbuf>::kSmemBytes;  // the kernel's own layout
  constexpr int threads = EC::kThreads;
  auto fn = moe_gemm_kernel<KIND, BN, EPI>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fn), smem);
  if (e == cudaSuccess && grid > 0) e = launch_pdl(fn, dim3(grid), dim3(threads), (size_t)smem, stream, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // the error is returned here; do not leave it for a later call to find
    // what the launch asked for against what the compiled kernel allows
    cudaFuncAttributes fa = {};
    cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(fn));
    std::snprintf(g_launch_diag, sizeof(g_launch_diag),
                  "gemm kind %d BN %d epilogue warps %d: grid %d x %d threads, %d B dynamic smem; kernel: %d regs, "
                  "max %d threads, max dynamic smem %d B",
                  KIND, BN, EPI, grid, threads, smem, fa.numRegs, fa.maxThreadsPerBlock,
                  fa.maxDynamicSharedSizeBytes);
  }
  return e;
}

template <int KIND, int EPI, bool POLL>
static cudaError_t launch_pair_one(const GemmParams& p, int pairs, cudaStream_t stream) {
  using SH = PairShape<KIND, EPI>;
  constexpr int smem = SH::kSmemBytes;
  auto fn = moe_dw_pair_kernel<KIND, EPI, POLL>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fn), smem);
  if (e == cudaSuccess && pairs > 0)
    e = launch_pdl(fn, dim3(2 * pairs), dim3(SH::kThreads), (size_t)smem, stream, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // the error is returned here; do not leave it for a later call to find
    cudaFuncAttributes fa = {};
    cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(fn));
    std::snprintf(g_launch_diag, sizeof(g_launch_diag),
                  "pair gemm kind %d epilogue warps %d: %d pairs x %d threads, %d B dynamic smem; kernel: %d regs, "
                  "max %d threads, max dynamic smem %d B",
                  KIND, EPI, pairs, SH::kThreads, smem, fa.numRegs, fa.maxThreadsPerBlock,
                  fa.maxDynamicSharedSizeBytes);
  }
  return e;
}

// Pairs of a 2-CTA cluster kernel that can be resident at once on this
// device (one CTA per SM; a cluster needs two SMs of one GPC), once per
// (function, device).  A persistent pair kernel launches no more, so that no
// pair waits for another to finish before it starts its share of the tiles.
static int resident_pairs(const void* fn, int threads, int smem) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> known;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  std::lock_guard<std::mutex> lk(mu);
  auto it = known.find({fn, dev});
  if (it != known.end()) return it->second;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (unsigned)(sms / 2 > 0 ? sms / 2 : 1));
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = (size_t)smem;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = sms / 2;
  }
  known[{fn, dev}] = n;
  return n;
}

template <int KIND, int EPI>
static cudaError_t launch_gm_pair_one(const GemmParams& p, int max_pairs, cudaStream_t stream) {
  using SH = PairMShape<KIND, EPI>;
  constexpr int smem = SH::kSmemBytes;
  auto fn = moe_gm_pair_kernel<KIND, EPI>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fn), smem);
  int pairs = 0;
  if (e == cudaSuccess) {
    pairs = resident_pairs(reinterpret_cast<const void*>(fn), SH::kThreads, smem);
    if (pairs > max_pairs) pairs = max_pairs;
    if (pairs > 0) e = launch_pdl(fn, dim3(2 * pairs), dim3(SH::kThreads), (size_t)smem, stream, p);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();  // the error is returned here; do not leave it for a later call to find
    cudaFuncAttributes fa = {};
    cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(fn));
    std::snprintf(g_launch_diag, sizeof(g_launch_diag),
                  "pair gemm (M) kind %d epilogue warps %d: %d pairs x %d threads, %d B dynamic smem; kernel: %d "
                  "regs, max %d threads, max dynamic smem %d B",
                  KIND, EPI, pairs, SH::kThreads, smem, fa.numRegs, fa.maxThreadsPerBlock,
                  fa.maxDynamicSharedSizeBytes);
  }
  return e;
}

// The dynamic shared-memory limit is a per-device property of a function: it
// is set once for each (function, device), under a lock, so that host threads
// driving different devices (or the same one) all see it set before they
// launch.  Callers pass the largest size the function is ever launched with.
cudaError_t set_max_dynamic_smem(const void* fn, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({fn, dev})) return cudaSuccess;
  e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  done.insert({fn, dev});
  return cudaSuccess;
}

// Role timeline of one GEMM kind (moe_trace_gemm): the next launches of that
// kind write their records into the selected buffer.
namespace {
std::mutex g_trace_mu;
int g_trace_kind = -1;
uint8_t* g_trace_buf = nullptr;
int g_trace_cap = 0;
}  // namespace

void set_gemm_trace(int kind, void* buf, int cap) {
  std::lock_guard<std::mutex> lk(g_trace_mu);
  g_trace_kind = buf ? kind : -1;
  g_trace_buf = static_cast<uint8_t*>(buf);
  g_trace_cap = cap;
}

cudaError_t launch_gemm(int kind, int bn, int epi, const GemmParams& p_in, int grid, cudaStream_t s, bool traced) {
  GemmParams p = p_in;
  if (traced) {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (kind == g_trace_kind) {
      p.trace = g_trace_buf;
      p.trace_cap = g_trace_cap;
    }
  }
#define MOE_CASE(K, B, W) \
  if (kind == K && bn == B && epi == W) return launch_one<K, B, W>(p, grid, s);
  MOE_CASE(G_UP, 128, 4)
  MOE_CASE(G_UP, 256, 4)
  MOE_CASE(G_DOWN, 128, 4)
  MOE_CASE(G_DOWN, 256, 4)
  MOE_CASE(G_DH, 64, 4)
  MOE_CASE(G_DH, 128, 4)
  MOE_CASE(G_DH, 256, 4)
  MOE_CASE(G_DH, 64, 8)
  MOE_CASE(G_DH, 128, 8)
  MOE_CASE(G_DH, 256, 8)
  MOE_CASE(G_DXT, 128, 4)
  MOE_CASE(G_DXT, 256, 4)
  MOE_CASE(G_DXT, 128, 8)
  MOE_CASE(G_DXT, 256, 8)
  MOE_CASE(G_DW1, 128, 4)
  MOE_CASE(G_DW1, 256, 4)
  MOE_CASE(G_DW1, 128, 8)
  MOE_CASE(G_DW1, 256, 8)
  MOE_CASE(G_DW2, 128, 4)
  MOE_CASE(G_DW2, 256, 4)
  MOE_CASE(G_DW2, 128, 8)
  MOE_CASE(G_DW2, 256, 8)
  MOE_CASE(G_UPQ, 128, 4)
  MOE_CASE(G_DOWNQ, 128, 4)
  MOE_CASE(G_RTR, 192, 4)
  MOE_CASE(G_RTR, 384, 4)
  MOE_CASE(G_DWR, 128, 4)
#undef MOE_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_pair(int kind, int epi, const GemmParams& p_in, int pairs, cudaStream_t s) {
  GemmParams p = p_in;
  {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (kind == g_trace_kind) {
      p.trace = g_trace_buf;
      p.trace_cap = g_trace_cap;
    }
  }
  static const bool poll = std::getenv("MOE_PAIR_POLL") && std::atoi(std::getenv("MOE_PAIR_POLL")) != 0;
  if (kind == G_DW1 && epi == 4) return poll ? launch_pair_one<G_DW1, 4, true>(p, pairs, s) : launch_pair_one<G_DW1, 4, false>(p, pairs, s);
  if (kind == G_DW1 && epi == 8) return poll ? launch_pair_one<G_DW1, 8, true>(p, pairs, s) : launch_pair_one<G_DW1, 8, false>(p, pairs, s);
  if (kind == G_DW2 && epi == 4) return poll ? launch_pair_one<G_DW2, 4, true>(p, pairs, s) : launch_pair_one<G_DW2, 4, false>(p, pairs, s);
  if (kind == G_DW2 && epi == 8) return poll ? launch_pair_one<G_DW2, 8, true>(p, pairs, s) : launch_pair_one<G_DW2, 8, false>(p, pairs, s);
  return cudaErrorInvalidValue;
}



cudaError_t launch_gemm_pair_m(int kind, int epi, const GemmParams& p_in, int max_pairs, cudaStream_t s) {
  GemmParams p = p_in;
  {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (kind == g_trace_kind) {
      p.trace = g_trace_buf;
      p.trace_cap = g_trace_cap;
    }
  }
  if (kind == G_DOWN && epi == 4) return launch_gm_pair_one<G_DOWN, 4>(p, max_pairs, s);
  if (kind == G_DXT && epi == 4) return launch_gm_pair_one<G_DXT, 4>(p, max_pairs, s);
  if (kind == G_DXT && epi == 8) return launch_gm_pair_one<G_DXT, 8>(p, max_pairs, s);
  return cudaErrorInvalidValue;
}

template <int KIND>
static cudaError_t launch_gm_wide_one(const GemmParams& p, int grid, cudaStream_t stream) {
  using SH = WideMShape<KIND>;
  constexpr int smem = SH::kSmemBytes;
  auto fn = moe_gm_wide_kernel<KIND>;
  cudaError_t e = set_max_dynamic_smem(reinterpret_cast<const void*>(fn), smem);
  if (e == cudaSuccess && grid > 0) e = launch_pdl(fn, dim3(grid), dim3(SH::kThreads), (size_t)smem, stream, p);
  if (e != cudaSuccess) {
    cudaGetLastError();  // the error is returned here; do not leave it for a later call to find
    cudaFuncAttributes fa = {};
    cudaFuncGetAttributes(&fa, reinterpret_cast<const void*>(fn));
    std::snprintf(g_launch_diag, sizeof(g_launch_diag),
                  "wide gemm (M) kind %d: grid %d x %d threads, %d B dynamic smem; kernel: %d regs, max %d threads, "
                  "max dynamic smem %d B",
                  KIND, grid, SH::kThreads, smem, fa.numRegs, fa.maxThreadsPerBlock, fa.maxDynamicSharedSizeBytes);
  }
  return e;
}

cudaError_t launch_gemm_wide_m(int kind, const GemmParams& p_in, int grid, cudaStream_t s) {
  GemmParams p = p_in;
  {
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (kind == g_trace_kind) {
      p.trace = g_trace_buf;
      p.trace_cap = g_trace_cap;
    }
  }
  if (kind == G_DOWN) return launch_gm_wide_one<G_DOWN>(p, grid, s);
  if (kind == G_DXT) return launch_gm_wide_one<G_DXT>(p, grid, s);
  return cudaErrorInvalidValue;
}

// The 256-row tile list (write_wide_list) as a launch of its own, for the dX~
// kernel on 256-row tiles (the down-proj's list comes from the up-proj kernel).
__global__ void __launch_bounds__(32) wide_list_kernel(const int* __restrict__ offsets, int E, int* __restrict__ list,
                                                       int* __restrict__ base) {
  pdl_wait();
  write_wide_list(offsets, E, list, base, (int)threadIdx.x);
}

cudaError_t launch_wide_list(const int* offsets, int E, int* list, int* base, cudaStream_t s) {
  if (E < 1) return cudaErrorInvalidValue;
  return launch_pdl(wide_list_kernel, dim3(1), dim3(32), 0, s, offsets, E, list, base);
}

// Pair and leftover lists of the grouped-M M tiles: for expert e, whose
// segment holds tiles [offsets[e] / 128, offsets[e + 1] / 128), the first
// tile of every pair of consecutive tiles goes to `pairs`, and the last tile
// of an odd count to `left`; both are [count, tile...] in expert order.  One
// block, a thread per expert (E <= 1024).
__global__ void __launch_bounds__(1024) pair_lists_kernel(const int* __restrict__ offsets, int E,
                                                         int* __restrict__ pairs, int* __restrict__ left) {
  __shared__ int wp[32], wl[32];
  const int e = threadIdx.x;
  const int lane = e & 31, w = e >> 5;
  pdl_wait();
  int t0 = 0, nt = 0;
  if (e < E) {
    const int o0 = __ldg(offsets + e), o1 = __ldg(offsets + e + 1);
    t0 = o0 / kBM;
    nt = (o1 - o0) / kBM;
  }
  const int np = nt >> 1, nl = nt & 1;
  int sp = np, sl = nl;  // inclusive scans within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, sp, o);
    const int b = __shfl_up_sync(0xffffffffu, sl, o);
    if (lane >= o) {
      sp += a;
      sl += b;
    }
  }
  if (lane == 31) {
    wp[w] = sp;
    wl[w] = sl;
  }
  __syncthreads();
  if (w == 0) {  // scan of the warp totals
    const int nw = (int)(blockDim.x >> 5);
    int a = lane < nw ? wp[lane] : 0, b = lane < nw ? wl[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, a, o);
      const int y = __shfl_up_sync(0xffffffffu, b, o);
      if (lane >= o) {
        a += x;
        b += y;
      }
    }
    wp[lane] = a;
    wl[lane] = b;
  }
  __syncthreads();
  const int bp = (w > 0 ? wp[w - 1] : 0) + sp - np;  // exclusive offsets
  const int bl = (w > 0 ? wl[w - 1] : 0) + sl - nl;
  for (int j = 0; j < np; ++j) pairs[1 + bp + j] = t0 + 2 * j;
  if (nl) left[1 + bl] = t0 + nt - 1;
  if (e == (int)blockDim.x - 1) {
    pairs[0] = bp + np;
    left[0] = bl + nl;
  }
}

cudaError_t launch_pair_lists(const int* offsets, int E, int* pairs, int* left, cudaStream_t s) {
  if (E < 1 || E > 1024) return cudaErrorInvalidValue;
  return launch_pdl(pair_lists_kernel, dim3(1), dim3(1024), 0, s, offsets, E, pairs, left);
}

}  // namespace moe
