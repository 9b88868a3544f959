// Instantiations and launcher of the tcgen05 grouped GEMM (see gemm.cuh).
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <set>
#include <utility>

#include "gemm.cuh"
#include "gemm_pair.cuh"
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

// The dynamic shared-memory limit is a per-device property of a function: it
// is set once for each (function, device), under a lock, so that host threads
// driving different devices (or the same one) all see it set before they
// launch.
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

cudaError_t launch_gemm(int kind, int bn, int epi, const GemmParams& p_in, int grid, cudaStream_t s) {
  GemmParams p = p_in;
  {
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




}  // namespace moe
