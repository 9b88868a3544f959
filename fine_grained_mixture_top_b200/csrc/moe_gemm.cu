// Instantiations and launcher of the tcgen05 grouped GEMM (see gemm.cuh).
#include <cuda_runtime.h>

#include "gemm.cuh"
#include "moe_internal.h"

namespace moe {

template <int KIND, int BN, int EPI>
static cudaError_t launch_one(const GemmParams& p, int grid, cudaStream_t stream) {
  using EC = EpiCfg<KIND, EPI>;
  constexpr int smem = GemmShape<KIND, BN, EPI * EC::kBufs>::kSmemBytes;
  constexpr int threads = EC::kThreads;
  auto fn = moe_gemm_kernel<KIND, BN, EPI>;
  static int configured_dev = -1;  // per-process; the library serves one device at a time
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    configured_dev = dev;
  }
  if (grid <= 0) return cudaSuccess;
  return launch_pdl(fn, dim3(grid), dim3(threads), (size_t)smem, stream, p);
}

cudaError_t launch_gemm(int kind, int bn, int epi, const GemmParams& p, int grid, cudaStream_t s) {
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




}  // namespace moe
