// Consistency checks of a routing, compiled into the debug build only
// (MOE_DEBUG=1, libmoe_debug.so).  The release build launches nothing here.
//
// The grouped GEMMs trust the routing completely: a row index past the
// segment, a token id past T or an expert id past E would make a TMA or
// cp.async copy read or write outside its tensor.  In the debug build every
// entry point that consumes a routing first runs validate_routing_kernel,
// which checks the routing's invariants and records the first violation in
// the status word (MOE_ERR_DEVICE_CHECK, `where` = 0x100 + the check's
// number below) instead of faulting; the entry point then waits for the check
// and, on a violation, returns MOE_ERR_DEVICE_CHECK without launching any
// kernel that would use the routing.  The GEMMs' gather warps also check
// each token id they load.  Every read of the check itself stays inside the
// routing's buffers whatever their contents.
#include <cuda_runtime.h>

#include "moe_internal.h"

namespace moe {

#if MOE_DEBUG
namespace {
__device__ __forceinline__ void fail(const DevStatus& st, int check) { raise_status(st, ST_DEVICE_CHECK, 0x100 + check); }

__global__ void validate_routing_kernel(RoutingView v, DevStatus st) {
  pdl_wait();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int E = v.E;
  const int64_t T = v.T;
  if (i == 0) {
    if (v.offsets[0] != 0) fail(st, 1);                      // first segment starts at row 0
    if (v.offsets[E] > v.R_max) fail(st, 2);                 // rows fit the row space
    if (v.tok_ptr[0] != 0 || v.tok_ptr[T] > v.P_max) fail(st, 3);  // pairs fit the pair space
  }
  if (i < E) {
    const int a = v.offsets[i], b = v.offsets[i + 1], c = v.counts[i];
    // segments 128-aligned, ordered, each exactly its count rounded up to 128
    if ((a & 127) || (b & 127) || c < 0 || b - a != ((c + 127) & ~127)) fail(st, 4);
  }
  if (i < T) {
    const int a = v.tok_ptr[i], b = v.tok_ptr[i + 1];
    if (b < a) fail(st, 5);                                  // token pair lists ordered
    for (int p = a; p < b && p < v.P_max; ++p) {
      const int e = v.pair_expert[p];
      if (e < 0 || e >= E) {
        fail(st, 6);                                         // expert id in range
        continue;
      }
      const int r = v.pair_row[p];
      if (r < v.offsets[e] || r >= v.offsets[e] + v.counts[e] || r >= v.R_max) fail(st, 7);  // row inside its segment
      else if (v.row_tok[r] != (int)i) fail(st, 8);          // the row maps back to its token
    }
  }
  if (i < v.R_max && i < v.offsets[E]) {
    const int t = v.row_tok[i];
    if (t < -1 || t >= T) fail(st, 9);                       // token id of a row in range (-1: padding)
    const int e = v.tile_expert[i / 128];
    if (e < 0 || e >= E || i < v.offsets[e] || i >= v.offsets[e + 1]) fail(st, 10);  // tile owner
    else if ((i - v.offsets[e] < v.counts[e]) != (t >= 0)) fail(st, 11);  // padding exactly past the count
  }
}
}  // namespace

cudaError_t launch_validate_routing(const RoutingView& v, DevStatus st, cudaStream_t s) {
  int64_t n = v.R_max;
  if (v.T + 1 > n) n = v.T + 1;
  if (v.E + 1 > n) n = v.E + 1;
  const int threads = 256;
  return launch_pdl(validate_routing_kernel, dim3((unsigned)((n + threads - 1) / threads)), dim3(threads), 0, s, v,
                    st);
}
#else
cudaError_t launch_validate_routing(const RoutingView&, DevStatus, cudaStream_t) { return cudaSuccess; }
#endif

}  // namespace moe
