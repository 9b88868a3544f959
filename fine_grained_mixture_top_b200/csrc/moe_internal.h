// Internal launch interface between the C-ABI layer (moe_api.cu) and the
// kernel translation units.  Not part of the public ABI.
#pragma once
#include <cuda_runtime.h>
#include <cstdint>
#include <utility>

#include "gemm.cuh"

namespace moe {

#ifndef MOE_PDL
#define MOE_PDL 1
#endif

// Launch on `s` with programmatic stream serialization (see pdl_wait): the
// kernel's blocks may be scheduled while the previous kernel of the stream
// finishes.  Every kernel of this library calls pdl_wait() before touching
// global memory.
template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              A&&... args) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = block;
  c.dynamicSmemBytes = smem;
  c.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = MOE_PDL;
  c.attrs = at;
  c.numAttrs = 1;
  return cudaLaunchKernelEx(&c, kernel, std::forward<A>(args)...);
}


constexpr int kTile = 128;        // rows per expert tile (segments are padded to it)
constexpr int kChunk = 256;       // tokens per ranking chunk of the permutation

// Sets `fn`'s dynamic shared-memory limit on the current device, once per
// (function, device); thread-safe.
cudaError_t set_max_dynamic_smem(const void* fn, int bytes);

// Role timeline of GEMM kind `kind` (GemmKind) into `buf` (null: off), `cap`
// records per CTA and role.
void set_gemm_trace(int kind, void* buf, int cap);

// The calling thread's last failed GEMM launch: what it asked for and what
// the kernel allows (empty if none failed).
extern thread_local char g_launch_diag[256];

// epi: epilogue warps (4, or 8 for the dH and dX~ kinds)
// traced = false: the launch writes no role timeline even while its kind is
// traced (the second launch of a kind that runs as two)
cudaError_t launch_gemm(int kind, int bn, int epi, const GemmParams& p, int grid, cudaStream_t s, bool traced = true);
// Weight-gradient kinds on CTA pairs (256 x 256 tiles, gemm_pair.cuh):
// p.num_m_tiles / p.num_n_tiles count 256-wide tiles; `pairs` clusters of 2.
cudaError_t launch_gemm_pair(int kind, int epi, const GemmParams& p, int pairs, cudaStream_t s);
// Down-proj and dX~ on CTA pairs (gemm_pair_m.cuh) over the pair list p.mlist;
// p.num_n_tiles counts 256-column tiles; at most `max_pairs` clusters of 2
// (fewer if fewer fit the device at once).
cudaError_t launch_gemm_pair_m(int kind, int epi, const GemmParams& p, int max_pairs, cudaStream_t s);
// Down-proj and dX~ with 256 x 256 tiles on one CTA (gemm_wide_m.cuh) over
// the list p.mlist of 256-row tiles; p.num_n_tiles counts 256-column tiles.
cudaError_t launch_gemm_wide_m(int kind, const GemmParams& p, int grid, cudaStream_t s);
// List of the grouped-M tiles in 256-row tiles from the segment offsets
// ([count, entry...]: up to R_max / 256 + E entries after the count) and each
// expert's first entry (base [E + 1]).
cudaError_t launch_wide_list(const int* offsets, int E, int* list, int* base, cudaStream_t s);
// Pair list and leftover list of the grouped-M tiles from the segment offsets
// (each [count, tile...]; `pairs` holds up to R_max / 256 + 1 entries after the
// count, `left` up to E).
cudaError_t launch_pair_lists(const int* offsets, int E, int* pairs, int* left, cudaStream_t s);

// Per-kernel timing (moe_profile_enable): while on, each launch site brackets
// its kernel with two CUDA events recorded on the launching stream.
// Every launch site also opens an NVTX range with the same name (a no-op
// unless a profiler is attached), so a profiler's timeline shows the kernel
// names the breakdown uses.
struct ProfScope {
  int slot = -1;
  cudaStream_t stream;
  ProfScope(cudaStream_t s, const char* name);
  ~ProfScope();
};
// An NVTX range over one call of the C ABI.
struct ApiRange {
  explicit ApiRange(const char* name);
  ~ApiRange();
};

// ---- routing (moe_route.cu)
struct RouteArgs {
  int T, d, E, K, Epad;
  const float* Wr;
  __nv_bfloat16* Wr_split;  // [d, 3*Epad]
  const float* logits;      // [T, E]
  float* probs;             // [T, E]
  int* topk_idx;            // [T, K]
  float* topk_gate;         // [T, K]
  int* tok_ptr;             // [T+1]
  int* pair_expert;         // [P_max]
  float* pair_gate;         // [P_max]
  int* pair_row;            // [P_max]
  int* counts;              // [E]
  int* offsets;             // [E+1]
  int* row_tok;             // [R_max]
  float* row_gate;          // [R_max]
  int* tile_expert;         // [R_max/128]
  int* sync;                // [1] blocks done (zeroed by the rank kernel)
  int* hist;                // [nchunks, E]
  int* local_rank;          // [P_max]
  int nchunks;
  DevStatus st;
};
cudaError_t launch_split_wr(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_softmax_topk(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_permute(const RouteArgs& a, cudaStream_t s);  // rank + scan + scatter

struct RoundArgs {
  int T, E, mode;
  unsigned long long seed;
  const float* probs;   // [T, E]
  float* probsT;        // [E, T]
  uint32_t* memberT;    // [E, ceil(T/32)] routed tokens of each expert
  uint32_t* finalT;     // [E, ceil(T/32)] tokens of each expert after rounding
  int* rowpre;          // [E, ceil(T/32)] final tokens of each expert before each word
  int* local;           // [T] pair count of each token, then its pairs' offset inside its block of 256
  int* blk;             // [ceil(T/256) + 1] block offsets, total last
  int* sync;            // [1] blocks done
};
cudaError_t launch_token_round(const RouteArgs& a, const RoundArgs& r, cudaStream_t s);

// ---- aggregation and router backward (moe_agg.cu)
cudaError_t launch_aggregate_fwd(int T, int d, const int* tok_ptr, const int* pair_row, const float* pair_gate,
                                 const __nv_bfloat16* Y, __nv_bfloat16* O, cudaStream_t s);
// Backward preparation (router backward, Wr^T, expert order), one launch.
struct BwdPrepArgs {
  int T, d, E, Epad, nds;  // nds: dS partials per row
  int router;              // router path on: dz, dz split and Wr^T
  const int* tok_ptr;
  const int* pair_row;
  const int* pair_expert;
  const float* pair_gate;
  const float* dS_part;
  float* dz_row;               // [R_max]
  __nv_bfloat16* dz_split;     // [T, 2 Epad]
  const float* Wr;             // [d, E]
  float* WrT;                  // [E, d]
  const int* counts;           // [E]
  int* expert_order;           // [E]
  int* sched;                  // [16] weight-gradient tile counters, zeroed here
  float* pair_dS;              // [P] dS of each pair, or null
  int K;                       // experts per token (pairs per token before rounding)
  int lanes, tok_blocks, tr_blocks;  // set by the launcher: lanes per token, block counts
};
cudaError_t launch_bwd_prep(const BwdPrepArgs& a, cudaStream_t s);
cudaError_t launch_dwr_reduce(int d, int E, int Epad, int splits, const float* part, float* dWr, cudaStream_t s);
cudaError_t launch_aggregate_bwd(int T, int d, const int* tok_ptr, const int* pair_row, const __nv_bfloat16* dXt,
                                 __nv_bfloat16* dX, cudaStream_t s);
cudaError_t launch_wait_selftest(int* flag, DevStatus st, cudaStream_t s);
cudaError_t launch_router_bwd_given(int T, int d, int E, int Epad, const int* tok_ptr, const int* pair_expert,
                                    const float* pair_gate, const float* dS, const int* pos, const float* Wr,
                                    float* WrT, __nv_bfloat16* dz_split, __nv_bfloat16* dX, cudaStream_t s);

// ---- caller-given routing and expert parallelism (moe_ep.cu)
cudaError_t launch_given_pairs(int T, int K, int E, const int* topk_idx, const float* topk_gate, int* tok_ptr,
                               int* pair_expert, float* pair_gate, DevStatus st, cudaStream_t s);
cudaError_t launch_ep_pack(int T, int d, int E, int64_t R_max, int64_t P_max, const int* tok_ptr,
                           const int* pair_expert, const int* pair_row, const int* counts, const int* offsets,
                           const int* tile_expert, const int* row_tok, const float* row_gate,
                           const __nv_bfloat16* src, __nv_bfloat16* send, float* send_gate, int* pair_pos, int* cum,
                           cudaStream_t s);

// ---- debug build only (moe_debug.cu): routing consistency checks
#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif
struct RoutingView {
  int64_t T, P_max, R_max;
  int E;
  const int *tok_ptr, *pair_expert, *pair_row, *counts, *offsets, *row_tok, *tile_expert;
};
// Checks the routing's invariants; a violation sets MOE_ERR_DEVICE_CHECK in
// the status word.  A no-op (no launch) unless built with MOE_DEBUG=1.
cudaError_t launch_validate_routing(const RoutingView& v, DevStatus st, cudaStream_t s);

// ---- MXFP8 quantization (moe_mx.cu)
cudaError_t launch_mx_quant_rows(const __nv_bfloat16* in, int64_t rows, int K, uint8_t* codes, uint8_t* scales,
                                 cudaStream_t s);
// codes [E][N][K] (K-major); scales linear [E][N][K/32] and/or (tiles != null,
// K % 128 == 0, N % 128 == 0) the block-scaled GEMM's 512-byte scale tiles
cudaError_t launch_mx_quant_cols(const __nv_bfloat16* in, int E, int K, int N, uint8_t* codes, uint8_t* scales,
                                 uint8_t* tiles, int split_half, cudaStream_t s);
}  // namespace moe
