// Persistent, warp-specialised tcgen05 GEMM for every contraction of the MoE
// layer: one main loop (TMA / cp.async gather -> shared-memory ring ->
// tcgen05.mma into a double-buffered TMEM accumulator) and one epilogue per
// kernel kind.
//
// Kernel kinds (rows r of the expert-major, 128-padded row space; e = expert):
//   UP   H_r = X[tok_r] W1[e]  (gather on A); epilogue stores H and SwiGLU(H)
//   DOWN Y_r = A_r W2[e]
//   DH   dA'_r = dO[tok_r] W2[e]^T (gather on A); epilogue reloads H, forms
//        dS partials, dSwiGLU -> dH, and A_hat = s_r * A_r
//   DXT  dX~_r = dH_r W1[e]^T (+ dz_r Wr[:, e]^T, the router path, when given)
//   DW1  dW1[e] = X[tok]^T dH   (K runs over the rows of expert e; gather on A)
//   DW2  dW2[e] = A_hat^T dO[tok] (K runs over the rows of expert e; gather on B)
//   RTR  router logits X Wr with Wr split into three bf16 parts (hi+mid+lo)
//   DWR  router weight gradient X^T dz, dz split into two bf16 parts, split-K
//   UPQ  UP with MXFP8 operands (E4M3 codes, one E8M0 scale per 32 K): the
//        epilogue stores H (bf16) and A quantized to MXFP8 with its scales
//   DOWNQ DOWN with MXFP8 operands
//
// Sources: page "SonicMoE：突破细粒度MoE硬件效率瓶颈，实现高稀疏性下的极致训练加速"
// (implementation paragraph: grouped GEMMs with modular fusion, eight kernels);
// page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", section
// "第二，IO 感知的算子融合" (gather fused into the GEMM, SwiGLU in the
// epilogue, dH kernel overlapping IO with MMA) and section "软件抽象层 QuACK"
// (every MoE GEMM = shared main loop + per-kernel epilogue).
//
// Roles: warp 0 lane 0 issues TMA loads; warp 1 allocates TMEM and issues the
// MMAs (one thread); warps 2-5 run the epilogue (one accumulator row each);
// warps 6-9 (gather kinds only) stream gathered rows with cp.async into the
// same 128-byte-swizzled layout TMA would produce.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "mx.cuh"
#include "ptx.cuh"

namespace moe {

enum GemmKind : int { G_UP = 0, G_DOWN, G_DH, G_DXT, G_DW1, G_DW2, G_RTR, G_DWR, G_UPQ, G_DOWNQ };

struct GemmParams {
  CUtensorMap tmA;   // TMA map of A (kinds whose A is not gathered)
  CUtensorMap tmB;   // TMA map of B (kinds whose B is not gathered)
  CUtensorMap tmC0;  // TMA store map of the first bf16 output (32 x 32 boxes, 64B swizzle)
  CUtensorMap tmC1;  // TMA store map of the second bf16 output (UP: A, DH: A_hat)
  DevStatus st;
  const int* offsets;      // [E+1] 128-aligned segment starts
  const int* counts;       // [E]
  const int* tile_expert;  // [R_max/128]
  const int* row_tok;      // [R_max]  token of each row, -1 for padding
  const float* row_gate;   // [R_max]
  const __nv_bfloat16* gsrc;  // gathered operand source [T, gld]
  int gld;
  int T, d, n, E, Epad;
  int num_n_tiles;
  int num_m_tiles;   // non-grouped-M kinds
  int ksplit;        // DWR
  int ksplit_rows;   // DWR, multiple of 64
  __nv_bfloat16* out0;
  __nv_bfloat16* out1;
  const __nv_bfloat16* hin;
  float* outf;
  const float* bias;
  int* sched;                // weight-gradient kinds: zeroed 64-bit tile counter (8-byte aligned)
  const int* expert_order;   // weight-gradient kinds: experts by descending token count
  int dual_ended;            // weight-gradient kinds: 0 every claim from the largest experts' end; 1 odd
                             // CTAs claim from the smallest experts' end; 2 every CTA alternates ends
  // grouped-M kinds: the 128-row M tiles to run, [count, tile...], or null
  // for all of them (the pair kernel's list: the first of each pair of tiles)
  const int* mlist;
  // up-proj only: where the first CTA writes the 256-row tile list of the
  // grouped-M tiles for the down-proj launch that follows (or null), and the
  // list's first entry of each expert [E + 1]
  int* wlist;
  int* wbase;
  // grouped-M tile order: 0 M-tile-major (the N tiles of one M tile run side
  // by side), 1 weight-stationary (within an expert, the M tiles of one N
  // tile run side by side, so each weight tile is read from DRAM once)
  int wstat;
  const float* rvec;         // DXT router path: Wr transposed [E, d], or null
  const float* rscale;       // DXT router path: dz of each row [R_max] (padding rows unset)
  // MXFP8 kinds.  Scale tiles are 512 bytes: 128 tile rows x 4 scales (one
  // K block of 128), the scale of row m, sub-block j at 16 (m % 32) + 4 (m / 32) + j.
  const uint8_t* sfa_src;    // UPQ: X scales [T, d/32] (gathered per row); DOWNQ: A scale tiles [R_max/128][n/128]
  const uint8_t* sfb_src;    // weight scale tiles [E][N tiles][K/128]
  uint8_t* aq_out;           // UPQ: A codes [R_max, n]
  uint8_t* sa_out;           // UPQ: A scale tiles [R_max/128][n/128]
  // Role timeline (moe_trace_gemm), null when off: per CTA and role, up to
  // trace_cap records of (globaltimer ns, clock64 low bits, tile << 8 | event)
  uint8_t* trace;
  int trace_cap;
};

// One timeline record; roles: 0 TMA producer, 1 MMA issuer, 2 epilogue
// (its first warp), 3 gather warps (their first thread).
struct TraceRec {
  unsigned long long ns;
  uint32_t clk;
  uint32_t info;  // tile << 8 | event
};
__device__ __forceinline__ void trace_ev(const GemmParams& p, int role, int& n, int tile, int ev) {
  if (p.trace && n < p.trace_cap) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    TraceRec* r = reinterpret_cast<TraceRec*>(p.trace) + ((size_t)blockIdx.x * 4 + role) * p.trace_cap + n;
    r->ns = t;
    r->clk = (uint32_t)clock64();
    r->info = ((uint32_t)tile << 8) | (uint32_t)ev;
    ++n;
  }
}

template <int KIND>
struct KindTraits {
  static constexpr bool kGroupedM =
      (KIND == G_UP || KIND == G_DOWN || KIND == G_DH || KIND == G_DXT || KIND == G_UPQ || KIND == G_DOWNQ);
  static constexpr bool kFp8 = (KIND == G_UPQ || KIND == G_DOWNQ);
  static constexpr bool kGroupedK = (KIND == G_DW1 || KIND == G_DW2);
  static constexpr bool kAGather = (KIND == G_UP || KIND == G_DH || KIND == G_DW1 || KIND == G_UPQ);
  static constexpr bool kBGather = (KIND == G_DW2);
  static constexpr bool kGather = kAGather || kBGather;
  static constexpr bool kAMN = (KIND == G_DW1 || KIND == G_DW2 || KIND == G_DWR);
  static constexpr bool kBMN = !(KIND == G_DH || KIND == G_DXT || KIND == G_UPQ || KIND == G_DOWNQ);
};

// Registers per thread at which a block of `threads` still launches: the
// register file is split over the SM's four sub-partitions (16384 each) and
// a block's warps are spread over them, so the sub-partition with the most
// warps, ceil(warps / 4), bounds the count (allocated in multiples of 8 per
// thread, at most 255): 128 for 14 warps, 168 for 10 or 12, 255 for 6.
__host__ __device__ constexpr int max_regs_for(int threads) {
  return ((16384 / (32 * ((threads / 32 + 3) / 4))) & ~7) > 255 ? 255
                                                                : ((16384 / (32 * ((threads / 32 + 3) / 4))) & ~7);
}

// Epilogue configuration: EPI = 4 or 8 epilogue warps.  With 8, two warps
// share each TMEM lane quarter and each takes half of the tile's columns;
// that pays where the epilogue, not the main loop, bounds a tile (the dH
// epilogue with its H reload and three outputs, or a short K loop).
template <int KIND, int EPI>
struct EpiCfg {
  static_assert(EPI == 4 || EPI == 8, "4 or 8 epilogue warps");
  static constexpr int kWarps = EPI;
  static constexpr int kColSplit = EPI / 4;
  // 2 KB staging buffers per warp: the up-proj and dH epilogues store three
  // outputs per chunk; the others ring through 3 buffers.  With 8 warps the
  // dX~ kernel keeps 2 (so that its stage ring keeps its depth), while the
  // weight-gradient kinds, which get 8 warps when their tiles are store-bound
  // (few rows per expert), keep 4 bulk stores in flight per warp.
  // One-output kinds (down-proj, dX~, dW1, dW2) stage 32 rows x 64 columns
  // per buffer (4 KB, 128-byte swizzle) so that each TMA store writes whole
  // 128-byte row segments: a 32-column box writes half-lines, twice the store
  // requests, and the per-SM store path then bounds store-heavy tiles.  They
  // keep 2 such buffers per warp.
  static constexpr bool kWide = (KIND == G_DOWN || KIND == G_DXT || KindTraits<KIND>::kGroupedK);
  static constexpr int kBufs = (KIND == G_UP || KIND == G_DH || KIND == G_UPQ)
                                   ? 3
                                   : (kWide ? 2 : (EPI == 8 ? 2 : 3));
  static constexpr int kBufBytes = kWide ? 4096 : 2048;
  // staging of all epilogue warps in 2 KB units: the GemmShape NBUF that both
  // the kernel's layout and its launch (the dynamic shared-memory size) use
  static constexpr int kNbuf = EPI * kBufs * (kBufBytes / 2048);
  static constexpr int kThreads = 32 * (2 + EPI + (KindTraits<KIND>::kGather ? 4 : 0));
  static constexpr int kMaxReg = max_regs_for(kThreads);
};

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kWideSecond = 1 << 30;  // 256-row tile list entry flag: the pair's second M tile exists

// The 256-row tile list of the grouped-M tiles, by one warp: for expert e,
// whose padded segment holds M tiles [offsets[e] / 128, offsets[e + 1] / 128),
// one entry per pair of consecutive tiles (its first tile, with kWideSecond)
// and one for the last tile of an odd count (without the flag);
// list = [count, entry...] in expert order, and base[e] = the index (after the
// count) of expert e's first entry, base[E] = the count.
__device__ __forceinline__ void write_wide_list(const int* __restrict__ offsets, int E, int* __restrict__ list,
                                                int* __restrict__ base_out, int lane) {
  int base = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    int t0 = 0, nt = 0;
    if (e < E) {
      const int o0 = __ldg(offsets + e), o1 = __ldg(offsets + e + 1);
      t0 = o0 / kBM;
      nt = (o1 - o0) / kBM;
    }
    const int nw = (nt + 1) >> 1;
    int sw = nw;  // inclusive scan over the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int a = __shfl_up_sync(0xffffffffu, sw, o);
      if (lane >= o) sw += a;
    }
    const int b = base + sw - nw;
    for (int j = 0; j < nw; ++j) list[1 + b + j] = (t0 + 2 * j) | (2 * j + 1 < nt ? kWideSecond : 0);
    if (e < E) base_out[e] = b;
    base += __shfl_sync(0xffffffffu, sw, 31);
  }
  if (lane == 0) {
    list[0] = base;
    base_out[E] = base;
  }
}
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kBoxBytes = 64 * 64 * 2;  // one 64x64 bf16 box (MN-major operand)
constexpr int kStageBudget = 200 * 1024;
constexpr int kSmemLimit = 227 * 1024;  // dynamic shared memory per block
constexpr int kRtrGroup = 4;  // router logits: k-blocks per promoted hi-part group
constexpr int kStoreBuf = 2048;  // one epilogue staging buffer: 32 rows x 32 bf16
constexpr int kTileQ = 4;        // depth of the dynamic scheduler's tile queue

// Shared-memory rings of k-blocks (A slots of 16 KB, B slots of BN x 64
// bf16).  The up-proj and dH kernels, whose A rows are gathered with cp.async
// and published a few k-blocks after they are issued, give A and B separate
// rings so that A's is deeper.  The other kinds keep one ring of (A, B)
// stages with one barrier pair per stage: fewer barrier operations per
// k-block where the main loop runs near the tensor-core rate.
template <int KIND, int BN, int NBUF = 12>
struct GemmShape {
  using KT = KindTraits<KIND>;
  static constexpr bool kSplit = (KIND == G_UP || KIND == G_DH || KIND == G_UPQ);
  // B slot: BN rows of 128 bytes (64 bf16 or 128 fp8 K elements)
  static constexpr int kBBytes = BN * kBK * 2;
  // MXFP8 kinds: one 512-byte scale tile per A slot and per 128 rows of a B slot
  static constexpr int kSFABytes = KT::kFp8 ? 512 : 0;
  static constexpr int kSFBBytes = KT::kFp8 ? 512 * (BN / 128) : 0;
  static constexpr int kASlot = kABytes + kSFABytes;  // budget per A slot
  static constexpr int kBSlot = kBBytes + kSFBBytes;  // budget per B slot
  static constexpr int kStoreBytes = NBUF * kStoreBuf;  // epilogue staging: NBUF buffers of 2 KB
  static constexpr int kBudget = (kSmemLimit - 2048 - kStoreBytes) < kStageBudget
                                     ? (kSmemLimit - 2048 - kStoreBytes) : kStageBudget;
  static constexpr int cap8(int x) { return x > 8 ? 8 : x; }
  static constexpr int kStages = cap8(kBudget / (kASlot + kBSlot));  // one (A, B) ring
  static constexpr int kSBs = (kBudget - 3 * kBSlot >= 5 * kASlot) ? (kBBytes >= 32768 ? 3 : 4) : 2;
  static constexpr int kSA = kSplit ? cap8((kBudget - kSBs * kBSlot) / kASlot) : kStages;
  static constexpr int kSB = kSplit ? kSBs : kStages;
  // cp.async publication lag of a gathered operand (k-blocks in flight per
  // thread = lag + 1; the MMA keeps ring - lag - 1 published k-blocks queued)
  static constexpr int kLag = kSplit ? ((kSA - 3 > 3) ? 3 : ((kSA - 3 < 1) ? 1 : kSA - 3)) : 1;
  static constexpr int kAOffset = 0;
  static constexpr int kBOffset = kSA * kABytes;
  // accumulator buffers start at power-of-two column offsets
  static constexpr int kAccStride = BN <= 64 ? 64 : (BN <= 128 ? 128 : 256);
  // MXFP8: the scale factors live in TMEM after the two accumulators
  static constexpr int kSFACol = 2 * kAccStride;      // 4 columns
  static constexpr int kSFBCol = 2 * kAccStride + 4;  // 4 columns per 128 B rows
  static constexpr int kTmemCols = KT::kFp8 ? 512 : 2 * kAccStride;
  static constexpr int kSFAOffset = kBOffset + kSB * kBBytes;      // MXFP8 scale-tile rings
  static constexpr int kSFBOffset = kSFAOffset + kSA * kSFABytes;
  static constexpr int kStoreOffset = kSFBOffset + kSB * kSFBBytes;  // epilogue staging
  static constexpr int kBarOffset = kStoreOffset + kStoreBytes;
  static constexpr int kSmemBytes = kBarOffset + 1024 + 1024;  // barriers + alignment slack
  static_assert(kSA >= 2 && kSB >= 2 && kSA <= 8 && kSB <= 8, "ring depths");
  static_assert(!KT::kFp8 || (BN == 128 && kSFBCol + 4 * (BN / 128) <= kTmemCols), "MXFP8 tiles are 128 wide");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

struct TileInfo {
  int e, mt, nt, m0, n0, krow0, nkb, split;
};

template <int KIND, int BN>
__device__ __forceinline__ int gemm_num_tiles(const GemmParams& p) {
  using KT = KindTraits<KIND>;
  if constexpr (KT::kGroupedM) {
    if (p.mlist) return __ldg(p.mlist) * p.num_n_tiles;
    return (__ldg(p.offsets + p.E) / kBM) * p.num_n_tiles;
  } else if constexpr (KT::kGroupedK) {
    return p.E * p.num_m_tiles * p.num_n_tiles;
  } else if constexpr (KIND == G_DWR) {
    return p.num_m_tiles * p.num_n_tiles * p.ksplit;
  } else {
    return p.num_m_tiles * p.num_n_tiles;
  }
}

template <int KIND, int BN>
__device__ __forceinline__ TileInfo gemm_tile(const GemmParams& p, int tile) {
  using KT = KindTraits<KIND>;
  TileInfo t;
  t.split = 0;
  t.krow0 = 0;
  if constexpr (KT::kGroupedM) {
    t.mt = tile / p.num_n_tiles;
    t.nt = tile - t.mt * p.num_n_tiles;
    if (p.mlist) t.mt = __ldg(p.mlist + 1 + t.mt);
    t.e = __ldg(p.tile_expert + t.mt);
    if (p.wstat && !p.mlist) {
      // the expert's tiles are [t0, t0 + m) x N tiles in either order; walk
      // its M tiles first within each N tile
      const int t0 = __ldg(p.offsets + t.e) / kBM;
      const int m = __ldg(p.offsets + t.e + 1) / kBM - t0;
      const int l = tile - t0 * p.num_n_tiles;
      t.nt = l / m;
      t.mt = t0 + (l - t.nt * m);
    }
    t.m0 = t.mt * kBM;
    if constexpr (KIND == G_UP || KIND == G_UPQ) t.n0 = t.nt * (BN / 2);
    else t.n0 = t.nt * BN;
    const int K = (KIND == G_UP || KIND == G_DH || KIND == G_UPQ) ? p.d
                  : ((KIND == G_DOWN || KIND == G_DOWNQ) ? p.n : 2 * p.n);
    t.nkb = KT::kFp8 ? K / 128 : K / kBK;  // a k-block is 128 bytes of K per row
  } else if constexpr (KT::kGroupedK) {
    const int per_e = p.num_m_tiles * p.num_n_tiles;
    const int ei = tile / per_e;
    t.e = p.expert_order ? __ldg(p.expert_order + ei) : ei;  // largest experts first
    const int rem = tile - ei * per_e;
    t.mt = rem / p.num_n_tiles;
    t.nt = rem - t.mt * p.num_n_tiles;
    t.m0 = t.mt * kBM;
    t.n0 = t.nt * BN;
    t.krow0 = __ldg(p.offsets + t.e);
    t.nkb = (__ldg(p.counts + t.e) + kBK - 1) / kBK;
  } else if constexpr (KIND == G_DWR) {
    const int per_s = p.num_m_tiles * p.num_n_tiles;
    t.split = tile / per_s;
    const int rem = tile - t.split * per_s;
    t.mt = rem / p.num_n_tiles;
    t.nt = rem - t.mt * p.num_n_tiles;
    t.e = 0;
    t.m0 = t.mt * kBM;
    t.n0 = t.nt * BN;
    t.krow0 = t.split * p.ksplit_rows;
    int rows = p.T - t.krow0;
    if (rows > p.ksplit_rows) rows = p.ksplit_rows;
    t.nkb = rows > 0 ? (rows + kBK - 1) / kBK : 0;
  } else {  // G_RTR
    t.mt = tile / p.num_n_tiles;
    t.nt = tile - t.mt * p.num_n_tiles;
    t.e = 0;
    t.m0 = t.mt * kBM;
    t.n0 = t.nt * BN;
    t.nkb = p.d / kBK;
  }
  return t;
}

// Weight-gradient kinds: the tile whose expert-dependent fields (expert id,
// first row, k-blocks) are already resolved -- the producer resolves them once
// and hands them to the other roles through the shared-memory tile queue.
template <int KIND, int BN>
__device__ __forceinline__ TileInfo gemm_tile_resolved(const GemmParams& p, int tile, int e, int krow0, int nkb) {
  TileInfo t;
  const int per_e = p.num_m_tiles * p.num_n_tiles;
  const int rem = tile - (tile / per_e) * per_e;
  t.e = e;
  t.mt = rem / p.num_n_tiles;
  t.nt = rem - t.mt * p.num_n_tiles;
  t.m0 = t.mt * kBM;
  t.n0 = t.nt * BN;
  t.krow0 = krow0;
  t.nkb = nkb;
  t.split = 0;
  return t;
}

// Token id of a gathered row.  The debug build (MOE_DEBUG=1) checks it and
// turns an out-of-range id into a padding row (zero fill) after recording
// the violation, so that no copy leaves the gathered tensor.
#ifndef MOE_DEBUG
#define MOE_DEBUG 0
#endif
template <int KIND>
__device__ __forceinline__ int gather_tok(const GemmParams& p, int r) {
  int tok = __ldg(p.row_tok + r);
#if MOE_DEBUG
  if (tok < -1 || tok >= p.T) {
    raise_status(p.st, ST_DEVICE_CHECK, 0x200 + KIND);
    tok = -1;
  }
#endif
  return tok;
}

// Byte offset of 16-byte chunk `c` of 128-byte line `i` in a 128B-swizzled tile.
__device__ __forceinline__ uint32_t sw128(int line, int chunk) {
  return (uint32_t)(line * 128 + ((chunk ^ (line & 7)) << 4));
}

// ----------------------------------------------------------------- producer
// TMA loads of k-block kb: A into a_s (completing on bar_a), B into b_s
// (completing on bar_b); an operand the gather warps stream is skipped.
template <int KIND, int BN>
__device__ __forceinline__ void issue_tma(const GemmParams& p, const TileInfo& t, int kb, uint32_t a_s,
                                          uint32_t bar_a, uint32_t b_s, uint32_t bar_b, uint32_t sfa_s,
                                          uint32_t sfb_s) {
  const void* tA = &p.tmA;
  const void* tB = &p.tmB;
  const int k0 = kb * kBK;
  constexpr int nb = BN / 64;
  using SHp = GemmShape<KIND, BN>;
  // one ring: a single arrive.expect_tx covers both operands' bytes
  constexpr bool kOne = !SHp::kSplit;
  constexpr uint32_t kTxA = (KIND == G_UP || KIND == G_DH || KIND == G_DW1 || KIND == G_UPQ)
                                ? 0u : (uint32_t)(kABytes + SHp::kSFABytes);
  constexpr uint32_t kTxB = (KIND == G_DW2) ? 0u : (uint32_t)(nb * kBoxBytes + SHp::kSFBBytes);
  (void)sfa_s;
  (void)sfb_s;
  if constexpr (kOne) {
    mbar_arrive_expect_tx(bar_a, kTxA + kTxB);
    bar_b = bar_a;
  }
  (void)bar_b;  // unused by the kinds whose B is gathered
  auto expect_a = [&](uint32_t bytes) {
    if constexpr (!kOne) mbar_arrive_expect_tx(bar_a, bytes);
  };
  auto expect_b = [&](uint32_t bytes) {
    if constexpr (!kOne) mbar_arrive_expect_tx(bar_b, bytes);
  };
  if constexpr (KIND == G_UP) {
    constexpr int half = nb / 2;
    expect_b(nb * kBoxBytes);
    for (int j = 0; j < nb; ++j) {
      const int col = (j < half) ? (t.n0 + 64 * j) : (p.n + t.n0 + 64 * (j - half));
      tma_load_2d(b_s + j * kBoxBytes, tB, bar_b, col, t.e * p.d + k0);
    }
  } else if constexpr (KIND == G_DOWN) {
    expect_a(kABytes);
    tma_load_2d(a_s, tA, bar_a, k0, t.m0);
    expect_b(nb * kBoxBytes);
    for (int j = 0; j < nb; ++j) tma_load_2d(b_s + j * kBoxBytes, tB, bar_b, t.n0 + 64 * j, t.e * p.n + k0);
  } else if constexpr (KIND == G_DH) {
    expect_b(BN * 128);
    tma_load_2d(b_s, tB, bar_b, k0, t.e * p.n + t.n0);
  } else if constexpr (KIND == G_DXT) {
    expect_a(kABytes);
    tma_load_2d(a_s, tA, bar_a, k0, t.m0);
    expect_b(BN * 128);
    tma_load_2d(b_s, tB, bar_b, k0, t.e * p.d + t.n0);
  } else if constexpr (KIND == G_DW1) {
    expect_b(nb * kBoxBytes);
    for (int j = 0; j < nb; ++j) tma_load_2d(b_s + j * kBoxBytes, tB, bar_b, t.n0 + 64 * j, t.krow0 + k0);
  } else if constexpr (KIND == G_DW2) {
    expect_a(2 * kBoxBytes);
    for (int h = 0; h < 2; ++h) tma_load_2d(a_s + h * kBoxBytes, tA, bar_a, t.m0 + 64 * h, t.krow0 + k0);
  } else if constexpr (KIND == G_UPQ) {
    // W1 codes transposed [E * 2n rows, d bytes]: 64 gate rows, then the
    // same 64 up rows; the scale tile of (expert, N tile, K block)
    const int x = kb * 128;
    expect_b((uint32_t)(BN * 128 + SHp::kSFBBytes));
    tma_load_2d(b_s, tB, bar_b, x, t.e * 2 * p.n + t.n0);
    tma_load_2d(b_s + 64 * 128, tB, bar_b, x, t.e * 2 * p.n + p.n + t.n0);
    bulk_load(sfb_s, p.sfb_src + ((size_t)(t.e * p.num_n_tiles + t.nt) * (p.d / 128) + kb) * 512, 512, bar_b);
  } else if constexpr (KIND == G_DOWNQ) {
    // A codes [R_max, n bytes] and its scale tiles; W2 codes transposed
    // [E * d rows, n bytes] and their scale tiles
    const int x = kb * 128;
    tma_load_2d(a_s, tA, bar_a, x, t.m0);
    bulk_load(sfa_s, p.sfa_src + ((size_t)t.mt * (p.n / 128) + kb) * 512, 512, bar_a);
    tma_load_2d(b_s, tB, bar_a, x, t.e * p.d + t.n0);
    bulk_load(sfb_s, p.sfb_src + ((size_t)(t.e * (p.d / 128) + t.nt) * (p.n / 128) + kb) * 512, 512, bar_a);
  } else if constexpr (KIND == G_RTR) {
    // Wr column box j = (group j / 3, part j % 3: hi, mid, lo) goes to slot
    // [hi of every group | mid, lo of group 0 | mid, lo of group 1 ...], so
    // that one MMA covers every group's hi part and one every mid and lo part
    constexpr int G = BN / 192;
    expect_a(kABytes);
    tma_load_2d(a_s, tA, bar_a, k0, t.m0);
    expect_b(nb * kBoxBytes);
    for (int j = 0; j < nb; ++j) {
      const int pos = (j % 3 == 0) ? j / 3 : G + 2 * (j / 3) + (j % 3 - 1);
      tma_load_2d(b_s + pos * kBoxBytes, tB, bar_b, t.n0 + 64 * j, k0);
    }
  } else {  // G_DWR
    expect_a(2 * kBoxBytes);
    for (int h = 0; h < 2; ++h) tma_load_2d(a_s + h * kBoxBytes, tA, bar_a, t.m0 + 64 * h, t.krow0 + k0);
    expect_b(nb * kBoxBytes);
    for (int j = 0; j < nb; ++j) tma_load_2d(b_s + j * kBoxBytes, tB, bar_b, t.n0 + 64 * j, t.krow0 + k0);
  }
}

// ----------------------------------------------------------------- epilogue helpers
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
    d4[q] = w;
  }
}
__device__ __forceinline__ void load_row32_bf16(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w = s4[q];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      v[8 * q + 2 * i] = f.x;
      v[8 * q + 2 * i + 1] = f.y;
    }
  }
}
__device__ __forceinline__ void zero32(float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = 0.f;
}
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }

// Epilogue staging: a 32-row x 32-column bf16 box laid out with the 64-byte
// swizzle the output tensor maps use; thread `row` writes its row.
__device__ __forceinline__ uint32_t sw64(int row, int chunk) {
  return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}
__device__ __forceinline__ uint4 pack8f(const float* v) {
  uint4 w;
  w.x = pack_bf16x2(v[0], v[1]);
  w.y = pack_bf16x2(v[2], v[3]);
  w.z = pack_bf16x2(v[4], v[5]);
  w.w = pack_bf16x2(v[6], v[7]);
  return w;
}
__device__ __forceinline__ void stage_row32(uint32_t buf, int row, const float (&v)[32]) {
#pragma unroll
  for (int c = 0; c < 4; ++c) st_shared_v4(buf + sw64(row, c), pack8f(v + 8 * c));
}

// ----------------------------------------------------------------- kernel
template <int KIND, int BN, int EPI>
__global__ void __maxnreg__((EpiCfg<KIND, EPI>::kMaxReg))
    moe_gemm_kernel(const __grid_constant__ GemmParams p) {
  using KT = KindTraits<KIND>;
  using EC = EpiCfg<KIND, EPI>;
  using SH = GemmShape<KIND, BN, EC::kNbuf>;
  constexpr int kEpiEnd = 2 + EPI;  // epilogue warps are [2, kEpiEnd)
  constexpr bool kSplit = SH::kSplit;  // separate A and B rings
  constexpr int SA = SH::kSA;      // A ring slots
  constexpr int SB = SH::kSB;      // B ring slots
  constexpr int kLag = SH::kLag;   // gathered k-blocks are published kLag k-blocks after issue
  constexpr uint32_t kIdesc = idesc_bf16_f32(BN, KT::kAMN, KT::kBMN);

  extern __shared__ uint8_t smem_raw[];
  // a launch with less shared memory than this layout needs stops here with
  // a status instead of touching memory past its allocation
  if (dynamic_smem_bytes() < (uint32_t)SH::kSmemBytes) {
    if (threadIdx.x == 0) raise_status(p.st, ST_DEVICE_CHECK, 0x300 + KIND);
    return;
  }
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::kBarOffset);
  uint64_t* full_a = bars;         // [SA] A ring (the (A, B) ring without kSplit)
  uint64_t* empty_a = bars + 8;
  uint64_t* full_b = kSplit ? bars + 16 : full_a;  // [SB] B ring
  uint64_t* empty_b = kSplit ? bars + 24 : empty_a;
  uint64_t* acc_full = bars + 32;
  uint64_t* acc_empty = bars + 34;
  uint64_t* hi_full = bars + 36;   // router logits: promoted hi-part groups
  uint64_t* hi_empty = bars + 38;
  uint64_t* tq_full = bars + 40;   // dynamic scheduler: tile queue
  uint64_t* tq_empty = bars + 44;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 48);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 49);
  // [kTileQ] queued tiles {tile, expert, first row, k-blocks}; written and
  // read between the queue's mbarrier arrive (release) and wait (acquire)
  int4* tq_info = reinterpret_cast<int4*>(bars + 50);
  auto a_slot = [&](int i) -> uint32_t { return base + SH::kAOffset + (uint32_t)(i * kABytes); };
  auto b_slot = [&](int i) -> uint32_t { return base + SH::kBOffset + (uint32_t)(i * SH::kBBytes); };
  // the router-logit kind covers G = BN / 192 groups of 64 experts per tile
  // in 256 G TMEM columns: two alternating hi slots of 64 G columns (every
  // group's hi part), then each group's mid and lo (128 columns per group)
  constexpr int kRtrG = (KIND == G_RTR) ? BN / 192 : 1;
  constexpr int kTmemCols = (KIND == G_RTR) ? 256 * kRtrG : SH::kTmemCols;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    if constexpr (kSplit) {  // A gathered (128 threads), B by the TMA thread
      for (int s = 0; s < SA; ++s) {
        mbar_init(&full_a[s], 128);
        mbar_init(&empty_a[s], 1);
      }
      for (int s = 0; s < SB; ++s) {
        mbar_init(&full_b[s], 1);
        mbar_init(&empty_b[s], 1);
      }
    } else {  // the TMA thread (+ 128 gather threads)
      for (int s = 0; s < SA; ++s) {
        mbar_init(&full_a[s], 1 + (KT::kGather ? 128 : 0));
        mbar_init(&empty_a[s], 1);
      }
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * EPI);
      mbar_init(&hi_full[b], 1);
      mbar_init(&hi_empty[b], 128);
    }
    for (int b = 0; b < kTileQ; ++b) {
      mbar_init(&tq_full[b], 1);
      mbar_init(&tq_empty[b], 1 + EPI + (KT::kGather ? 4 : 0));  // consumer warps: MMA, epilogue, gather
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (!KT::kAGather) tma_prefetch_desc(&p.tmA);
    if constexpr (!KT::kBGather) tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above touched only shared memory, TMEM and the kernel's own
  // parameters; global reads and writes start once the predecessor is done
  pdl_wait();

  const int num_tiles = gemm_num_tiles<KIND, BN>(p);

  // Tile order.  Static kinds walk tiles round-robin.  The weight-gradient
  // kinds, whose tiles differ in length with the expert's token count, take
  // tiles dynamically from a list ordered by expert, largest first.  Claims
  // come from both ends of the list: the front holds the long, L2-bound tiles
  // of the busiest experts, the back the short tiles of the smallest experts,
  // bound by storing their results.  With dual_ended = 1, even CTAs claim from
  // the front and odd CTAs from the back, so both kinds run at once on
  // different SMs; with 2, every CTA takes its first tile from the front and
  // then alternates ends, so that a short tile's stores run under the next
  // long tile's main loop on the same SM.  One 64-bit counter holds both ends
  // (front claims in the low word, back claims in the high word); claim k
  // (the sum of both before the increment) is valid iff k < tiles, and the
  // last tiles taken are the middle-sized ones.  The TMA thread claims a tile
  // one tile ahead (the atomic's latency hides behind the current tile's
  // loads), resolves its expert once, and hands it to the other roles through
  // a shared-memory queue.
  constexpr bool kDyn = KT::kGroupedK;
  const bool alternate = p.dual_ended == 2;
  const bool front_cta = p.dual_ended != 1 || (blockIdx.x & 1u) == 0u;
  // the end that claim i (the claim of this CTA's tile i >= 1) takes
  auto front_of = [&](int i) -> bool { return alternate ? (i & 1) == 0 : front_cta; };
  const int nfront0 = p.dual_ended == 1 ? ((int)gridDim.x + 1) / 2 : (int)gridDim.x;  // first tiles, unclaimed
  const int nback0 = (int)gridDim.x - nfront0;
  auto claim = [&](bool front) -> unsigned long long {
    return atomicAdd(reinterpret_cast<unsigned long long*>(p.sched), front ? 1ull : (1ull << 32));
  };
  auto claimed_tile = [&](unsigned long long old, bool front) -> int {
    const int f = (int)(old & 0xffffffffull) + nfront0;
    const int b = (int)(old >> 32) + nback0;
    if (f + b >= num_tiles) return num_tiles;
    return front ? f : num_tiles - 1 - b;
  };
  unsigned long long next_claim = 0;
  int res_ei = -1, res_e = 0, res_krow0 = 0, res_nkb = 0;  // the producer's last resolved expert
  auto produce_tile = [&](int i, bool& good, TileInfo& t) -> int {
    if constexpr (kDyn) {
      int tile;
      if (i == 0) {
        const int j = p.dual_ended == 1 ? ((int)blockIdx.x >> 1) : (int)blockIdx.x;
        tile = front_cta ? j : num_tiles - 1 - j;
      } else {
        tile = claimed_tile(next_claim, front_of(i));
      }
      if (tile < num_tiles) next_claim = claim(front_of(i + 1));  // the next tile's claim, in flight meanwhile
      int e = 0, krow0 = 0, nkb = 0;
      if (tile < num_tiles) {
        const int ei = tile / (p.num_m_tiles * p.num_n_tiles);
        if (ei != res_ei) {
          res_ei = ei;
          res_e = p.expert_order ? __ldg(p.expert_order + ei) : ei;
          res_krow0 = __ldg(p.offsets + res_e);
          res_nkb = (__ldg(p.counts + res_e) + kBK - 1) / kBK;
        }
        e = res_e;
        krow0 = res_krow0;
        nkb = res_nkb;
        t = gemm_tile_resolved<KIND, BN>(p, tile, e, krow0, nkb);
      }
      const int slot = i % kTileQ;
      if (!mbar_wait(smem_u32(&tq_empty[slot]), ((i / kTileQ) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 10)) {
        good = false;
        return num_tiles;
      }
      tq_info[slot] = make_int4(tile, e, krow0, nkb);
      mbar_arrive(smem_u32(&tq_full[slot]));
      return tile;
    } else {
      const int tile = (int)blockIdx.x + i * (int)gridDim.x;
      if (tile < num_tiles) t = gemm_tile<KIND, BN>(p, tile);
      return tile;
    }
  };
  auto consume_tile = [&](int i, bool& good, TileInfo& t) -> int {
    if constexpr (kDyn) {
      const int slot = i % kTileQ;
      if (!mbar_wait(smem_u32(&tq_full[slot]), (i / kTileQ) & 1, abort_flag, p.st, KIND * 16 + 11)) {
        good = false;
        return num_tiles;
      }
      const int4 q = tq_info[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tq_empty[slot]));
      if (q.x < num_tiles) t = gemm_tile_resolved<KIND, BN>(p, q.x, q.y, q.z, q.w);
      return q.x;
    } else {
      const int tile = (int)blockIdx.x + i * (int)gridDim.x;
      if (tile < num_tiles) t = gemm_tile<KIND, BN>(p, tile);
      return tile;
    }
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int it = 0, ntr = 0;
      bool ok = true;
      for (int ti = 0; ok; ++ti) {
        TileInfo t;
        const int tile = produce_tile(ti, ok, t);
        if (!ok || tile >= num_tiles) break;
        trace_ev(p, 0, ntr, tile, 0);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int sa = it % SA, sb = it % SB;
          if constexpr (!kSplit) {
            if (!mbar_wait(smem_u32(&empty_a[sa]), ((it / SA) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 1)) {
              ok = false;
              break;
            }
          } else {
            if (!mbar_wait(smem_u32(&empty_b[sb]), ((it / SB) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 12)) {
              ok = false;
              break;
            }
          }
          issue_tma<KIND, BN>(p, t, kb, a_slot(sa), smem_u32(&full_a[sa]), b_slot(sb), smem_u32(&full_b[sb]),
                              base + SH::kSFAOffset + (uint32_t)(sa * SH::kSFABytes),
                              base + SH::kSFBOffset + (uint32_t)(sb * SH::kSFBBytes));
          if (ti == 0) trace_ev(p, 0, ntr, kb, 16);  // first tile: each k-block's issue
        }
        trace_ev(p, 0, ntr, tile, 1);
      }
    }
  } else if (warp == 1 && KIND == G_RTR) {
    // ---------------- MMA issuer, router logits.  The hi part of Wr (which
    // carries almost all of each logit) is accumulated in groups of kRtrGroup
    // k-blocks into two alternating TMEM slots; the epilogue adds every group
    // into fp32 registers, so the tensor core's long accumulation chain is cut
    // into short ones.  The mid and lo parts accumulate over the whole K.
    constexpr uint32_t kIdescHi = idesc_bf16_f32(64 * kRtrG, KT::kAMN, KT::kBMN);
    constexpr uint32_t kIdescMl = idesc_bf16_f32(128 * kRtrG, KT::kAMN, KT::kBMN);
    int it = 0, tcount = 0, hg = 0;
    bool ok = true;
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (!mbar_wait(smem_u32(&acc_empty[0]), (tcount & 1) ^ 1, abort_flag, p.st, KIND * 16 + 7)) {
        ok = false;
        break;
      }
      tc_fence_after();
      int slot = 0;
      for (int kb = 0; kb < t.nkb && ok; ++kb, ++it) {
        const bool first = (kb % kRtrGroup) == 0;
        const bool last = (kb % kRtrGroup) == kRtrGroup - 1 || kb == t.nkb - 1;
        if (first) {
          slot = hg & 1;
          if (!mbar_wait(smem_u32(&hi_empty[slot]), ((hg >> 1) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 8)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const int sa = it % SA, sb = it % SB;
        if (!mbar_wait(smem_u32(&full_a[sa]), (it / SA) & 1, abort_flag, p.st, KIND * 16 + 3) ||
            (kSplit && !mbar_wait(smem_u32(&full_b[sb]), (it / SB) & 1, abort_flag, p.st, KIND * 16 + 13))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a_s = a_slot(sa);
          const uint32_t b_s = b_slot(sb);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(a_s + kk * 32, 16, 1024);
            const uint64_t bhi = smem_desc_sw128(b_s + kk * 2048, kBoxBytes, 1024);
            const uint64_t bml = smem_desc_sw128(b_s + kRtrG * kBoxBytes + kk * 2048, kBoxBytes, 1024);
            tc_mma_bf16(tmem_base + (uint32_t)(slot * 64 * kRtrG), ad, bhi, kIdescHi, (first && kk == 0) ? 0u : 1u);
            tc_mma_bf16(tmem_base + (uint32_t)(128 * kRtrG), ad, bml, kIdescMl, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(smem_u32(&empty_a[sa]));
          if (kSplit) tc_commit(smem_u32(&empty_b[sb]));
          if (last) tc_commit(smem_u32(&hi_full[slot]));
        }
        __syncwarp();
        if (last) ++hg;
      }
      if (!ok) break;
      if (lane == 0) tc_commit(smem_u32(&acc_full[0]));
      __syncwarp();
      ++tcount;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    int it = 0, tcount = 0, ntr = 0;
    bool ok = true;
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (t.nkb == 0) continue;
      if (lane == 0) trace_ev(p, 1, ntr, tile, 0);
      const int b = tcount & 1;
      const int use = tcount >> 1;
      if (!mbar_wait(smem_u32(&acc_empty[b]), (use & 1) ^ 1, abort_flag, p.st, KIND * 16 + 2)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) trace_ev(p, 1, ntr, tile, 1);
      const uint32_t d_tmem = tmem_base + (uint32_t)(b * SH::kAccStride);
      for (int kb = 0; kb < t.nkb; ++kb, ++it) {
        const int sa = it % SA, sb = it % SB;
        if (!mbar_wait(smem_u32(&full_a[sa]), (it / SA) & 1, abort_flag, p.st, KIND * 16 + 3) ||
            (kSplit && !mbar_wait(smem_u32(&full_b[sb]), (it / SB) & 1, abort_flag, p.st, KIND * 16 + 13))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (kb == 0 && lane == 0) trace_ev(p, 1, ntr, tile, 2);
        if (ti == 0 && lane == 0) trace_ev(p, 1, ntr, kb, 16);  // first tile: each k-block's operands ready
        if (lane == 0) {
          const uint32_t a_s = a_slot(sa);
          const uint32_t b_s = b_slot(sb);
          if constexpr (KT::kFp8) {
            // scale tiles into TMEM (in issue order with the MMAs that read them),
            // then 4 MMAs of K = 32 fp8 elements, each with its scale byte
            const uint32_t sfa_t = tmem_base + (uint32_t)SH::kSFACol;
            const uint32_t sfb_t = tmem_base + (uint32_t)SH::kSFBCol;
            tc_cp_32x128b_x4(sfa_t, smem_desc_rows16(base + SH::kSFAOffset + (uint32_t)(sa * SH::kSFABytes)));
            tc_cp_32x128b_x4(sfb_t, smem_desc_rows16(base + SH::kSFBOffset + (uint32_t)(sb * SH::kSFBBytes)));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = smem_desc_sw128(a_s + kk * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(b_s + kk * 32, 16, 1024);
              const uint32_t sel = (uint32_t)kk << 30;
              tc_mma_mxf8(d_tmem, ad, bd, idesc_mxf8(BN, (uint32_t)kk, (uint32_t)kk), sfa_t | sel, sfb_t | sel,
                          (kb > 0 || kk > 0) ? 1u : 0u);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = KT::kAMN ? smem_desc_sw128(a_s + kk * 2048, kBoxBytes, 1024)
                                           : smem_desc_sw128(a_s + kk * 32, 16, 1024);
              const uint64_t bd = KT::kBMN ? smem_desc_sw128(b_s + kk * 2048, kBoxBytes, 1024)
                                           : smem_desc_sw128(b_s + kk * 32, 16, 1024);
              tc_mma_bf16(d_tmem, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
          }
          tc_commit(smem_u32(&empty_a[sa]));
          if (kSplit) tc_commit(smem_u32(&empty_b[sb]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) {
        tc_commit(smem_u32(&acc_full[b]));
        trace_ev(p, 1, ntr, tile, 3);
      }
      __syncwarp();
      ++tcount;
    }
  } else if (warp < kEpiEnd && KIND == G_RTR) {
    // ---------------- epilogue, router logits: z = sum of promoted hi groups + mid + lo + bias
    const int q = warp & 3;
    const int rloc = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    int tcount = 0, hg = 0;
    bool ok = true;
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      float hs[kRtrG][64];
#pragma unroll
      for (int g = 0; g < kRtrG; ++g)
#pragma unroll
        for (int i = 0; i < 64; ++i) hs[g][i] = 0.f;
      const int ngroups = (t.nkb + kRtrGroup - 1) / kRtrGroup;
      for (int grp = 0; grp < ngroups; ++grp, ++hg) {
        const int slot = hg & 1;
        if (!mbar_wait(smem_u32(&hi_full[slot]), (hg >> 1) & 1, abort_flag, p.st, KIND * 16 + 9)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int g = 0; g < kRtrG; ++g) {
          uint32_t r0[32], r1[32];
          tmem_ld32(lane_addr + slot * 64 * kRtrG + 64 * g, r0);
          tmem_ld32(lane_addr + slot * 64 * kRtrG + 64 * g + 32, r1);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            hs[g][i] += __uint_as_float(r0[i]);
            hs[g][32 + i] += __uint_as_float(r1[i]);
          }
        }
        tc_fence_before();
        mbar_arrive(smem_u32(&hi_empty[slot]));
      }
      if (!ok) break;
      if (!mbar_wait(smem_u32(&acc_full[0]), tcount & 1, abort_flag, p.st, KIND * 16 + 4)) break;
      tc_fence_after();
      // each warp's 32 rows x 32 logits go through shared memory (padded
      // rows, conflict-free both ways) and leave as 128-byte row pieces
      float* stg = reinterpret_cast<float*>(smem + SH::kStoreOffset + (warp - 2) * (EC::kBufs * kStoreBuf));
#pragma unroll
      for (int gc = 0; gc < 2 * kRtrG; ++gc) {  // 32 columns of group gc / 2 at a time
        const int g = gc >> 1, c = 32 * (gc & 1);
        uint32_t mid[32], lo[32];
        tmem_ld32(lane_addr + 128 * kRtrG + 128 * g + c, mid);
        tmem_ld32(lane_addr + 128 * kRtrG + 128 * g + 64 + c, lo);
        tc_wait_ld();
        const int e0 = (t.nt * kRtrG + g) * 64 + c;  // first expert of these columns
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = e0 + i;
          float z = hs[g][c + i] + (__uint_as_float(mid[i]) + __uint_as_float(lo[i]));
          if (p.bias && e < p.E) z += __ldg(p.bias + e);
          stg[lane * 33 + i] = z;
        }
        __syncwarp();
        const int e = e0 + lane;
#pragma unroll 4
        for (int r = 0; r < 32; ++r) {
          const int trow = t.m0 + q * 32 + r;
          if (trow < p.T && e < p.E) p.outf[(size_t)trow * p.E + e] = stg[r * 33 + lane];
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[0]));
      ++tcount;
    }
  } else if (warp < kEpiEnd) {
    // ---------------- epilogue: one accumulator row per thread.  bf16 results
    // are staged per warp in shared memory (32 rows x 32 columns) and written
    // with TMA tensor stores; each warp owns three 2 KB staging buffers.  A
    // warp reaches TMEM lanes [32 (warp % 4), +32) only.
    const int q = warp & 3;
    const int ew = warp - 2;
    const int half = ew >> 2;  // column part of this warp (EC::kColSplit parts)
    const int rloc = q * 32 + lane;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t stg = base + SH::kStoreOffset + ew * (EC::kBufs * EC::kBufBytes);
    int ring = 0;  // next staging buffer for one-output kinds
    // Make staging buffer(s) free: `pending` store groups may still be reading.
    auto stage_wait = [&](auto pending_tag) {
      constexpr int kPend = decltype(pending_tag)::value;
      if (lane == 0) bulk_wait_read<kPend>();
      __syncwarp();
    };
    auto stage_publish = [&]() {
      fence_proxy_async_smem();
      __syncwarp();
    };
    int tcount = 0, ntr = 0;
    const bool tracer = (warp == 2 && lane == 0);
    bool ok = true;
    if constexpr (KIND == G_UP) {
      // the first CTA's first epilogue warp writes the down-proj's tile list
      // while the first tile's main loop runs
      if (p.wlist && blockIdx.x == 0 && warp == 2) write_wide_list(p.offsets, p.E, p.wlist, p.wbase, lane);
    }
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (tracer) trace_ev(p, 2, ntr, tile, 0);
      const int row0 = t.m0 + q * 32;  // first output row of this warp's slice
      if constexpr (KT::kGroupedK) {
        if (t.nkb == 0) {  // expert without tokens: its weight gradient is zero
          // one staged box of zeros, stored to each 32-column chunk of this
          // warp's rows as one bulk group
          const int M = (KIND == G_DW1) ? p.d : p.n;
          if (row0 < M) {
            constexpr int kC = BN / EC::kColSplit;
            const uint32_t buf = stg + ring * EC::kBufBytes;
            stage_wait(std::integral_constant<int, EC::kBufs - 1>{});
#pragma unroll
            for (int j = 0; j < 8; ++j) st_shared_v4(buf + sw128(lane, j), make_uint4(0u, 0u, 0u, 0u));
            stage_publish();
            if (lane == 0) {
              for (int c = half * kC; c < half * kC + kC; c += 64)
                tma_store_2d(&p.tmC0, buf, t.n0 + c, t.e * M + row0);
              bulk_commit();
            }
            ring = ring + 1 == EC::kBufs ? 0 : ring + 1;
          }
          continue;
        }
      } else if constexpr (KIND == G_DWR) {
        if (t.nkb == 0) {
          const int m = t.m0 + rloc;
          if (m < p.d) {
            float* dst = p.outf + ((size_t)t.split * p.d + m) * p.Epad + t.nt * 64;
            for (int c = 0; c < 64; ++c) dst[c] = 0.f;
          }
          continue;
        }
      }
      // dH epilogue: start loading this row's first 16 columns of H (gate
      // and up) while the MMAs run
      uint4 h_nx[4];
      constexpr int kCols = BN / EC::kColSplit;  // accumulator columns of this warp
      if constexpr (KIND == G_DH) {
        const uint4* h4 =
            reinterpret_cast<const uint4*>(p.hin + (size_t)(t.m0 + rloc) * (2 * p.n) + t.n0 + half * kCols);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          h_nx[i] = __ldg(h4 + i);
          h_nx[2 + i] = __ldg(h4 + p.n / 8 + i);
        }
      }
      // dX~ router path: load this tile's first 32 values of row e of Wr^T
      // (the same for every row of the tile) while the MMAs run
      float rz = 0.f;
      const float4* rv = nullptr;
      if constexpr (KIND == G_DXT) {
        if (p.rvec) {
          const int r = t.m0 + rloc;
          rz = __ldg(p.row_tok + r) >= 0 ? __ldg(p.rscale + r) : 0.f;
          rv = reinterpret_cast<const float4*>(p.rvec + (size_t)t.e * p.d + t.n0);
        }
      }
      const int b = tcount & 1;
      const int use = tcount >> 1;
      if (!mbar_wait(smem_u32(&acc_full[b]), use & 1, abort_flag, p.st, KIND * 16 + 4)) break;
      tc_fence_after();
      if (tracer) trace_ev(p, 2, ntr, tile, 1);
      const uint32_t tacc = lane_addr + (uint32_t)(b * SH::kAccStride);

      if constexpr (KIND == G_UP) {
        constexpr int BNh = BN / 2;  // gate columns [0, BNh), up columns [BNh, BN)
        constexpr int kHalfCols = BNh / EC::kColSplit;
        const int c0 = half * kHalfCols;
#pragma unroll 1
        for (int c = c0; c < c0 + kHalfCols; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tacc + c, g);
          tmem_ld32(tacc + BNh + c, u);
          tc_wait_ld();
          float gv[32], uv[32], av[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            gv[i] = bf16_round(__uint_as_float(g[i]));
            uv[i] = bf16_round(__uint_as_float(u[i]));
            av[i] = gv[i] * sigmoidf_(gv[i]) * uv[i];
          }
          stage_wait(std::integral_constant<int, 0>{});
          stage_row32(stg, lane, gv);
          stage_row32(stg + kStoreBuf, lane, uv);
          stage_row32(stg + 2 * kStoreBuf, lane, av);
          stage_publish();
          if (lane == 0) {
            tma_store_2d(&p.tmC0, stg, t.n0 + c, row0);
            tma_store_2d(&p.tmC0, stg + kStoreBuf, p.n + t.n0 + c, row0);
            tma_store_2d(&p.tmC1, stg + 2 * kStoreBuf, t.n0 + c, row0);
            bulk_commit();
          }
        }
      } else if constexpr (KIND == G_UPQ) {
        // H (bf16, kept for the backward) through the staging boxes; A
        // quantized per row in blocks of 32 to E4M3 codes with an E8M0 scale
        // (the smallest exponent at which nothing saturates), the codes
        // stored straight from registers, the two scales of this tile's 64
        // columns into the scale tile of (M tile, K block t.n0 / 128)
        constexpr int BNh = BN / 2;  // gate columns [0, BNh), up columns [BNh, BN)
        const int r = t.m0 + rloc;
        uint32_t sc2 = 0u;
#pragma unroll 1
        for (int c = 0; c < BNh; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tacc + c, g);
          tmem_ld32(tacc + BNh + c, u);
          tc_wait_ld();
          float gv[32], uv[32], av[32];
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            gv[i] = bf16_round(__uint_as_float(g[i]));
            uv[i] = bf16_round(__uint_as_float(u[i]));
            av[i] = gv[i] * sigmoidf_(gv[i]) * uv[i];
            amax = fmaxf(amax, fabsf(av[i]));
          }
          stage_wait(std::integral_constant<int, 0>{});
          stage_row32(stg, lane, gv);
          stage_row32(stg + kStoreBuf, lane, uv);
          stage_publish();
          if (lane == 0) {
            tma_store_2d(&p.tmC0, stg, t.n0 + c, row0);
            tma_store_2d(&p.tmC0, stg + kStoreBuf, p.n + t.n0 + c, row0);
            bulk_commit();
          }
          const uint32_t code = mx_scale_code(amax);
          const float sinv = mx_inv_scale(code);
          uint32_t w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            w[i] = mx_e4m3x2(av[4 * i] * sinv, av[4 * i + 1] * sinv) |
                   (mx_e4m3x2(av[4 * i + 2] * sinv, av[4 * i + 3] * sinv) << 16);
          uint4* dst = reinterpret_cast<uint4*>(p.aq_out + (size_t)r * p.n + t.n0 + c);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
          sc2 |= code << (8 * (c / 32));
        }
        *reinterpret_cast<uint16_t*>(p.sa_out + ((size_t)t.mt * (p.n / 128) + t.n0 / 128) * 512 +
                                     16 * (rloc & 31) + 4 * (rloc >> 5) + (t.n0 % 128) / 32) = (uint16_t)sc2;
      } else if constexpr (KIND == G_DOWNQ) {
        const int c0 = half * kCols;
#pragma unroll 1
        for (int c = c0; c < c0 + kCols; c += 32) {
          uint32_t a[32];
          tmem_ld32(tacc + c, a);
          tc_wait_ld();
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(a[i]);
          const uint32_t buf = stg + ring * EC::kBufBytes;
          stage_wait(std::integral_constant<int, EC::kBufs - 1>{});
          stage_row32(buf, lane, v);
          stage_publish();
          if (lane == 0) {
            tma_store_2d(&p.tmC0, buf, t.n0 + c, row0);
            bulk_commit();
          }
          ring = ring + 1 == EC::kBufs ? 0 : ring + 1;
        }
      } else if constexpr (KIND == G_DOWN || KIND == G_DXT || KT::kGroupedK) {
        int orow = row0;
        bool live = true;
        if constexpr (KT::kGroupedK) {
          const int M = (KIND == G_DW1) ? p.d : p.n;
          live = row0 < M;
          orow = t.e * M + row0;
        }
        const int c0 = half * kCols;  // this warp's columns: [c0, c0 + kCols)
        static_assert(!EC::kWide || (BN / EC::kColSplit) % 64 == 0, "64-column store chunks");
#pragma unroll 1
        for (int c = c0; c < c0 + kCols; c += 64) {
          uint32_t a[32], a2[32];
          tmem_ld32(tacc + c, a);
          tmem_ld32(tacc + c + 32, a2);
          float4 r_cur[16];
          if constexpr (KIND == G_DXT) {
            if (rv) {  // router path: this chunk's Wr^T values (the same for every row), loaded
                       // while the accumulator loads are in flight
#pragma unroll
              for (int i = 0; i < 16; ++i) r_cur[i] = __ldg(rv + c / 4 + i);
            }
          }
          tc_wait_ld();
          if (live) {
            const uint32_t buf = stg + ring * EC::kBufBytes;
            stage_wait(std::integral_constant<int, EC::kBufs - 1>{});
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // 8 columns per 16-byte chunk of the 128-byte row
              float v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(j < 4 ? a[8 * j + i] : a2[8 * (j - 4) + i]);
              if constexpr (KIND == G_DXT) {
                if (rv) {  // + dz_r * Wr[n0 + c + 8 j + i, e]
                  const float4 w0 = r_cur[2 * j], w1 = r_cur[2 * j + 1];
                  v[0] = fmaf(rz, w0.x, v[0]);
                  v[1] = fmaf(rz, w0.y, v[1]);
                  v[2] = fmaf(rz, w0.z, v[2]);
                  v[3] = fmaf(rz, w0.w, v[3]);
                  v[4] = fmaf(rz, w1.x, v[4]);
                  v[5] = fmaf(rz, w1.y, v[5]);
                  v[6] = fmaf(rz, w1.z, v[6]);
                  v[7] = fmaf(rz, w1.w, v[7]);
                }
              }
              st_shared_v4(buf + sw128(lane, j), pack8f(v));
            }
            stage_publish();
            if (lane == 0) {
              tma_store_2d(&p.tmC0, buf, t.n0 + c, orow);
              bulk_commit();
            }
            ring = ring + 1 == EC::kBufs ? 0 : ring + 1;
          }
        }
      } else if constexpr (KIND == G_DH) {
        // 16 columns at a time (register budget of 8 epilogue warps); the H
        // values of the next 16 columns are loaded one step ahead
        const int r = t.m0 + rloc;
        const float s = __ldg(p.row_gate + r);
        const int c0 = half * kCols;  // this warp's first column in the tile
        const uint4* h4 = reinterpret_cast<const uint4*>(p.hin + (size_t)r * (2 * p.n) + t.n0 + c0);
        const int up8 = p.n / 8;  // offset of the up half in 16-byte units
        float dsum = 0.f;
#pragma unroll 1
        for (int c = 0; c < kCols; c += 32) {
          stage_wait(std::integral_constant<int, 0>{});
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int cc = c + 16 * sub;
            uint32_t a[16];
            tmem_ld16(tacc + c0 + cc, a);
            uint4 hc[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) hc[i] = h_nx[i];
            if (cc + 16 < kCols) {  // prefetch the next 16 columns of H
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                h_nx[i] = __ldg(h4 + (cc + 16) / 8 + i);
                h_nx[2 + i] = __ldg(h4 + up8 + (cc + 16) / 8 + i);
              }
            }
            tc_wait_ld();
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
              const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&hc[qq]);
              const __nv_bfloat162* u2 = reinterpret_cast<const __nv_bfloat162*>(&hc[2 + qq]);
              float dg[8], du[8], ah[8];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 gf = __bfloat1622float2(g2[i]);
                const float2 uf = __bfloat1622float2(u2[i]);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const float g = h ? gf.y : gf.x;
                  const float u = h ? uf.y : uf.x;
                  const float dap = __uint_as_float(a[8 * qq + 2 * i + h]);
                  const float sg = sigmoidf_(g);
                  const float silu = g * sg;
                  const float A = silu * u;
                  dsum = fmaf(dap, A, dsum);
                  const float dA = s * dap;
                  dg[2 * i + h] = dA * u * sg * (1.0f + g * (1.0f - sg));
                  du[2 * i + h] = dA * silu;
                  ah[2 * i + h] = s * A;
                }
              }
              const int q16 = 2 * sub + qq;  // 16-byte unit of the 32-column staging row
              st_shared_v4(stg + sw64(lane, q16), pack8f(dg));
              st_shared_v4(stg + kStoreBuf + sw64(lane, q16), pack8f(du));
              st_shared_v4(stg + 2 * kStoreBuf + sw64(lane, q16), pack8f(ah));
            }
          }
          stage_publish();
          if (lane == 0) {
            tma_store_2d(&p.tmC0, stg, t.n0 + c0 + c, row0);
            tma_store_2d(&p.tmC0, stg + kStoreBuf, p.n + t.n0 + c0 + c, row0);
            tma_store_2d(&p.tmC1, stg + 2 * kStoreBuf, t.n0 + c0 + c, row0);
            bulk_commit();
          }
        }
        // one dS partial per (N tile, column part)
        p.outf[((size_t)r * p.num_n_tiles + t.nt) * EC::kColSplit + half] = dsum;
      } else {  // G_DWR
        const int m = t.m0 + rloc;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          uint32_t hi[32], lo[32];
          tmem_ld32(tacc + c, hi);
          tmem_ld32(tacc + 64 + c, lo);
          tc_wait_ld();
          if (m < p.d) {
            float* dst = p.outf + ((size_t)t.split * p.d + m) * p.Epad + t.nt * 64 + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
              float4 v = make_float4(__uint_as_float(hi[i]) + __uint_as_float(lo[i]),
                                     __uint_as_float(hi[i + 1]) + __uint_as_float(lo[i + 1]),
                                     __uint_as_float(hi[i + 2]) + __uint_as_float(lo[i + 2]),
                                     __uint_as_float(hi[i + 3]) + __uint_as_float(lo[i + 3]));
              *reinterpret_cast<float4*>(dst + i) = v;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&acc_empty[b]));
      if (tracer) trace_ev(p, 2, ntr, tile, 2);
      ++tcount;
    }
    if (lane == 0) bulk_wait_all();  // stores finished before the CTA exits
  } else if constexpr (KT::kGather) {
    // ---------------- gather producers (the last 4 warps): cp.async rows into the swizzled ring
    const int gt = threadIdx.x - 32 * kEpiEnd;  // 0..127
    const int chunk = gt & 7;
    const int line0 = gt >> 3;         // 0..15
    // the gathered operand's ring: A for up-proj, dH and dW1; B for dW2
    // (dW1 and dW2 share one ring with the TMA operand)
    constexpr int GS = KT::kAGather ? SA : SB;
    uint64_t* g_full = KT::kAGather ? full_a : full_b;
    uint64_t* g_empty = KT::kAGather ? empty_a : empty_b;
    int it = 0, ntr = 0;
    int pending = 0;
    bool ok = true;
    int first_tk[2][4];                    // weight-gradient kinds: row tokens of the
    int first_krow0 = -1, first_nkb = -1;  // last expert's first two k-blocks
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (gt == 0) trace_ev(p, 3, ntr, tile, 0);
      if constexpr (KIND == G_UP || KIND == G_DH || KIND == G_UPQ) {
        // A tile = 128 gathered rows x 128 bytes of K; this thread: lines
        // line0 + 16 j (MXFP8: the codes are read as pairs of bytes, so the
        // same 16-byte chunks apply; the chunk-0 threads also copy each row's
        // 4 scale bytes of the k-block into the scale tile)
        const __nv_bfloat16* src[8];
        uint32_t nbytes[8];
        int toks[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int tok = gather_tok<KIND>(p, t.m0 + line0 + 16 * j);
          toks[j] = tok;
          src[j] = p.gsrc + (size_t)(tok < 0 ? 0 : tok) * p.gld + chunk * 8;
          nbytes[j] = tok < 0 ? 0u : 16u;
        }
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % GS;
          if (!mbar_wait(smem_u32(&g_empty[s]), ((it / GS) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 5)) {
            ok = false;
            break;
          }
          const uint32_t a_s = a_slot(s);
#pragma unroll
          for (int j = 0; j < 8; ++j) cp_async_16(a_s + sw128(line0 + 16 * j, chunk), src[j] + kb * kBK, nbytes[j]);
          if constexpr (KIND == G_UPQ) {
            if (chunk == 0) {
              const uint32_t sf_s = base + SH::kSFAOffset + (uint32_t)(s * SH::kSFABytes);
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int r = line0 + 16 * j;
                const int tok = toks[j];
                const uint8_t* ssrc = p.sfa_src + (size_t)(tok < 0 ? 0 : tok) * (p.d / 32) + kb * 4;
                cp_async_4(sf_s + 16 * (r & 31) + 4 * (r >> 5), ssrc, tok < 0 ? 0u : 4u);
              }
            }
          }
          cp_async_commit();
          if (pending == kLag) {
            cp_async_wait<kLag>();
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&g_full[(it - kLag) % GS]));
          } else {
            ++pending;
          }
        }
        if (gt == 0) trace_ev(p, 3, ntr, tile, 1);
      } else {
        // MN-major gathered operand: 64 K-rows (tokens) per k-block.  The row
        // indices of the next two k-blocks are loaded ahead, so the dependent
        // index load does not sit in front of every k-block's copies.
        constexpr int nbox = (KIND == G_DW1) ? 2 : BN / 64;
        int tk[3][4];
        if (t.krow0 == first_krow0 && t.nkb == first_nkb) {
          // same expert as this warp's previous tile (an expert has many
          // tiles): its first two k-blocks' row tokens are already known
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int j = 0; j < 4; ++j) tk[q + 1][j] = first_tk[q][j];
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tk[q + 1][j] = q < t.nkb ? gather_tok<KIND>(p, t.krow0 + q * kBK + line0 + 16 * j) : -1;
              first_tk[q][j] = tk[q + 1][j];
            }
          first_krow0 = t.krow0;
          first_nkb = t.nkb;
        }
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % GS;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tk[0][j] = tk[1][j];
            tk[1][j] = tk[2][j];
          }
          if (kb + 2 < t.nkb) {
#pragma unroll
            for (int j = 0; j < 4; ++j) tk[2][j] = gather_tok<KIND>(p, t.krow0 + (kb + 2) * kBK + line0 + 16 * j);
          }
          if (!mbar_wait(smem_u32(&g_empty[s]), ((it / GS) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 6)) {
            ok = false;
            break;
          }
          const uint32_t dst0 = KT::kAGather ? a_slot(s) : b_slot(s);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i = line0 + 16 * j;
            const int tok = tk[0][j];
#pragma unroll
            for (int bx = 0; bx < nbox; ++bx) {
              const int col = (KIND == G_DW1 ? t.m0 : t.n0) + 64 * bx + chunk * 8;
              const bool valid = tok >= 0 && (KIND != G_DW1 || col < p.d);
              const __nv_bfloat16* src = p.gsrc + (valid ? ((size_t)tok * p.gld + col) : 0);
              cp_async_16(dst0 + bx * kBoxBytes + sw128(i, chunk), src, valid ? 16u : 0u);
            }
          }
          cp_async_commit();
          if (pending == kLag) {
            cp_async_wait<kLag>();
            fence_proxy_async_smem();
            mbar_arrive(smem_u32(&g_full[(it - kLag) % GS]));
          } else {
            ++pending;
          }
        }
        if (gt == 0) trace_ev(p, 3, ntr, tile, 1);
        if constexpr (kDyn) {
          // Before blocking on the queue for the next tile, publish this
          // tile's last k-blocks: a stage held back while this warp waits on
          // the queue would make the MMA wait on it while the queue, full of
          // tiles the MMA has not taken, cannot move.  When the next tile is
          // already queued nothing blocks, and the held k-blocks are
          // published as that tile's first copies go out, so the copy
          // pipeline runs on across the tile boundary.
          if (ok && pending > 0 &&
              !mbar_test_wait(smem_u32(&tq_full[(ti + 1) % kTileQ]), ((ti + 1) / kTileQ) & 1)) {
            cp_async_wait<0>();
            fence_proxy_async_smem();
            for (int k = pending; k > 0; --k) mbar_arrive(smem_u32(&g_full[(it - k) % GS]));
            pending = 0;
          }
        }
      }
    }
    // drain: the last `pending` k-blocks are complete after wait_group 0
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (ok) {
      for (int k = pending; k > 0; --k) mbar_arrive(smem_u32(&g_full[(it - k) % GS]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace moe
