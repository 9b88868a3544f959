// Down-projection and dX~ GEMMs on CTA pairs: one 256 x 256 output tile --
// two 128-row M tiles of one expert by 256 columns -- per pair of CTAs (a
// 2-CTA cluster), the MMAs issued by the pair's first CTA with cta_group::2.
//
//   DOWN  Y[rows]   = A[rows] W2[e]      K = n,  N = d   (W2 rows are K: B MN-major)
//   DXT   dX~[rows] = dH[rows] W1[e]^T   K = 2n, N = d   (W1 rows are N: B K-major)
//                   (+ dz_r Wr[:, e] per row with the router path)
//
// Every grouped GEMM of the layer fills shared memory from L2 at a fixed rate
// per SM, and with 128 x 256 tiles on one CTA that rate, not the tensor core,
// sets the pace: 48 KB of operands per 64-deep k-block.  In a pair each CTA
// loads its own 128 rows of A and half of B's 256 columns, 32 KB per k-block
// for the same MMA work per CTA.  Page "DeepSeek做大→Mega MoE，Tri Dao团队加快→
// SonicMoE", section "实验结果", credits the Blackwell grouped GEMM's 2-CTA MMA
// for part of the method's speed-up.
//
// Both operands come by TMA, so no stage needs forwarding: each CTA's loads
// complete on the first CTA's full barrier (the cta_group::2 form of the
// tensor load), whose single arrival -- the first CTA's producer, expecting
// both CTAs' bytes -- opens the stage to the MMA.  No load multicasts: each
// CTA reads its own operand halves from global memory.
//
// Tiles: the pair list p.mlist holds the first 128-row tile of every pair of
// consecutive M tiles of one expert; an expert with an odd number of M tiles
// leaves its last one to moe_gemm_kernel (a second launch over the list of
// leftover tiles).  Pair tile j = (list entry j / N tiles, N tile), taken
// round-robin by the pairs, the same sequence in both CTAs.
//
// Roles (both CTAs):
//   warp 0 lane 0   TMA loads of this CTA's halves of A and B
//   warp 1          TMEM allocation (both CTAs); MMA issue (first CTA)
//   warps 2..2+EPI  epilogue: this CTA's 128 accumulator rows, 256 columns,
//                   stored through 32-row x 64-column staging boxes
// Every wait is a CTA-scope wait on the waiting CTA's own barrier, as the
// tensor-core pipeline needs no more: the stage's data is written by TMA and
// read by the MMA (both async-proxy operations ordered by the transaction
// count), and the accumulator hand-offs are ordered by the tcgen05 fences
// around them.
// Barriers:
//   full[s]      first CTA's: one arrival (with both CTAs' bytes) + the bytes
//   empty[s]     both CTAs': the MMA's commit (two commits, one per CTA)
//   acc_full[b]  both CTAs': the MMA's commit at the end of a tile
//   acc_empty[b] first CTA's: one arrival per epilogue warp of both CTAs
#pragma once
#include "gemm.cuh"

namespace moe {

template <int KIND, int EPI>
struct PairMShape {
  static_assert(KIND == G_DOWN || KIND == G_DXT, "pair tiles over M: down-proj and dX~");
  static constexpr int kHalf = 128;                // rows of A and columns of B per CTA
  static constexpr int kABytes = kHalf * kBK * 2;  // 16 KB
  static constexpr int kBBytes = kHalf * kBK * 2;  // 16 KB
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kBoxBytesOut = 32 * 64 * 2;  // one staging box: 32 rows x 64 columns
  static constexpr int kBufs = 2;
  static constexpr int kStoreBytes = EPI * kBufs * kBoxBytesOut;
  static constexpr int kBudget = (kSmemLimit - 2048 - kStoreBytes) < 200 * 1024 ? (kSmemLimit - 2048 - kStoreBytes)
                                                                                   : 200 * 1024;
  static constexpr int kStagesRaw = kBudget / kStage;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kAOffset = 0;
  static constexpr int kBOffset = kStages * kABytes;
  static constexpr int kStoreOffset = kBOffset + kStages * kBBytes;
  static constexpr int kBarOffset = kStoreOffset + kStoreBytes;
  static constexpr int kSmemBytes = kBarOffset + 1024 + 1024;
  static constexpr int kThreads = 32 * (2 + EPI);
  static constexpr int kMaxReg = max_regs_for(kThreads);
  static_assert(kStages >= 4, "pair ring depth");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

template <int KIND, int EPI>
__global__ void __maxnreg__((PairMShape<KIND, EPI>::kMaxReg)) __cluster_dims__(2, 1, 1)
    moe_gm_pair_kernel(const __grid_constant__ GemmParams p) {
  using SH = PairMShape<KIND, EPI>;
  constexpr int S = SH::kStages;
  constexpr int kEpiEnd = 2 + EPI;
  constexpr int kColSplit = EPI / 4;
  constexpr int kBufs = SH::kBufs;
  constexpr bool kBMN = (KIND == G_DOWN);
  // M = 256 over the pair, N = 256; A K-major
  constexpr uint32_t kIdesc = idesc_bf16_f32(256, false, kBMN, 256);
  constexpr int kAccStride = 256;
  constexpr int kTmemCols = 512;

  extern __shared__ uint8_t smem_raw[];
  if (dynamic_smem_bytes() < (uint32_t)SH::kSmemBytes) {  // both CTAs of the pair leave alike
    if (threadIdx.x == 0) raise_status(p.st, ST_DEVICE_CHECK, 0x300 + KIND);
    return;
  }
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  const uint32_t rank = cluster_ctarank();  // 0: the pair's first CTA
  const bool lead = rank == 0;
  const int pair = (int)blockIdx.x >> 1;
  const int npairs = (int)gridDim.x >> 1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::kBarOffset);
  uint64_t* full = bars;            // [S]   (the first CTA's are the ones used)
  uint64_t* empty = bars + 8;       // [S]
  uint64_t* acc_full = bars + 16;   // [2]
  uint64_t* acc_empty = bars + 18;  // [2]   (the first CTA's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 21);
  auto a_slot = [&](int i) -> uint32_t { return base + SH::kAOffset + (uint32_t)(i * SH::kABytes); };
  auto b_slot = [&](int i) -> uint32_t { return base + SH::kBOffset + (uint32_t)(i * SH::kBBytes); };
  auto lead_bar = [&](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 0); };
  auto peer_bar = [&](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 1); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);   // the first CTA's producer (arrive + expect both CTAs' bytes)
      mbar_init(&empty[s], 1);  // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI);  // one arrive per epilogue warp of both CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any remote arrive or load
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int ntn = p.num_n_tiles;  // 256-column tiles
  const int num_tiles = __ldg(p.mlist) * ntn;
  const int nkb = (KIND == G_DOWN) ? p.n / kBK : 2 * p.n / kBK;
  auto decode = [&](int tile) -> TileInfo {
    TileInfo t;
    const int j = tile / ntn;
    t.nt = tile - j * ntn;
    t.mt = __ldg(p.mlist + 1 + j);
    t.e = __ldg(p.tile_expert + t.mt);
    t.m0 = t.mt * kBM;  // the pair's first row; this CTA's rows start at m0 + half0
    t.n0 = t.nt * 256;
    t.krow0 = 0;
    t.nkb = nkb;
    t.split = 0;
    return t;
  };
  const int half0 = (int)rank * SH::kHalf;

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs): this CTA's 128 rows of A and
    // 128 of B's 256 columns; completion counted on the first CTA's full[s]
    if (lane == 0) {
      int it = 0, ntr = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const TileInfo t = decode(tile);
        trace_ev(p, 0, ntr, tile, 0);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(smem_u32(&empty[s]), ((it / S) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = lead_bar(&full[s]);
          if (lead) mbar_arrive_expect_tx(smem_u32(&full[s]), 2u * SH::kStage);
          const int k0 = kb * kBK;
          tma_load_2d_pair(a_slot(s), &p.tmA, fb, k0, t.m0 + half0);
          if constexpr (KIND == G_DOWN) {  // W2[e] rows k0.., columns n0 + half0 + [0, 128): two 64-column boxes
            tma_load_2d_pair(b_slot(s), &p.tmB, fb, t.n0 + half0, t.e * p.n + k0);
            tma_load_2d_pair(b_slot(s) + kBoxBytes, &p.tmB, fb, t.n0 + half0 + 64, t.e * p.n + k0);
          } else {  // W1[e] rows n0 + half0 + [0, 128) (the N index), K columns k0..
            tma_load_2d_pair(b_slot(s), &p.tmB, fb, k0, t.e * p.d + t.n0 + half0);
          }
          if (tile == pair) trace_ev(p, 0, ntr, kb, 16);  // first tile: each k-block's issue
        }
        trace_ev(p, 0, ntr, tile, 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (first CTA only)
    if (lead) {
      int it = 0, tcount = 0, ntr = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
        const TileInfo t = decode(tile);
        if (lane == 0) trace_ev(p, 1, ntr, tile, 0);
        const int b = tcount & 1;
        const int use = tcount >> 1;
        if (!mbar_wait(smem_u32(&acc_empty[b]), (use & 1) ^ 1, abort_flag, p.st, KIND * 16 + 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) trace_ev(p, 1, ntr, tile, 1);
        const uint32_t d_tmem = tmem_base + (uint32_t)(b * kAccStride);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(smem_u32(&full[s]), (it / S) & 1, abort_flag, p.st, KIND * 16 + 3)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (kb == 0 && lane == 0) trace_ev(p, 1, ntr, tile, 2);
          if (tile == pair && lane == 0) trace_ev(p, 1, ntr, kb, 16);  // first tile: each k-block's operands ready
          if (lane == 0) {
            const uint32_t a_s = a_slot(s);
            const uint32_t b_s = b_slot(s);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(a_s + kk * 32, 16, 1024);
              const uint64_t bd = kBMN ? smem_desc_sw128(b_s + kk * 2048, kBoxBytes, 1024)
                                       : smem_desc_sw128(b_s + kk * 32, 16, 1024);
              tc_mma_bf16_pair(d_tmem, ad, bd, kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit_pair(smem_u32(&empty[s]));
            tc_commit_pair(peer_bar(&empty[s]));
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) {
          tc_commit_pair(smem_u32(&acc_full[b]));
          tc_commit_pair(peer_bar(&acc_full[b]));
          trace_ev(p, 1, ntr, tile, 3);
        }
        __syncwarp();
        ++tcount;
      }
    }
  } else if (warp < kEpiEnd) {
    // ---------------- epilogue: this CTA's 128 accumulator rows, 256 columns
    const int q = warp & 3;
    const int ew = warp - 2;
    const int part = ew >> 2;  // column part of this warp (kColSplit parts)
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t stg = base + SH::kStoreOffset + ew * (kBufs * SH::kBoxBytesOut);
    constexpr int kCols = 256 / kColSplit;
    int ring = 0, tcount = 0, ntr = 0;
    const bool tracer = (warp == 2 && lane == 0);
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
      const TileInfo t = decode(tile);
      if (tracer) trace_ev(p, 2, ntr, tile, 0);
      const int row0 = t.m0 + half0 + q * 32;  // first output row of this warp's slice
      const int r = row0 + lane;
      // dX~ router path: dz of this row and row e of Wr^T (the same for every
      // row of the tile), loaded while the MMAs run
      float rz = 0.f;
      const float4* rv = nullptr;
      if constexpr (KIND == G_DXT) {
        if (p.rvec) {
          rz = __ldg(p.row_tok + r) >= 0 ? __ldg(p.rscale + r) : 0.f;
          rv = reinterpret_cast<const float4*>(p.rvec + (size_t)t.e * p.d + t.n0);
        }
      }
      const int b = tcount & 1;
      const int use = tcount >> 1;
      if (!mbar_wait(smem_u32(&acc_full[b]), use & 1, abort_flag, p.st, KIND * 16 + 4)) break;
      tc_fence_after();
      if (tracer) trace_ev(p, 2, ntr, tile, 1);
      const uint32_t tacc = lane_addr + (uint32_t)(b * kAccStride);
      const int c0 = part * kCols;
#pragma unroll 1
      for (int c = c0; c < c0 + kCols; c += 64) {
        uint32_t a[32], a2[32];
        tmem_ld32(tacc + c, a);
        tmem_ld32(tacc + c + 32, a2);
        float4 r_cur[16];
        if constexpr (KIND == G_DXT) {
          if (rv) {
#pragma unroll
            for (int i = 0; i < 16; ++i) r_cur[i] = __ldg(rv + c / 4 + i);
          }
        }
        tc_wait_ld();
        const uint32_t buf = stg + ring * SH::kBoxBytesOut;
        if (lane == 0) bulk_wait_read<kBufs - 1>();
        __syncwarp();
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
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmC0, buf, t.n0 + c, row0);
          bulk_commit();
        }
        ring = ring + 1 == kBufs ? 0 : ring + 1;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(lead_bar(&acc_empty[b]));
      if (tracer) trace_ev(p, 2, ntr, tile, 2);
      ++tcount;
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still read its shared memory or arrive on its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
