// Down-projection and dX~ GEMMs with 256 x 256 output tiles on one CTA: two
// consecutive 128-row M tiles of one expert share every k-block's B tile.
//
//   DOWN  Y[rows]   = A[rows] W2[e]      K = n,  N = d   (W2 rows are K: B MN-major)
//   DXT   dX~[rows] = dH[rows] W1[e]^T   K = 2n, N = d   (W1 rows are N: B K-major)
//                   (+ dz_r Wr[:, e] per row with the router path)
//
// Every grouped GEMM of the layer fills shared memory from L2 at a rate per
// SM that its bytes in flight and the load latency set; with 128 x 256 tiles
// that rate, not the tensor core, paces the long main loops of the large
// layers: 48 KB of operands per 64-deep k-block, 85 flop per byte.  Here a
// k-block is 2 x 16 KB of A and 32 KB of B for twice the MMA work, 128 flop
// per byte, with the same shared-memory ring.  This is the operand sharing of
// a 2-CTA (cta_group::2) tile kept inside one SM, so no stage waits on a
// signal from another SM.  The price is TMEM: the two 128 x 256 fp32
// accumulators fill all 512 columns, so they are not double-buffered.  The
// epilogue drains the first half while the second half's last MMAs run, and
// the next tile's first MMAs on a half wait only for that half to drain; the
// stage ring keeps loading meanwhile.
//
// Tiles: the list p.mlist holds one entry per pair of consecutive M tiles of
// an expert, its first tile index with bit 30 set when the second tile
// exists (an expert with an odd number of M tiles ends with a single tile).
// The CTAs walk the tiles round-robin, an expert's tiles either entry-major
// (tile = entry x N tiles + N tile: neighbouring CTAs share one pair's A rows
// through L2) or, with p.wstat, N-tile-major (neighbouring CTAs share one
// weight tile, read from DRAM once).
//
// Roles:
//   warp 0 lane 0   TMA loads: A (one or two 128-row boxes) and B
//   warp 1          TMEM allocation; MMA issue (lane 0)
//   warps 2..5      epilogue: one accumulator row per thread and half, 256
//                   columns, stored through 32-row x 64-column staging boxes
// Barriers:
//   full[s]       the producer's arrive.expect_tx + the bytes
//   empty[s]      the MMA's commit
//   acc_full[h]   the MMA's commit after half h's last k-block
//   acc_empty[h]  one arrival per epilogue warp after draining half h
#pragma once
#include "gemm.cuh"

namespace moe {

template <int KIND>
struct WideMShape {
  static_assert(KIND == G_DOWN || KIND == G_DXT, "256-row tiles: down-proj and dX~");
  static constexpr int kEpi = 4;                        // epilogue warps
  static constexpr int kHalfA = kBM * kBK * 2;          // 16 KB: one 128-row A box
  static constexpr int kABytes = 2 * kHalfA;            // 32 KB
  static constexpr int kBBytes = 256 * kBK * 2;         // 32 KB
  static constexpr int kStage = kABytes + kBBytes;      // 64 KB
  static constexpr int kBoxBytesOut = 32 * 64 * 2;      // one staging box: 32 rows x 64 columns
  static constexpr int kBufs = 2;                       // staging boxes per epilogue warp
  static constexpr int kStoreBytes = kEpi * kBufs * kBoxBytesOut;
  static constexpr int kBudget = kSmemLimit - 2048 - kStoreBytes;
  static constexpr int kStagesRaw = kBudget / kStage;
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kAOffset = 0;
  static constexpr int kBOffset = kStages * kABytes;
  static constexpr int kStoreOffset = kBOffset + kStages * kBBytes;
  static constexpr int kBarOffset = kStoreOffset + kStoreBytes;
  static constexpr int kSmemBytes = kBarOffset + 1024 + 1024;  // barriers + alignment slack
  static constexpr int kThreads = 32 * (2 + kEpi);
  static constexpr int kMaxReg = max_regs_for(kThreads);
  static_assert(kStages >= 3, "wide ring depth");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

template <int KIND>
__global__ void __maxnreg__((WideMShape<KIND>::kMaxReg)) moe_gm_wide_kernel(const __grid_constant__ GemmParams p) {
  using SH = WideMShape<KIND>;
  constexpr int S = SH::kStages;
  constexpr int kEpiEnd = 2 + SH::kEpi;
  constexpr int kBufs = SH::kBufs;
  constexpr bool kBMN = (KIND == G_DOWN);
  constexpr uint32_t kIdesc = idesc_bf16_f32(256, false, kBMN);  // M = 128 per half, N = 256
  constexpr int kTmemCols = 512;                                  // half h at column 256 h

  extern __shared__ uint8_t smem_raw[];
  if (dynamic_smem_bytes() < (uint32_t)SH::kSmemBytes) {
    if (threadIdx.x == 0) raise_status(p.st, ST_DEVICE_CHECK, 0x300 + KIND);
    return;
  }
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SH::kBarOffset);
  uint64_t* full = bars;            // [S]
  uint64_t* empty = bars + 8;       // [S]
  uint64_t* acc_full = bars + 16;   // [2] per half
  uint64_t* acc_empty = bars + 18;  // [2] per half
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 20);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 21);
  auto a_slot = [&](int i) -> uint32_t { return base + SH::kAOffset + (uint32_t)(i * SH::kABytes); };
  auto b_slot = [&](int i) -> uint32_t { return base + SH::kBOffset + (uint32_t)(i * SH::kBBytes); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&acc_full[h], 1);
      mbar_init(&acc_empty[h], SH::kEpi);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.tmA);
    tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int ntn = p.num_n_tiles;  // 256-column tiles
  const int num_tiles = __ldg(p.mlist) * ntn;
  const int nkb = (KIND == G_DOWN) ? p.n / kBK : 2 * p.n / kBK;
  // tile -> (first M tile, whether the second exists, expert, N tile).  With
  // p.wstat an expert's tiles, [b, b + w) entries x N tiles, walk its entries
  // first within each N tile (each weight tile read from DRAM once).
  auto decode = [&](int tile, bool& two) -> TileInfo {
    TileInfo t;
    int j = tile / ntn;
    t.nt = tile - j * ntn;
    if (p.wstat) {
      const int e = __ldg(p.tile_expert + (__ldg(p.mlist + 1 + j) & (kWideSecond - 1)));
      const int b = __ldg(p.wbase + e);
      const int w = __ldg(p.wbase + e + 1) - b;
      const int l = tile - b * ntn;
      t.nt = l / w;
      j = b + (l - t.nt * w);
    }
    const int ent = __ldg(p.mlist + 1 + j);
    two = (ent & kWideSecond) != 0;
    t.mt = ent & (kWideSecond - 1);
    t.e = __ldg(p.tile_expert + t.mt);
    t.m0 = t.mt * kBM;
    t.n0 = t.nt * 256;
    t.krow0 = 0;
    t.nkb = nkb;
    t.split = 0;
    return t;
  };

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int it = 0, ntr = 0;
      bool ok = true;
      for (int tile = (int)blockIdx.x; tile < num_tiles && ok; tile += (int)gridDim.x) {
        bool two;
        const TileInfo t = decode(tile, two);
        trace_ev(p, 0, ntr, tile, 0);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!mbar_wait(smem_u32(&empty[s]), ((it / S) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, (uint32_t)((two ? 2 : 1) * SH::kHalfA + SH::kBBytes));
          const int k0 = kb * kBK;
          tma_load_2d(a_slot(s), &p.tmA, fb, k0, t.m0);
          if (two) tma_load_2d(a_slot(s) + SH::kHalfA, &p.tmA, fb, k0, t.m0 + kBM);
          if constexpr (KIND == G_DOWN) {  // W2[e] rows k0.., columns n0 + [0, 256): four 64-column boxes
#pragma unroll
            for (int j = 0; j < 4; ++j) tma_load_2d(b_slot(s) + j * kBoxBytes, &p.tmB, fb, t.n0 + 64 * j, t.e * p.n + k0);
          } else {  // W1[e] rows n0 + [0, 256) (the N index), K columns k0..
            tma_load_2d(b_slot(s), &p.tmB, fb, k0, t.e * p.d + t.n0);
          }
          if (tile == (int)blockIdx.x) trace_ev(p, 0, ntr, kb, 16);  // first tile: each k-block's issue
        }
        trace_ev(p, 0, ntr, tile, 1);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: per k-block, half 0's MMAs, then half 1's
    // with the same B descriptors.  Half 0's accumulator is committed ahead
    // of half 1's last MMAs so that its drain starts early.
    int it = 0, u0 = 0, u1 = 0, ntr = 0;
    bool ok = true;
    for (int tile = (int)blockIdx.x; tile < num_tiles && ok; tile += (int)gridDim.x) {
      bool two;
      const TileInfo t = decode(tile, two);
      if (lane == 0) trace_ev(p, 1, ntr, tile, 0);
      for (int kb = 0; kb < t.nkb; ++kb, ++it) {
        const int s = it % S;
        if (!mbar_wait(smem_u32(&full[s]), (it / S) & 1, abort_flag, p.st, KIND * 16 + 3)) {
          ok = false;
          break;
        }
        if (kb == 0) {  // half 0's accumulator drained by the previous tile's epilogue
          if (!mbar_wait(smem_u32(&acc_empty[0]), (u0 & 1) ^ 1, abort_flag, p.st, KIND * 16 + 2)) {
            ok = false;
            break;
          }
          if (lane == 0) trace_ev(p, 1, ntr, tile, 1);
        }
        tc_fence_after();
        if (kb == 0 && lane == 0) trace_ev(p, 1, ntr, tile, 2);
        if (tile == (int)blockIdx.x && lane == 0) trace_ev(p, 1, ntr, kb, 16);  // first tile: operands ready
        const uint32_t a_s = a_slot(s);
        const uint32_t b_s = b_slot(s);
        auto bdesc = [&](int kk) -> uint64_t {
          return kBMN ? smem_desc_sw128(b_s + kk * 2048, kBoxBytes, 1024) : smem_desc_sw128(b_s + kk * 32, 16, 1024);
        };
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_bf16(tmem_base, smem_desc_sw128(a_s + kk * 32, 16, 1024), bdesc(kk), kIdesc,
                        (kb > 0 || kk > 0) ? 1u : 0u);
          if (kb == t.nkb - 1) tc_commit(smem_u32(&acc_full[0]));
        }
        __syncwarp();
        if (two) {
          if (kb == 0) {
            if (!mbar_wait(smem_u32(&acc_empty[1]), (u1 & 1) ^ 1, abort_flag, p.st, KIND * 16 + 5)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              tc_mma_bf16(tmem_base + 256u, smem_desc_sw128(a_s + SH::kHalfA + kk * 32, 16, 1024), bdesc(kk),
                          kIdesc, (kb > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (lane == 0) {
          tc_commit(smem_u32(&empty[s]));
          if (two && kb == t.nkb - 1) tc_commit(smem_u32(&acc_full[1]));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) trace_ev(p, 1, ntr, tile, 3);
      ++u0;
      if (two) ++u1;
    }
  } else if (warp < kEpiEnd) {
    // ---------------- epilogue: TMEM lane quarter q of each half
    const int q = warp & 3;
    const int ew = warp - 2;
    const uint32_t lane_addr = tmem_base + ((uint32_t)(q * 32) << 16);
    const uint32_t stg = base + SH::kStoreOffset + ew * (kBufs * SH::kBoxBytesOut);
    int ring = 0, u0 = 0, u1 = 0, ntr = 0;
    const bool tracer = (warp == 2 && lane == 0);
    bool ok = true;
    for (int tile = (int)blockIdx.x; tile < num_tiles && ok; tile += (int)gridDim.x) {
      bool two;
      const TileInfo t = decode(tile, two);
      if (tracer) trace_ev(p, 2, ntr, tile, 0);
      const float4* rv = nullptr;  // dX~ router path: row e of Wr^T, the same for every row
      if constexpr (KIND == G_DXT) {
        if (p.rvec) rv = reinterpret_cast<const float4*>(p.rvec + (size_t)t.e * p.d + t.n0);
      }
      for (int h = 0; h < (two ? 2 : 1); ++h) {
        const int row0 = t.m0 + h * kBM + q * 32;  // first output row of this warp's slice
        float rz = 0.f;
        if constexpr (KIND == G_DXT) {
          if (rv) {
            const int r = row0 + lane;
            rz = __ldg(p.row_tok + r) >= 0 ? __ldg(p.rscale + r) : 0.f;
          }
        }
        const int use = h == 0 ? u0 : u1;
        if (!mbar_wait(smem_u32(&acc_full[h]), use & 1, abort_flag, p.st, KIND * 16 + 4)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (tracer && h == 0) trace_ev(p, 2, ntr, tile, 1);
        const uint32_t tacc = lane_addr + (uint32_t)(h * 256);
#pragma unroll 1
        for (int c = 0; c < 256; c += 64) {
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
        if (lane == 0) mbar_arrive(smem_u32(&acc_empty[h]));
      }
      if (!ok) break;
      if (tracer) trace_ev(p, 2, ntr, tile, 2);
      ++u0;
      if (two) ++u1;
    }
    if (lane == 0) bulk_wait_all();  // stores finished before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace moe
