// Weight-gradient GEMMs (dW1, dW2) on CTA pairs: one 256 x 256 output tile
// per pair of CTAs (a 2-CTA cluster), the MMAs issued by the pair's first
// CTA with cta_group::2.
//
//   DW1  dW1[e] = X[tok]^T dH    M = d rows, N = 2n columns, K = rows of e
//   DW2  dW2[e] = A_hat^T dO[tok] M = n rows, N = d columns, K = rows of e
//
// Why pairs: every grouped GEMM of the layer streams its operands from L2
// into shared memory at a fixed rate per SM, and with 128 x 256 tiles on one
// CTA that rate, not the tensor core, sets the pace (48 KB of operands per
// 64-deep k-block).  In a pair, each CTA loads its own 128 rows of A and only
// half of B's 256 columns -- 32 KB per k-block for the same MMA work per CTA.
// Page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", section "实验结果",
// credits the Blackwell grouped GEMM's 2-CTA MMA (with its tile scheduler)
// for part of the speed-up.  No load here multicasts: each CTA loads its own
// operand halves from global memory.
//
// Roles (both CTAs, same warp layout as moe_gemm_kernel):
//   warp 0 lane 0   TMA loads of this CTA's half of the TMA operand; in the
//                   first CTA also the tile claims (one queue for the pair)
//   warp 1          TMEM allocation (both CTAs); MMA issue (first CTA); in
//                   the second CTA, lane 0 forwards each stage once it is
//                   complete there to the first CTA's full barrier
//   warps 2..2+EPI  epilogue: this CTA's 128 accumulator rows (p.tmC1: a store
//                   map of 32-row x 64-column boxes with the 128-byte swizzle)
//   last 4 warps    cp.async gather of this CTA's half of the gathered operand
// Each CTA fills its own stage and completes its own full[s] (its TMA bytes +
// its 128 gather threads, as in moe_gemm_kernel).  The forwarding thread has
// no copies in flight, so its cluster-scope release (which waits for the
// issuing thread's outstanding memory operations) costs nothing; a gather
// thread releasing at cluster scope itself would wait for its next k-block's
// copies each time and serialise the copy pipeline.
// Barriers that pair members arrive on remotely live in the first CTA:
//   full[s]      (also) the second CTA's forwarded stage
//   acc_empty[b] the epilogue warps of both CTAs
//   tq_empty[q]  every queue consumer of both CTAs
// Barriers the first CTA's MMA thread completes in both CTAs (two commits):
//   empty[s], acc_full[b]; the tile queue's tq_full[q] is arrived on in both
//   CTAs by the first CTA's producer, which also writes both queues.
#pragma once
#include "gemm.cuh"

namespace moe {

template <int KIND, int EPI>
struct PairShape {
  static_assert(KIND == G_DW1 || KIND == G_DW2, "pair kernel: weight-gradient kinds");
  static constexpr int kHalf = 128;                  // rows of A and columns of B per CTA
  static constexpr int kABytes = kHalf * kBK * 2;    // 16 KB: two 64 x 64 MN-major boxes
  static constexpr int kBBytes = kHalf * kBK * 2;    // 16 KB
  static constexpr int kStage = kABytes + kBBytes;
  // Epilogue staging: per warp, kBufs boxes of 32 rows x 64 columns (4 KB,
  // 128-byte swizzle), each leaving as one TMA store of whole 128-byte row
  // segments (a 32-column box writes half-lines, twice the store requests).
  static constexpr int kBoxBytesOut = 32 * 64 * 2;
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
  static constexpr int kThreads = 32 * (2 + EPI + 4);
  static constexpr int kMaxReg = max_regs_for(kThreads);
  static_assert(kStages >= 3, "pair ring depth");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
};

// POLL: the waits whose last arrival crosses the pair (the MMA's wait for a
// forwarded stage, the second CTA's waits for the MMA's commits and the
// forwarder's wait) poll instead of suspending.
template <int KIND, int EPI, bool POLL>
__global__ void __maxnreg__((PairShape<KIND, EPI>::kMaxReg)) __cluster_dims__(2, 1, 1)
    moe_dw_pair_kernel(const __grid_constant__ GemmParams p) {
  using SH = PairShape<KIND, EPI>;
  constexpr int S = SH::kStages;
  constexpr int kEpiEnd = 2 + EPI;
  constexpr int kColSplit = EPI / 4;
  constexpr int kBufs = SH::kBufs;
  // M = 256 over the pair, N = 256, both operands MN-major
  constexpr uint32_t kIdesc = idesc_bf16_f32(256, true, true, 256);
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
  uint64_t* full = bars;           // [S]   (first CTA's are the ones used)
  uint64_t* empty = bars + 8;      // [S]
  uint64_t* acc_full = bars + 16;  // [2]
  uint64_t* acc_empty = bars + 18; // [2]   (first CTA's)
  uint64_t* tq_full = bars + 20;   // [kTileQ]
  uint64_t* tq_empty = bars + 24;  // [kTileQ] (first CTA's)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 29);
  int4* tq_info = reinterpret_cast<int4*>(bars + 30);  // [kTileQ]
  auto a_slot = [&](int i) -> uint32_t { return base + SH::kAOffset + (uint32_t)(i * SH::kABytes); };
  auto b_slot = [&](int i) -> uint32_t { return base + SH::kBOffset + (uint32_t)(i * SH::kBBytes); };
  // the first CTA's copy of a barrier (a shared::cluster address)
  auto lead_bar = [&](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 0); };
  auto peer_bar = [&](uint64_t* b) -> uint32_t { return mapa_shared(smem_u32(b), 1); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  auto xwait = [&](uint32_t bar, uint32_t parity, int where) -> bool {
    return POLL ? mbar_poll(bar, parity, abort_flag, p.st, where) : mbar_wait(bar, parity, abort_flag, p.st, where);
  };
  // queue consumers: the first CTA's MMA warp, epilogue and gather warps; the
  // second CTA's producer, forwarder, epilogue and gather warps
  constexpr int kQConsumers = (1 + EPI + 4) + (2 + EPI + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // own producer (expect_tx of own TMA bytes) + 128 own gather threads,
      // + in the first CTA the second CTA's forwarded stage
      mbar_init(&full[s], 1 + 128 + (lead ? 1 : 0));
      mbar_init(&empty[s], 1);  // the MMA commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI);  // one arrive per epilogue warp of both CTAs
    }
    for (int b = 0; b < kTileQ; ++b) {
      mbar_init(&tq_full[b], 1);
      mbar_init(&tq_empty[b], kQConsumers);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (KIND == G_DW2) tma_prefetch_desc(&p.tmA);
    else tma_prefetch_desc(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();

  const int mt_count = p.num_m_tiles;  // 256-row tiles
  const int nt_count = p.num_n_tiles;  // 256-column tiles
  const int per_e = mt_count * nt_count;
  const int num_tiles = p.E * per_e;

  // Tile claims (first CTA's producer), as in moe_gemm_kernel with
  // dual_ended = 1 (any nonzero mode here): pairs of even index from the
  // largest experts' end of the order, odd pairs from the smallest experts' end.
  const bool front_end = !p.dual_ended || (pair & 1) == 0;
  const int nfront0 = p.dual_ended ? (npairs + 1) / 2 : npairs;
  const int nback0 = npairs - nfront0;
  auto decode = [&](int tile, int e, int krow0, int nkb) -> TileInfo {
    TileInfo t;
    const int rem = tile - (tile / per_e) * per_e;
    t.e = e;
    t.mt = rem / nt_count;
    t.nt = rem - t.mt * nt_count;
    t.m0 = t.mt * 256;
    t.n0 = t.nt * 256;
    t.krow0 = krow0;
    t.nkb = nkb;
    t.split = 0;
    return t;
  };
  // consume the pair's queue (every role but the first CTA's producer); a
  // whole warp calls it, except the second CTA's producer (its lane 0 alone)
  auto consume_tile = [&](int i, bool& good, TileInfo& t, bool whole_warp = true) -> int {
    const int slot = i % kTileQ;
    if (!mbar_wait_cl(smem_u32(&tq_full[slot]), (i / kTileQ) & 1, abort_flag, p.st, KIND * 16 + 11)) {
      good = false;
      return num_tiles;
    }
    const int4 q = tq_info[slot];
    if (whole_warp) __syncwarp();
    if (lane == 0) mbar_arrive_remote(lead_bar(&tq_empty[slot]));
    if (q.x < num_tiles) t = decode(q.x, q.y, q.z, q.w);
    return q.x;
  };
  // this CTA's half: rows of A (its M offset) and columns of B (its N offset)
  const int half0 = (int)rank * SH::kHalf;

  if (warp == 0) {
    // ---------------- TMA producer (and, in the first CTA, the tile claims)
    if (lane == 0) {
      const void* tm = (KIND == G_DW2) ? static_cast<const void*>(&p.tmA) : static_cast<const void*>(&p.tmB);
      const uint32_t tma_dst0 = (KIND == G_DW2) ? a_slot(0) : b_slot(0);
      const uint32_t tma_step = (KIND == G_DW2) ? (uint32_t)SH::kABytes : (uint32_t)SH::kBBytes;
      int it = 0, ntr = 0;
      bool ok = true;
      unsigned long long next_claim = 0;
      int res_ei = -1, res_e = 0, res_krow0 = 0, res_nkb = 0;
      for (int ti = 0; ok; ++ti) {
        TileInfo t;
        int tile;
        if (lead) {
          if (ti == 0) {
            const int j = p.dual_ended ? (pair >> 1) : pair;
            tile = front_end ? j : num_tiles - 1 - j;
          } else {
            const int f = (int)(next_claim & 0xffffffffull) + nfront0;
            const int b = (int)(next_claim >> 32) + nback0;
            tile = (f + b >= num_tiles) ? num_tiles : (front_end ? f : num_tiles - 1 - b);
          }
          if (tile < num_tiles)
            next_claim = atomicAdd(reinterpret_cast<unsigned long long*>(p.sched), front_end ? 1ull : (1ull << 32));
          int e = 0, krow0 = 0, nkb = 0;
          if (tile < num_tiles) {
            const int ei = tile / per_e;
            if (ei != res_ei) {
              res_ei = ei;
              res_e = p.expert_order ? __ldg(p.expert_order + ei) : ei;
              res_krow0 = __ldg(p.offsets + res_e);
              res_nkb = (__ldg(p.counts + res_e) + kBK - 1) / kBK;
            }
            e = res_e;
            krow0 = res_krow0;
            nkb = res_nkb;
            t = decode(tile, e, krow0, nkb);
          }
          const int slot = ti % kTileQ;
          if (!mbar_wait_cl(smem_u32(&tq_empty[slot]), ((ti / kTileQ) & 1) ^ 1, abort_flag, p.st, KIND * 16 + 10)) {
            ok = false;
            break;
          }
          const int4 q = make_int4(tile, e, krow0, nkb);
          tq_info[slot] = q;
          st_cluster_v4(mapa_shared(smem_u32(&tq_info[slot]), 1), q);
          mbar_arrive(smem_u32(&tq_full[slot]));
          mbar_arrive_cluster(peer_bar(&tq_full[slot]));
        } else {
          tile = consume_tile(ti, ok, t, false);
        }
        if (!ok || tile >= num_tiles) break;
        trace_ev(p, 0, ntr, tile, 0);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!xwait(smem_u32(&empty[s]), ((it / S) & 1) ^ 1, KIND * 16 + 1)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(&full[s]);
          mbar_arrive_expect_tx(fb, (uint32_t)tma_step);  // this CTA's TMA bytes
          const uint32_t dst = tma_dst0 + (uint32_t)s * tma_step;
          const int krow = t.krow0 + kb * kBK;
          const int col = ((KIND == G_DW2) ? t.m0 : t.n0) + half0;
          tma_load_2d(dst, tm, fb, col, krow);
          tma_load_2d(dst + kBoxBytes, tm, fb, col + 64, krow);
          if (ti == 0) trace_ev(p, 0, ntr, kb, 16);  // first tile: each k-block's issue
        }
        trace_ev(p, 0, ntr, tile, 1);
      }
    }
  } else if (warp == 1 && !lead) {
    // ---------------- forwarder (second CTA): each stage, once complete here
    // (this CTA's TMA bytes and gather copies), is signalled on the first
    // CTA's full barrier
    if (lane == 0) {
      int it = 0, ntr = 0;
      bool ok = true;
      for (int ti = 0; ok; ++ti) {
        TileInfo t;
        const int tile = consume_tile(ti, ok, t, false);
        if (!ok || tile >= num_tiles) break;
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!xwait(smem_u32(&full[s]), (it / S) & 1, KIND * 16 + 14)) {
            ok = false;
            break;
          }
          mbar_arrive_cluster(lead_bar(&full[s]));
          if (ti == 0) trace_ev(p, 1, ntr, kb, 16);  // first tile: stage complete here, forwarded
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (first CTA only)
    {
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
        if (!mbar_wait_cl(smem_u32(&acc_empty[b]), (use & 1) ^ 1, abort_flag, p.st, KIND * 16 + 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) trace_ev(p, 1, ntr, tile, 1);
        const uint32_t d_tmem = tmem_base + (uint32_t)(b * kAccStride);
        for (int kb = 0; kb < t.nkb; ++kb, ++it) {
          const int s = it % S;
          if (!(POLL ? mbar_poll(smem_u32(&full[s]), (it / S) & 1, abort_flag, p.st, KIND * 16 + 3)
                     : mbar_wait_cl(smem_u32(&full[s]), (it / S) & 1, abort_flag, p.st, KIND * 16 + 3))) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (kb == 0 && lane == 0) trace_ev(p, 1, ntr, tile, 2);
          if (ti == 0 && lane == 0) trace_ev(p, 1, ntr, kb, 16);  // first tile: each k-block's operands ready
          if (lane == 0) {
            const uint32_t a_s = a_slot(s);
            const uint32_t b_s = b_slot(s);
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(a_s + kk * 2048, kBoxBytes, 1024);
              const uint64_t bd = smem_desc_sw128(b_s + kk * 2048, kBoxBytes, 1024);
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
    const int M = (KIND == G_DW1) ? p.d : p.n;
    constexpr int kCols = 256 / kColSplit;
    int ring = 0, tcount = 0, ntr = 0;
    const bool tracer = (warp == 2 && lane == 0);
    bool ok = true;
    auto stage_wait = [&]() {
      if (lane == 0) bulk_wait_read<kBufs - 1>();
      __syncwarp();
    };
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (tracer) trace_ev(p, 2, ntr, tile, 0);
      const int row0 = t.m0 + half0 + q * 32;  // first output row of this warp's slice
      const int orow = t.e * M + row0;
      const int c0 = part * kCols;
      if (t.nkb == 0) {  // expert without tokens: its weight gradient is zero
        const uint32_t buf = stg + ring * SH::kBoxBytesOut;
        stage_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j) st_shared_v4(buf + sw128(lane, j), make_uint4(0u, 0u, 0u, 0u));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int c = c0; c < c0 + kCols; c += 64) tma_store_2d(&p.tmC1, buf, t.n0 + c, orow);
          bulk_commit();
        }
        ring = ring + 1 == kBufs ? 0 : ring + 1;
        continue;
      }
      const int b = tcount & 1;
      const int use = tcount >> 1;
      if (!mbar_wait(smem_u32(&acc_full[b]), use & 1, abort_flag, p.st, KIND * 16 + 4)) break;
      tc_fence_after();
      if (tracer) trace_ev(p, 2, ntr, tile, 1);
      const uint32_t tacc = lane_addr + (uint32_t)(b * kAccStride);
#pragma unroll 1
      for (int c = c0; c < c0 + kCols; c += 64) {
        uint32_t a[32], a2[32];
        tmem_ld32(tacc + c, a);
        tmem_ld32(tacc + c + 32, a2);
        tc_wait_ld();
        const uint32_t buf = stg + ring * SH::kBoxBytesOut;
        stage_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[8], w[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[i] = __uint_as_float(a[8 * j + i]);
            w[i] = __uint_as_float(a2[8 * j + i]);
          }
          st_shared_v4(buf + sw128(lane, j), pack8f(v));
          st_shared_v4(buf + sw128(lane, 4 + j), pack8f(w));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&p.tmC1, buf, t.n0 + c, orow);
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
  } else {
    // ---------------- gather warps: this CTA's half of the gathered operand
    // (DW1: A = X columns [m0 + half0, +128); DW2: B = dO columns
    // [n0 + half0, +128)) for 64 routed rows per k-block, cp.async into the
    // 128B-swizzled MN-major layout TMA would produce; each thread publishes
    // its k-blocks on this CTA's full barrier one k-block after issuing them.
    const int gt = threadIdx.x - 32 * kEpiEnd;  // 0..127
    const int chunk = gt & 7;
    const int line0 = gt >> 3;  // 0..15
    constexpr int kLag = 1;
    int it = 0, ntr = 0, pending = 0;
    bool ok = true;
    int first_tk[2][4];
    int first_krow0 = -1, first_nkb = -1;
    auto publish = [&](int k_it) {  // k-block k_it of this thread's copies is complete
      fence_proxy_async_smem();
      mbar_arrive(smem_u32(&full[k_it % S]));
    };
    for (int ti = 0; ok; ++ti) {
      TileInfo t;
      const int tile = consume_tile(ti, ok, t);
      if (!ok || tile >= num_tiles) break;
      if (gt == 0) trace_ev(p, 3, ntr, tile, 0);
      int tk[3][4];
      if (t.krow0 == first_krow0 && t.nkb == first_nkb) {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq)
#pragma unroll
          for (int j = 0; j < 4; ++j) tk[qq + 1][j] = first_tk[qq][j];
      } else {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tk[qq + 1][j] = qq < t.nkb ? gather_tok<KIND>(p, t.krow0 + qq * kBK + line0 + 16 * j) : -1;
            first_tk[qq][j] = tk[qq + 1][j];
          }
        first_krow0 = t.krow0;
        first_nkb = t.nkb;
      }
      const int colbase = ((KIND == G_DW1) ? t.m0 : t.n0) + half0;
      for (int kb = 0; kb < t.nkb; ++kb, ++it) {
        const int s = it % S;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          tk[0][j] = tk[1][j];
          tk[1][j] = tk[2][j];
        }
        if (kb + 2 < t.nkb) {
#pragma unroll
          for (int j = 0; j < 4; ++j) tk[2][j] = gather_tok<KIND>(p, t.krow0 + (kb + 2) * kBK + line0 + 16 * j);
        }
        if (!xwait(smem_u32(&empty[s]), ((it / S) & 1) ^ 1, KIND * 16 + 6)) {
          ok = false;
          break;
        }
        const uint32_t dst0 = (KIND == G_DW1) ? a_slot(s) : b_slot(s);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = line0 + 16 * j;
          const int tok = tk[0][j];
#pragma unroll
          for (int bx = 0; bx < 2; ++bx) {
            const int col = colbase + 64 * bx + chunk * 8;
            const bool valid = tok >= 0;
            const __nv_bfloat16* src = p.gsrc + (valid ? ((size_t)tok * p.gld + col) : 0);
            cp_async_16(dst0 + bx * kBoxBytes + sw128(i, chunk), src, valid ? 16u : 0u);
          }
        }
        cp_async_commit();
        if (ti == 0 && gt == 0) trace_ev(p, 3, ntr, kb, 16);  // first tile: each k-block's copies issued
        if (pending == kLag) {
          cp_async_wait<kLag>();
          publish(it - kLag);
          if (ti == 0 && gt == 0) trace_ev(p, 3, ntr, kb - kLag, 17);  // ... and published
        } else {
          ++pending;
        }
      }
      if (gt == 0) trace_ev(p, 3, ntr, tile, 1);
      // publish this tile's last k-block before taking the next tile unless
      // the next tile is already queued (see moe_gemm_kernel)
      if (ok && pending > 0 && !mbar_test_wait(smem_u32(&tq_full[(ti + 1) % kTileQ]), ((ti + 1) / kTileQ) & 1)) {
        cp_async_wait<0>();
        publish(it - 1);
        pending = 0;
      }
    }
    cp_async_wait<0>();
    if (ok && pending > 0) publish(it - 1);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still arrive on its barriers
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace moe
