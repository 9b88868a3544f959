// C-ABI layer (include/moe.h): argument checks, workspace carving, TMA
// descriptor encoding and the launch order of the layer's kernels.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <set>
#include <tuple>

#include <nvtx3/nvToolsExt.h>

#include "moe.h"
#include "moe_internal.h"

using namespace moe;

namespace {

// ----------------------------------------------------------------- status word
__device__ int g_status_word[2];  // [0] first error code, [1] where it happened

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};
long long g_spin_limit = 1ll << 31;
int g_sm_budget = 0;  // CTAs of a persistent GEMM at most (0: one per SM)
std::mutex g_mu;

bool device_state(int* dev_out, int** status_out, int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return false;
    g_status_ptr[dev] = static_cast<int*>(p);
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
    g_num_sms[dev] = sms;
  }
  *dev_out = dev;
  *status_out = g_status_ptr[dev];
  *sms_out = (g_sm_budget > 0 && g_sm_budget < g_num_sms[dev]) ? g_sm_budget : g_num_sms[dev];
  return true;
}

// ----------------------------------------------------------------- profiler
constexpr int kProfCap = 1 << 15;
struct ProfRec {
  cudaEvent_t a, b;
  const char* name;
};
ProfRec g_prof[kProfCap];
int g_prof_n = 0;        // records taken since the last enable
int g_prof_created = 0;  // event pairs created so far (reused across enables)
bool g_prof_on = false;
char g_prof_only[64] = {0};  // when set, only launches of this name are recorded

// ----------------------------------------------------------------- TMA encoding
using EncodeFn = decltype(&cuTensorMapEncodeTiled);
EncodeFn g_encode = nullptr;

bool get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<EncodeFn>(fn);
  return true;
}

// 2-D bf16 row-major tensor [rows, cols], box [box_rows, box_cols]; operand
// loads use the 128-byte swizzle, epilogue stores 32 x 32 boxes with the
// 64-byte swizzle.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
               uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
// Byte matrix [rows, cols] (MXFP8 codes), 128-byte swizzle.
bool make_tmap_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                  uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}
bool make_store_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return make_tmap(m, base, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}
// Store map of the one-output epilogues: 32-row x 64-column boxes, 128-byte
// swizzle (whole 128-byte row segments per store).
bool make_store_map_wide(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  return make_tmap(m, base, rows, cols, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B);
}

// ----------------------------------------------------------------- shapes
struct Plan {
  int64_t T;
  int d, E, n, K, Epad, Ew, nchunks;
  int64_t P_max, R_max;
  int bn_up, bn_down, bn_dh, bn_dxt, bn_dw1, bn_dw2;
  int nts;  // N tiles of the dH kernel
  int nds;  // dS partials per row: N tiles x column parts of the dH epilogue
  int epi_dh, epi_dxt;  // epilogue warps of the dH and dX~ kernels
  int epi_dw;           // epilogue warps of the weight-gradient kernels
  int dw_dual;          // weight-gradient tile claims: 0 largest experts first, 1 from both ends by CTA parity,
                        // 2 every CTA alternating ends
  int dw1_pair, dw2_pair;  // weight-gradient GEMMs on CTA pairs (256 x 256 tiles)
  int gm_pair;             // down-proj and dX~ on CTA pairs (256 x 256 tiles of two M tiles)
  int wide_down, wide_dxt;  // down-proj / dX~ with 256 x 256 tiles (two M tiles) on one CTA
  int wstat;                // grouped-M tile order: 1 weight-stationary, 0 M-tile-major
  int ksplit, ksplit_rows;
};

inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Column width of the router-logit tiles: 384 (two 64-expert groups, all 512
// TMEM columns) where the padded expert count is a multiple of 128, so that
// every 128-row tile of X is read once per two groups; else 192 (one group).
// On the DeepSeek-V3-shaped layer (Epad = 256, 64 row tiles) that is 128 tiles
// in one wave instead of 256 in 1.73.
inline int router_bn(int Epad) { return Epad % 128 == 0 ? 384 : 192; }

moe_status make_plan(const moe_dims* dims, const moe_opts* opts, Plan* pl) {
  if (!dims || !opts) return MOE_ERR_INVALID_ARG;
  if (opts->round_mode < 0 || opts->round_mode > 2 || (opts->router_grad != 0 && opts->router_grad != 1))
    return MOE_ERR_INVALID_ARG;
  const int64_t T = dims->T;
  const int d = dims->d, E = dims->E, n = dims->n, K = dims->K;
  if (T < 1 || d < 128 || n < 64 || E < 1 || K < 1) return MOE_ERR_UNSUPPORTED;
  if (d % 128 != 0 || n % 64 != 0 || K > 32 || K > E || E > 1024) return MOE_ERR_UNSUPPORTED;
  if (T * (int64_t)std::max(K, E) >= (int64_t(1) << 31) - 4096 * 1024) return MOE_ERR_UNSUPPORTED;
  if ((int64_t)d * 2 * n * E >= (int64_t(1) << 40)) return MOE_ERR_UNSUPPORTED;
  Plan p;
  p.T = T;
  p.d = d;
  p.E = E;
  p.n = n;
  p.K = K;
  p.Epad = (int)cdiv(E, 64) * 64;
  p.Ew = (int)cdiv(E, 32);
  p.nchunks = (int)cdiv(T, kChunk);
  p.P_max = T * K;
  if (opts->round_mode != 0) p.P_max = std::min<int64_t>(T * E, T * K + (int64_t)(kTile - 1) * E);
  p.R_max = cdiv(p.P_max + (int64_t)(kTile - 1) * E, kTile) * kTile;
  p.bn_up = (n % 128 == 0) ? 256 : 128;
  p.bn_down = (d % 256 == 0) ? 256 : 128;
  p.bn_dh = (n % 256 == 0) ? 256 : ((n % 128 == 0) ? 128 : 64);
  p.bn_dxt = p.bn_down;
  p.bn_dw1 = ((2 * n) % 256 == 0) ? 256 : 128;
  p.bn_dw2 = p.bn_down;
  p.nts = n / p.bn_dh;
  // Eight epilogue warps only where the epilogue outlasts a short main loop;
  // otherwise 4 warps, whose smaller staging leaves room for a deeper stage
  // ring.  Measured: dH with 4 warps 4 % faster at d = 1536 (24 k-blocks) and
  // at d = 2048; dX~ with 4 warps 7 % faster at 2n = 512 (8 k-blocks), with 8
  // warps 25 % faster at 2n = 256 (4 k-blocks: a 64 KB store plus the router
  // path per tile).  The dH threshold (12 k-blocks) is half the shortest main
  // loop measured to prefer 4.  (The down-proj kernel measured slower with 8:
  // its short main loop is bound by the Y stores, not the epilogue.)
  p.epi_dh = (d / 64 <= 12) ? 8 : 4;
  p.epi_dxt = (2 * n / 64 <= 4) ? 8 : 4;
  // The weight-gradient kernels keep 4 epilogue warps.  Their short tiles
  // (an expert's few rows) are bound by storing the 128 x BN result, but with
  // claims alternating between long and short tiles those stores run under
  // the long tiles' main loops, and the fourth ring stage that 4 warps' staging
  // leaves room for pays more: dW1 3-6 % faster than with 8 warps on the
  // DeepSeek-V3-shaped, E = 256 and small-expert layers (8 warps with one
  // staging buffer each, also 4 stages, measured level with 4 warps).
  p.epi_dw = 4;
  p.dw_dual = 2;  // every CTA alternates ends: short tiles' stores run under long tiles' main loops
  // tuning overrides, for measurements: MOE_EPI_DW, MOE_EPI_DH, MOE_EPI_DXT
  // (4 or 8 epilogue warps), MOE_DW_DUAL (0 to 2)
  auto epi_override = [](const char* name, int& field) {
    if (const char* v = std::getenv(name)) {
      const int x = std::atoi(v);
      if (x == 4 || x == 8) field = x;
    }
  };
  epi_override("MOE_EPI_DW", p.epi_dw);
  epi_override("MOE_EPI_DH", p.epi_dh);
  epi_override("MOE_EPI_DXT", p.epi_dxt);
  if (const char* v = std::getenv("MOE_DW_DUAL")) {
    const int x = std::atoi(v);
    if (x >= 0 && x <= 2) p.dw_dual = x;
  }
  // 256 x 256 pair tiles where both output dimensions are multiples of 256
  // (MOE_DW_PAIR=1 turns them on)
  const bool pair_on = std::getenv("MOE_DW_PAIR") && std::atoi(std::getenv("MOE_DW_PAIR")) != 0;
  p.dw1_pair = pair_on && (d % 256 == 0) && ((2 * n) % 256 == 0);
  p.dw2_pair = pair_on && (d % 256 == 0) && (n % 256 == 0);
  // Down-proj and dX~ on CTA pairs (MOE_GM_PAIR=1, where N = d splits into
  // 256-column tiles).  Off by default: measured no faster than one CTA per
  // 128 x 256 tile on any workload here, and slower on the balanced ones.
  p.gm_pair = 0;
  if (const char* v = std::getenv("MOE_GM_PAIR")) p.gm_pair = (d % 256 == 0) && std::atoi(v) != 0;
  // Down-proj with 256 x 256 tiles on one CTA (two M tiles sharing B) where N
  // = d splits into 256-column tiles and the main loop (n / 64 k-blocks) is
  // long enough for the single-buffered accumulator.  Measured against the
  // 128 x 256 tiles: 1.5-5 % faster at n = 768..2048 (12-32 k-blocks), 5 %
  // slower at n = 256 (4).  dX~ on the same tiles measured level or slower on
  // the balanced layers (+3 % at 2n = 1536) and 1.4 % faster on the
  // DeepSeek-V3-shaped one, so it stays opt-in: MOE_GM_WIDE=1 turns both on,
  // MOE_GM_WIDE=0 both off.
  p.wide_down = (d % 256 == 0) && (n / 64 >= 12);
  p.wide_dxt = 0;
  if (const char* v = std::getenv("MOE_GM_WIDE")) {
    const int x = std::atoi(v);
    p.wide_down = (d % 256 == 0) && x != 0;
    p.wide_dxt = (d % 256 == 0) && x != 0;
  }
  if (p.gm_pair) p.wide_down = p.wide_dxt = 0;
  // Grouped-M tile order.  Weight-stationary (within an expert, the M tiles of
  // one N tile side by side, so that each tile of the expert's weights is read
  // from DRAM once and served from L2 to all of them) where an expert's
  // weights outweigh its rows several times over (2n > 4 T K / E: the
  // DeepSeek-V3-shaped layer, 16x): there its DRAM reads fell by 3-15 % per
  // kernel.  Elsewhere M-tile-major (the N tiles of one M tile side by side,
  // sharing its gathered rows), which measured 1-5 % faster per kernel on the
  // 7B-class, Qwen3- and OLMoE-shaped layers.  MOE_TILE_ORDER=0/1 overrides.
  p.wstat = (2 * (int64_t)n * E > 4 * T * K) ? 1 : 0;
  if (const char* v = std::getenv("MOE_TILE_ORDER")) p.wstat = std::atoi(v) != 0;
  p.nds = p.nts * (p.epi_dh / 4);
  // split-K of the router-weight gradient: the split count with the shortest
  // critical path of the persistent launch on 148 SMs -- tiles round-robin,
  // so (waves of tiles) x (k-blocks per tile) -- plus the reduction's read of
  // the fp32 partials (about 450 KB per k-block of one tile's load time).
  // A fixed "two tiles per SM" left 3.03 waves on the DeepSeek-V3-shaped layer
  // and 2.1 on the 7B-class one.
  {
    const int64_t mn_tiles = cdiv(d, 128) * (p.Epad / 64);
    double best = 0.0;
    const int64_t ks_max = std::min<int64_t>(64, cdiv(T, 64));
    for (int64_t ks = 1; ks <= ks_max; ++ks) {
      const int64_t rows = cdiv(cdiv(T, ks), 64) * 64;
      const int64_t splits = cdiv(T, rows);
      const double cost =
          (double)cdiv(mn_tiles * splits, 148) * (double)(rows / 64) + (double)splits * d * p.Epad / 450000.0;
      if (ks == 1 || cost < best) {
        best = cost;
        p.ksplit_rows = (int)rows;
        p.ksplit = (int)splits;
      }
    }
  }
  // MOE_LOG=1: the tile plan of each new shape, once, on stderr
  if (const char* v = std::getenv("MOE_LOG")) {
    if (std::atoi(v) != 0) {
      static std::mutex mu;
      static std::set<std::tuple<int64_t, int, int, int, int, int>> seen;
      std::lock_guard<std::mutex> lk(mu);
      if (seen.insert({T, d, E, n, K, opts->round_mode}).second)
        std::fprintf(stderr,
                     "moe plan T=%lld d=%d E=%d n=%d K=%d round=%d: P_max=%lld R_max=%lld; BN up %d down %d dH %d "
                     "dX~ %d dW1 %d dW2 %d; epilogue warps dH %d dX~ %d dW %d; dW tiles from both ends %d; CTA pairs "
                     "dW1 %d dW2 %d down/dX~ %d; 256-row tiles on one CTA down %d dX~ %d; router tile %d columns; "
                     "dWr split-K %d x %d rows\n",
                     (long long)T, d, E, n, K, opts->round_mode, (long long)p.P_max, (long long)p.R_max, p.bn_up,
                     p.bn_down, p.bn_dh, p.bn_dxt, p.bn_dw1, p.bn_dw2, p.epi_dh, p.epi_dxt, p.epi_dw, p.dw_dual,
                     p.dw1_pair, p.dw2_pair, p.gm_pair, p.wide_down, p.wide_dxt, router_bn(p.Epad), p.ksplit,
                     p.ksplit_rows);
    }
  }
  *pl = p;
  return MOE_OK;
}

struct Carve {
  char* base;
  size_t off = 0;
  template <class T>
  T* take(size_t count) {
    T* r = reinterpret_cast<T*>(base ? base + off : nullptr);
    off = align256(off + count * sizeof(T));
    return r;
  }
};

struct RouteWs {
  __nv_bfloat16* Wr_split;
  float* logits;
  int* sync;  // [1] blocks done, for the last-block offsets scan of the permutation
  int* hist;
  int* local_rank;
  uint32_t* memberT;  // token rounding: [E, ceil(T/32)]
  uint32_t* finalT;   // token rounding: [E, ceil(T/32)]
  float* probsT;      // token rounding: [E, T]
  int* rowpre;        // token rounding: [E, ceil(T/32)]
  int* local;         // token rounding: [T]
  int* blk;           // token rounding: [ceil(T/256) + 1]
};
size_t carve_route(const Plan& p, void* ws, RouteWs* w) {
  Carve c{static_cast<char*>(ws)};
  w->Wr_split = c.take<__nv_bfloat16>((size_t)p.d * 3 * p.Epad);
  w->logits = c.take<float>((size_t)p.T * p.E);
  w->sync = c.take<int>(4);
  w->hist = c.take<int>((size_t)p.nchunks * p.E);
  w->local_rank = c.take<int>((size_t)p.P_max);
  const size_t W = (size_t)cdiv(p.T, 32);
  w->memberT = c.take<uint32_t>((size_t)p.E * W);
  w->finalT = c.take<uint32_t>((size_t)p.E * W);
  w->probsT = c.take<float>((size_t)p.E * p.T);
  w->rowpre = c.take<int>((size_t)p.E * W);
  w->local = c.take<int>((size_t)p.T);
  w->blk = c.take<int>((size_t)cdiv(p.T, 256) + 1);
  return c.off;
}

struct FwdWs {
  __nv_bfloat16* A;
  __nv_bfloat16* Y;
  int *mpair, *mleft;  // pair and leftover lists of the M tiles (CTA-pair down-proj)
  int* mwide;          // 256-row tile list of the M tiles (one-CTA 256 x 256 down-proj)
  int* mwbase;         // its first entry of each expert [E + 1]
};
// MXFP8 forward: codes and scales of X, W1, W2 and A, and Y
// MXFP8 expert weights: codes K-major and scales in the MMA's tile layout
struct MxWeights {
  uint8_t *W1q, *SW1t;         // [E, 2n, d], scale tiles [E][n/64][d/128]
  uint8_t *W2q, *SW2t;         // [E, d, n], scale tiles [E][d/128][n/128]
};
struct MxFwdWs {
  MxWeights wt;                // filled by the quantizing forward; unused with pre-quantized weights
  uint8_t *Xq, *SX;            // [T, d], [T, d/32]
  uint8_t *Aq, *SA;            // [R_max, n], scale tiles [R_max/128][n/128]
  __nv_bfloat16* Y;            // [R_max, d]
};
size_t carve_fwd(const Plan& p, void* ws, FwdWs* w) {
  Carve c{static_cast<char*>(ws)};
  w->A = c.take<__nv_bfloat16>((size_t)p.R_max * p.n);
  w->Y = c.take<__nv_bfloat16>((size_t)p.R_max * p.d);
  w->mpair = c.take<int>((size_t)(p.R_max / 256 + 2));
  w->mleft = c.take<int>((size_t)p.E + 1);
  w->mwide = c.take<int>((size_t)(p.R_max / 256 + p.E + 2));
  w->mwbase = c.take<int>((size_t)p.E + 1);
  return c.off;
}

bool mx_supported(const Plan& p) { return p.n % 128 == 0; }

size_t carve_mx_weights(const Plan& p, Carve& c, MxWeights* w) {
  const size_t d = p.d, n = p.n, E = p.E;
  w->W1q = c.take<uint8_t>(E * 2 * n * d);
  w->SW1t = c.take<uint8_t>(E * (n / 64) * (d / 128) * 512);
  w->W2q = c.take<uint8_t>(E * d * n);
  w->SW2t = c.take<uint8_t>(E * (d / 128) * (n / 128) * 512);
  return c.off;
}
size_t mx_weights_bytes(const Plan& p) {
  Carve c{nullptr};
  MxWeights w;
  return carve_mx_weights(p, c, &w);
}

size_t carve_fwd_mx(const Plan& p, void* ws, MxFwdWs* w) {
  Carve c{static_cast<char*>(ws)};
  const size_t T = (size_t)p.T, d = p.d, n = p.n, R = (size_t)p.R_max;
  carve_mx_weights(p, c, &w->wt);
  w->Xq = c.take<uint8_t>(T * d);
  w->SX = c.take<uint8_t>(T * (d / 32));
  w->Aq = c.take<uint8_t>(R * n);
  w->SA = c.take<uint8_t>((R / 128) * (n / 128) * 512);
  w->Y = c.take<__nv_bfloat16>(R * d);
  return c.off;
}

struct BwdWs {
  __nv_bfloat16 *dH, *Ahat, *dXt, *dz_split;
  float *dS_part, *dz_row, *WrT, *dWr_part;
  int *sched, *expert_order;
  int *mpair, *mleft;  // pair and leftover lists of the M tiles (CTA-pair dX~)
  int* mwide;          // 256-row tile list of the M tiles (one-CTA 256 x 256 dX~)
  int* mwbase;         // its first entry of each expert [E + 1]
};
size_t carve_bwd(const Plan& p, void* ws, BwdWs* w) {
  Carve c{static_cast<char*>(ws)};
  w->dH = c.take<__nv_bfloat16>((size_t)p.R_max * 2 * p.n);
  w->Ahat = c.take<__nv_bfloat16>((size_t)p.R_max * p.n);
  w->dXt = c.take<__nv_bfloat16>((size_t)p.R_max * p.d);
  // sized for 8 dH epilogue warps whatever the plan picked, so that the
  // MOE_EPI_DH override cannot outgrow a workspace sized before it was set
  w->dS_part = c.take<float>((size_t)p.R_max * p.nts * 2);
  w->dz_split = c.take<__nv_bfloat16>((size_t)p.T * 2 * p.Epad);
  w->dz_row = c.take<float>((size_t)p.R_max);
  w->WrT = c.take<float>((size_t)p.E * p.d);
  w->dWr_part = c.take<float>((size_t)p.ksplit * p.d * p.Epad);
  w->sched = c.take<int>(16);
  w->expert_order = c.take<int>((size_t)p.E);
  w->mpair = c.take<int>((size_t)(p.R_max / 256 + 2));
  w->mleft = c.take<int>((size_t)p.E + 1);
  w->mwide = c.take<int>((size_t)(p.R_max / 256 + p.E + 2));
  w->mwbase = c.take<int>((size_t)p.E + 1);
  return c.off;
}

inline bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool routing_ok(const moe_routing* rt, const Plan& p, bool need_probs) {
  if (!rt) return false;
  const void* req[] = {rt->topk_idx, rt->topk_gate, rt->tok_ptr, rt->pair_expert, rt->pair_gate, rt->pair_row,
                       rt->counts, rt->offsets, rt->row_tok, rt->row_gate, rt->tile_expert};
  for (const void* q : req)
    if (!q || !aligned16(q)) return false;
  if (need_probs && (!rt->probs || !aligned16(rt->probs))) return false;
  if (rt->logits && !aligned16(rt->logits)) return false;
  return rt->P_max >= p.P_max && rt->R_max >= p.R_max;
}

RouteArgs route_args(const Plan& p, const moe_routing* rt, const RouteWs& w) {
  RouteArgs a;
  a.T = (int)p.T;
  a.d = p.d;
  a.E = p.E;
  a.K = p.K;
  a.Epad = p.Epad;
  a.Wr = nullptr;
  a.Wr_split = w.Wr_split;
  a.logits = rt->logits ? rt->logits : w.logits;
  a.probs = rt->probs;
  a.topk_idx = rt->topk_idx;
  a.topk_gate = rt->topk_gate;
  a.tok_ptr = rt->tok_ptr;
  a.pair_expert = rt->pair_expert;
  a.pair_gate = rt->pair_gate;
  a.pair_row = rt->pair_row;
  a.counts = rt->counts;
  a.offsets = rt->offsets;
  a.row_tok = rt->row_tok;
  a.row_gate = rt->row_gate;
  a.tile_expert = rt->tile_expert;
  a.sync = w.sync;
  a.hist = w.hist;
  a.local_rank = w.local_rank;
  a.nchunks = p.nchunks;
  a.st = DevStatus{nullptr, g_spin_limit};
  return a;
}

GemmParams base_params(const Plan& p, const moe_routing* rt, int* status) {
  GemmParams g;
  std::memset(&g, 0, sizeof(g));
  g.st = DevStatus{status, g_spin_limit};
  g.offsets = rt ? rt->offsets : nullptr;
  g.counts = rt ? rt->counts : nullptr;
  g.tile_expert = rt ? rt->tile_expert : nullptr;
  g.row_tok = rt ? rt->row_tok : nullptr;
  g.row_gate = rt ? rt->row_gate : nullptr;
  g.T = (int)p.T;
  g.d = p.d;
  g.n = p.n;
  g.E = p.E;
  g.Epad = p.Epad;
  g.wstat = p.wstat;
  return g;
}

// Debug build: check the routing's invariants on the device before (or
// after) a step uses (or builds) it, wait for the check and report a
// violation as cudaErrorInvalidValue (the caller returns MOE_ERR_DEVICE_CHECK
// through moe_get_status, and launches nothing more).  Nothing is launched,
// and nothing waits, in the release build.
cudaError_t validate_routing(const Plan& p, const moe_routing* rt, int* status, cudaStream_t st) {
  if (!MOE_DEBUG) return cudaSuccess;
  RoutingView v;
  v.T = p.T;
  v.P_max = p.P_max;
  v.R_max = p.R_max;
  v.E = p.E;
  v.tok_ptr = rt->tok_ptr;
  v.pair_expert = rt->pair_expert;
  v.pair_row = rt->pair_row;
  v.counts = rt->counts;
  v.offsets = rt->offsets;
  v.row_tok = rt->row_tok;
  v.tile_expert = rt->tile_expert;
  {
    ProfScope ps(st, "validate_routing");
    cudaError_t e = launch_validate_routing(v, DevStatus{status, g_spin_limit}, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  int h = 0;
  e = cudaMemcpy(&h, status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return e;
  return h == 0 ? cudaSuccess : cudaErrorInvalidValue;
}
#define MOE_VALIDATE(p, rt, status, st)                              \
  do {                                                               \
    const cudaError_t moe_v_ = validate_routing(p, rt, status, st);  \
    if (moe_v_ == cudaErrorInvalidValue) return MOE_ERR_DEVICE_CHECK; \
    if (moe_v_ != cudaSuccess) return cuda_failed(moe_v_, __LINE__);  \
  } while (0)

// Records event grad_ready[i] (a cudaEvent_t, may be null) on the stream.
// Recording cannot fail on a valid event; a failure surfaces at the next sync.
inline void record_ready(void* const* grad_ready, int i, cudaStream_t st) {
  if (grad_ready && grad_ready[i]) cudaEventRecord(static_cast<cudaEvent_t>(grad_ready[i]), st);
}

inline int grid_for(int64_t max_tiles, int sms) { return (int)std::max<int64_t>(1, std::min<int64_t>(max_tiles, sms)); }

// The last CUDA runtime error a call returned, with the source line that saw
// it (read back through moe_last_error).
thread_local char g_last_error[512] = "";

moe_status cuda_failed(cudaError_t e, int line) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s (%s) at moe_api.cu:%d%s%s", cudaGetErrorName(e),
                cudaGetErrorString(e), line, g_launch_diag[0] ? "; " : "", g_launch_diag);
  g_launch_diag[0] = 0;
  return MOE_ERR_CUDA;
}

#define MOE_TRY_CUDA(x)                                   \
  do {                                                    \
    const cudaError_t moe_e_ = (x);                       \
    if (moe_e_ != cudaSuccess) return cuda_failed(moe_e_, __LINE__); \
  } while (0)
#define MOE_TRY_MAP(x)                                 \
  do {                                                 \
    if (!(x)) return MOE_ERR_INVALID_ARG;              \
  } while (0)

}  // namespace

namespace moe {
ApiRange::ApiRange(const char* name) { nvtxRangePushA(name); }
ApiRange::~ApiRange() { nvtxRangePop(); }

ProfScope::ProfScope(cudaStream_t s, const char* name) : stream(s) {
  nvtxRangePushA(name);
  if (!g_prof_on || g_prof_n >= kProfCap) return;
  if (g_prof_only[0] && std::strcmp(g_prof_only, name) != 0) return;
  ProfRec& r = g_prof[g_prof_n];
  if (g_prof_n >= g_prof_created) {
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return;
    ++g_prof_created;
  }
  r.name = name;
  slot = g_prof_n++;
  cudaEventRecord(r.a, stream);
}
ProfScope::~ProfScope() {
  if (slot >= 0) cudaEventRecord(g_prof[slot].b, stream);
  nvtxRangePop();
}
}  // namespace moe

extern "C" {

moe_status moe_query_sizes(const moe_dims* dims, const moe_opts* opts, moe_sizes* out) {
  if (!out) return MOE_ERR_INVALID_ARG;
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  RouteWs rw;
  FwdWs fw;
  BwdWs bw;
  out->P_max = p.P_max;
  out->R_max = p.R_max;
  out->route_ws = carve_route(p, nullptr, &rw);
  out->fwd_ws = carve_fwd(p, nullptr, &fw);
  out->bwd_ws = carve_bwd(p, nullptr, &bw);
  out->h_elems = p.R_max * 2 * p.n;
  MxFwdWs mw;
  out->fwd_mx_ws = mx_supported(p) ? carve_fwd_mx(p, nullptr, &mw) : 0;
  out->mx_weights_bytes = mx_supported(p) ? mx_weights_bytes(p) : 0;
  return MOE_OK;
}

moe_status moe_route(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr, const float* bias,
                     const moe_routing* rt, void* ws, size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_route");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (!X || !Wr || !aligned16(X) || !aligned16(Wr) || (bias && !aligned16(bias)) || !routing_ok(rt, p, true))
    return MOE_ERR_INVALID_ARG;
  RouteWs w;
  if (!ws || ws_bytes < carve_route(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_route(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  RouteArgs a = route_args(p, rt, w);
  a.Wr = Wr;
  a.st.word = status;
  {
    ProfScope ps(st, "router_split_wr");
    MOE_TRY_CUDA(launch_split_wr(a, st));
  }

  GemmParams g = base_params(p, rt, status);
  MOE_TRY_MAP(make_tmap(&g.tmA, X, (uint64_t)p.T, (uint64_t)p.d, 64, 128));
  MOE_TRY_MAP(make_tmap(&g.tmB, w.Wr_split, (uint64_t)p.d, (uint64_t)3 * p.Epad, 64, 64));
  // one tile covers both groups of 64 experts where E <= 128 (TMEM holds two
  // groups' hi slots and mid/lo accumulators), so X is read once per row tile
  const int bn_rtr = router_bn(p.Epad);
  g.num_m_tiles = (int)cdiv(p.T, 128);
  g.num_n_tiles = 3 * p.Epad / bn_rtr;
  g.outf = const_cast<float*>(a.logits);
  g.bias = bias;
  {
    ProfScope ps(st, "router_logits_gemm");
    MOE_TRY_CUDA(launch_gemm(G_RTR, bn_rtr, 4, g, grid_for((int64_t)g.num_m_tiles * g.num_n_tiles, sms), st));
  }

  {
    ProfScope ps(st, "router_softmax_topk");
    MOE_TRY_CUDA(launch_softmax_topk(a, st));
  }
  // with token rounding to follow, the permutation is left to moe_token_round
  // (it rebuilds counts, segments and rows from the rounded expert sets)
  if (opts->round_mode != 0) return MOE_OK;
  MOE_TRY_CUDA(launch_permute(a, st));
  MOE_VALIDATE(p, rt, status, st);
  return MOE_OK;
}

moe_status moe_token_round(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, void* ws,
                           size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_token_round");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (opts->round_mode == 0) return MOE_ERR_INVALID_ARG;
  if (!routing_ok(rt, p, true)) return MOE_ERR_INVALID_ARG;
  RouteWs w;
  if (!ws || ws_bytes < carve_route(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_route(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  RouteArgs a = route_args(p, rt, w);
  a.st.word = status;
  RoundArgs r;
  r.T = (int)p.T;
  r.E = p.E;
  r.mode = opts->round_mode;
  r.seed = (unsigned long long)opts->seed;
  r.probs = rt->probs;
  r.probsT = w.probsT;
  r.memberT = w.memberT;
  r.finalT = w.finalT;
  r.rowpre = w.rowpre;
  r.local = w.local;
  r.blk = w.blk;
  r.sync = w.sync + 1;
  MOE_TRY_CUDA(launch_token_round(a, r, static_cast<cudaStream_t>(stream)));
  MOE_VALIDATE(p, rt, status, static_cast<cudaStream_t>(stream));
  return MOE_OK;
}

moe_status moe_forward(const moe_dims* dims, const moe_opts* opts, const void* X, const void* W1, const void* W2,
                       const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_forward");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  const void* ptrs[] = {X, W1, W2, O, H};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  FwdWs w;
  if (!ws || ws_bytes < carve_fwd(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_fwd(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t mtiles = p.R_max / kTile;
  MOE_VALIDATE(p, rt, status, st);

  // up-projection: H = X[tok] W1[e], A = SwiGLU(H)
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmB, W1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n, 64, 64));
    g.gsrc = static_cast<const __nv_bfloat16*>(X);
    g.gld = p.d;
    g.num_n_tiles = p.n / (p.bn_up / 2);
    g.out0 = static_cast<__nv_bfloat16*>(H);
    g.out1 = w.A;
    MOE_TRY_MAP(make_store_map(&g.tmC0, H, (uint64_t)p.R_max, (uint64_t)2 * p.n));
    MOE_TRY_MAP(make_store_map(&g.tmC1, w.A, (uint64_t)p.R_max, (uint64_t)p.n));
    if (p.wide_down) {  // the down-proj's 256-row tile list, written by the first CTA
      g.wlist = w.mwide;
      g.wbase = w.mwbase;
    }
    ProfScope ps(st, "up_proj_gemm");
    MOE_TRY_CUDA(launch_gemm(G_UP, p.bn_up, 4, g, grid_for(mtiles * g.num_n_tiles, sms), st));
  }
  // down-projection: Y = A W2[e]
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmA, w.A, (uint64_t)p.R_max, (uint64_t)p.n, 64, 128));
    MOE_TRY_MAP(make_tmap(&g.tmB, W2, (uint64_t)p.E * p.n, (uint64_t)p.d, 64, 64));
    g.num_n_tiles = p.d / p.bn_down;
    g.out0 = w.Y;
    MOE_TRY_MAP(make_store_map_wide(&g.tmC0, w.Y, (uint64_t)p.R_max, (uint64_t)p.d));
    ProfScope ps(st, "down_proj_gemm");
    if (p.gm_pair) {
      // pairs of M tiles on CTA pairs, then each expert's odd last M tile on one CTA
      MOE_TRY_CUDA(launch_pair_lists(rt->offsets, p.E, w.mpair, w.mleft, st));
      g.num_n_tiles = p.d / 256;
      g.mlist = w.mpair;
      MOE_TRY_CUDA(launch_gemm_pair_m(G_DOWN, 4, g, (int)std::min<int64_t>(sms / 2, (mtiles / 2) * g.num_n_tiles), st));
      g.mlist = w.mleft;
      MOE_TRY_CUDA(launch_gemm(G_DOWN, 256, 4, g, grid_for(std::min<int64_t>(p.E, mtiles) * g.num_n_tiles, sms), st,
                               false));
    } else if (p.wide_down) {  // over the tile list the up-proj kernel wrote
      g.num_n_tiles = p.d / 256;
      g.mlist = w.mwide;
      g.wbase = w.mwbase;
      MOE_TRY_CUDA(launch_gemm_wide_m(G_DOWN, g, grid_for((mtiles / 2 + p.E) * g.num_n_tiles, sms), st));
    } else {
      MOE_TRY_CUDA(launch_gemm(G_DOWN, p.bn_down, 4, g, grid_for(mtiles * g.num_n_tiles, sms), st));
    }
  }
  {
    ProfScope ps(st, "aggregate_fwd");
    MOE_TRY_CUDA(launch_aggregate_fwd((int)p.T, p.d, rt->tok_ptr, rt->pair_row, rt->pair_gate, w.Y,
                                      static_cast<__nv_bfloat16*>(O), st));
  }
  return MOE_OK;
}

}  // extern "C"

namespace {
// W1, W2 (bf16) to MXFP8 codes, K-major, with their scales in the MMA's tile
// layout: W1 along d per output column (its tiles hold 64 gate and the same
// 64 up columns), W2 along n per output column.
cudaError_t quantize_mx_weights(const Plan& p, const void* W1, const void* W2, const MxWeights& wt, cudaStream_t st) {
  ProfScope ps(st, "mx_quant_w");
  cudaError_t e = launch_mx_quant_cols(static_cast<const __nv_bfloat16*>(W1), p.E, p.d, 2 * p.n, wt.W1q, nullptr,
                                       wt.SW1t, 1, st);
  if (e != cudaSuccess) return e;
  return launch_mx_quant_cols(static_cast<const __nv_bfloat16*>(W2), p.E, p.n, p.d, wt.W2q, nullptr, wt.SW2t, 0, st);
}

// The MXFP8 forward on quantized weights: X to MXFP8 per row, then the
// block-scaled up-projection (H bf16 out, A quantized in its epilogue), the
// block-scaled down-projection and the aggregation.
moe_status forward_mx(const Plan& p, const void* X, const MxWeights& wt, const moe_routing* rt, void* O, void* H,
                      const MxFwdWs& w, int* status, int sms, cudaStream_t st) {
  const int64_t mtiles = p.R_max / kTile;
  const int E = p.E, d = p.d, n = p.n;
  MOE_VALIDATE(p, rt, status, st);
  {
    ProfScope ps(st, "mx_quant_x");
    MOE_TRY_CUDA(launch_mx_quant_rows(static_cast<const __nv_bfloat16*>(X), p.T, d, w.Xq, w.SX, st));
  }
  // up-projection on MXFP8 operands: H = X[tok] W1[e] (bf16 out), A = SwiGLU(H)
  // quantized to MXFP8 with its scale tiles
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap_u8(&g.tmB, wt.W1q, (uint64_t)E * 2 * n, (uint64_t)d, 128, 64));
    g.gsrc = reinterpret_cast<const __nv_bfloat16*>(w.Xq);  // rows of d bytes, gathered in 16-byte chunks
    g.gld = d / 2;
    g.sfa_src = w.SX;
    g.sfb_src = wt.SW1t;
    g.num_n_tiles = n / 64;
    g.out0 = static_cast<__nv_bfloat16*>(H);
    g.aq_out = w.Aq;
    g.sa_out = w.SA;
    MOE_TRY_MAP(make_store_map(&g.tmC0, H, (uint64_t)p.R_max, (uint64_t)2 * n));
    ProfScope ps(st, "up_proj_gemm_mx");
    MOE_TRY_CUDA(launch_gemm(G_UPQ, 128, 4, g, grid_for(mtiles * g.num_n_tiles, sms), st));
  }
  // down-projection on MXFP8 operands: Y = A W2[e]
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap_u8(&g.tmA, w.Aq, (uint64_t)p.R_max, (uint64_t)n, 128, 128));
    MOE_TRY_MAP(make_tmap_u8(&g.tmB, wt.W2q, (uint64_t)E * d, (uint64_t)n, 128, 128));
    g.sfa_src = w.SA;
    g.sfb_src = wt.SW2t;
    g.num_n_tiles = d / 128;
    g.out0 = w.Y;
    MOE_TRY_MAP(make_store_map(&g.tmC0, w.Y, (uint64_t)p.R_max, (uint64_t)d));
    ProfScope ps(st, "down_proj_gemm_mx");
    MOE_TRY_CUDA(launch_gemm(G_DOWNQ, 128, 4, g, grid_for(mtiles * g.num_n_tiles, sms), st));
  }
  {
    ProfScope ps(st, "aggregate_fwd");
    MOE_TRY_CUDA(launch_aggregate_fwd((int)p.T, d, rt->tok_ptr, rt->pair_row, rt->pair_gate, w.Y,
                                      static_cast<__nv_bfloat16*>(O), st));
  }
  return MOE_OK;
}

// Shape, pointer and workspace checks shared by the MXFP8 forward entries.
moe_status mx_forward_setup(const moe_dims* dims, const moe_opts* opts, const void* X, const moe_routing* rt,
                            void* O, void* H, void* ws, size_t ws_bytes, Plan* p, MxFwdWs* w) {
  moe_status s = make_plan(dims, opts, p);
  if (s != MOE_OK) return s;
  if (!mx_supported(*p)) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {X, O, H};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (!routing_ok(rt, *p, false)) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < carve_fwd_mx(*p, nullptr, w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_fwd_mx(*p, ws, w);
  return MOE_OK;
}
}  // namespace

extern "C" {

moe_status moe_forward_mxfp8(const moe_dims* dims, const moe_opts* opts, const void* X, const void* W1,
                             const void* W2, const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes,
                             void* stream) {
  ApiRange api_range("moe_forward_mxfp8");
  if (!W1 || !W2 || !aligned16(W1) || !aligned16(W2)) {
    Plan p;
    const moe_status s = make_plan(dims, opts, &p);
    if (s != MOE_OK) return s;
    return mx_supported(p) ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  }
  Plan p;
  MxFwdWs w;
  moe_status s = mx_forward_setup(dims, opts, X, rt, O, H, ws, ws_bytes, &p, &w);
  if (s != MOE_OK) return s;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  MOE_TRY_CUDA(quantize_mx_weights(p, W1, W2, w.wt, st));
  return forward_mx(p, X, w.wt, rt, O, H, w, status, sms, st);
}

moe_status moe_mx_quantize_weights(const moe_dims* dims, const moe_opts* opts, const void* W1, const void* W2,
                                   void* wq, size_t wq_bytes, void* stream) {
  ApiRange api_range("moe_mx_quantize_weights");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (!mx_supported(p)) return MOE_ERR_UNSUPPORTED;
  const void* ptrs[] = {W1, W2, wq};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (wq_bytes < mx_weights_bytes(p)) return MOE_ERR_WORKSPACE;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  Carve c{static_cast<char*>(wq)};
  MxWeights wt;
  carve_mx_weights(p, c, &wt);
  MOE_TRY_CUDA(quantize_mx_weights(p, W1, W2, wt, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_forward_mxfp8_q(const moe_dims* dims, const moe_opts* opts, const void* X, const void* wq,
                               const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_forward_mxfp8_q");
  if (!wq || !aligned16(wq)) {
    Plan p;
    const moe_status s = make_plan(dims, opts, &p);
    if (s != MOE_OK) return s;
    return mx_supported(p) ? MOE_ERR_INVALID_ARG : MOE_ERR_UNSUPPORTED;
  }
  Plan p;
  MxFwdWs w;
  moe_status s = mx_forward_setup(dims, opts, X, rt, O, H, ws, ws_bytes, &p, &w);
  if (s != MOE_OK) return s;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  Carve c{static_cast<char*>(const_cast<void*>(wq))};
  MxWeights wt;
  carve_mx_weights(p, c, &wt);
  return forward_mx(p, X, wt, rt, O, H, w, status, sms, static_cast<cudaStream_t>(stream));
}

}  // extern "C"



namespace {
// dWr = X^T dz: the split-K tensor-core GEMM over the bf16 hi/lo split of dz
// (w.dz_split, written before), then the reduction of the splits in order.
// Returns the first failing CUDA status (tensor-map failures as
// cudaErrorInvalidValue).
cudaError_t run_dwr(const Plan& p, const moe_routing* rt, const BwdWs& w, const void* X, float* dWr, int* status,
                    int sms, cudaStream_t st) {
  GemmParams g = base_params(p, rt, status);
  if (!make_tmap(&g.tmA, X, (uint64_t)p.T, (uint64_t)p.d, 64, 64) ||
      !make_tmap(&g.tmB, w.dz_split, (uint64_t)p.T, (uint64_t)2 * p.Epad, 64, 64))
    return cudaErrorInvalidValue;
  g.num_m_tiles = (int)cdiv(p.d, 128);
  g.num_n_tiles = p.Epad / 64;
  g.ksplit = p.ksplit;
  g.ksplit_rows = p.ksplit_rows;
  g.outf = w.dWr_part;
  {
    ProfScope ps(st, "router_dwr_gemm");
    cudaError_t e = launch_gemm(G_DWR, 128, 4, g, grid_for((int64_t)g.num_m_tiles * g.num_n_tiles * p.ksplit, sms), st);
    if (e != cudaSuccess) return e;
  }
  ProfScope ps(st, "router_dwr_reduce");
  return launch_dwr_reduce(p.d, p.E, p.Epad, p.ksplit, w.dWr_part, dWr, st);
}
}  // namespace

extern "C" {

moe_status moe_backward(const moe_dims* dims, const moe_opts* opts, const void* dO, const void* X, const float* Wr,
                        const void* W1, const void* W2, const moe_routing* rt, const void* H, void* dX, void* dW1,
                        void* dW2, float* dWr, void* ws, size_t ws_bytes, void* stream) {
  return moe_backward_ev(dims, opts, dO, X, Wr, W1, W2, rt, H, dX, dW1, dW2, dWr, ws, ws_bytes, nullptr, stream);
}

moe_status moe_backward_ev(const moe_dims* dims, const moe_opts* opts, const void* dO, const void* X, const float* Wr,
                           const void* W1, const void* W2, const moe_routing* rt, const void* H, void* dX,
                           void* dW1, void* dW2, float* dWr, void* ws, size_t ws_bytes, void* const* grad_ready,
                           void* stream) {
  ApiRange api_range("moe_backward_ev");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  const void* ptrs[] = {dO, X, W1, W2, H, dX, dW1, dW2};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  const bool rg = opts->router_grad != 0;
  if (rg && (!Wr || !dWr || !aligned16(Wr) || !aligned16(dWr))) return MOE_ERR_INVALID_ARG;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  BwdWs w;
  if (!ws || ws_bytes < carve_bwd(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_bwd(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t mtiles = p.R_max / kTile;
  const __nv_bfloat16* dOb = static_cast<const __nv_bfloat16*>(dO);
  const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
  MOE_VALIDATE(p, rt, status, st);
  // dH kernel: dA' = dO[tok] W2[e]^T; epilogue: H -> A, dS partials, dSwiGLU, A_hat
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmB, W2, (uint64_t)p.E * p.n, (uint64_t)p.d, 64, (uint32_t)p.bn_dh));
    g.gsrc = dOb;
    g.gld = p.d;
    g.num_n_tiles = p.nts;
    g.hin = static_cast<const __nv_bfloat16*>(H);
    g.out0 = w.dH;
    g.out1 = w.Ahat;
    g.outf = w.dS_part;
    MOE_TRY_MAP(make_store_map(&g.tmC0, w.dH, (uint64_t)p.R_max, (uint64_t)2 * p.n));
    MOE_TRY_MAP(make_store_map(&g.tmC1, w.Ahat, (uint64_t)p.R_max, (uint64_t)p.n));
    ProfScope ps(st, "dh_gemm");
    MOE_TRY_CUDA(launch_gemm(G_DH, p.bn_dh, p.epi_dh, g, grid_for(mtiles * g.num_n_tiles, sms), st));
  }
  // Router path, dz = s * (dS - sum_j s_j dS_j), and Wr^T, both consumed by
  // the dX~ epilogue; the expert order (largest first) in which the
  // weight-gradient GEMMs take their tiles, and their zeroed tile counters.
  {
    BwdPrepArgs a{};
    a.T = (int)p.T;
    a.d = p.d;
    a.E = p.E;
    a.Epad = p.Epad;
    a.nds = p.nds;
    a.K = p.K;
    a.router = rg ? 1 : 0;
    a.tok_ptr = rt->tok_ptr;
    a.pair_row = rt->pair_row;
    a.pair_expert = rt->pair_expert;
    a.pair_gate = rt->pair_gate;
    a.dS_part = w.dS_part;
    a.dz_row = w.dz_row;
    a.dz_split = w.dz_split;
    a.Wr = Wr;
    a.WrT = w.WrT;
    a.counts = rt->counts;
    a.expert_order = w.expert_order;
    a.sched = w.sched;
    a.pair_dS = rt->pair_dS;
    ProfScope ps(st, "bwd_prep");
    MOE_TRY_CUDA(launch_bwd_prep(a, st));
  }
  // dW2[e] = A_hat^T dO[tok]
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmA, w.Ahat, (uint64_t)p.R_max, (uint64_t)p.n, 64, 64));
    g.gsrc = dOb;
    g.gld = p.d;
    g.num_m_tiles = (int)cdiv(p.n, 128);
    g.num_n_tiles = p.d / p.bn_dw2;
    g.out0 = static_cast<__nv_bfloat16*>(dW2);
    g.sched = w.sched + 0;  // 64-bit tile counter (front and back claims)
    g.dual_ended = p.dw_dual;
    g.expert_order = w.expert_order;
    MOE_TRY_MAP(make_store_map_wide(&g.tmC0, dW2, (uint64_t)p.E * p.n, (uint64_t)p.d));
    ProfScope ps(st, "dw2_gemm");
    if (p.dw2_pair) {
      MOE_TRY_MAP(make_tmap(&g.tmC1, dW2, (uint64_t)p.E * p.n, (uint64_t)p.d, 64, 32));
      g.num_m_tiles = p.n / 256;
      g.num_n_tiles = p.d / 256;
      MOE_TRY_CUDA(launch_gemm_pair(G_DW2, p.epi_dw, g,
                                    grid_for((int64_t)p.E * g.num_m_tiles * g.num_n_tiles, sms / 2), st));
    } else {
      MOE_TRY_CUDA(launch_gemm(G_DW2, p.bn_dw2, p.epi_dw, g,
                               grid_for((int64_t)p.E * g.num_m_tiles * g.num_n_tiles, sms), st));
    }
  }
  record_ready(grad_ready, 0, st);  // dW2 final
  // dW1[e] = X[tok]^T dH
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmB, w.dH, (uint64_t)p.R_max, (uint64_t)2 * p.n, 64, 64));
    g.gsrc = Xb;
    g.gld = p.d;
    g.num_m_tiles = (int)cdiv(p.d, 128);
    g.num_n_tiles = 2 * p.n / p.bn_dw1;
    g.out0 = static_cast<__nv_bfloat16*>(dW1);
    g.sched = w.sched + 2;  // a 64-bit counter of its own
    g.dual_ended = p.dw_dual;
    g.expert_order = w.expert_order;
    MOE_TRY_MAP(make_store_map_wide(&g.tmC0, dW1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n));
    ProfScope ps(st, "dw1_gemm");
    if (p.dw1_pair) {
      MOE_TRY_MAP(make_tmap(&g.tmC1, dW1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n, 64, 32));
      g.num_m_tiles = p.d / 256;
      g.num_n_tiles = 2 * p.n / 256;
      MOE_TRY_CUDA(launch_gemm_pair(G_DW1, p.epi_dw, g,
                                    grid_for((int64_t)p.E * g.num_m_tiles * g.num_n_tiles, sms / 2), st));
    } else {
      MOE_TRY_CUDA(launch_gemm(G_DW1, p.bn_dw1, p.epi_dw, g,
                               grid_for((int64_t)p.E * g.num_m_tiles * g.num_n_tiles, sms), st));
    }
  }
  record_ready(grad_ready, 1, st);  // dW1 final
  // dX~ = dH W1[e]^T
  {
    GemmParams g = base_params(p, rt, status);
    MOE_TRY_MAP(make_tmap(&g.tmA, w.dH, (uint64_t)p.R_max, (uint64_t)2 * p.n, 64, 128));
    MOE_TRY_MAP(make_tmap(&g.tmB, W1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n, 64, (uint32_t)p.bn_dxt));
    g.num_n_tiles = p.d / p.bn_dxt;
    g.out0 = w.dXt;
    if (rg) {
      g.rvec = w.WrT;
      g.rscale = w.dz_row;
    }
    MOE_TRY_MAP(make_store_map_wide(&g.tmC0, w.dXt, (uint64_t)p.R_max, (uint64_t)p.d));
    if (p.wide_dxt) {
      ProfScope pl(st, "dxt_tile_list");
      MOE_TRY_CUDA(launch_wide_list(rt->offsets, p.E, w.mwide, w.mwbase, st));
    }
    ProfScope ps(st, "dxt_gemm");
    if (p.gm_pair) {
      // pairs of M tiles on CTA pairs (each CTA loading 128 of a tile's 256 W1
      // rows), then each expert's odd last M tile on one CTA
      MOE_TRY_CUDA(launch_pair_lists(rt->offsets, p.E, w.mpair, w.mleft, st));
      GemmParams gp = g;
      MOE_TRY_MAP(make_tmap(&gp.tmB, W1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n, 64, 128));
      gp.num_n_tiles = p.d / 256;
      gp.mlist = w.mpair;
      MOE_TRY_CUDA(
          launch_gemm_pair_m(G_DXT, p.epi_dxt, gp, (int)std::min<int64_t>(sms / 2, (mtiles / 2) * gp.num_n_tiles), st));
      g.num_n_tiles = p.d / 256;
      g.mlist = w.mleft;
      MOE_TRY_CUDA(
          launch_gemm(G_DXT, 256, p.epi_dxt, g, grid_for(std::min<int64_t>(p.E, mtiles) * g.num_n_tiles, sms), st,
                      false));
    } else if (p.wide_dxt) {
      GemmParams gw = g;
      MOE_TRY_MAP(make_tmap(&gw.tmB, W1, (uint64_t)p.E * p.d, (uint64_t)2 * p.n, 64, 256));
      gw.num_n_tiles = p.d / 256;
      gw.mlist = w.mwide;
      gw.wbase = w.mwbase;
      MOE_TRY_CUDA(launch_gemm_wide_m(G_DXT, gw, grid_for((mtiles / 2 + p.E) * gw.num_n_tiles, sms), st));
    } else {
      MOE_TRY_CUDA(launch_gemm(G_DXT, p.bn_dxt, p.epi_dxt, g, grid_for(mtiles * g.num_n_tiles, sms), st));
    }
  }
  if (rg) MOE_TRY_CUDA(run_dwr(p, rt, w, X, dWr, status, sms, st));
  record_ready(grad_ready, 2, st);  // dWr final (or nothing to wait for without the router path)
  {
    ProfScope ps(st, "aggregate_bwd");
    MOE_TRY_CUDA(launch_aggregate_bwd((int)p.T, p.d, rt->tok_ptr, rt->pair_row, w.dXt,
                                      static_cast<__nv_bfloat16*>(dX), st));
  }
  return MOE_OK;
}

moe_status moe_route_given(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, void* ws,
                           size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_route_given");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  RouteWs w;
  if (!ws || ws_bytes < carve_route(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_route(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouteArgs a = route_args(p, rt, w);
  a.st.word = status;
  {
    ProfScope ps(st, "given_pairs");
    MOE_TRY_CUDA(launch_given_pairs((int)p.T, p.K, p.E, rt->topk_idx, rt->topk_gate, rt->tok_ptr, rt->pair_expert,
                                    rt->pair_gate, a.st, st));
  }
  MOE_TRY_CUDA(launch_permute(a, st));
  MOE_VALIDATE(p, rt, status, st);
  return MOE_OK;
}

moe_status moe_ep_pack(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, const void* src,
                       void* send_rows, float* send_gate, int32_t* pair_pos, void* ws, size_t ws_bytes,
                       void* stream) {
  ApiRange api_range("moe_ep_pack");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  if (send_rows && (!src || !aligned16(src) || !aligned16(send_rows))) return MOE_ERR_INVALID_ARG;
  if ((send_gate && !aligned16(send_gate)) || (pair_pos && !aligned16(pair_pos))) return MOE_ERR_INVALID_ARG;
  if (!ws || ws_bytes < (size_t)(p.E + 1) * sizeof(int)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope ps(st, "ep_pack");
  MOE_TRY_CUDA(launch_ep_pack((int)p.T, p.d, p.E, p.R_max, p.P_max, rt->tok_ptr, rt->pair_expert, rt->pair_row,
                              rt->counts, rt->offsets, rt->tile_expert, rt->row_tok, rt->row_gate,
                              static_cast<const __nv_bfloat16*>(src), static_cast<__nv_bfloat16*>(send_rows),
                              send_gate, pair_pos, static_cast<int*>(ws), st));
  return MOE_OK;
}

moe_status moe_ep_combine(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, const int32_t* pair_pos,
                          const void* rows, void* out, void* stream) {
  ApiRange api_range("moe_ep_combine");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  const void* ptrs[] = {pair_pos, rows, out};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  ProfScope ps(st, "ep_combine");
  MOE_TRY_CUDA(launch_aggregate_bwd((int)p.T, p.d, rt->tok_ptr, pair_pos, static_cast<const __nv_bfloat16*>(rows),
                                    static_cast<__nv_bfloat16*>(out), st));
  return MOE_OK;
}

moe_status moe_router_backward(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr,
                               const moe_routing* rt, const float* dS, const int32_t* pair_pos, void* dX, float* dWr,
                               void* ws, size_t ws_bytes, void* stream) {
  ApiRange api_range("moe_router_backward");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  const void* ptrs[] = {X, Wr, dS, dX, dWr};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return MOE_ERR_INVALID_ARG;
  if (pair_pos && !aligned16(pair_pos)) return MOE_ERR_INVALID_ARG;
  if (!routing_ok(rt, p, false)) return MOE_ERR_INVALID_ARG;
  BwdWs w;
  if (!ws || ws_bytes < carve_bwd(p, nullptr, &w)) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  carve_bwd(p, ws, &w);
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  {
    ProfScope ps(st, "router_bwd_given");
    MOE_TRY_CUDA(launch_router_bwd_given((int)p.T, p.d, p.E, p.Epad, rt->tok_ptr, rt->pair_expert, rt->pair_gate, dS,
                                         pair_pos, Wr, w.WrT, w.dz_split, static_cast<__nv_bfloat16*>(dX), st));
  }
  MOE_TRY_CUDA(run_dwr(p, rt, w, X, dWr, status, sms, st));
  return MOE_OK;
}

moe_status moe_get_status(void* stream, int32_t* where) {
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MOE_ERR_CUDA;
  int h[2] = {0, 0};
  if (cudaMemcpy(h, status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero[2] = {0, 0};
  if (cudaMemcpy(status, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return MOE_ERR_CUDA;
  if (where) *where = h[1];
  return static_cast<moe_status>(h[0]);
}

moe_status moe_mx_quantize_rows(const void* in, int64_t rows, int32_t K, void* codes, void* scales, void* stream) {
  if (rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (K % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (!in || !codes || !scales || !aligned16(in) || !aligned16(codes) || !aligned16(scales))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY_CUDA(launch_mx_quant_rows(static_cast<const __nv_bfloat16*>(in), rows, K, static_cast<uint8_t*>(codes),
                                    static_cast<uint8_t*>(scales), static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_mx_quantize_cols(const void* in, int32_t E, int32_t K, int32_t N, void* codes, void* scales,
                                void* stream) {
  if (E < 0 || K <= 0 || N < 0) return MOE_ERR_INVALID_ARG;
  if (K % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (!in || !codes || !scales || !aligned16(in) || !aligned16(codes) || !aligned16(scales))
    return MOE_ERR_INVALID_ARG;
  MOE_TRY_CUDA(launch_mx_quant_cols(static_cast<const __nv_bfloat16*>(in), E, K, N, static_cast<uint8_t*>(codes),
                                    static_cast<uint8_t*>(scales), nullptr, 0, static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

moe_status moe_set_sm_budget(int32_t sms) {
  if (sms < 0) return MOE_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_mu);
  g_sm_budget = sms;
  return MOE_OK;
}

moe_status moe_set_spin_limit(int64_t cycles) {
  if (cycles < 1000) return MOE_ERR_INVALID_ARG;
  g_spin_limit = cycles;
  return MOE_OK;
}

moe_status moe_selftest_wait_timeout(int32_t* waited_ok, void* stream) {
  if (!waited_ok) return MOE_ERR_INVALID_ARG;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms)) return MOE_ERR_CUDA;
  if (launch_wait_selftest(waited_ok, DevStatus{status, g_spin_limit}, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_profile_enable(int32_t on) {
  if (on != 0 && on != 1) return MOE_ERR_INVALID_ARG;
  if (on) g_prof_n = 0;
  g_prof_on = on != 0;
  return MOE_OK;
}

moe_status moe_profile_select(const char* name) {
  if (!name) {
    g_prof_only[0] = 0;
    return MOE_OK;
  }
  if (std::strlen(name) >= sizeof(g_prof_only)) return MOE_ERR_INVALID_ARG;
  std::strcpy(g_prof_only, name);
  return MOE_OK;
}

int32_t moe_profile_count(void) { return g_prof_n; }

moe_status moe_profile_read(int32_t i, const char** name, float* ms) {
  if (i < 0 || i >= g_prof_n || !name || !ms) return MOE_ERR_INVALID_ARG;
  *name = g_prof[i].name;
  if (cudaEventElapsedTime(ms, g_prof[i].a, g_prof[i].b) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_trace_gemm(int32_t kind, void* buf, int64_t records_per_role) {
  if (kind < -1 || kind > G_DOWNQ) return MOE_ERR_INVALID_ARG;
  if (buf && kind >= 0 && (records_per_role < 1 || records_per_role > (1 << 24) || !aligned16(buf)))
    return MOE_ERR_INVALID_ARG;
  set_gemm_trace(kind, kind >= 0 ? buf : nullptr, (int)records_per_role);
  return MOE_OK;
}

const char* moe_last_error(void) { return g_last_error; }

const char* moe_status_str(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_DEVICE_CHECK: return "device consistency check failed";
    case MOE_ERR_SCRATCH_LIMIT: return "shape needs more scratch than the static array holds";
  }
  return "unknown status";
}

}  // extern "C"

// ----------------------------------------------------------------- routing without caller scratch
// moe_route_noalloc serves callers that cannot allocate device memory at all,
// such as a plugin that is handed only its input and output buffers by a host
// runtime, or code running under an allocator that owns the whole device pool
// and cannot carve out a workspace.  Its scratch (Wr split, per-chunk expert
// histograms, per-pair ranks) lives in the file-scope array below instead of
// the caller's ws.  Every byte of it that a call reads is first written by the
// same call, so the contents left by an earlier call never matter and nothing
// needs clearing.  All calls on a device share the one array: calls whose GPU
// work overlaps (different streams, no ordering between them) race.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_scratch_ptr[kMaxDevices] = {nullptr};

// Set-up, once per device, with that device current: the host-side symbol is
// only a stand-in, so resolve the array's device address.
bool noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return false;
    g_noalloc_scratch_ptr[dev] = ptr;
  }
  *out = g_noalloc_scratch_ptr[dev];
  return true;
}

size_t carve_noalloc_route(const Plan& p, void* base, RouteWs* w) {
  Carve c{static_cast<char*>(base)};
  w->Wr_split = c.take<__nv_bfloat16>((size_t)p.d * 3 * p.Epad);
  w->sync = c.take<int>(4);
  w->hist = c.take<int>((size_t)p.nchunks * p.E);
  w->local_rank = c.take<int>((size_t)p.T * p.K);
  w->logits = nullptr;
  w->memberT = nullptr;
  w->finalT = nullptr;
  w->probsT = nullptr;
  w->local = nullptr;
  w->blk = nullptr;
  return c.off;
}
}  // namespace

extern "C" moe_status moe_route_noalloc(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr,
                                        const float* bias, const moe_routing* rt, void* stream) {
  ApiRange api_range("moe_route_noalloc");
  Plan p;
  moe_status s = make_plan(dims, opts, &p);
  if (s != MOE_OK) return s;
  RouteWs w;
  if (carve_noalloc_route(p, nullptr, &w) > kNoAllocScratchBytes) return MOE_ERR_SCRATCH_LIMIT;
  if (!X || !Wr || !aligned16(X) || !aligned16(Wr) || (bias && !aligned16(bias)) || !routing_ok(rt, p, true) ||
      !rt->logits)
    return MOE_ERR_INVALID_ARG;
  int dev, sms;
  int* status;
  if (!device_state(&dev, &status, &sms) || !get_encode()) return MOE_ERR_CUDA;
  void* scratch = nullptr;
  if (!noalloc_scratch(dev, &scratch)) return MOE_ERR_CUDA;
  carve_noalloc_route(p, scratch, &w);
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  RouteArgs a = route_args(p, rt, w);
  a.Wr = Wr;
  a.st.word = status;
  MOE_TRY_CUDA(launch_split_wr(a, st));
  GemmParams g = base_params(p, rt, status);
  MOE_TRY_MAP(make_tmap(&g.tmA, X, (uint64_t)p.T, (uint64_t)p.d, 64, 128));
  MOE_TRY_MAP(make_tmap(&g.tmB, w.Wr_split, (uint64_t)p.d, (uint64_t)3 * p.Epad, 64, 64));
  const int bn_rtr = router_bn(p.Epad);
  g.num_m_tiles = (int)cdiv(p.T, 128);
  g.num_n_tiles = 3 * p.Epad / bn_rtr;
  g.outf = rt->logits;
  g.bias = bias;
  MOE_TRY_CUDA(launch_gemm(G_RTR, bn_rtr, 4, g, grid_for((int64_t)g.num_m_tiles * g.num_n_tiles, sms), st));
  MOE_TRY_CUDA(launch_softmax_topk(a, st));
  MOE_TRY_CUDA(launch_permute(a, st));
  MOE_VALIDATE(p, rt, status, st);
  return MOE_OK;
}
