/*
 * moe.h -- C ABI of the B200 (sm_100a) fine-grained MoE expert layer:
 * top-K routing, permutation into per-expert segments, grouped-GEMM
 * up-projection with gather and SwiGLU fused, grouped-GEMM down-projection,
 * gate-weighted aggregation, and the full backward pass with the router-score
 * gradient computed without caching any per-expert output.
 *
 * Sources (scraped pages on SonicMoE):
 *   [P1] "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE" (news article on the
 *        SonicMoE Blackwell blog), sections "MoE 与它的隐患",
 *        "核心创新：一次算法级的重新设计", "软件抽象层 QuACK".
 *   [P2] "SonicMoE：突破细粒度MoE硬件效率瓶颈，实现高稀疏性下的极致训练加速",
 *        paragraphs on the algorithm (router gradient without cached
 *        activations), scheduling (token rounding) and implementation (the
 *        eight kernels).
 *
 * Conventions for every entry point
 *   - Every tensor pointer is a DEVICE pointer owned by the caller; the library
 *     allocates and frees nothing.  Scratch memory is the caller's `ws` buffer,
 *     sized by moe_query_sizes().  All pointers must be 16-byte aligned.
 *   - bf16 tensors are passed as `void*` holding IEEE bfloat16 bit patterns.
 *   - Row-major layouts: X[T,d], Wr[d,E] (fp32), W1[E,d,2n] with columns
 *     [0,n) the gate projection and [n,2n) the up projection, W2[E,n,d].
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; argument errors are returned synchronously,
 *     device-side errors (a bounded wait that ran out, a failed check) are
 *     recorded in a device status word read by moe_get_status().
 *   - Supported shapes: d % 128 == 0, n % 64 == 0, 1 <= K <= min(E, 32),
 *     1 <= E <= 1024, 1 <= T < 2^31 / max(K, E).  Anything else returns
 *     MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* NULL where a pointer is required, misaligned pointer, bad option */
  MOE_ERR_UNSUPPORTED = 2,   /* shape outside the supported range */
  MOE_ERR_WORKSPACE = 3,     /* ws NULL or smaller than moe_query_sizes() asks */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch error, no device) */
  MOE_ERR_TIMEOUT = 5,       /* device: a bounded wait inside a kernel ran out */
  MOE_ERR_DEVICE_CHECK = 6,  /* device: an internal consistency check failed */
  MOE_ERR_SCRATCH_LIMIT = 7  /* moe_route_noalloc: the shape needs more than its static scratch */
} moe_status;

/* Layer shape: T tokens, model width d, E experts of intermediate width n, top-K. */
typedef struct {
  int64_t T;
  int32_t d, E, n, K;
} moe_dims;

typedef struct {
  int32_t round_mode;  /* token rounding used by moe_token_round: 1 nearest, 2 stochastic (0: off) */
  int32_t router_grad; /* 1: moe_backward adds the router path to dX and writes dWr */
  uint64_t seed;       /* seed of the stochastic rounding decision */
} moe_opts;

/*
 * Routing state, produced by moe_route (and rewritten by moe_token_round),
 * read by moe_forward / moe_backward.  All device pointers, caller-allocated
 * with the capacities P_max (pairs) and R_max (rows) from moe_query_sizes.
 *
 *   logits[T,E] f32, probs[T,E] f32   router logits z = X Wr (+ bias) and
 *                                      p = softmax(z) over all E experts
 *   topk_idx[T,K] i32, topk_gate[T,K]  the K largest logits per token (ties to
 *                                      the lower expert index, slots in
 *                                      descending order) and their gates, a
 *                                      softmax over the selected logits
 *   tok_ptr[T+1], pair_expert[P_max], pair_gate[P_max], pair_row[P_max]
 *                                      (token, expert) pairs as CSR over tokens
 *                                      and the expert-major row of each pair
 *   counts[E], offsets[E+1]            tokens per expert; segment starts, each
 *                                      a multiple of 128 (segments are padded
 *                                      to whole 128-row tiles); offsets[E] is
 *                                      the number of rows in use
 *   row_tok[R_max], row_gate[R_max]    token and gate of every row; padding
 *                                      rows hold token -1 and gate 0; inside a
 *                                      segment rows ascend in token order
 *   tile_expert[R_max/128]             expert of each 128-row tile
 *   pair_dS[P_max] (nullable)          if set, moe_backward writes the router
 *                                      score gradient dS of every pair there
 *                                      (fp32), with or without router_grad
 */
typedef struct {
  float* logits;
  float* probs;
  int32_t* topk_idx;
  float* topk_gate;
  int32_t* tok_ptr;
  int32_t* pair_expert;
  float* pair_gate;
  int32_t* pair_row;
  int32_t* counts;
  int32_t* offsets;
  int32_t* row_tok;
  float* row_gate;
  int32_t* tile_expert;
  int64_t P_max;
  int64_t R_max;
  float* pair_dS;
} moe_routing;

typedef struct {
  int64_t P_max;        /* capacity of the pair arrays */
  int64_t R_max;        /* capacity of the row arrays (a multiple of 128) */
  size_t route_ws;      /* bytes of ws for moe_route and moe_token_round */
  size_t fwd_ws;        /* bytes of ws for moe_forward */
  size_t bwd_ws;        /* bytes of ws for moe_backward */
  int64_t h_elems;      /* elements of the saved activation H = R_max * 2n (bf16) */
  size_t fwd_mx_ws;     /* bytes of ws for moe_forward_mxfp8(_q); 0 where that shape is unsupported */
  size_t mx_weights_bytes; /* bytes of the MXFP8 expert weights of moe_mx_quantize_weights; 0 if unsupported */
} moe_sizes;

/* Capacities and workspace sizes for a shape.  Host only; no GPU work. */
moe_status moe_query_sizes(const moe_dims* dims, const moe_opts* opts, moe_sizes* out);

/*
 * Router and permutation ([P1] "MoE 与它的隐患": each token is sent to a few
 * experts chosen by the router; [P1] "第二，IO 感知的算子融合": the grouped
 * GEMMs gather the routed rows themselves, so routing only produces indices).
 *   X[T,d] bf16, Wr[d,E] f32, bias[E] f32 (nullable; added to the logits
 *   before the softmax).  Fills every array of *rt except pair_row's unused
 *   tail.  rt->logits may be NULL (then kept in ws only).
 *   With opts->round_mode != 0 it stops after the top-K selection (logits,
 *   probs, topk_idx, topk_gate, tok_ptr, pair_expert, pair_gate): the rounded
 *   routing replaces the rest, and moe_token_round, which must follow on the
 *   same stream, builds it.
 */
moe_status moe_route(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr,
                     const float* bias, const moe_routing* rt, void* ws, size_t ws_bytes, void* stream);

/*
 * Routing given by the caller: rt->topk_idx[T,K] (experts, distinct within a
 * token, each in [0, E)) and rt->topk_gate[T,K] are inputs here.  Builds the
 * pairs (token t's pairs are t*K .. t*K+K-1, in slot order) and the
 * permutation exactly as moe_route does after its top-K; logits and probs
 * are neither read nor written (so moe_token_round and the router path of
 * moe_backward do not apply).  A token whose selection breaks the rules is
 * replaced by experts 0..K-1 with gate 0 and reported as
 * MOE_ERR_DEVICE_CHECK by moe_get_status.  ws of moe_sizes.route_ws bytes.
 * Used by the expert ranks of expert parallelism, whose "tokens" are the
 * rows they receive, each with one expert (K = 1) and its gate.
 */
moe_status moe_route_given(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Token rounding ([P2] scheduling paragraph): rounds every expert's token
 * count to a multiple of the 128-row GEMM tile with at most one tile of
 * deviation, keeping the total in expectation (opts->round_mode 2) or rounding
 * to the nearest multiple (mode 1).  Rounding down drops the routed tokens of
 * least probability, rounding up adds the unrouted tokens of largest
 * probability; gates become p renormalised over each token's final experts,
 * listed in ascending expert order.  Rewrites tok_ptr, pair_*, counts,
 * offsets, row_*, tile_expert of *rt (topk_idx/topk_gate keep the unrounded
 * selection).  Must follow moe_route on the same stream; it needs only the
 * top-K selection of that call (tok_ptr, pair_expert, probs).
 */
moe_status moe_token_round(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, void* ws,
                           size_t ws_bytes, void* stream);

/*
 * Forward ([P2] implementation paragraph: up-proj (A), down-proj (Y) and
 * expert aggregation (O) kernels):
 *   H_r = X[tok_r] W1[e_r]  (gather fused into the GEMM), A_r = silu(g)*u
 *   fused in its epilogue; Y_r = A_r W2[e_r];  O_t = sum_k gate * Y_row.
 *   O[T,d] bf16 out.  H[R_max,2n] bf16 out: the only per-row activation kept
 *   for the backward.  A and Y live in ws only.
 */
moe_status moe_forward(const moe_dims* dims, const moe_opts* opts, const void* X, const void* W1, const void* W2,
                       const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes, void* stream);

/*
 * Forward with MXFP8 GEMM operands (MXFP8 precision is named as future work
 * of the method, page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE",
 * closing paragraph; format and scale rule as for moe_mx_quantize_rows).
 * X is quantized along d per row, W1 along d and W2 along n per output
 * column, A = SwiGLU(H) along n per row; the GEMMs multiply E4M3 codes with
 * their E8M0 block scales on the tensor cores (kind::mxf8f6f4) and
 * accumulate in fp32.  Same arguments and outputs as moe_forward (O bf16;
 * H bf16 kept for moe_backward, which is unchanged); ws of
 * moe_sizes.fwd_mx_ws bytes.  Needs n % 128 == 0 (MOE_ERR_UNSUPPORTED
 * otherwise).
 */
moe_status moe_forward_mxfp8(const moe_dims* dims, const moe_opts* opts, const void* X, const void* W1,
                             const void* W2, const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes,
                             void* stream);

/*
 * The MXFP8 forward in two parts, for weights that stay fixed over many
 * calls (inference): moe_mx_quantize_weights writes W1 and W2 as MXFP8 (E4M3
 * codes, K-major, and their E8M0 scales in the layout the block-scaled MMA
 * reads) into wq, moe_sizes.mx_weights_bytes bytes of caller memory;
 * moe_forward_mxfp8_q is moe_forward_mxfp8 on those quantized weights (X
 * is still quantized per call).  The results are those of moe_forward_mxfp8
 * on the same W1, W2, bit for bit.  Same shape rule (n % 128 == 0) and
 * errors; ws of moe_sizes.fwd_mx_ws bytes.
 */
moe_status moe_mx_quantize_weights(const moe_dims* dims, const moe_opts* opts, const void* W1, const void* W2,
                                   void* wq, size_t wq_bytes, void* stream);
moe_status moe_forward_mxfp8_q(const moe_dims* dims, const moe_opts* opts, const void* X, const void* wq,
                               const moe_routing* rt, void* O, void* H, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward given dO[T,d] bf16 ([P2] implementation and algorithm paragraphs;
 * [P1] "第一，激活内存与专家粒度解耦"): dH kernel dA'_r = dO[tok_r] W2[e]^T
 * with H reloaded in its epilogue, the router score gradient
 * dS_r = <dA'_r, SwiGLU(H_r)> (no Y needed), dSwiGLU; dW2[e] = sum s_r A_r^T
 * dO[tok_r]; dX~_r = dH_r W1[e]^T; dW1[e] = sum X[tok_r]^T dH_r; dX
 * aggregation.  Router path (opts->router_grad): dz = s (dS - sum s dS) over
 * each token's experts, dWr = X^T dz (fp32 out, may be NULL only when
 * router_grad is 0), dX += dz Wr^T.
 *   dX[T,d], dW1[E,d,2n], dW2[E,n,d] bf16 out (overwritten, not accumulated).
 */
moe_status moe_backward(const moe_dims* dims, const moe_opts* opts, const void* dO, const void* X,
                        const float* Wr, const void* W1, const void* W2, const moe_routing* rt, const void* H,
                        void* dX, void* dW1, void* dW2, float* dWr, void* ws, size_t ws_bytes, void* stream);

/*
 * moe_backward that also reports when each weight gradient is final, so that
 * a data-parallel caller can start reducing it across ranks while the rest of
 * the backward runs (the pages train their layer data-parallel; the reduction
 * is the caller's).  grad_ready may be NULL, else it points to three
 * cudaEvent_t handles (each may be NULL), recorded on `stream`:
 *   grad_ready[0] once dW2 is written, grad_ready[1] once dW1 is written,
 *   grad_ready[2] once dWr is written (router_grad = 0: at the same point).
 * dW2 and dW1 are computed before dX~, so their reductions overlap the dX~
 * GEMM and the dX aggregation.  Events are caller-owned; everything else is
 * as for moe_backward.
 */
moe_status moe_backward_ev(const moe_dims* dims, const moe_opts* opts, const void* dO, const void* X,
                           const float* Wr, const void* W1, const void* W2, const moe_routing* rt, const void* H,
                           void* dX, void* dW1, void* dW2, float* dWr, void* ws, size_t ws_bytes,
                           void* const* grad_ready, void* stream);

/*
 * Expert parallelism (named as future work of the method, page
 * "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing paragraph: a token
 * all-to-all before the up-projection and after the down-projection).  The
 * exchange is the caller's; these calls lay the rows out for it.  The send
 * order is expert-major without padding: expert e's rows (its tokens in
 * ascending order) start at sum_{e'<e} counts[e'], so experts owned by one
 * rank form one contiguous block per destination.
 *
 * moe_ep_pack: send_rows[j] = src[token of row j] for the P routed rows
 *   (src[T,d] bf16: X in the forward, dO in the backward; send_rows [P,d]
 *   bf16, may be NULL), send_gate[j] = its gate (f32, may be NULL) and
 *   pair_pos[p] = j for each pair p (i32, may be NULL).  ws: at least
 *   4*(E+1) bytes (moe_sizes.route_ws is enough).
 * moe_ep_combine: out[t] = sum over token t's pairs p of rows[pair_pos[p]]
 *   (rows [P,d] bf16 in send order, as they come back; out [T,d] bf16,
 *   overwritten; fp32 sums in pair order).  The expert ranks apply the gates.
 */
moe_status moe_ep_pack(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, const void* src,
                       void* send_rows, float* send_gate, int32_t* pair_pos, void* ws, size_t ws_bytes,
                       void* stream);
moe_status moe_ep_combine(const moe_dims* dims, const moe_opts* opts, const moe_routing* rt, const int32_t* pair_pos,
                          const void* rows, void* out, void* stream);

/*
 * The router path of the backward from router score gradients computed
 * elsewhere (under expert parallelism, by the ranks that own the experts):
 *   dS: fp32, dS of pair p at dS[pair_pos[p]] (pair_pos may be NULL: dS[p]);
 *   dz = s (dS - sum s dS) over each token's experts ([P1] "MoE 与它的隐患";
 *   [P2] algorithm paragraph: the router gradient from dS without Y);
 *   dX[T,d] bf16 += dz Wr^T (read, updated, written back);
 *   dWr[d,E] f32 = X^T dz (overwritten).
 * X[T,d] bf16, Wr[d,E] f32, rt: the routing of moe_route.  ws of
 * moe_sizes.bwd_ws bytes.
 */
moe_status moe_router_backward(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr,
                               const moe_routing* rt, const float* dS, const int32_t* pair_pos, void* dX, float* dWr,
                               void* ws, size_t ws_bytes, void* stream);

/*
 * At most `sms` CTAs for each persistent GEMM kernel launched from now on by
 * this process (0, the default: one per SM).  A caller that overlaps a
 * communication kernel with the backward leaves SMs for it this way; results
 * do not depend on the budget.  Negative values: MOE_ERR_INVALID_ARG.
 */
moe_status moe_set_sm_budget(int32_t sms);

/*
 * MXFP8 quantization (the pages list MXFP8 precision as future work of the
 * method, page "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", closing
 * paragraph; the element and scale encodings are those of the OCP
 * Microscaling formats): E4M3 codes with one E8M0 scale per 32 consecutive
 * elements along K.  The scale is the smallest power of two at which no
 * element of the block saturates.  This departs from the OCP MX v1.0 scale
 * rule (section 6.3: shared exponent floor(log2 amax) - 8, elements above 448
 * clamped), which gives a scale half as large, and clamps the block maximum,
 * whenever the block maximum's significand exceeds 1.75; here no element is
 * ever clamped.
 *
 * moe_mx_quantize_rows: in[rows, K] bf16 -> codes[rows, K] u8 and
 *   scales[rows, K/32] u8, quantized along each row.
 * moe_mx_quantize_cols: in[E, K, N] bf16 (an expert weight stack, K rows) ->
 *   codes[E, N, K] u8 (transposed: K contiguous) and scales[E, N, K/32] u8,
 *   quantized along K for each column.
 * K must be a multiple of 32 (MOE_ERR_UNSUPPORTED otherwise); pointers must
 * be 16-byte aligned device pointers (MOE_ERR_INVALID_ARG).  Asynchronous on
 * `stream`.
 */
moe_status moe_mx_quantize_rows(const void* in, int64_t rows, int32_t K, void* codes, void* scales, void* stream);
moe_status moe_mx_quantize_cols(const void* in, int32_t E, int32_t K, int32_t N, void* codes, void* scales,
                                void* stream);

/*
 * Synchronises `stream`, returns the device status word (MOE_OK if no kernel
 * reported an error since the last call) and clears it.  *where (nullable)
 * receives the code of the wait or check that failed.
 */
moe_status moe_get_status(void* stream, int32_t* where);

/* Number of clock cycles a bounded wait spins before giving up (default 2^31,
 * about a second).  Values < 1000 are rejected with MOE_ERR_INVALID_ARG. */
moe_status moe_set_spin_limit(int64_t cycles);

/*
 * Failure-detection self test: launches one thread that waits, through the
 * kernels' bounded-wait primitive, on a barrier nothing completes.  On return
 * (after a stream sync) *waited_ok (device int) is 0 and moe_get_status()
 * reports MOE_ERR_TIMEOUT.  Meant for tests with a small spin limit.
 */
moe_status moe_selftest_wait_timeout(int32_t* waited_ok, void* stream);

/*
 * Per-kernel timing for benchmarks.  While enabled, every kernel the library
 * launches is bracketed by two CUDA events recorded on its launching stream
 * (host-side bookkeeping only; the events are created once and reused).
 * moe_profile_enable(1) clears earlier records; moe_profile_count() gives the
 * number of kernel launches recorded; moe_profile_read(i, ...) returns the
 * name and duration in ms of launch i once its stream has completed.  Not
 * thread-safe; meant for one benchmarking thread.
 */
moe_status moe_profile_enable(int32_t on);
/* Restrict recording to launches of one kernel name (as reported by
 * moe_profile_read); NULL records every launch again.  Bracketing a single
 * kernel keeps the event overhead out of the rest of the timed work. */
moe_status moe_profile_select(const char* name);
int32_t moe_profile_count(void);
moe_status moe_profile_read(int32_t i, const char** name, float* ms);

/*
 * Role timeline of one grouped-GEMM kind (tracing; the pages report per-kernel
 * tensor-core utilisation and HBM traffic of their kernels, page
 * "DeepSeek做大→Mega MoE，Tri Dao团队加快→SonicMoE", section "第二，IO 感知的
 * 算子融合" -- this shows where inside one of these kernels the time goes).
 * kind: 0 up-proj, 1 down-proj, 2 dH, 3 dX~, 4 dW1, 5 dW2, 6 router logits,
 * 7 router dWr, 8 MXFP8 up-proj, 9 MXFP8 down-proj; -1 (or buf NULL) turns
 * tracing off.  While on, every launch of that kind writes, per CTA and role
 * (0 TMA producer, 1 MMA issuer, 2 epilogue, 3 gather warps), up to
 * `records_per_role` 16-byte records {u64 %globaltimer ns, u32 clock64 low
 * bits, u32 tile << 8 | event} at
 *   buf + 16 * ((cta * 4 + role) * records_per_role + i),
 * so buf needs 64 * grid * records_per_role bytes (grid <= the SM count).
 * The caller zeroes buf (a zero record is unused).  Events per tile:
 * producer 0 tile taken, 1 last k-block issued; MMA 0 tile taken,
 * 1 accumulator free, 2 first k-block's operands ready, 3 last MMA committed;
 * epilogue 0 tile taken, 1 accumulator full, 2 accumulator released (its
 * stores issued); gather 0 tile taken, 1 last k-block's copies issued.
 * Where a kind runs as two launches -- down-proj and dX~ with d % 256 == 0:
 * pairs of M tiles on 2-CTA clusters, then each expert's odd last M tile on
 * single CTAs -- the first (pair) launch is the one traced.
 * Launches in flight keep the buffer: turn tracing off or synchronize before
 * freeing it.  Results do not depend on tracing.
 */
moe_status moe_trace_gemm(int32_t kind, void* buf, int64_t records_per_role);

/*
 * moe_route_noalloc -- moe_route for callers that cannot allocate device
 * memory.  Such callers exist: a plugin that a host runtime hands only its
 * input and output buffers, or code running under an allocator that owns the
 * whole device pool and cannot give out a workspace.  The pages have no
 * counterpart to this entry point; it is a deployment convenience.
 *
 * Same inputs and outputs as moe_route (rt->logits must be non-NULL here),
 * but no ws: the scratch (Wr split, chunk histograms, pair ranks) lives in a
 * 16 MiB static device array inside the library.  Every GPU that loads the
 * library holds that array until the process exits.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on each device resolves the array's device address (a
 *     set-up step done once per device, with that device current); make that
 *     first call before any stream capture.
 *   - All calls on a device share the array, and it keeps the previous call's
 *     contents (each call writes every scratch byte it reads first).  Calls
 *     whose GPU work overlaps race on it: order them (one stream, or events).
 *   - Returns MOE_ERR_SCRATCH_LIMIT, without touching the GPU, when the shape
 *     needs more than 16 MiB (16777216 bytes) of scratch, namely the sum of
 *       2*d*3*ceil(E/64)*64    (Wr split)
 *       16                     (block-completion counters)
 *       4*ceil(T/256)*E        (chunk histograms)
 *       4*T*K                  (pair ranks)
 *     bytes, each of the four parts rounded up to a multiple of 256.
 */
moe_status moe_route_noalloc(const moe_dims* dims, const moe_opts* opts, const void* X, const float* Wr,
                             const float* bias, const moe_routing* rt, void* stream);

/* Static description of a status code. */
const char* moe_status_str(moe_status s);

/* The CUDA runtime error behind the calling thread's most recent
 * MOE_ERR_CUDA: error name, message and the library source line that saw it.
 * Empty if no call on this thread has failed that way.  The string is owned
 * by the library and stays valid until the thread's next failing call. */
const char* moe_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
