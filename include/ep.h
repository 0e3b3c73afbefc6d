/*
 * ep.h -- C ABI of the B200 MoE token-routing library (libep.so).
 *
 * The library computes the data-parallel hot path of expert-parallel token
 * routing as the DeepEP pages describe it, with all R ranks simulated inside
 * one GPU's HBM: every "rank" is a slice of one allocation, and a copy to a
 * rank is a store into that rank's slice.  There is no inter-GPU transfer.
 *
 * General rules (all entry points):
 *   - Every pointer argument is DEVICE memory owned by the caller, except
 *     where a comment says "host".  The library never allocates device memory
 *     and never frees what it is given.  Scratch memory ("workspace") is sized
 *     by ep_*_workspace_bytes() and passed in by the caller; the library clears
 *     it on the stream at the start of each call.
 *   - Every call is asynchronous on `stream` and never synchronises the host.
 *     The caller orders calls with events.  Calls are stateless and may run
 *     concurrently if they use distinct output and workspace buffers.
 *   - Kernels are launched with programmatic stream serialization
 *     (programmatic dependent launch): each one waits for the previous grid
 *     on the stream before it touches memory, and lets the next one be
 *     scheduled early.  Ordinary launches, copies and events that follow on
 *     the stream see every output as usual.  A kernel of the caller's that
 *     follows with the same launch attribute must itself wait
 *     (cudaGridDependencySynchronize) before it reads the outputs.
 *   - The return value is a host-side status (EP_OK ... EP_ERR_UNSUPPORTED).
 *     Argument checks happen before anything is launched; on an error nothing
 *     is launched and no output is touched.
 *   - Errors the GPU detects (a bad expert id, a receive buffer too small, a
 *     bounded wait that ran out) are never trapped.  The kernels skip the
 *     offending access and OR an EP_STATUS_* bit into the optional device word
 *     `status` (int32), which the caller zeroes beforehand and reads after its
 *     own synchronisation.  A NULL `status` discards these reports.
 *   - Layouts are row-major and contiguous.  "[R, T, H]" means R*T*H elements,
 *     the last index fastest.  bf16 data is passed as raw 16-bit patterns
 *     (void*), e4m3 data as bytes.
 *
 * Notation: R ranks (every rank is a source and a destination), T tokens per
 * source rank, H hidden size, K top-k slots per token, E experts in total,
 * E_l = E / R experts per rank (expert e lives on rank e / E_l, local id
 * e % E_l), cap = rows per destination rank in the normal receive buffer.
 *
 * Limits (from the get_dispatch_layout specification: 1 <= K <= 16,
 * 1 <= E <= 512 with E % R == 0, R <= 384): calls outside them return
 * EP_ERR_INVALID_ARG.
 */
#ifndef EP_H_
#define EP_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

/* Host-side return codes. */
#define EP_OK               0  /* launched                                   */
#define EP_ERR_INVALID_ARG  1  /* a size, pointer or alignment check failed  */
#define EP_ERR_CUDA         2  /* the CUDA runtime reported a launch error   */
#define EP_ERR_UNSUPPORTED  3  /* valid call, shape the library cannot run   */

/* Device-side status bits, OR-ed into `status`. */
#define EP_STATUS_BAD_EXPERT       1  /* a top-k id outside [-1, E); slot ignored      */
#define EP_STATUS_CAPACITY         2  /* a copy's row >= cap; copy not written         */
#define EP_STATUS_WAIT_TIMEOUT     4  /* a bounded wait ran out; results are invalid   */
#define EP_STATUS_BAD_POSITION     8  /* a send_pos / ll_pos entry outside its buffer  */

/* Flags of ep_ll_dispatch (fp8_flags). */
#define EP_LL_FP8          1  /* e4m3 payload with one scale per 128 channels      */
#define EP_LL_ROUND_SCALE  2  /* scales rounded up to powers of two (needs FP8)    */
#define EP_LL_UE8M0        4  /* scales stored as UE8M0 exponent bytes (needs
                                 ROUND_SCALE): value 2^(byte - 127)              */

/* Debug flags for ep_set_debug_flags(). */
#define EP_DEBUG_SUPPRESS_PUBLISH  1u /* scan tiles publish nothing, so every tile but
                                         the first waits until its limit runs out:
                                         exercises EP_STATUS_WAIT_TIMEOUT            */

/* Text for a host return code. */
EP_API const char *ep_status_string(int code);

/* Library version (major * 10000 + minor * 100 + patch). */
EP_API int ep_version(void);

/* Process-wide limit of every bounded device wait, in nanoseconds of
 * %globaltimer (default 1e9, i.e. one second).  Applies to launches issued
 * after the call.  Returns EP_ERR_INVALID_ARG for a negative value. */
EP_API int ep_set_wait_timeout_ns(long long ns);

/* Process-wide debug flags (EP_DEBUG_*); 0 restores normal operation. */
EP_API int ep_set_debug_flags(unsigned flags);

/*
 * Opt-in full-grid phase timers of the single-GPU entry points.
 * Passage: DeepEP PR #720 page, "Notify full-kernel duration": thread 0 of
 * every block publishes its %globaltimer at entry, a complemented atomicMax
 * keeps the earliest block start, and the last block to complete records the
 * interval from that start to its own completion and counts the launch.
 * Here a phase may span chained kernels: it starts at the earliest block of
 * its first kernel (after that kernel's wait for the previous grid in the
 * stream) and ends at the last block of its last kernel.
 *
 *   timers      device memory, 8-byte aligned, num_phases x 8 uint64 (zeroed
 *               by the caller before the first timed launch), or NULL to turn
 *               the timers off.  Phase p owns timers[8p .. 8p+7]:
 *                 p = 0  notify (ep_notify_dispatch, and the notify half of
 *                        ep_dispatch / ep_dispatch_noalloc): zeroing, scan and
 *                        finish kernels;
 *                 p = 1  row copy (ep_dispatch_cached, ep_dispatch_cached_fp8,
 *                        the copy half of ep_dispatch / ep_dispatch_noalloc);
 *                 p = 2  combine (ep_combine);
 *                 p = 3  LL dispatch (ep_ll_dispatch): zeroing, scan and the
 *                        dispatch kernel that runs beside the scan;
 *                 p = 4  LL combine (ep_ll_combine);
 *               [8p+0] and [8p+1] are working slots (the complemented earliest
 *               start and the finished-block count of the launch in progress;
 *               each launch returns them to 0), [8p+2] the cumulative duration
 *               in ns, [8p+3] the number of phases timed, [8p+4] and [8p+5] the
 *               last phase's start and end (%globaltimer ns).
 *   num_phases  1..5: phases p >= num_phases are not timed (ignored for NULL).
 *
 * Process-wide; read when a call launches its kernels, so it applies to the
 * calls issued after it (a CUDA graph keeps what its capture saw).  The
 * sharded (ep_shard_*) entry points never time.  Phases of one timer must not
 * overlap: time one stream.  The memory must stay valid while calls that saw
 * it may still run.  Returns EP_ERR_INVALID_ARG for a pointer that is not
 * 8-byte aligned or num_phases outside 1..5.
 */
EP_API int ep_set_phase_timers(unsigned long long *timers, int num_phases);

/*
 * A1: get_dispatch_layout.
 * Passage: the get_dispatch_layout API (GET_DISPATCH_LAYOUT_API page,
 * "Parameters" and "Return Values"; DeepEP "Python 接口" page, Dispatch API
 * inputs num_tokens_per_rank, is_token_in_rank, num_tokens_per_expert).
 *
 *   topk_idx               in  int64 [S, T, K]; -1 marks an unselected slot
 *   num_src_ranks (S)      source ranks whose tokens are in topk_idx (S >= 1;
 *                          S = 1 is the pages' single-rank call)
 *   num_tokens (T) >= 0, num_topk (K), num_experts (E), num_ranks (R)
 *   num_tokens_per_rank    out int32 [S, R]: tokens of s with >= 1 expert on d
 *   num_tokens_per_expert  out int32 [S, E]: slots of s that select e
 *   is_token_in_rank       out uint8 [S, T, R]: 1 if (s,t) goes to d, else 0
 *
 * A repeated expert in one token counts twice in num_tokens_per_expert and
 * once in is_token_in_rank.  Ids outside [-1, E) are ignored and reported as
 * EP_STATUS_BAD_EXPERT.
 */
EP_API int ep_get_dispatch_layout(const int64_t *topk_idx, int num_src_ranks,
                                  int num_tokens, int num_topk, int num_experts,
                                  int num_ranks, int32_t *num_tokens_per_rank,
                                  int32_t *num_tokens_per_expert,
                                  uint8_t *is_token_in_rank, int32_t *status,
                                  cudaStream_t stream);

/* Workspace bytes ep_dispatch needs for R ranks, T tokens and E experts. */
EP_API size_t ep_dispatch_workspace_bytes(int num_ranks, int num_tokens,
                                          int num_experts);

/*
 * A2 + A3: rank prefix matrix, positions, and the dispatch scatter.
 * Passage: Buffer.dispatch (DeepEP "Python 接口" page, Dispatch API inputs
 * and outputs; intranode handle tuple and check_data's inclusive
 * recv_gbl_rank_prefix_sum walk on the DeepEP legacy-test analysis page).
 *
 * Inputs:
 *   x                  bf16 [R, T, H], H % 8 == 0, 16-byte aligned
 *   topk_idx           int64 [R, T, K] or NULL (then is_token_in_rank is
 *                      required and no metadata or expert counts are written)
 *   topk_weights       fp32 [R, T, K] or NULL
 *   is_token_in_rank   uint8 [R, T, R] or NULL.  If given it decides which
 *                      ranks receive each token (topk_idx then only fills the
 *                      received metadata); if NULL the routing is computed
 *                      from topk_idx (rank of each valid slot's expert).
 *   expert_alignment   >= 1; capacity (cap) >= 0 rows per destination rank
 *                      (cap = R*T can never overflow)
 * Outputs (rows of destination d are numbered by source rank, then token):
 *   recv_x             bf16 [R, cap, H]: row p of d = x of the p-th token
 *                      d receives.  Rows >= recv_count[d] are not touched.
 *   recv_topk_idx      int64 [R, cap, K] or NULL: local expert id (e - d*E_l)
 *                      for slots whose expert lives on d, else -1
 *   recv_topk_weights  fp32 [R, cap, K] or NULL: the weight for local slots,
 *                      else 0.0 (needs topk_weights)
 *   recv_src_idx       int32 [R, cap]: source token index t of each row
 *   rank_prefix_matrix int32 [R, R]: P[s][d] = tokens ranks 0..s send to d
 *   recv_count         int32 [R]: P[R-1][d]
 *   num_recv_tokens_per_expert int32 [R, E_l] or NULL: slots received per
 *                      local expert, rounded up to expert_alignment (needs
 *                      topk_idx)
 *   send_pos           int32 [R, T, R]: row of (s,t) inside d, or -1.
 *                      (rank_prefix_matrix, recv_src_idx, is_token_in_rank,
 *                      send_pos and recv_count form the dispatch handle.)
 *   workspace          ep_dispatch_workspace_bytes(R, T, E) bytes, any content
 * A copy whose row is >= cap is not written and sets EP_STATUS_CAPACITY;
 * send_pos still holds its row.  With a fixed capacity this is the pages'
 * num_worst_tokens mode: recv_topk_idx rows from recv_count[d] to cap - 1 read
 * -1 (DeepEP legacy-test analysis page, the num_worst_tokens check), and no
 * count has to travel to the host.  ep_dispatch = ep_notify_dispatch followed
 * by ep_dispatch_cached on the handle it produced.
 */
EP_API int ep_dispatch(const void *x, const int64_t *topk_idx,
                       const float *topk_weights,
                       const uint8_t *is_token_in_rank, int num_ranks,
                       int num_tokens, int hidden, int num_topk,
                       int num_experts, int expert_alignment, int capacity,
                       void *recv_x, int64_t *recv_topk_idx,
                       float *recv_topk_weights, int32_t *recv_src_idx,
                       int32_t *rank_prefix_matrix, int32_t *recv_count,
                       int32_t *num_recv_tokens_per_expert, int32_t *send_pos,
                       void *workspace, size_t workspace_bytes,
                       int32_t *status, cudaStream_t stream);

/*
 * A2 + received metadata: the first half of ep_dispatch (the notify step of
 * the pages' dispatch, reduced to a prefix scan because all ranks share one
 * HBM).  Arguments, outputs and rules are ep_dispatch's, without x and
 * recv_x; it computes the handle (send_pos, rank_prefix_matrix, recv_count,
 * recv_src_idx), recv_topk_idx / recv_topk_weights and
 * num_recv_tokens_per_expert.
 *
 * Optionally, when the routing comes from topk_idx (is_token_in_rank NULL),
 * the same kernel also returns the layout of ep_get_dispatch_layout for all
 * R source ranks (A1 fused into A2): num_tokens_per_rank int32 [R, R],
 * num_tokens_per_expert int32 [R, E], is_token_in_rank_out uint8 [R, T, R];
 * each may be NULL.  Requesting them with is_token_in_rank given returns
 * EP_ERR_INVALID_ARG.
 */
EP_API int ep_notify_dispatch(const int64_t *topk_idx, const float *topk_weights,
                              const uint8_t *is_token_in_rank, int num_ranks,
                              int num_tokens, int num_topk, int num_experts,
                              int expert_alignment, int capacity,
                              int64_t *recv_topk_idx, float *recv_topk_weights,
                              int32_t *recv_src_idx, int32_t *rank_prefix_matrix,
                              int32_t *recv_count,
                              int32_t *num_recv_tokens_per_expert,
                              int32_t *send_pos, int32_t *num_tokens_per_rank,
                              int32_t *num_tokens_per_expert,
                              uint8_t *is_token_in_rank_out, void *workspace,
                              size_t workspace_bytes, int32_t *status,
                              cudaStream_t stream);

/*
 * A3 rows: cached-mode dispatch.  Passage: Buffer.dispatch with a handle
 * (DeepEP "Python 接口" page, Dispatch API, cached mode: the layout step is
 * skipped and only recv_x is returned; legacy-test analysis page, the cached
 * re-dispatch check that reproduces recv_x).
 *
 *   x         bf16 [R, T, H] (H % 8 == 0, 16-byte aligned)
 *   send_pos  int32 [R, T, R] from ep_dispatch / ep_notify_dispatch
 *   recv_x    out bf16 [R, cap, H]: row send_pos[s][t][d] of d = x[s][t]
 * Only the rows named by send_pos are written; entries >= cap are skipped
 * and set EP_STATUS_CAPACITY.
 */
EP_API int ep_dispatch_cached(const void *x, const int32_t *send_pos,
                              int num_ranks, int num_tokens, int hidden,
                              int capacity, void *recv_x, int32_t *status,
                              cudaStream_t stream);

/*
 * A3 rows for FP8 input (the pages' x = (x_e4m3, x_scales) form; DeepEP
 * "Python 接口" page, Dispatch API, FP8 tuple input; legacy-test analysis
 * page, the column-major scale layout prepared for TMA).  Cached mode: the
 * handle comes from ep_notify_dispatch (FP8 dispatch = ep_notify_dispatch +
 * this call).
 *
 *   x_e4m3            e4m3 bytes [R, T, H], H % 128 == 0, 16-byte aligned
 *   x_scales          fp32 per 128 channels: [R, T, H/128] (row-major) or,
 *                     with scales_col_major = 1, [R, H/128, T]
 *   recv_x            out e4m3 [R, cap, H]; recv_scales out fp32
 *                     [R, cap, H/128] (row-major)
 * Bytes are copied unchanged.
 */
EP_API int ep_dispatch_cached_fp8(const void *x_e4m3, const float *x_scales,
                                  int scales_col_major, const int32_t *send_pos,
                                  int num_ranks, int num_tokens, int hidden,
                                  int capacity, void *recv_x,
                                  float *recv_scales, int32_t *status,
                                  cudaStream_t stream);

/*
 * ep_dispatch without a workspace argument.  The routing method has no
 * counterpart of this call: it exists for callers that cannot allocate device
 * memory when they call -- a host program whose device memory belongs to
 * another allocator, or a latency-critical loop that cannot afford
 * cudaMalloc/cudaFree (they can synchronise the device).
 *
 * Arguments, outputs and results are those of ep_dispatch; its argument
 * checks come first (an invalid call returns EP_ERR_INVALID_ARG whatever its
 * size).  The scratch lives in a 2 MiB static device array inside the
 * library, held on every GPU that loads the library until the process exits;
 * this call allocates nothing.  Calls needing more than that
 * (ep_dispatch_workspace_bytes(R, T, E) > 2 MiB, with E = 0 when topk_idx is
 * NULL) return EP_ERR_UNSUPPORTED.
 * The first call on a device, with that device current, looks up the array's
 * device address (cudaGetSymbolAddress); make that first call before any
 * stream capture.  Later calls outside stream capture look it up again (so a
 * device reset, after which the array may sit elsewhere, does no harm); a call
 * whose stream is capturing uses the address of the last call outside capture.
 * Every call on a device shares the array and it keeps the last call's
 * contents (the call clears what it uses on `stream` first): calls that
 * overlap on the GPU, e.g. on two streams at once, race on it.
 */
EP_API int ep_dispatch_noalloc(const void *x, const int64_t *topk_idx,
                               const float *topk_weights,
                               const uint8_t *is_token_in_rank, int num_ranks,
                               int num_tokens, int hidden, int num_topk,
                               int num_experts, int expert_alignment,
                               int capacity, void *recv_x,
                               int64_t *recv_topk_idx,
                               float *recv_topk_weights,
                               int32_t *recv_src_idx,
                               int32_t *rank_prefix_matrix,
                               int32_t *recv_count,
                               int32_t *num_recv_tokens_per_expert,
                               int32_t *send_pos, int32_t *status,
                               cudaStream_t stream);

/*
 * A4: combine (gather-reduce).
 * Passage: Buffer.combine (DeepEP legacy-test analysis page, combine_args and
 * the check that (combined_x - bias) / is_token_in_rank.sum(1) equals x).
 *
 *   y                      bf16 [R, cap, H], the experts' outputs, row for row
 *                          as ep_dispatch laid out recv_x (identity experts:
 *                          y = recv_x); H % 8 == 0, 16-byte aligned
 *   recv_topk_weights      fp32 [R, cap, K] or NULL
 *   send_pos               int32 [R, T, R] from ep_dispatch
 *   bias_0, bias_1         bf16 [R, T, H] or NULL (the pages' bias tuple),
 *                          16-byte aligned
 *   combined_x             out bf16 [R, T, H]:
 *                          bf16_rne( sum over d ascending with send_pos >= 0
 *                          of float(y[d][send_pos]), then + bias_0, then +
 *                          bias_1 ), fp32 accumulation from +0.0; a token with
 *                          no destination gives +0.0 (+ its biases)
 *   combined_topk_weights  out fp32 [R, T, K] or NULL: the same ascending sum
 *                          of recv_topk_weights (needs recv_topk_weights)
 * A send_pos entry outside [-1, cap) is skipped and sets
 * EP_STATUS_BAD_POSITION.
 */
EP_API int ep_combine(const void *y, const float *recv_topk_weights,
                      const int32_t *send_pos, const void *bias_0,
                      const void *bias_1, int num_ranks, int num_tokens,
                      int hidden, int num_topk, int capacity, void *combined_x,
                      float *combined_topk_weights, int32_t *status,
                      cudaStream_t stream);

/* Workspace bytes ep_ll_dispatch needs for R ranks, T tokens, E experts. */
EP_API size_t ep_ll_workspace_bytes(int num_ranks, int num_tokens,
                                    int num_experts);

/*
 * A5: low-latency dispatch with fused FP8 quantisation.
 * Passage: Buffer.low_latency_dispatch (DeepEP legacy-test analysis page, the
 * low_latency_dispatch call, its handle (recv_src_info, recv_layout_range)
 * and its per-expert count and per-source-rank checks; FP8 input described on
 * the "Python 接口" page as e4m3 values with fp32 scales per 128 channels).
 *
 * Each (token, expert) pair gets one row of that expert's slab; rows are
 * ordered by source rank, then token.  Slabs hold R*T rows, so they never
 * overflow.
 *   x              bf16 [R, T, H]; H % 128 == 0 for FP8, H % 8 == 0 for bf16
 *   topk_idx       int64 [R, T, K]
 *   rank_mask      int32 [R] or NULL: non-zero marks a failed rank (the pages'
 *                  shrink mode, low_latency_query_mask_buffer): a failed source
 *                  rank sends nothing, and slots whose expert lives on a
 *                  failed rank are dropped (ll_pos -1, not counted)
 *   fp8_flags      0: recv_x is bf16 [R, E_l, R*T, H], recv_scales unused;
 *                  EP_LL_FP8: recv_x is e4m3 [R, E_l, R*T, H] and recv_scales
 *                  fp32 [R, E_l, R*T, H/128] with, per 128-channel block,
 *                  amax' = max(max|x|, 1e-4), q = e4m3_rne_satfinite(x *
 *                  (448 / amax')), scale = amax' / 448;
 *                  | EP_LL_ROUND_SCALE: scale = the smallest power of two
 *                  >= amax' / 448 and q = e4m3(x * (1 / scale)) (exact
 *                  reciprocal); | EP_LL_UE8M0: recv_scales is uint8
 *                  [R, E_l, R*T, H/128] holding each scale's biased exponent
 *   recv_count     out int32 [R, E_l]: rows of each local expert
 *   recv_src_info  out int32 [R, E_l, R*T]: source token index of each row
 *   layout_range   out int32 [R, E_l, R, 2]: (first row, rows) per source rank
 *   ll_pos         out int32 [R, T, K]: slab row of each slot, -1 if the slot
 *                  is unselected, invalid or dropped (a repeated expert in a
 *                  token shares its first slot's row)
 *   cumulative_local_expert_recv_stats  int32 [R, E_l] or NULL: each call adds
 *                  its recv_count (the pages' cumulative per-expert counter)
 *   workspace      ep_ll_workspace_bytes(R, T, E) bytes, any content
 * H is limited by shared memory (at least two bf16 input rows staged per
 * CTA): H <= 57792 (FP8: H <= 57728, a multiple of 128); larger returns
 * EP_ERR_UNSUPPORTED.
 */
EP_API int ep_ll_dispatch(const void *x, const int64_t *topk_idx,
                          const int32_t *rank_mask, int num_ranks,
                          int num_tokens, int hidden, int num_topk,
                          int num_experts, int fp8_flags, void *recv_x,
                          void *recv_scales, int32_t *recv_count,
                          int32_t *recv_src_info, int32_t *layout_range,
                          int32_t *ll_pos,
                          int32_t *cumulative_local_expert_recv_stats,
                          void *workspace, size_t workspace_bytes,
                          int32_t *status, cudaStream_t stream);

/*
 * A6: low-latency combine with top-k weights.
 * Passage: Buffer.low_latency_combine (DeepEP legacy-test analysis page, the
 * low_latency_combine call and the check that the result equals x times the
 * sum of the top-k weights with unselected slots masked to 0).
 *
 *   y              bf16 [R, E_l, R*T, H], the experts' outputs laid out as
 *                  ep_ll_dispatch laid out its slabs; H % 8 == 0
 *   topk_idx, topk_weights  int64 / fp32 [R, T, K]
 *   ll_pos         int32 [R, T, K] from ep_ll_dispatch
 *   rank_mask      int32 [R] or NULL: slots of failed source ranks and slots
 *                  whose expert lives on a failed rank contribute nothing
 *   out            bf16 [R, T, H]: bf16_rne(acc), acc = +0.0 then, for k
 *                  ascending over valid slots, acc = fmaf(float(y[e][ll_pos]),
 *                  w[k], acc)
 * A slot with ll_pos -1 (dropped at dispatch) contributes nothing; a valid
 * expert with ll_pos outside [-1, R*T) is skipped and sets
 * EP_STATUS_BAD_POSITION.
 */
EP_API int ep_ll_combine(const void *y, const int64_t *topk_idx,
                         const float *topk_weights, const int32_t *ll_pos,
                         const int32_t *rank_mask, int num_ranks,
                         int num_tokens, int hidden, int num_topk,
                         int num_experts, void *out, int32_t *status,
                         cudaStream_t stream);

/* ==========================================================================
 * One rank per GPU (sharded job).
 *
 * Passage: the Buffer of the DeepEP "Python 接口" page ("Distributed /
 * ProcessGroup"): every rank allocates its communication buffer, the ranks
 * all-gather device ids and IPC handles over a torch.distributed group, and
 * each rank then writes into its peers' buffers directly; the dispatch notify
 * step exchanges per-rank token counts before the data moves (DeepEP PR #720
 * page, "Notify full-kernel duration", non-cached dispatch notify).
 *
 * Here each process holds ONE source rank `rank` of R, with its T tokens.
 * The path of one dispatch + combine:
 *   1. ep_get_dispatch_layout on the rank's own tokens (S = 1): its row of
 *      num_tokens_per_rank [R] and num_tokens_per_expert [E];
 *   2. the caller all-gathers those rows over its process group into
 *      counts [R, R] and expert_counts [R, E] (the notify exchange);
 *   3. ep_shard_notify: rank prefix matrix, this rank's send positions, and
 *      the received metadata written into every destination's buffers;
 *   4. ep_shard_dispatch: the token rows written into the destinations'
 *      receive buffers;
 *   5. a cross-rank synchronisation by the caller (a collective on the
 *      stream, or stream sync + barrier) before receive buffers are read;
 *   6. ep_shard_combine: each rank gathers its tokens' rows back from the
 *      destinations' expert outputs and reduces them exactly as ep_combine
 *      (fp32, ascending destination rank, one rounding), so the results are
 *      bit-identical to the single-GPU path on the same inputs;
 *   7. a synchronisation before any rank overwrites buffers peers still read.
 * No kernel waits on another rank: all cross-rank ordering is the caller's
 * synchronisation.  Peers' memory is written with plain and bulk (TMA)
 * stores and read with plain loads; no multicast form is used.
 *
 * "Peer tables" are DEVICE arrays of R device pointers, entry d pointing at
 * rank d's buffer as mapped in this process (this rank's own buffer at entry
 * `rank`), built once from ep_ipc_open.
 * ========================================================================== */

#define EP_IPC_HANDLE_BYTES 64

/* Allocate `bytes` of device memory on the current device for buffers that
 * peers map (zeroed; a plain cudaMalloc allocation, so its IPC handle covers
 * it from its first byte).  The one allocating call of the library; it
 * synchronises the device.  Free with ep_shard_free. */
EP_API int ep_shard_alloc(size_t bytes, void **ptr);
EP_API int ep_shard_free(void *ptr);

/* The IPC handle (EP_IPC_HANDLE_BYTES host bytes) of an allocation made by
 * ep_shard_alloc, for the other ranks of the job. */
EP_API int ep_ipc_handle(const void *ptr, void *handle);

/* Map another process's allocation from its handle (peer access enabled
 * lazily); *ptr is its first byte in this process.  A handle cannot be opened
 * in the process that made it.  Unmap with ep_ipc_close. */
EP_API int ep_ipc_open(const void *handle, void **ptr);
EP_API int ep_ipc_close(void *ptr);

/* Workspace bytes of ep_shard_notify for R ranks and T tokens on this rank. */
EP_API size_t ep_shard_workspace_bytes(int num_ranks, int num_tokens);

/*
 * Notify + received metadata of one rank of a sharded job.
 *
 *   topk_idx, topk_weights  int64 / fp32 [T, K], this rank's tokens
 *   counts            int32 [R, R]: counts[s][d] = tokens rank s sends to d
 *                     (every rank's num_tokens_per_rank row, gathered)
 *   expert_counts     int32 [R, E] (every rank's num_tokens_per_expert) or
 *                     NULL (then num_recv_tokens_per_expert must be NULL)
 *   rank              this process's rank, 0 <= rank < R
 *   recv_src_idx_peers     peer table of int32 [cap] receive buffers
 *   recv_topk_idx_peers    peer table of int64 [cap, K] buffers, or NULL
 *   recv_topk_weights_peers peer table of fp32 [cap, K] buffers, or NULL
 *   recv_topk_idx     this rank's own int64 [cap, K] buffer (entry `rank` of
 *                     recv_topk_idx_peers; NULL iff that table is NULL): its
 *                     rows from recv_count to cap - 1 are set to -1
 * Outputs (this rank's device memory):
 *   rank_prefix_matrix int32 [R, R], P[s][d] = sum over s' <= s of counts
 *   recv_count        int32 [1]: rows this rank receives, P[R-1][rank]
 *   num_recv_tokens_per_expert int32 [E_l] or NULL: slots this rank's
 *                     experts receive, rounded up to expert_alignment
 *   send_pos          int32 [T, R]: row of (rank, t) in destination d
 *                     (P[rank-1][d] + earlier tokens of this rank to d), or -1
 *   notify_probe      uint64 [4] or NULL: a full-grid timer of the notify
 *                     scan kernel, from the earliest block start to the
 *                     last block end in %globaltimer ns: [0] += duration,
 *                     [1] += 1 launch, [2] = that launch's earliest start,
 *                     [3] = its end (absolute ns; comparing [2] across
 *                     ranks shows their arrival skew).  Zero it once.
 * In the destinations' buffers (rows in rank order, then token order, as the
 * single-GPU path numbers them): recv_src_idx = t, recv_topk_idx = local
 * expert id or -1, recv_topk_weights = weight or 0.0.  Rows >= cap are not
 * written and set EP_STATUS_CAPACITY.
 */
EP_API int ep_shard_notify(const int64_t *topk_idx, const float *topk_weights,
                           const int32_t *counts, const int32_t *expert_counts,
                           int rank, int num_ranks, int num_tokens, int num_topk,
                           int num_experts, int expert_alignment, int capacity,
                           int32_t *const *recv_src_idx_peers,
                           int64_t *const *recv_topk_idx_peers,
                           float *const *recv_topk_weights_peers,
                           int64_t *recv_topk_idx, int32_t *rank_prefix_matrix,
                           int32_t *recv_count,
                           int32_t *num_recv_tokens_per_expert,
                           int32_t *send_pos, unsigned long long *notify_probe,
                           void *workspace, size_t workspace_bytes,
                           int32_t *status, cudaStream_t stream);

/*
 * Rows of one rank of a sharded job: x bf16 [T, H] (H % 8 == 0, 16-byte
 * aligned); row t goes to row send_pos[t][d] of rank d's bf16 [cap, H]
 * receive buffer (peer table recv_x_peers), for every d with a position.
 */
EP_API int ep_shard_dispatch(const void *x, const int32_t *send_pos,
                             int num_ranks, int num_tokens, int hidden,
                             int capacity, void *const *recv_x_peers,
                             int32_t *status, cudaStream_t stream);

/*
 * Combine of one rank of a sharded job: combined_x bf16 [T, H] =
 * bf16_rne(sum over d ascending with send_pos[t][d] >= 0 of
 * float(y_d[send_pos[t][d]]), + bias_0, + bias_1), y_d rank d's bf16
 * [cap, H] expert outputs (peer table y_peers); combined_topk_weights fp32
 * [T, K] (or NULL) the same sum over the peers' recv_topk_weights rows.
 */
EP_API int ep_shard_combine(const void *const *y_peers,
                            const float *const *recv_topk_weights_peers,
                            const int32_t *send_pos, const void *bias_0,
                            const void *bias_1, int num_ranks, int num_tokens,
                            int hidden, int num_topk, int capacity,
                            void *combined_x, float *combined_topk_weights,
                            int32_t *status, cudaStream_t stream);

/* --------------------------------------------------------------------------
 * The low-latency pair, one rank per GPU.
 *
 * Passage: the legacy-test page's low_latency_dispatch / low_latency_combine
 * (per-expert slabs [E_l, R * T, H], the handle (recv_src_info,
 * recv_layout_range), per-expert counts) and, for the exchange, the sharding
 * of the Buffer as above.  Each process holds source rank `rank`'s T tokens
 * and, as destination `rank`, the slabs of its E_l = E / R experts:
 *   1. ep_shard_ll_counts: counts[E] = rows this rank sends to each expert;
 *   2. the caller all-gathers them into counts [R, E];
 *   3. ep_shard_ll_dispatch: positions, quantised rows and handle entries
 *      written into every destination's slabs (through the peer tables);
 *   4. a cross-rank synchronisation by the caller; experts run on their slabs;
 *   5. ep_shard_ll_combine: each rank reads its tokens' rows back from the
 *      destinations' expert-output slabs and takes the weighted sum.
 * Every output equals the single-GPU ep_ll_dispatch / ep_ll_combine on the
 * stacked inputs, restricted to the rank: ll_pos rows of source `rank`, the
 * slab rows, recv_src_info and layout_range of destination d in d's memory,
 * recv_count of the rank's own experts.  Slab rows are ordered by source rank,
 * then token, so rank r's rows of expert e follow those of ranks 0..r-1.
 *
 * Peer tables are device arrays of R device pointers, entry d = rank d's
 * buffer mapped in this process: recv_x_peers [R] -> e4m3 or bf16 [E_l, R*T, H];
 * recv_scales_peers [R] -> fp32 or UE8M0 bytes [E_l, R*T, H/128] (FP8 only);
 * recv_src_info_peers [R] -> int32 [E_l, R*T]; layout_range_peers [R] ->
 * int32 [E_l, R, 2]; y_peers [R] -> bf16 [E_l, R*T, H].  Nothing here waits
 * for another rank's kernels.  rank_mask: as in ep_ll_dispatch (nullable).
 * ========================================================================== */

/* counts [E] int32, written (zeroed first) with this rank's rows per expert:
 * its tokens whose distinct valid slots hold the expert, none if `rank`
 * fails, none to a failed rank's experts.  topk_idx [T, K] int64. */
EP_API int ep_shard_ll_counts(const int64_t *topk_idx, const int32_t *rank_mask,
                              int rank, int num_ranks, int num_tokens,
                              int num_topk, int num_experts, int32_t *counts,
                              int32_t *status, cudaStream_t stream);

/* Workspace bytes of ep_shard_ll_dispatch (any content). */
EP_API size_t ep_shard_ll_workspace_bytes(int num_ranks, int num_tokens,
                                          int num_experts);

/* x bf16 [T, H] (16-byte aligned), topk_idx int64 [T, K], counts int32
 * [R, E] (every rank's ep_shard_ll_counts, in rank order).  fp8_flags as in
 * ep_ll_dispatch.  Writes through the peer tables (see above); locally
 * recv_count int32 [E_l] (rows received by this rank's experts), ll_pos int32
 * [T, K] (slab row of each slot, -1 when dropped) and, if non-null,
 * cumulative_local_expert_recv_stats int32 [E_l] += recv_count.  Returns
 * before anything is launched on a bad argument. */
EP_API int ep_shard_ll_dispatch(const void *x, const int64_t *topk_idx,
                                const int32_t *rank_mask, const int32_t *counts,
                                int rank, int num_ranks, int num_tokens,
                                int hidden, int num_topk, int num_experts,
                                int fp8_flags, void *const *recv_x_peers,
                                void *const *recv_scales_peers,
                                int32_t *const *recv_src_info_peers,
                                int32_t *const *layout_range_peers,
                                int32_t *recv_count, int32_t *ll_pos,
                                int32_t *cumulative_local_expert_recv_stats,
                                void *workspace, size_t workspace_bytes,
                                int32_t *status, cudaStream_t stream);

/* out bf16 [T, H] (16-byte aligned): for each token, sum over its slots k in
 * ascending order of fmaf(y[row of slot k], topk_weights[k], acc), one bf16
 * rounding, where the rows are read from y_peers (the destinations'
 * expert-output slabs) at ll_pos.  topk_weights fp32 [T, K]. */
EP_API int ep_shard_ll_combine(const void *const *y_peers, const int64_t *topk_idx,
                               const float *topk_weights, const int32_t *ll_pos,
                               const int32_t *rank_mask, int rank, int num_ranks,
                               int num_tokens, int hidden, int num_topk,
                               int num_experts, void *out, int32_t *status,
                               cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* EP_H_ */
