/*
 * ep_a2a.h — C ABI of libep_a2a.so: rank-major MoE expert-parallel token
 * dispatch and combine for one NVIDIA B200 (sm_100a), all EP ranks virtual.
 *
 * Every EP rank is a virtual rank whose receive arrays live in one GPU's HBM,
 * inside one caller-owned workspace.  A "send" from rank src to rank d is a
 * copy into rank d's slice of that workspace.  All entry points take plain
 * pointers and sizes; device pointers are CUDA device addresses on the current
 * device, host pointers are ordinary process memory.  No entry point allocates
 * device memory, and none throws: each returns an ep_a2a_status, and on failure
 * ep_a2a_last_error() gives a one-line message (per calling thread).
 *
 * GPU work is enqueued asynchronously on the caller's stream (a cudaStream_t
 * passed as void*; NULL = the legacy default stream).  Arguments are validated
 * synchronously on the host before anything is enqueued; a call that returns an
 * error has enqueued nothing.
 *
 * Sources (page title, then section):
 *   flashinfer.moe_ep.NVLinkOneSidedConfig — options paragraph
 *     (extra_payload_bytes_per_token, eplb_stats_num_experts, enable_rank_mask,
 *     use_low_precision_combine) and the `lamport` paragraph (slot
 *     src * tokens_per_rank + t; tokens_per_rank = runtime_max_tokens_per_rank).
 *   flashinfer.moe_ep.NVLinkTwoSidedAlltoAll — class constraints (num_experts a
 *     multiple of 4; the EPLB stats span every expert), dispatch(), combine(),
 *     destroy().
 *   flashinfer.comm.moe_a2a_dispatch — Parameters (token_selected_experts,
 *     input_payloads, workspace, runtime_max_tokens_per_rank, eplb_local_stats,
 *     enable_rank_mask, active_rank_mask) and Returns.
 *   vllm.distributed.device_communicators.all2all —
 *     FlashInferNVLinkTwoSidedManager.get_communication (invalid_expert_id =
 *     num_experts for received rows past a source's token count).
 */
#ifndef EP_A2A_H
#define EP_A2A_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Limits of this implementation. */
#define EP_A2A_MAX_RANKS 256          /* ep_size */
#define EP_A2A_RANK_MASK_WORDS 4      /* uint64 words of active_rank_mask */
#define EP_A2A_MAX_PAYLOADS 8         /* entries of the payload list */
#define EP_A2A_MAX_TOP_K 32

typedef struct ep_a2a_handle_s* ep_a2a_handle;   /* opaque, library-owned host object */

typedef enum {
  EP_A2A_OK = 0,
  EP_A2A_ERR_INVALID_ARG = 1,     /* a size, pointer or flag breaks a rule below */
  EP_A2A_ERR_CAPACITY = 2,        /* step larger than the capacity given at init */
  EP_A2A_ERR_UNSUPPORTED = 3,     /* beyond this implementation's limits */
  EP_A2A_ERR_CUDA = 4,            /* a CUDA runtime call failed (launch, device query) */
  EP_A2A_ERR_NOT_INITIALIZED = 5, /* NULL or destroyed handle */
  EP_A2A_ERR_NO_PLAN = 6,         /* combine without a preceding dispatch */
  EP_A2A_ERR_DEVICE_TIMEOUT = 7,  /* a bounded wait inside a kernel ran out */
  EP_A2A_ERR_DEVICE_BOUNDS = 8    /* checked build (libep_a2a_checked.so, compiled with
                                     EP_A2A_CHECKS=1) only: a combine kernel found a
                                     plan entry in the workspace out of range (a
                                     destination rank >= ep_size or more destinations
                                     than the plan holds) and skipped that token */
} ep_a2a_status;

typedef enum {
  EP_A2A_COMBINE_BF16 = 0,        /* expert_output is bf16 */
  EP_A2A_COMBINE_FP8_E4M3 = 1     /* expert_output is E4M3 (fn), unscaled */
} ep_a2a_combine_dtype;

/*
 * Sizes fixed at init (the pages' MoEEpCommParams plus the one-sided config
 * options).  Capacity values bound every later step.
 */
typedef struct {
  int32_t ep_size;                /* 1..EP_A2A_MAX_RANKS */
  int32_t num_experts;            /* E: divisible by 4 (NVLinkTwoSidedAlltoAll) and by
                                     ep_size; expert e is owned by rank e / (E / ep_size) */
  int32_t top_k;                  /* 1..EP_A2A_MAX_TOP_K */
  int32_t max_tokens_per_rank;    /* capacity: largest runtime_max_tokens_per_rank */
  int32_t hidden_size;            /* elements per combine row (bf16 or E4M3) */
  int32_t num_payloads;           /* 0..EP_A2A_MAX_PAYLOADS dispatch payloads */
  int64_t payload_row_bytes[EP_A2A_MAX_PAYLOADS];  /* capacity of each payload's row,
                                     bytes (> 0): token rows, block scales, topk_weights,
                                     extra_payload_bytes_per_token, ... */
  int32_t eplb_stats_num_experts; /* 0 = no EPLB gather; else must equal num_experts */
  int32_t enable_rank_mask;       /* 0: every rank always active and no mask may be
                                     passed; 1: dispatch accepts active_rank_mask */
  int32_t invalid_expert_id;      /* id written into invalid received rows; < 0 means
                                     num_experts (no rank owns it) */
  int32_t reserved;               /* must be 0 */
} ep_a2a_params;

/*
 * Everything dispatch produced, as device pointers into the workspace (views of
 * the workspace, as the pages return them).  They stay valid, and keep their contents,
 * until the next dispatch on the same handle or its destruction.  Every
 * per-rank array of rank d sits at (rank-0 pointer + d * rank_stride_bytes).
 * Let tpr = tokens_per_rank and slot s = src * tpr + t.
 */
typedef struct {
  int32_t tokens_per_rank;        /* this step's runtime_max_tokens_per_rank */
  int32_t num_payloads;
  int64_t rank_stride_bytes;      /* bytes between consecutive ranks' arrays */
  void* recv_payloads[EP_A2A_MAX_PAYLOADS]; /* [ep*tpr, row_bytes_i]: row s = payload i of
                                     token t of rank src, for valid s; invalid rows are
                                     not written */
  int32_t* recv_topk_ids;         /* [ep*tpr, top_k]: the token's global ids for valid s,
                                     else invalid_expert_id in all top_k entries */
  uint8_t* recv_valid;            /* [ep*tpr]: 1 if row s was received, else 0 */
  int32_t* eplb_gathered_stats;   /* [ep, E] per rank: row r = rank r's eplb_local_stats
                                     (zeros for a masked-off r); NULL if not gathered */
  int32_t* send_counts;           /* [ep(src), ep(dst)]: tokens src sent to dst (one
                                     array, not per rank) */
  uint8_t* plan_num_dst;          /* [ep(src), tpr]: distinct destination ranks of token
                                     (src, t); 0xFF if the token does not exist */
  uint8_t* plan_dst_ranks;        /* [ep(src), tpr, plan_stride]: those ranks ascending;
                                     entries past plan_num_dst are 0xFF */
  int32_t plan_stride;            /* bytes per plan_dst_ranks row: top_k rounded up to 8 */
  int32_t reserved;
} ep_a2a_dispatch_result;

/*
 * Bytes of device workspace needed for `params` (flashinfer.comm.moe_a2a_dispatch,
 * Parameters, `workspace`: one workspace of [ep_size, size_per_rank] bytes; here
 * a control region followed by ep_size rank regions, each holding that rank's
 * receive arrays for ep_size * max_tokens_per_rank slots).  Host only; no CUDA
 * call.  INVALID_ARG / UNSUPPORTED when params break the rules of ep_a2a_params.
 */
ep_a2a_status ep_a2a_workspace_size(const ep_a2a_params* params, size_t* bytes);

/*
 * Bind a caller-owned device workspace (>= ep_a2a_workspace_size bytes, 256-byte
 * aligned) and create a handle.  The pages' moe_a2a_initialize / create_communication,
 * for all virtual ranks at once.  Clears the workspace's small control region on
 * `stream` (the caller keeps the workspace alive until ep_a2a_destroy).
 * The library owns the returned handle; free it with ep_a2a_destroy.
 */
ep_a2a_status ep_a2a_init(const ep_a2a_params* params, void* workspace,
                          size_t workspace_bytes, void* stream, ep_a2a_handle* out_handle);

/*
 * Dispatch (flashinfer.comm.moe_a2a_dispatch; NVLinkTwoSidedAlltoAll.dispatch()):
 * send each token of every live source rank, with all its payload rows, once to
 * every live rank owning any of its top_k experts, landing at slot
 * src * tokens_per_rank + t of that rank's receive arrays.
 *
 *   token_selected_experts  device int32 [ep, tpr, top_k]: global expert ids; an id
 *                           outside [0, E) is owned by no rank and not routed.
 *   local_num_tokens        host int32 [ep]: tokens of each rank, <= tpr.  Rows
 *                           t >= local_num_tokens[r] of the inputs are ignored.
 *   runtime_max_tokens_per_rank  tpr of this step, <= max_tokens_per_rank; <= 0
 *                           means max_tokens_per_rank.
 *   payloads                host array of num_payloads device pointers; payload i is
 *                           [ep, tpr, payload_row_bytes[i]] bytes, rank-major.  The
 *                           bytes are copied verbatim (no sentinel rewriting: NaN,
 *                           -0 and any other pattern arrive unchanged).
 *   payload_row_bytes       host int64 [num_payloads]: this step's row bytes
 *                           (<= the init capacity); NULL = the init values.
 *   num_payloads            <= the init num_payloads.
 *   eplb_local_stats        device int32 [ep, eplb_stats_num_experts], or NULL.
 *                           Must be NULL when init had eplb_stats_num_experts = 0.
 *   active_rank_mask        host uint64 [EP_A2A_RANK_MASK_WORDS] (bit r = rank r
 *                           alive), or NULL = all alive.  Needs enable_rank_mask and
 *                           at least one live rank below ep_size; bits >= ep_size are
 *                           ignored.  A masked-off rank neither sends nor receives:
 *                           tokens routed to it are dropped, its receive arrays are
 *                           not written, its tokens are not sent.
 *   result                  filled on success (pointers into the workspace).
 *
 * The routing plan is kept in the workspace for the next ep_a2a_combine.
 * Input buffers must stay untouched until the enqueued work has run.
 */
ep_a2a_status ep_a2a_dispatch(ep_a2a_handle handle, const int32_t* token_selected_experts,
                              const int32_t* local_num_tokens,
                              int32_t runtime_max_tokens_per_rank,
                              const void* const* payloads, const int64_t* payload_row_bytes,
                              int32_t num_payloads, const int32_t* eplb_local_stats,
                              const uint64_t* active_rank_mask, void* stream,
                              ep_a2a_dispatch_result* result);

/*
 * Combine (NVLinkTwoSidedAlltoAll.combine()): for each existing token (src, t) of
 * the last dispatch, out[src][t][:] = bf16 of the fp32 sum, in ascending
 * destination-rank order starting from +0.0f, of expert_output[d][src*tpr + t][:]
 * over the token's destination ranks d; one round-to-nearest-even at the end.
 * A token whose destinations were all masked off gets +0.0.
 *
 *   expert_output   device [ep, ep*tpr, hidden_size] of `dtype` (bf16 or E4M3):
 *                   row (d, s) is rank d's result for the token in slot s, its
 *                   experts' outputs with the routing weights applied and summed
 *                   on that rank.  Only rows of valid slots are read.  (hidden_size
 *                   is the handle's combine row length, see
 *                   ep_a2a_set_combine_hidden.)
 *   output          device bf16 [ep, tpr, hidden_size].  Rows of tokens that do
 *                   not exist (t >= local_num_tokens[src], masked-off src) are not
 *                   written.
 * NO_PLAN if no dispatch has run on this handle.
 */
ep_a2a_status ep_a2a_combine(ep_a2a_handle handle, const void* expert_output,
                             ep_a2a_combine_dtype dtype, void* output, void* stream);

/*
 * Combine of per-expert outputs: the step that makes the combine's input
 * (NVLinkTwoSidedAlltoAll.combine(): each rank's row is its own experts'
 * outputs, weighted and summed) fused into the combine, so the per-rank rows
 * are never written to memory.  For each existing token (src, t) of the last
 * dispatch:
 *   z_d = bf16( fp32 sum over the token's slots j whose expert rank d owns,
 *               ascending j, of topk_weights[j] * y[j] (one fused multiply-add
 *               per term, accumulator starting at +0.0f) )
 *   out[src][t] = bf16( fp32 sum of z_d over the token's destination ranks d in
 *                       ascending order, starting at +0.0f )
 * which equals ep_a2a_combine applied to the rows z.  Slots whose expert is
 * owned by no rank or by a masked-off rank take no part.
 *
 *   topk_weights            device fp32 [ep, tpr, top_k] (source layout)
 *   expert_output_per_slot  device bf16 [ep, tpr, top_k, hidden_size]: row
 *                           (src, t, j) = output of expert j of token t of src;
 *                           rows of slots that take no part are not read
 *   output                  device bf16 [ep, tpr, hidden_size]; rows of tokens that
 *                           do not exist are not written
 * The routing ids are the ones the last dispatch received (read from the
 * workspace).  NO_PLAN if no dispatch has run on this handle.
 */
ep_a2a_status ep_a2a_combine_experts(ep_a2a_handle handle, const float* topk_weights,
                                     const void* expert_output_per_slot, void* output,
                                     void* stream);

/*
 * Low-precision combine of per-expert outputs with the quantisation on the
 * sending side (flashinfer.moe_ep.NVLinkOneSidedConfig, use_low_precision_combine:
 * the combine rows travel as FP8; NVLinkTwoSidedAlltoAll.combine(): each rank's
 * row is its own experts' weighted outputs, summed).  For each existing token
 * (src, t) of the last dispatch and each destination rank d, in one kernel:
 *   z_d     = the row of ep_a2a_combine_experts (bf16, one fma per term)
 *   amax_d  = max |z_d|; scale_d = amax_d / 448, inv_d = 448 / amax_d (fp32,
 *             rounded to nearest; 1 and 1 for an all-zero row)
 *   q_d     = E4M3(z_d * inv_d), nearest even, saturating
 *   out[src][t] = bf16( acc ),  acc = fmaf(decode(q_d), scale_d, acc) over the
 *             token's destination ranks in ascending order, from +0.0f
 * which equals ep_a2a_quantize_e4m3_rows applied to the rows z_d followed by
 * ep_a2a_combine_scaled.  The rows, codes and scales are never written to
 * memory.  Arguments, layouts and errors as ep_a2a_combine_experts.
 */
ep_a2a_status ep_a2a_combine_experts_fp8(ep_a2a_handle handle, const float* topk_weights,
                                         const void* expert_output_per_slot, void* output,
                                         void* stream);

/*
 * FP8 helper (flashinfer.moe_ep.NVLinkOneSidedConfig, use_low_precision_combine):
 * e4m3_out[i] = E4M3(bf16_in[i]), round to nearest even, saturating to +-448.
 * Device pointers; n elements.  Not part of a dispatch / combine step.
 */
ep_a2a_status ep_a2a_quantize_e4m3(const void* bf16_in, void* e4m3_out, int64_t n,
                                   void* stream);

/*
 * FP8 combine with one scale per row (flashinfer.moe_ep.NVLinkOneSidedConfig,
 * use_low_precision_combine; the pages fix no scale convention, this is one):
 * as ep_a2a_combine with E4M3 rows, each row (d, s) also carrying an fp32 scale:
 *   out[src][t] = bf16( acc ),  acc = fmaf(decode(q[d][s]), row_scales[d][s], acc)
 * over the token's destination ranks d in ascending order, from +0.0f.
 *   expert_output_e4m3  device [ep, ep*tpr, hidden_size] E4M3 codes
 *   row_scales          device fp32 [ep, ep*tpr] (only valid rows are read)
 *   output              device bf16 [ep, tpr, hidden_size]
 */
ep_a2a_status ep_a2a_combine_scaled(ep_a2a_handle handle, const void* expert_output_e4m3,
                                    const float* row_scales, void* output, void* stream);

/*
 * Rows to E4M3 with one scale per row, the sender side of the scaled FP8
 * combine: per row of `hidden` bf16 values, amax = max |x|, scale = amax / 448
 * and inv = 448 / amax (fp32, rounded to nearest; 1 and 1 for an all-zero row),
 * code = E4M3(x * inv) rounded to nearest even and saturating.  Device
 * pointers: bf16_in [rows, hidden], e4m3_out [rows, hidden], row_scales [rows].
 */
ep_a2a_status ep_a2a_quantize_e4m3_rows(const void* bf16_in, void* e4m3_out, float* row_scales,
                                        int64_t rows, int32_t hidden, void* stream);

/*
 * Dense variant (vllm.distributed.device_communicators.all2all,
 * AgRsAll2AllManager: dispatch by all-gather, combine by reduce-scatter), for
 * comparison with the rank-major path on the same arrays; no handle, no plan.
 *
 * ep_a2a_allgather: every live rank receives every token of every live rank,
 * recv_payloads[i] + d * recv_rank_stride_bytes + (src * tpr + t) * row_bytes[i]
 * = payloads[i] + (src * tpr + t) * row_bytes[i] for live d, live src and
 * t < local_num_tokens[src].  local_num_tokens and active_rank_mask (NULL = all
 * live) are host arrays; payloads and recv_payloads are host arrays of device
 * pointers (rank 0's receive array per payload); other rows are not written.
 *
 * ep_a2a_reduce_scatter: out[src][t] = bf16( fp32 sum over live ranks d,
 * ascending, from +0.0f, of x[d][src * tpr + t] ) for live src and
 * t < local_num_tokens[src]; x is device bf16 [ep, ep*tpr, hidden], out device
 * bf16 [ep, tpr, hidden]; other rows are not written.
 */
ep_a2a_status ep_a2a_allgather(int32_t ep_size, int32_t tokens_per_rank,
                               const int32_t* local_num_tokens,
                               const uint64_t* active_rank_mask, const void* const* payloads,
                               const int64_t* payload_row_bytes, int32_t num_payloads,
                               void* const* recv_payloads, int64_t recv_rank_stride_bytes,
                               void* stream);
ep_a2a_status ep_a2a_reduce_scatter(int32_t ep_size, int32_t tokens_per_rank, int32_t hidden,
                                    const int32_t* local_num_tokens,
                                    const uint64_t* active_rank_mask, const void* x, void* out,
                                    void* stream);

/*
 * Synchronise `stream`, then read and clear the handle's device error word.
 * DEVICE_TIMEOUT if a kernel's bounded wait ran out since the last check;
 * DEVICE_BOUNDS (checked build only) if a kernel skipped an out-of-range index.
 */
ep_a2a_status ep_a2a_get_status(ep_a2a_handle handle, void* stream);

/*
 * Failure-detection check (the pages' timeout_sec bounds waits on peers,
 * flashinfer.moe_ep.NVLinkOneSidedConfig, `timeout_sec`; here a wait that runs
 * out returns an error status instead of trapping): enqueues one kernel whose
 * bounded wait on a shared-memory barrier can never complete; after limit_ns
 * (1..1e10) of GPU time it sets the handle's error word and returns, leaving the
 * context usable.  ep_a2a_get_status then reports EP_A2A_ERR_DEVICE_TIMEOUT.
 */
ep_a2a_status ep_a2a_debug_wait_probe(ep_a2a_handle handle, int64_t limit_ns, void* stream);

/* Tuning knobs of the kernels (performance only; results never change). */
typedef enum {
  EP_A2A_OPT_COPY_PATH = 0,       /* 1 = vector load/store copy for every payload
                                     (default); for rows that are 16-byte multiples at
                                     16-byte-aligned addresses: 0 = bulk-async loads into
                                     shared memory + vector stores, 2 = bulk-async loads
                                     and bulk-async stores (other rows take the vector
                                     copy) */
  EP_A2A_OPT_COPY_CTAS_PER_SM = 1,/* CTAs per SM of the bulk copy kernel (1..8) */
  EP_A2A_OPT_COPY_STAGES = 2,     /* shared-memory row stages per copy CTA (2..32; 0 = as
                                     many as fit, up to 8 / 16) */
  EP_A2A_OPT_COMBINE_THREADS = 3, /* threads per CTA of the combine kernels (64..512);
                                     0 (default) = automatic, from the combine kind and
                                     the token slots (64, 128 or 256) */
  EP_A2A_OPT_BULK_MIN_ROW_BYTES = 4, /* rows shorter than this take the vector copy (0..2^24) */
  EP_A2A_OPT_COMBINE_CTAS_PER_SM = 5, /* combine grid = min(tokens, SMs x this) (1..1024);
                                       0 (default) = automatic (16 or 128) */
  EP_A2A_OPT_COPY_CONSUMER_WARPS = 6, /* store warps per CTA of copy path 0 (4, 8 or 16) */
  EP_A2A_OPT_COPY_INTERLEAVE = 7, /* paths 0 and 2: 1 = CTA b copies tokens b, b + grid, ...
                                     (default); 0 = each CTA copies a contiguous chunk */
  EP_A2A_OPT_VEC_UNROLL = 8,      /* vector copy: vectors per lane in flight (2, 4, 8; 0 =
                                     default: the fewest that move the largest row in
                                     two rounds) */
  EP_A2A_OPT_VEC_CTAS_PER_SM = 9, /* vector copy grid = SMs x this (1..64); 0 (default) =
                                     automatic: 4 with at most 8 token slots per SM and
                                     256 threads per token, else 32 */
  EP_A2A_OPT_STORE_STREAMING = 10,/* vector copy: 1 = evict-first (.cs) stores
                                     (default), 0 = plain stores */
  EP_A2A_OPT_PDL = 11,            /* 1 (default): each kernel of the path may start while
                                     the one before it finishes (programmatic dependent
                                     launch; flashinfer.moe_ep.NVLinkOneSidedConfig,
                                     enable_pdl); each waits for its predecessor before
                                     it touches memory, so results do not change */
  EP_A2A_OPT_VEC_THREADS_PER_TOKEN = 12,/* vector copy: threads per token (32, 64, 128,
                                     256); 0 (default) = from the token count and the
                                     largest row */
  EP_A2A_OPT_COMBINE_PREFETCH = 13,/* combines: p in 1..4 = each CTA asks for the rows of
                                     its token p grid strides ahead to be brought into L2
                                     (cp.async.bulk.prefetch.L2) while it sums the current
                                     one; 0 = never; -1 (default) = automatic: 1 for the
                                     FP8 combines from 8192 token slots, the BF16
                                     combine from 8192 to 16383 and the sender-side FP8
                                     expert combine (its split kernel) from 8192, else 0 */
  EP_A2A_OPT_COPY_PREFETCH = 14,  /* vector copy: 1 = the same for the next token's rows;
                                     0 = never; -1 (default) = automatic: 1 where the
                                     automatic grid is 4 CTAs per SM, else 0 */
  EP_A2A_OPT_COMBINE_PIPELINE = 15,/* BF16 / FP8 / scaled FP8 combines of 16-byte vectors
                                     with at most 8 destinations per token (top_k or
                                     ep_size <= 8): 1 = each thread keeps the loads of its
                                     next column vector in flight while it adds the
                                     current one; 2 = the rows are staged in shared
                                     memory by bulk-async copies (4 KB chunks of every
                                     destination row, or slot row for the expert-output
                                     combine, per stage) and summed from there; 0 = one
                                     vector at
                                     a time; -1 (default) = 1 for the FP8, scaled FP8
                                     and expert-output combines, 0 for BF16 */
  EP_A2A_OPT_COPY_VEC_BYTES = 16, /* vector copy: widest access per thread, 16 or 32
                                     (default) bytes (sm_100 256-bit loads and stores,
                                     for rows and addresses that are 32-byte multiples) */
  EP_A2A_OPT_ROUTE_IN_COPY = 17,  /* vector copy path (COPY_PATH 1): 1 = the copy kernel
                                     also writes the routing plan, valid bytes, received
                                     ids, send counts and EPLB gather, so a dispatch is
                                     one kernel; 0 (default, measured faster) = a
                                     separate routing kernel runs first, beside the copy
                                     (the bulk paths always use it) */
  EP_A2A_OPT_FP8_EXPERTS_KERNEL = 18 /* ep_a2a_combine_experts_fp8 with top_k <= 8 and
                                     hidden a multiple of 8: 0 (default) = a cluster of
                                     CTAs per token, each a slice of the row with its
                                     rows z_d in shared memory, the row maxima exchanged
                                     through distributed shared memory; 1 = a cluster per
                                     token with one column vector per thread and the rows
                                     in registers (hidden up to 16384); 2 = one CTA per
                                     token with the whole rows in shared memory */
} ep_a2a_option;
ep_a2a_status ep_a2a_set_option(ep_a2a_handle handle, ep_a2a_option option, int64_t value);

/*
 * Per-kernel device timing.  Between ep_a2a_profile_start and ep_a2a_profile_stop
 * every kernel this handle launches is bracketed by two CUDA events recorded on
 * the launch stream; stop waits for them and returns, per kernel, the launch count
 * and the summed event-to-event milliseconds.  Meant for benchmarks: recording
 * adds two event records per launch.  At most max_launches launches are timed
 * (later ones run untimed); start allocates the events (host-side CUDA objects,
 * no device memory), stop frees them.
 */
typedef enum {
  EP_A2A_KERNEL_ROUTE_PLAN = 0,   /* routing plan + EPLB gather */
  EP_A2A_KERNEL_COPY_BULK = 1,    /* dispatch rows, bulk-async loads and stores */
  EP_A2A_KERNEL_COPY_VEC = 2,     /* dispatch rows, vector path */
  EP_A2A_KERNEL_COMBINE = 3,
  EP_A2A_KERNEL_COPY_STAGED = 4,  /* dispatch rows, bulk-async loads + vector stores */
  EP_A2A_KERNEL_COMBINE_EXPERTS = 5, /* combine of per-expert outputs */
  EP_A2A_KERNEL_COMBINE_EXPERTS_FP8 = 6, /* the same, quantised on the sending side */
  EP_A2A_KERNEL_COUNT = 7
} ep_a2a_kernel;
typedef struct {
  int64_t launches[EP_A2A_KERNEL_COUNT];
  double total_ms[EP_A2A_KERNEL_COUNT];
} ep_a2a_kernel_times;
ep_a2a_status ep_a2a_profile_start(ep_a2a_handle handle, int32_t max_launches);
ep_a2a_status ep_a2a_profile_stop(ep_a2a_handle handle, ep_a2a_kernel_times* times);

/*
 * Release the handle (NVLinkTwoSidedAlltoAll.destroy(): idempotent).  Sets
 * *handle to NULL; NULL or *handle == NULL is a no-op returning OK.  Does not
 * free the workspace, which the caller owns.
 */
ep_a2a_status ep_a2a_destroy(ep_a2a_handle* handle);

/*
 * Capacity growth (vllm.distributed.device_communicators.all2all,
 * FlashInferNVLinkOneSidedManager.initialize): the MoE layers of a model share
 * one handle, sized for the largest of them, and a layer whose request does not
 * fit replaces it with a larger one.  Given the parameters of the current handle
 * and of a new request, writes to *out the parameters that serve both and to
 * *grown 1 if they differ from `current` (a new handle is needed), else 0
 * (*out = *current with invalid_expert_id resolved).
 *   ep_size, num_experts, top_k   must be equal (INVALID_ARG otherwise: a handle
 *                                 serves one top_k and one expert count)
 *   max_tokens_per_rank,
 *   hidden_size                   the larger of the two
 *   payload_row_bytes[i]          the larger of the two, a payload that one side
 *                                 lacks counting as 0; num_payloads the larger
 *   eplb_stats_num_experts        num_experts if either side gathers, else 0
 *   enable_rank_mask              1 if either side is 1
 *   invalid_expert_id             must resolve (< 0 = num_experts) to the same id
 * Both inputs are checked as by ep_a2a_init.  Host only: no CUDA call.  To
 * grow, the caller synchronises the streams that use the old handle, destroys
 * it, allocates a workspace of ep_a2a_workspace_size(out) bytes and calls
 * ep_a2a_init on it; the old workspace's views and plan are gone, so the next
 * combine needs a new dispatch.
 */
ep_a2a_status ep_a2a_grow_params(const ep_a2a_params* current, const ep_a2a_params* request,
                                 ep_a2a_params* out, int32_t* grown);

/*
 * Row length of this handle's combines.  A handle grown to the largest hidden
 * size also serves layers with smaller ones, whose combine reads and writes rows
 * of their own length (the combine takes it from its payload in
 * vllm.distributed.device_communicators.all2all,
 * FlashInferNVLinkOneSidedManager.initialize).  ep_a2a_combine,
 * ep_a2a_combine_experts and ep_a2a_combine_scaled called after this returns use
 * rows of `hidden` elements: 1..params.hidden_size, which init sets.  Host state
 * only, nothing is enqueued.  INVALID_ARG for hidden < 1, CAPACITY above
 * params.hidden_size.
 */
ep_a2a_status ep_a2a_set_combine_hidden(ep_a2a_handle handle, int32_t hidden);

const char* ep_a2a_status_string(ep_a2a_status status);
const char* ep_a2a_last_error(void);

/*
 * Routing plan without a workspace, for callers that cannot allocate device
 * memory.  The pages have no counterpart: it exists for callers whose device
 * memory belongs to an outer allocator (for example a serving engine that
 * reserves nearly all of HBM for its own pools at start-up, or a host
 * application that does not let plug-in libraries call cudaMalloc) and who
 * therefore cannot give ep_a2a_init a workspace that includes the routing
 * kernel's scratch.  This call runs the same routing-plan kernel as
 * ep_a2a_dispatch with that scratch (send-count accumulators and tickets) in a
 * fixed array inside the library, and allocates nothing: no cudaMalloc, no
 * cudaFree, no allocating library routine.  The caller passes every input and
 * output.  It writes what ep_a2a_dispatch writes into plan_num_dst,
 * plan_dst_ranks, send_counts, recv_topk_ids and recv_valid (no EPLB gather,
 * no payload copy), with the same meaning and layout:
 *
 *   token_selected_experts  device int32 [ep, tpr, top_k]
 *   local_num_tokens        host int32 [ep], each 0..tpr
 *   active_rank_mask        host uint64 [EP_A2A_RANK_MASK_WORDS] or NULL (all active)
 *   invalid_expert_id       < 0 means num_experts
 *   plan_num_dst            device [ep, tpr]
 *   plan_dst_ranks          device [ep, tpr, round_up(top_k, 8)]
 *   send_counts             device int32 [ep, ep]
 *   recv_topk_ids           device, rank 0's int32 [ep*tpr, top_k]; 4-byte aligned
 *   recv_valid              device, rank 0's uint8 [ep*tpr]
 *   recv_rank_stride_bytes  bytes from rank d's recv_topk_ids / recv_valid to rank
 *                           d+1's (the same for both arrays; a multiple of 4)
 *
 * recv_valid must not overlap recv_topk_ids, and with ep_size > 1 the two
 * arrays of one rank must fit together inside recv_rank_stride_bytes
 * (INVALID_ARG otherwise), so that no write lands on another array or rank.
 *
 * Limit: ep_size <= EP_A2A_NOALLOC_MAX_RANKS (64); larger sizes return
 * EP_A2A_ERR_UNSUPPORTED.  The array takes 16,640 bytes on every GPU that loads
 * the library, until the process exits.  The first call in each CUDA context of
 * a device looks up the array's device address with that device current
 * (cudaGetSymbolAddress) and caches it with the context's id; after a device
 * reset the device has a new context, and the next call looks the address up
 * again.  Make that first call before any stream capture.  Every call shares
 * the array and clears the part it uses on `stream` before its kernel, so calls
 * in stream order are independent; calls whose work overlaps on the GPU race
 * on the array.
 */
#define EP_A2A_NOALLOC_MAX_RANKS 64
ep_a2a_status ep_a2a_route_plan_noalloc(
    int32_t ep_size, int32_t num_experts, int32_t top_k, int32_t tokens_per_rank,
    int32_t invalid_expert_id, const int32_t* token_selected_experts,
    const int32_t* local_num_tokens, const uint64_t* active_rank_mask, uint8_t* plan_num_dst,
    uint8_t* plan_dst_ranks, int32_t* send_counts, int32_t* recv_topk_ids, uint8_t* recv_valid,
    int64_t recv_rank_stride_bytes, void* stream);

/*
 * ---------------------------------------------------------------------------
 * Expert parallelism between real ranks: one process per EP rank.
 *
 * The same dispatch and combine as above (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll,
 * dispatch() / combine(); slots src * tokens_per_rank + t, OneSidedConfig
 * `lamport`), with each EP rank a process that owns one device "window" for
 * what its peers send it.  Windows are exported with CUDA IPC handles and
 * mapped by every peer; senders write rows into peer windows with plain
 * stores (no rank ever loads from a peer's memory) and then set one flag per
 * (source, destination) pair with a release store at system scope.
 * Receivers check those flags with acquire loads in a bounded wait
 * (NVLinkOneSidedConfig, `timeout_sec`: there a kernel traps on expiry; here
 * the wait gives up, sets the handle's error word and ep_mp_get_status returns
 * EP_A2A_ERR_DEVICE_TIMEOUT, leaving the context usable).
 *
 * The library does no host communication.  The caller exchanges the IPC
 * handles (ep_mp_export on every rank, then all-gather) and separates the
 * phases with a host barrier after synchronising its stream:
 *   init (every rank) | barrier | dispatch | barrier | dispatch_wait,
 *   experts, combine_send | barrier | combine_finish
 * so that no kernel ever waits for a kernel of another process to run: the
 * flags are already set when a wait starts, unless a rank skipped its send.
 * Every live rank must make the same calls in the same order with the same
 * active_rank_mask; a masked-off rank makes none of the step's calls.
 * ---------------------------------------------------------------------------
 */
typedef struct ep_mp_handle_s* ep_mp_handle;   /* opaque, library-owned host object */

typedef struct {
  uint8_t handle[64];             /* cudaIpcMemHandle_t of the window's allocation */
  int64_t offset;                 /* window start minus allocation start (bytes) */
} ep_mp_ipc_handle;

/*
 * Bytes of one rank's window for `params` (the same params on every rank; the
 * rules of ep_a2a_params).  It holds the rank's own plan and counters, the
 * flags, the receive arrays [ep*cap] of every payload, ids and valid bytes,
 * the EPLB rows [ep, E], and the combine landing rows [ep, cap, hidden] of
 * 2-byte elements.  Host only.
 */
ep_a2a_status ep_mp_window_size(const ep_a2a_params* params, size_t* bytes);

/*
 * IPC handle of `window` (device memory from cudaMalloc, e.g. a torch
 * tensor; not from a stream-ordered pool or a virtual-memory mapping) for the
 * peers' ep_mp_init.  Host only, no device work.
 */
ep_a2a_status ep_mp_export(void* window, ep_mp_ipc_handle* out);

/*
 * Create rank `rank`'s handle: `window` (>= ep_mp_window_size bytes, 256-byte
 * aligned, caller-owned, kept alive until ep_mp_destroy on every rank) is
 * this rank's; peers[r] (r != rank) are the other ranks' exported handles
 * (peers[rank] is ignored).  Opens every peer window, clears this window's
 * control region and flags, and synchronises `stream`.  Every rank must
 * finish init before any rank dispatches (a host barrier).
 */
ep_a2a_status ep_mp_init(const ep_a2a_params* params, int32_t rank, void* window,
                         size_t window_bytes, const ep_mp_ipc_handle* peers, void* stream,
                         ep_mp_handle* out_handle);

/*
 * Send this rank's tokens (as ep_a2a_dispatch for source rank `rank`):
 *   token_selected_experts  device int32 [tpr, top_k] (this rank's tokens)
 *   local_num_tokens        this rank's token count, 0..tpr
 *   payloads                host array of device pointers, each [tpr, row_bytes_i]
 *   eplb_local_stats        device int32 [E] or NULL
 *   active_rank_mask        host uint64 [EP_A2A_RANK_MASK_WORDS] or NULL; this rank
 *                           must be live in it
 * Fills `result` with views of this rank's window: recv_payloads[i] [ep*tpr, rb_i],
 * recv_topk_ids [ep*tpr, k], recv_valid [ep*tpr], eplb_gathered_stats [ep, E]
 * (what peers sent this rank, complete once every live rank has dispatched and
 * ep_mp_dispatch_wait has succeeded), send_counts [ep] (tokens this rank sent to
 * each rank), plan_num_dst [tpr] and plan_dst_ranks [tpr, plan_stride] (this
 * rank's plan); rank_stride_bytes is 0.
 */
ep_a2a_status ep_mp_dispatch(ep_mp_handle handle, const int32_t* token_selected_experts,
                             int32_t local_num_tokens, int32_t runtime_max_tokens_per_rank,
                             const void* const* payloads, const int64_t* payload_row_bytes,
                             int32_t num_payloads, const int32_t* eplb_local_stats,
                             const uint64_t* active_rank_mask, void* stream,
                             ep_a2a_dispatch_result* result);

/*
 * Receive side of the dispatch: wait (bounded by timeout_ns, 1..1e10, of GPU
 * time) until every live rank's flag of this step has arrived.  On expiry the
 * handle's error word is set (ep_mp_get_status: EP_A2A_ERR_DEVICE_TIMEOUT).
 */
ep_a2a_status ep_mp_dispatch_wait(ep_mp_handle handle, int64_t timeout_ns, void* stream);

/*
 * Return rows: expert_output device [ep*tpr, hidden] of `dtype` holds this
 * rank's row for each slot it received (rank src's token t at src*tpr + t: its
 * own experts' outputs, weighted and summed); each valid slot's row is written
 * to source src's landing rows, then one flag per live rank.
 */
ep_a2a_status ep_mp_combine_send(ep_mp_handle handle, const void* expert_output,
                                 ep_a2a_combine_dtype dtype, void* stream);

/*
 * Wait (bounded, as ep_mp_dispatch_wait) for every live rank's combine flag,
 * then output device bf16 [tpr, hidden] = for each of this rank's tokens, the
 * fp32 sum in ascending destination-rank order, from +0.0f, of the rows its
 * destinations returned, rounded once to bf16 (the arithmetic of
 * ep_a2a_combine).  Rows of tokens t >= local_num_tokens are not written.
 */
ep_a2a_status ep_mp_combine_finish(ep_mp_handle handle, void* output, ep_a2a_combine_dtype dtype,
                                   int64_t timeout_ns, void* stream);

/* Synchronise `stream`, then read and clear the handle's error word. */
ep_a2a_status ep_mp_get_status(ep_mp_handle handle, void* stream);

/*
 * Close the peer mappings and free the handle (idempotent, NULL ok).  Every
 * rank's kernels that write into this rank's window must have completed, and
 * every rank must destroy before any rank frees its window (host barriers).
 */
ep_a2a_status ep_mp_destroy(ep_mp_handle* handle);

#ifdef __cplusplus
}
#endif

#endif /* EP_A2A_H */
