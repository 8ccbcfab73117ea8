// Internal declarations of libep_a2a: kernel argument blocks, launchers and
// small PTX wrappers (mbarrier, bulk-async copies).  Not part of the C ABI.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <utility>

#include "ep_a2a.h"

namespace ep_a2a {

constexpr int kMaxRanks = EP_A2A_MAX_RANKS;
constexpr int kMaskWords = EP_A2A_RANK_MASK_WORDS;
constexpr int kMaxPayloads = EP_A2A_MAX_PAYLOADS;
constexpr int kMaxTopK = EP_A2A_MAX_TOP_K;
constexpr uint8_t kNoToken = 0xFF;       // plan_num_dst of a token that does not exist
constexpr uint8_t kPad = 0xFF;           // plan_dst_ranks entries past the count
constexpr int kMaxStages = 32;           // shared-memory row stages per bulk-copy CTA

// Bits of the device error word.
enum : uint32_t { kErrWaitTimeout = 1u, kErrBounds = 2u };

// Checked builds (-DEP_A2A_CHECKS=1, libep_a2a_checked.so) test indices that
// come from device memory (the plan another kernel or the caller left in the
// workspace) before using them; a bad one sets kErrBounds and the access is
// skipped.  In the default build the checks compile to nothing.
#ifndef EP_A2A_CHECKS
#define EP_A2A_CHECKS 0
#endif

// Whether a token's plan row is usable: at most plan_stride destinations, each
// one a rank below ep.  Always true unless checks are compiled in.
__device__ __forceinline__ bool plan_row_ok(int nd, uint64_t w0, uint64_t w1, uint64_t w2,
                                            uint64_t w3, int ep, int plan_stride,
                                            uint32_t* err) {
  if (!EP_A2A_CHECKS) return true;
  bool ok = nd <= plan_stride && nd <= 32;
  for (int q = 0; ok && q < nd; ++q) {
    const uint64_t w = q < 8 ? w0 : (q < 16 ? w1 : (q < 24 ? w2 : w3));
    ok = (int)((w >> ((q & 7) * 8)) & 0xFFu) < ep;
  }
  if (!ok && err) atomicOr(err, kErrBounds);
  return ok;
}

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__host__ __device__ inline int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Routing plan (+ EPLB gather)
// ---------------------------------------------------------------------------
struct RouteArgs {
  const int32_t* ids;          // [ep, tpr, k]
  const int32_t* eplb_stats;   // [ep, eplb_n] or nullptr
  uint8_t* plan_nd;            // [ep*tpr]
  uint8_t* plan_dst;           // [ep*tpr, plan_stride]
  int32_t* count_acc;          // [ep*ep] scratch; zero between calls
  uint32_t* count_ticket;      // [ep] scratch; zero between calls
  int32_t* send_counts;        // [ep*ep]
  uint8_t* rank0;              // rank 0's region of the workspace
  int64_t rank_stride;         // bytes between rank regions
  int64_t off_ids, off_valid, off_eplb;  // offsets inside a rank region
  int ep, E, k, tpr, epr, plan_stride, eplb_n;
  int32_t invalid_id;
  int32_t n[kMaxRanks];        // local_num_tokens, 0 for masked-off ranks
  uint64_t live[kMaskWords];   // bit r = rank r active
  int vec_ids;                 // set by launch_route_plan: ids rows as 16-byte stores
};

cudaError_t launch_route_plan(const RouteArgs& a, bool use_mask, cudaStream_t stream,
                              bool pdl = false);

// ---------------------------------------------------------------------------
// Dispatch row copy
// ---------------------------------------------------------------------------
struct CopyArgs {
  const uint8_t* plan_nd;
  const uint8_t* plan_dst;
  uint8_t* rank0;
  int64_t rank_stride;
  int64_t ntok;                          // ep * tpr token slots
  int plan_stride;
  int np;                                // payloads handled by this launch
  const uint8_t* src[kMaxPayloads];      // [ep*tpr, rb] each
  int64_t rb[kMaxPayloads];              // row bytes
  int64_t dst_off[kMaxPayloads];         // receive array offset inside a rank region
  uint32_t smem_off[kMaxPayloads];       // bulk path: offset of the row in a stage
  uint32_t vec[kMaxPayloads];            // vector path: bytes per access (32/16/8/4/2/1)
  uint32_t stage_bytes;                  // bulk path: bytes of one stage
  uint32_t tx_bytes;                     // bulk path: bytes one token brings in
  int stages;                            // bulk path
  int interleave;                        // bulk paths: 1 = CTA b takes tokens b, b+grid, ...
  uint32_t* err;
  // vector path: the routing inputs, so that it finds each token's
  // destinations itself instead of reading the plan
  const int32_t* ids;                    // [ep, tpr, k]
  int E, k, epr, tpr, use_mask;
  int prefetch;                          // vector path: prefetch the next token's rows into L2
  // vector path with `route` set: the kernel also writes the routing plan,
  // the per-destination valid bytes and received ids, the send counts and the
  // EPLB gather (what launch_route_plan writes), so a dispatch is one launch
  int route;
  int ep;
  int32_t invalid_id;
  int32_t* count_acc;                    // [ep*ep] scratch; zero between calls
  uint32_t* count_ticket;                // [1] scratch; zero between calls
  int32_t* send_counts;                  // [ep*ep]
  int64_t off_ids, off_valid, off_eplb;  // inside a rank region
  const int32_t* eplb_stats;             // [ep, eplb_n] or nullptr
  int eplb_n;
  int32_t n[kMaxRanks];                  // local_num_tokens (0 for masked-off ranks)
  uint64_t live[kMaskWords];
};

cudaError_t launch_dispatch_bulk(const CopyArgs& a, int grid, cudaStream_t stream, bool pdl);
cudaError_t launch_dispatch_staged(const CopyArgs& a, int consumer_warps, int grid,
                                   cudaStream_t stream, bool pdl);
constexpr int kStagedMaxVec = 8;         // 16-byte vectors per consumer thread per token
cudaError_t launch_dispatch_vec(const CopyArgs& a, int grid, int unroll, int threads_per_token,
                                bool streaming, cudaStream_t stream, bool pdl);
int bulk_queue_depth(int stages);        // groups allowed in flight for `stages`

// ---------------------------------------------------------------------------
// Combine and the E4M3 helper
// ---------------------------------------------------------------------------
struct CombineArgs {
  const uint8_t* plan_nd;
  const uint8_t* plan_dst;
  const uint8_t* x;            // [ep, ep*tpr, H] bf16 or E4M3
  uint16_t* out;               // [ep, tpr, H] bf16
  int64_t ntok;                // ep * tpr
  int H;
  int plan_stride;
  int prefetch;                // p > 0: prefetch the rows of the CTA's token p
                               // grid strides ahead into L2
  int ep;
  uint32_t* err;               // device error word (checked builds)
  int out32;                   // pipelined E4M3 combines: one 32-byte store per
                               // vector (output 32-byte aligned)
};

// pipe: the two-deep pipelined kernel (needs at most 8 destinations per token);
// tight with 128 threads: the BF16 one-vector instance held to seven CTAs per SM
cudaError_t launch_combine(const CombineArgs& a, bool fp8, bool vec, bool pipe, int threads,
                           int grid, cudaStream_t stream, bool pdl, bool tight = false);

// Combine of per-(token, slot) expert outputs: the weighted reduction over each
// destination's local experts fused into the combine.
struct CombineExpertsArgs {
  const uint8_t* plan_nd;
  const uint8_t* plan_dst;
  const uint8_t* recv_ids0;    // rank 0's recv_topk_ids ([ep*tpr, k] int32 per rank)
  int64_t rank_stride;         // bytes between ranks' recv_topk_ids
  const float* w;              // topk_weights [ep*tpr, k]
  const uint16_t* y;           // bf16 [ep*tpr, k, H]
  uint16_t* out;               // bf16 [ep*tpr, H]
  int64_t ntok;
  int H, k, E, epr, plan_stride;
  int prefetch;                // p > 0: prefetch the slot rows of the CTA's token p
                               // grid strides ahead into L2
  int ep;
  uint32_t* err;               // device error word (checked builds)
};

cudaError_t launch_combine_experts(const CombineExpertsArgs& a, bool vec, bool pipe, int threads,
                                   int grid, cudaStream_t stream, bool pdl);
// The same with the slot rows staged in shared memory by bulk-async copies
// (top_k <= 8, hidden % 8 == 0, 16-byte aligned rows).
cudaError_t launch_combine_experts_staged(const CombineExpertsArgs& a, int grid, int ctas_per_sm,
                                          int max_smem, cudaStream_t stream, bool pdl);
// The same with each destination's row quantised to E4M3 with one scale per row
// before the sum.  smem_rows: the kernel that keeps the token's rows in `smem`
// bytes of shared memory (top_k <= 8, hidden % 8 == 0, 16-byte aligned rows);
// else the element kernel (threads <= 256).
cudaError_t launch_combine_experts_fp8(const CombineExpertsArgs& a, bool smem_rows, int threads,
                                       int grid, size_t smem, cudaStream_t stream, bool pdl);
// The same with a cluster of `cluster` (1, 2, 4, 8) CTAs of `threads` (<= 256)
// threads per token, each thread one 16-byte column vector (top_k <= 8, hidden
// % 8 == 0, hidden / 8 <= cluster * threads, 16-byte aligned rows); `clusters`
// clusters stride over the tokens.
cudaError_t launch_combine_experts_fp8_cluster(const CombineExpertsArgs& a, int cluster,
                                               int threads, int clusters, cudaStream_t stream,
                                               bool pdl);
// The same split over a cluster of `cluster` CTAs per token, each a slice of
// `cols` elements (two 16-byte vectors per thread, threads <= 256) with its
// rows z_d in `smem` bytes of shared memory (min(top_k, ep) rows x cols bf16).
cudaError_t launch_combine_experts_fp8_split(const CombineExpertsArgs& a, int cluster, int threads,
                                             int cols, int clusters, size_t smem,
                                             cudaStream_t stream, bool pdl);
cudaError_t launch_quantize_e4m3(const uint16_t* in, uint8_t* out, int64_t n, cudaStream_t stream);
cudaError_t launch_quantize_e4m3_rows(const uint16_t* in, uint8_t* out, float* scales,
                                      int64_t rows, int hidden, cudaStream_t stream);
// The BF16 (mode 0), FP8 (1) or scaled FP8 (2, scales [ep, ep*tpr]) combine with
// the rows staged in shared memory by bulk-async copies; at most 8 destinations
// per token, rows of 16-byte multiples at 16-byte aligned addresses.
cudaError_t launch_combine_staged(const CombineArgs& a, int mode, const float* scales,
                                  int grid, int ctas_per_sm, int max_smem, cudaStream_t stream,
                                  bool pdl);
// FP8 combine with one fp32 scale per row (scales [ep, ep*tpr]).
cudaError_t launch_combine_scaled(const CombineArgs& a, const float* scales, bool vec, bool pipe,
                                  int threads, int grid, cudaStream_t stream, bool pdl);
cudaError_t launch_wait_timeout_probe(uint32_t* err, unsigned long long limit_ns,
                                      cudaStream_t stream);

// Message returned by ep_a2a_last_error() on the calling thread.
void record_last_error(const char* msg);

// Launch `kernel` on `stream`; with `pdl` the launch may begin while the
// previous kernel of the stream finishes (programmatic dependent launch), and
// the kernel itself waits for that kernel (pdl_wait) before touching memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, bool pdl, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------------------
// PTX wrappers (sm_90+; built for sm_100a).  All forms are CTA-local.
// ---------------------------------------------------------------------------
#if defined(__CUDACC__)
// Wait until the grid this one depends on (programmatic dependent launch) has
// completed and its writes are visible; returns at once otherwise.  Every
// kernel of the path calls it before its first global memory access.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel of the stream (if launched with programmatic
// dependent launch) to start; it still waits for this grid with pdl_wait
// before it reads anything this grid writes.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// Make barrier initialisation visible to the async proxy (the bulk-copy unit).
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for phase `parity` of the barrier, for at most limit_ns.  Returns false
// if the limit ran out (the caller records an error and stops).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst_smem, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst_smem),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// This CTA's shared memory -> global, tracked by bulk groups.
__device__ __forceinline__ void bulk_store(void* dst, uint32_t src_smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
               "r"(src_smem), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// At most N committed groups may still be reading shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// All committed groups complete (writes performed).
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Ask the copy engine to bring `bytes` (a multiple of 16, 16-byte aligned)
// into L2 ahead of use; no registers or shared memory are involved.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
#endif  // __CUDACC__

}  // namespace ep_a2a
