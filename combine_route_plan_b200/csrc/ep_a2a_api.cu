// Host side of the C ABI declared in include/ep_a2a.h: argument validation,
// workspace layout, and kernel launches.  No device memory is allocated here;
// the caller owns the workspace and every input / output buffer.
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "ep_a2a_internal.cuh"

#define EP_API extern "C" __attribute__((visibility("default")))

namespace ep_a2a {
namespace {

constexpr uint32_t kMagic = 0x45504132u;   // "EPA2"
constexpr int64_t kAlign = 256;

thread_local std::string g_last_error;

ep_a2a_status fail(ep_a2a_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ep_a2a_status fail(ep_a2a_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

ep_a2a_status cuda_fail(cudaError_t e, const char* what) {
  return fail(EP_A2A_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Byte offsets of everything in the workspace.
struct Layout {
  int64_t off_err, off_count_acc, off_ticket, off_counts, off_plan_nd, off_plan_dst;
  int64_t ctrl_bytes;        // [0, ctrl_bytes) is cleared at init
  int64_t rank_base;         // rank 0's region
  int64_t rank_stride;       // bytes per rank region
  int64_t off_payload[kMaxPayloads];
  int64_t off_ids, off_valid, off_eplb;   // inside a rank region
  int64_t total;
  int plan_stride;
};

ep_a2a_status check_params(const ep_a2a_params* p) {
  if (!p) return fail(EP_A2A_ERR_INVALID_ARG, "params is NULL");
  if (p->ep_size < 1 || p->ep_size > kMaxRanks)
    return fail(EP_A2A_ERR_UNSUPPORTED, "ep_size %d outside 1..%d", p->ep_size, kMaxRanks);
  if (p->num_experts <= 0 || p->num_experts % 4 != 0)
    return fail(EP_A2A_ERR_INVALID_ARG, "num_experts %d must be a positive multiple of 4",
                p->num_experts);
  if (p->num_experts % p->ep_size != 0)
    return fail(EP_A2A_ERR_INVALID_ARG, "num_experts %d must be divisible by ep_size %d",
                p->num_experts, p->ep_size);
  if (p->top_k < 1 || p->top_k > kMaxTopK)
    return fail(EP_A2A_ERR_UNSUPPORTED, "top_k %d outside 1..%d", p->top_k, kMaxTopK);
  if (p->max_tokens_per_rank < 1)
    return fail(EP_A2A_ERR_INVALID_ARG, "max_tokens_per_rank %d must be >= 1",
                p->max_tokens_per_rank);
  if ((int64_t)p->ep_size * p->max_tokens_per_rank > (int64_t)1 << 30)
    return fail(EP_A2A_ERR_UNSUPPORTED, "ep_size * max_tokens_per_rank too large");
  if (p->hidden_size < 1)
    return fail(EP_A2A_ERR_INVALID_ARG, "hidden_size %d must be >= 1", p->hidden_size);
  if (p->num_payloads < 0 || p->num_payloads > kMaxPayloads)
    return fail(EP_A2A_ERR_UNSUPPORTED, "num_payloads %d outside 0..%d", p->num_payloads,
                kMaxPayloads);
  for (int i = 0; i < p->num_payloads; ++i)
    if (p->payload_row_bytes[i] < 1 || p->payload_row_bytes[i] > ((int64_t)1 << 24))
      return fail(EP_A2A_ERR_INVALID_ARG, "payload_row_bytes[%d] = %lld outside 1..2^24", i,
                  (long long)p->payload_row_bytes[i]);
  if (p->eplb_stats_num_experts != 0 && p->eplb_stats_num_experts != p->num_experts)
    return fail(EP_A2A_ERR_INVALID_ARG,
                "eplb_stats_num_experts %d must be 0 or num_experts %d (statistics must cover "
                "all experts)",
                p->eplb_stats_num_experts, p->num_experts);
  if (p->enable_rank_mask != 0 && p->enable_rank_mask != 1)
    return fail(EP_A2A_ERR_INVALID_ARG, "enable_rank_mask must be 0 or 1");
  if (p->reserved != 0) return fail(EP_A2A_ERR_INVALID_ARG, "reserved must be 0");
  return EP_A2A_OK;
}

Layout make_layout(const ep_a2a_params& p) {
  Layout L{};
  const int64_t ep = p.ep_size, cap = p.max_tokens_per_rank, slots = ep * cap;
  L.plan_stride = (int)align_up(p.top_k, 8);
  int64_t c = 0;
  L.off_err = c;        c = align_up(c + 16, kAlign);
  L.off_count_acc = c;  c = align_up(c + ep * ep * 4, kAlign);
  L.off_ticket = c;     c = align_up(c + ep * 4, kAlign);
  L.off_counts = c;     c = align_up(c + ep * ep * 4, kAlign);
  L.off_plan_nd = c;    c = align_up(c + slots, kAlign);
  L.off_plan_dst = c;   c = align_up(c + slots * L.plan_stride, kAlign);
  L.ctrl_bytes = c;
  L.rank_base = c;
  int64_t r = 0;
  for (int i = 0; i < kMaxPayloads; ++i) {
    L.off_payload[i] = r;
    if (i < p.num_payloads) r = align_up(r + slots * p.payload_row_bytes[i], kAlign);
  }
  L.off_ids = r;    r = align_up(r + slots * p.top_k * 4, kAlign);
  L.off_valid = r;  r = align_up(r + slots, kAlign);
  L.off_eplb = r;   r = align_up(r + ep * p.eplb_stats_num_experts * 4, kAlign);
  L.rank_stride = r;
  L.total = L.rank_base + ep * L.rank_stride;
  return L;
}

}  // namespace

void record_last_error(const char* msg) { g_last_error = msg; }

}  // namespace ep_a2a

using namespace ep_a2a;

struct ep_a2a_handle_s {
  uint32_t magic;
  ep_a2a_params p;
  Layout L;
  uint8_t* ws;
  size_t ws_bytes;
  int device;
  int num_sms;
  int max_smem_optin;
  bool have_plan;
  int last_tpr;
  int combine_hidden;     // row length of the combines, 1..p.hidden_size
  // tuning
  int copy_path;          // 0 staged, 1 vector only, 2 bulk loads + bulk stores
  int copy_consumer_warps;
  int copy_interleave;
  int vec_unroll;
  int vec_ctas_per_sm;
  int store_streaming;
  int pdl;                // programmatic dependent launch for the path's kernels
  int vec_threads_per_token;  // 0 = from the token count and the largest row
  // combine launch shape; -1 / 0 = automatic (combine_launch)
  int combine_prefetch;       // tokens ahead (grid strides) whose rows go to L2
  int copy_prefetch;          // vector copy: prefetch the next token's rows
  int copy_vec_bytes;         // vector copy: widest access, 16 or 32 bytes
  int combine_pipeline;       // 1: the two-deep pipelined kernels
  int copy_ctas_per_sm;
  int route_in_copy;      // vector copy path: 1 = the copy kernel also routes (one launch)
  int fp8_experts_kernel;   // sender-side FP8 expert combine: 0 split, 1 cluster, 2 one CTA
  int copy_stages;        // 0 = choose from the row size
  int combine_threads;
  int64_t bulk_min_row;   // rows below this go to the vector copy
  int combine_ctas_per_sm;
  // profiling (ep_a2a_profile_start / _stop)
  bool profiling;
  int prof_max;
  std::vector<cudaEvent_t> prof_events;   // 2 per timed launch
  std::vector<int> prof_kernel;           // kernel id per timed launch
};

namespace {

ep_a2a_status check_handle(ep_a2a_handle h) {
  if (!h || h->magic != kMagic)
    return fail(EP_A2A_ERR_NOT_INITIALIZED, "handle is NULL or destroyed");
  return EP_A2A_OK;
}

// Record the start event of a timed launch; returns the slot or -1.
int prof_begin(ep_a2a_handle h, int kernel, cudaStream_t stream) {
  if (!h->profiling || (int)h->prof_kernel.size() >= h->prof_max) return -1;
  const int slot = (int)h->prof_kernel.size();
  if (cudaEventRecord(h->prof_events[2 * slot], stream) != cudaSuccess) return -1;
  h->prof_kernel.push_back(kernel);
  return slot;
}

void prof_end(ep_a2a_handle h, int slot, cudaStream_t stream) {
  if (slot >= 0) cudaEventRecord(h->prof_events[2 * slot + 1], stream);
}

void prof_free(ep_a2a_handle h) {
  for (cudaEvent_t e : h->prof_events) cudaEventDestroy(e);
  h->prof_events.clear();
  h->prof_kernel.clear();
  h->profiling = false;
}

// Threads per token of the vector copy, given the vectors in the largest row.
// Measured on the workloads: with 16384 or more token slots a warp per token
// is fastest (enough tokens to fill the GPU; 32 beat 64-256 by 2-30 % at
// prefill); with fewer, the fewest threads (32..256) that hold the row in
// about two vectors each (Zipf step, 8192 slots: 224-vector MXFP8 rows 7 %
// faster on 128 threads than on a warp, 112-vector NVFP4 rows 1 % on 64;
// decode and wide-EP steps: 448-vector rows on 256).
int copy_threads_per_token(int64_t tokens, int64_t row_vectors) {
  if (tokens >= 16384) return 32;
  int t = 32;
  while (t < 256 && 2 * t < row_vectors) t *= 2;
  return t;
}

// Vectors in the largest row of a vector-copy launch.
int64_t largest_row_vectors(const CopyArgs& c) {
  int64_t most = 0;
  for (int p = 0; p < c.np; ++p) most = std::max<int64_t>(most, c.rb[p] / (int64_t)c.vec[p]);
  return most;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

enum CombineKind { kKindBf16, kKindFp8, kKindExperts };

struct CombineLaunch {
  bool pipe;
  bool staged;               // rows staged in shared memory by bulk-async copies
  int threads, grid, prefetch;
  bool tight;                // BF16, 128 threads: the instance held to 7 CTAs per SM
  int staged_ctas_per_sm;
};

// Launch shape of a combine: the options where set, else the defaults measured
// on the decode (1024 token slots), wide-EP (4096), Zipf (8192) and prefill
// (32768) workloads at hidden 7168:
//  * BF16: one vector at a time (pipelining was 1-12 % slower); from 16384
//    token slots 64 threads, 128 CTAs per SM requested, no prefetch; from 8192
//    128 threads and a one-token prefetch (Zipf step: 98 against 103 us);
//    below that 16 CTAs per SM and no prefetch, with 256 threads (wide-EP
//    step: 51 against 55 us), or at up to 8 token slots per SM 128 threads in
//    the instance held to 72 registers, seven CTAs per SM: every token of the
//    decode step in one wave, seven rounds of column vectors per token
//    (combine 23.6 against 24.8 us with 192 threads, two waves of five rounds,
//    and 25.6 with 256, three waves of four);
//  * FP8 and scaled FP8: pipelined (27-54 % faster); 64 threads up to 16
//    token slots per SM, 128 above (wide-EP step: 94.6 against 96.4 us); from
//    8192 slots on, prefetch one token ahead (faster by 5-10 %, slower by 5-10 %
//    on the small steps); 16 CTAs per SM requested from 16384 slots on
//    (scaled: 291 against 310 us), else 128;
//  * expert outputs: pipelined (24-28 % faster), no prefetch; 128 threads
//    below 8192 token slots with more than 16 per SM (wide-EP step: 129.8
//    against 132.7 us), else 64.
// The pipelined kernels hold at most 8 destination rows per token, and a token
// has at most min(top_k, ep_size) destinations.
CombineLaunch combine_launch(ep_a2a_handle h, CombineKind kind, int64_t ntok) {
  const bool fits = std::min(h->p.top_k, h->p.ep_size) <= 8;
  const bool big = ntok >= 16384;
  CombineLaunch c;
  c.pipe = fits && (h->combine_pipeline < 0 ? kind != kKindBf16 : h->combine_pipeline == 1);
  c.staged = fits && h->combine_pipeline == 2;
  // a staged CTA needs two stages of 32 KB: at most three CTAs per SM
  c.staged_ctas_per_sm = h->combine_ctas_per_sm > 0 ? std::min(h->combine_ctas_per_sm, 3) : 2;
  const bool mid = !big && ntok >= 8192;
  const bool small = ntok < 8192;
  const int64_t per_sm = ntok / std::max(1, h->num_sms);     // token slots per SM
  int threads = (small && per_sm > 16) ? 128 : 64, cps = 128, prefetch = 0;
  bool tight = false;
  if (kind == kKindFp8) {
    threads = big ? 128 : threads;
    cps = big ? 16 : 128;
    prefetch = ntok >= 8192 ? 1 : 0;
  } else if (kind == kKindBf16) {
    threads = big ? 64 : (mid ? 128 : (per_sm <= 8 ? 128 : 256));
    tight = !big && !mid && per_sm <= 8;
    cps = (big || mid) ? 128 : 16;
    prefetch = mid ? 1 : 0;
  }
  c.threads = h->combine_threads > 0 ? h->combine_threads : threads;
  c.tight = tight && c.threads == 128;
  if (h->combine_ctas_per_sm > 0) cps = h->combine_ctas_per_sm;
  c.grid = (int)std::max<int64_t>(1, std::min<int64_t>(ntok, (int64_t)h->num_sms * cps));
  c.prefetch = h->combine_prefetch >= 0 ? h->combine_prefetch : prefetch;
  return c;
}

// Vectors per thread in flight in the vector copy: the fewest of 2, 4, 8 with
// which a token group moves its largest row in at most two rounds (measured:
// 8 for the prefill rows of 448 32-byte vectors over a warp, 2 for the
// 3.5-14 KB rows of the decode, Zipf and wide-EP steps; a group with more
// vectors in flight than its row has only ties up registers).
int copy_unroll(int64_t row_vectors, int tpt) {
  const int64_t per_thread = (row_vectors + tpt - 1) / tpt;
  if (per_thread <= 4) return 2;
  if (per_thread <= 8) return 4;
  return 8;
}

// Widest access (up to `widest` bytes) that every row of a payload allows.
uint32_t vec_bytes(const void* src, const void* dst_base, int64_t rank_stride, int64_t rb,
                   uint32_t widest) {
  for (uint32_t v : {32u, 16u, 8u, 4u, 2u}) {
    if (v > widest) continue;
    if (rb % v == 0 && aligned(src, v) && aligned(dst_base, v) && rank_stride % v == 0) return v;
  }
  return 1u;
}

}  // namespace

EP_API const char* ep_a2a_status_string(ep_a2a_status s) {
  switch (s) {
    case EP_A2A_OK: return "ok";
    case EP_A2A_ERR_INVALID_ARG: return "invalid argument";
    case EP_A2A_ERR_CAPACITY: return "step exceeds the capacity given at init";
    case EP_A2A_ERR_UNSUPPORTED: return "unsupported size";
    case EP_A2A_ERR_CUDA: return "CUDA runtime error";
    case EP_A2A_ERR_NOT_INITIALIZED: return "handle not initialised";
    case EP_A2A_ERR_NO_PLAN: return "combine called before any dispatch";
    case EP_A2A_ERR_DEVICE_TIMEOUT: return "a bounded device wait ran out";
    case EP_A2A_ERR_DEVICE_BOUNDS: return "a device index check failed (checked build)";
  }
  return "unknown status";
}

EP_API const char* ep_a2a_last_error(void) { return g_last_error.c_str(); }

EP_API ep_a2a_status ep_a2a_workspace_size(const ep_a2a_params* params, size_t* bytes) {
  ep_a2a_status st = check_params(params);
  if (st != EP_A2A_OK) return st;
  if (!bytes) return fail(EP_A2A_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = (size_t)make_layout(*params).total;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_init(const ep_a2a_params* params, void* workspace,
                                 size_t workspace_bytes, void* stream,
                                 ep_a2a_handle* out_handle) {
  ep_a2a_status st = check_params(params);
  if (st != EP_A2A_OK) return st;
  if (!out_handle) return fail(EP_A2A_ERR_INVALID_ARG, "out_handle is NULL");
  *out_handle = nullptr;
  if (!workspace) return fail(EP_A2A_ERR_INVALID_ARG, "workspace is NULL");
  if (!aligned(workspace, kAlign))
    return fail(EP_A2A_ERR_INVALID_ARG, "workspace must be %lld-byte aligned", (long long)kAlign);
  const Layout L = make_layout(*params);
  if ((int64_t)workspace_bytes < L.total)
    return fail(EP_A2A_ERR_INVALID_ARG, "workspace has %zu bytes, needs %lld", workspace_bytes,
                (long long)L.total);
  cudaPointerAttributes attr;
  cudaError_t e = cudaPointerGetAttributes(&attr, workspace);
  if (e != cudaSuccess) return cuda_fail(e, "cudaPointerGetAttributes(workspace)");
  if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
    return fail(EP_A2A_ERR_INVALID_ARG, "workspace is not device memory");
  int dev = 0, sms = 0, smem = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (attr.device != dev)
    return fail(EP_A2A_ERR_INVALID_ARG, "workspace is on device %d, current device is %d",
                attr.device, dev);
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
  if ((e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) !=
      cudaSuccess)
    return cuda_fail(e, "cudaDeviceGetAttribute(shared memory)");
  e = cudaMemsetAsync(workspace, 0, (size_t)L.ctrl_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(control region)");

  ep_a2a_handle h = new (std::nothrow) ep_a2a_handle_s();
  if (!h) return fail(EP_A2A_ERR_INVALID_ARG, "out of host memory");
  h->magic = kMagic;
  h->p = *params;
  if (h->p.invalid_expert_id < 0) h->p.invalid_expert_id = h->p.num_experts;
  h->L = L;
  h->ws = static_cast<uint8_t*>(workspace);
  h->ws_bytes = workspace_bytes;
  h->device = dev;
  h->num_sms = sms;
  h->max_smem_optin = smem;
  h->have_plan = false;
  h->last_tpr = 0;
  h->combine_hidden = params->hidden_size;
  // Defaults measured on the prefill workload (ep 8, 4096 tokens/rank, 14.4 KB
  // rows): the vector copy with 32 CTAs per SM requested and evict-first stores
  // moved the rows fastest (487 us with 16-byte vectors, against 527 us for the
  // staged bulk-load path and 539 us for bulk loads + stores); 32-byte vectors
  // took it to 475 us (decode, Zipf and wide-EP workloads: 1-4 % faster too).
  h->copy_path = 1;
  h->copy_consumer_warps = 4;
  h->copy_interleave = 1;
  h->vec_unroll = 0;
  h->vec_ctas_per_sm = 0;        // automatic (copy launch below)
  h->store_streaming = 1;
  h->pdl = 1;
  h->vec_threads_per_token = 0;
  h->combine_prefetch = -1;       // automatic (combine_launch)
  h->copy_prefetch = -1;         // automatic
  h->copy_vec_bytes = 32;
  h->combine_pipeline = -1;
  h->copy_ctas_per_sm = 1;
  // Measured on the decode, Zipf, wide-EP and prefill workloads: the separate
  // routing kernel, running beside the copy (programmatic dependent launch), beat
  // routing inside the copy kernel on every one (decode 47.2 against 49.4 us,
  // wide EP 115.9 against 123.9 us, Zipf 135.6 against 146.8 us per step), and
  // the sender-side FP8 expert combine with its rows in shared memory beat the
  // cluster kernel (decode 83 against 175 us).
  h->route_in_copy = 0;
  h->fp8_experts_kernel = 0;
  h->copy_stages = 4;
  h->combine_threads = 0;
  h->bulk_min_row = 0;
  h->combine_ctas_per_sm = 0;
  h->profiling = false;
  h->prof_max = 0;
  *out_handle = h;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_set_option(ep_a2a_handle h, ep_a2a_option option, int64_t value) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  switch (option) {
    case EP_A2A_OPT_COPY_PATH:
      if (value < 0 || value > 2)
        return fail(EP_A2A_ERR_INVALID_ARG, "copy path must be 0, 1 or 2");
      h->copy_path = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_CTAS_PER_SM:
      if (value < 1 || value > 8) return fail(EP_A2A_ERR_INVALID_ARG, "CTAs per SM must be 1..8");
      h->copy_ctas_per_sm = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_STAGES:
      if (value != 0 && (value < 2 || value > kMaxStages))
        return fail(EP_A2A_ERR_INVALID_ARG, "stages must be 0 (automatic) or 2..%d", kMaxStages);
      h->copy_stages = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COMBINE_THREADS:
      if (value != 0 && (value < 64 || value > 512 || value % 32 != 0))
        return fail(EP_A2A_ERR_INVALID_ARG,
                    "combine threads must be 0 (automatic) or a multiple of 32 in 64..512");
      h->combine_threads = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_CONSUMER_WARPS:
      if (value != 4 && value != 8 && value != 16)
        return fail(EP_A2A_ERR_INVALID_ARG, "consumer warps must be 4, 8 or 16");
      h->copy_consumer_warps = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_INTERLEAVE:
      if (value != 0 && value != 1)
        return fail(EP_A2A_ERR_INVALID_ARG, "interleave must be 0 or 1");
      h->copy_interleave = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_VEC_UNROLL:
      if (value != 0 && value != 2 && value != 4 && value != 8)
        return fail(EP_A2A_ERR_INVALID_ARG, "vector unroll must be 0 (automatic), 2, 4 or 8");
      h->vec_unroll = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_VEC_CTAS_PER_SM:
      if (value < 0 || value > 64)
        return fail(EP_A2A_ERR_INVALID_ARG,
                    "vector copy CTAs per SM must be 0 (automatic) or 1..64");
      h->vec_ctas_per_sm = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_STORE_STREAMING:
      if (value != 0 && value != 1) return fail(EP_A2A_ERR_INVALID_ARG, "streaming must be 0 or 1");
      h->store_streaming = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_VEC_THREADS_PER_TOKEN:
      if (value != 0 && value != 32 && value != 64 && value != 128 && value != 256)
        return fail(EP_A2A_ERR_INVALID_ARG, "threads per token must be 0, 32, 64, 128 or 256");
      h->vec_threads_per_token = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COMBINE_PREFETCH:
      if (value < -1 || value > 4)
        return fail(EP_A2A_ERR_INVALID_ARG, "prefetch must be -1 (FP8 only), 0 or 1..4");
      h->combine_prefetch = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_VEC_BYTES:
      if (value != 16 && value != 32)
        return fail(EP_A2A_ERR_INVALID_ARG, "vector copy width must be 16 or 32 bytes");
      h->copy_vec_bytes = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COMBINE_PIPELINE:
      if (value < -1 || value > 2)
        return fail(EP_A2A_ERR_INVALID_ARG,
                    "combine pipeline must be -1 (automatic), 0, 1 or 2 (staged)");
      h->combine_pipeline = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COPY_PREFETCH:
      if (value < -1 || value > 1)
        return fail(EP_A2A_ERR_INVALID_ARG, "prefetch must be -1 (automatic), 0 or 1");
      h->copy_prefetch = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_PDL:
      if (value != 0 && value != 1) return fail(EP_A2A_ERR_INVALID_ARG, "pdl must be 0 or 1");
      h->pdl = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_BULK_MIN_ROW_BYTES:
      if (value < 0 || value > (1 << 24))
        return fail(EP_A2A_ERR_INVALID_ARG, "bulk minimum row bytes must be 0..2^24");
      h->bulk_min_row = value;
      return EP_A2A_OK;
    case EP_A2A_OPT_COMBINE_CTAS_PER_SM:
      if (value < 0 || value > 1024)
        return fail(EP_A2A_ERR_INVALID_ARG, "combine CTAs per SM must be 0..1024");
      h->combine_ctas_per_sm = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_FP8_EXPERTS_KERNEL:
      if (value < 0 || value > 2)
        return fail(EP_A2A_ERR_INVALID_ARG, "FP8 experts kernel must be 0, 1 or 2");
      h->fp8_experts_kernel = (int)value;
      return EP_A2A_OK;
    case EP_A2A_OPT_ROUTE_IN_COPY:
      if (value != 0 && value != 1)
        return fail(EP_A2A_ERR_INVALID_ARG, "route in copy must be 0 or 1");
      h->route_in_copy = (int)value;
      return EP_A2A_OK;
  }
  return fail(EP_A2A_ERR_INVALID_ARG, "unknown option %d", (int)option);
}

EP_API ep_a2a_status ep_a2a_dispatch(ep_a2a_handle h, const int32_t* token_selected_experts,
                                     const int32_t* local_num_tokens,
                                     int32_t runtime_max_tokens_per_rank,
                                     const void* const* payloads,
                                     const int64_t* payload_row_bytes, int32_t num_payloads,
                                     const int32_t* eplb_local_stats,
                                     const uint64_t* active_rank_mask, void* stream_v,
                                     ep_a2a_dispatch_result* result) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  const ep_a2a_params& p = h->p;
  const Layout& L = h->L;
  cudaStream_t stream = (cudaStream_t)stream_v;
  const int ep = p.ep_size;
  if (!token_selected_experts) return fail(EP_A2A_ERR_INVALID_ARG, "token_selected_experts is NULL");
  if (!local_num_tokens) return fail(EP_A2A_ERR_INVALID_ARG, "local_num_tokens is NULL");
  if (!result) return fail(EP_A2A_ERR_INVALID_ARG, "result is NULL");
  const int tpr = runtime_max_tokens_per_rank <= 0 ? p.max_tokens_per_rank
                                                   : runtime_max_tokens_per_rank;
  if (tpr > p.max_tokens_per_rank)
    return fail(EP_A2A_ERR_CAPACITY, "runtime_max_tokens_per_rank %d exceeds capacity %d", tpr,
                p.max_tokens_per_rank);
  if (num_payloads < 0 || num_payloads > p.num_payloads)
    return fail(EP_A2A_ERR_INVALID_ARG, "num_payloads %d outside 0..%d", num_payloads,
                p.num_payloads);
  if (num_payloads > 0 && !payloads) return fail(EP_A2A_ERR_INVALID_ARG, "payloads is NULL");
  int64_t rb[kMaxPayloads] = {0};
  for (int i = 0; i < num_payloads; ++i) {
    rb[i] = payload_row_bytes ? payload_row_bytes[i] : p.payload_row_bytes[i];
    if (rb[i] < 1 || rb[i] > p.payload_row_bytes[i])
      return fail(EP_A2A_ERR_CAPACITY, "payload %d row bytes %lld outside 1..%lld", i,
                  (long long)rb[i], (long long)p.payload_row_bytes[i]);
    if (!payloads[i]) return fail(EP_A2A_ERR_INVALID_ARG, "payload %d is NULL", i);
  }
  if (eplb_local_stats && p.eplb_stats_num_experts == 0)
    return fail(EP_A2A_ERR_INVALID_ARG,
                "eplb_local_stats given but the handle was created with eplb_stats_num_experts=0");
  if (eplb_local_stats && !aligned(eplb_local_stats, 16))
    return fail(EP_A2A_ERR_INVALID_ARG, "eplb_local_stats must be 16-byte aligned");
  if (active_rank_mask && !p.enable_rank_mask)
    return fail(EP_A2A_ERR_INVALID_ARG, "active_rank_mask needs enable_rank_mask");

  RouteArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  for (int w = 0; w < kMaskWords; ++w) ra.live[w] = ~0ull;
  if (active_rank_mask) {
    bool any = false;
    for (int w = 0; w < kMaskWords; ++w) ra.live[w] = active_rank_mask[w];
    for (int r = 0; r < ep; ++r) any |= ((ra.live[r >> 6] >> (r & 63)) & 1ull) != 0;
    if (!any) return fail(EP_A2A_ERR_INVALID_ARG, "active_rank_mask has no active rank");
  }
  for (int r = 0; r < ep; ++r) {
    const int n = local_num_tokens[r];
    if (n < 0 || n > tpr)
      return fail(EP_A2A_ERR_INVALID_ARG, "local_num_tokens[%d] = %d outside 0..%d", r, n, tpr);
    const bool live = ((ra.live[r >> 6] >> (r & 63)) & 1ull) != 0;
    ra.n[r] = live ? n : 0;
  }

  uint8_t* ws = h->ws;
  uint8_t* rank0 = ws + L.rank_base;
  const int64_t ntok = (int64_t)ep * tpr;
  ra.ids = token_selected_experts;
  ra.eplb_stats = eplb_local_stats;
  ra.plan_nd = ws + L.off_plan_nd;
  ra.plan_dst = ws + L.off_plan_dst;
  ra.count_acc = reinterpret_cast<int32_t*>(ws + L.off_count_acc);
  ra.count_ticket = reinterpret_cast<uint32_t*>(ws + L.off_ticket);
  ra.send_counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
  ra.rank0 = rank0;
  ra.rank_stride = L.rank_stride;
  ra.off_ids = L.off_ids;
  ra.off_valid = L.off_valid;
  ra.off_eplb = L.off_eplb;
  ra.ep = ep;
  ra.E = p.num_experts;
  ra.k = p.top_k;
  ra.tpr = tpr;
  ra.epr = p.num_experts / ep;
  ra.plan_stride = L.plan_stride;
  ra.eplb_n = p.eplb_stats_num_experts;
  ra.invalid_id = p.invalid_expert_id;
  // On the vector copy path the copy kernel routes each token itself and writes
  // everything the routing kernel would (one launch per dispatch); the bulk
  // paths read the plan, so they run after the routing kernel.
  const bool fused = h->copy_path == 1 && h->route_in_copy != 0;
  int slot = -1;
  const bool pdl = h->pdl != 0;
  cudaError_t e = cudaSuccess;
  if (!fused) {
    slot = prof_begin(h, EP_A2A_KERNEL_ROUTE_PLAN, stream);
    e = launch_route_plan(ra, active_rank_mask != nullptr, stream, pdl);
    prof_end(h, slot, stream);
    if (e != cudaSuccess) return cuda_fail(e, "routing-plan kernel launch");
  }

  // split payloads between the bulk-async copy and the vector copy
  CopyArgs bulk, vec;
  std::memset(&bulk, 0, sizeof(bulk));
  bulk.plan_nd = ra.plan_nd;
  bulk.plan_dst = ra.plan_dst;
  bulk.rank0 = rank0;
  bulk.rank_stride = L.rank_stride;
  bulk.ntok = ntok;
  bulk.plan_stride = L.plan_stride;
  bulk.err = reinterpret_cast<uint32_t*>(ws + L.off_err);
  bulk.interleave = h->copy_interleave;
  bulk.ids = token_selected_experts;
  bulk.E = p.num_experts;
  bulk.k = p.top_k;
  bulk.epr = p.num_experts / ep;
  bulk.tpr = tpr;
  bulk.use_mask = active_rank_mask != nullptr;
  bulk.prefetch = h->copy_prefetch;
  std::memcpy(bulk.n, ra.n, sizeof(bulk.n));
  std::memcpy(bulk.live, ra.live, sizeof(bulk.live));
  bulk.ep = ep;
  vec = bulk;
  if (fused) {
    vec.route = 1;
    vec.invalid_id = ra.invalid_id;
    vec.count_acc = ra.count_acc;
    vec.count_ticket = ra.count_ticket;
    vec.send_counts = ra.send_counts;
    vec.off_ids = ra.off_ids;
    vec.off_valid = ra.off_valid;
    vec.off_eplb = ra.off_eplb;
    vec.eplb_stats = ra.eplb_stats;
    vec.eplb_n = ra.eplb_n;
  }
  uint32_t stage = 0;
  for (int i = 0; i < num_payloads; ++i) {
    const uint8_t* src = static_cast<const uint8_t*>(payloads[i]);
    const bool bulk_ok =
        h->copy_path != 1 && rb[i] % 16 == 0 && aligned(src, 16) && rb[i] >= h->bulk_min_row;
    CopyArgs& c = bulk_ok ? bulk : vec;
    const int j = c.np++;
    c.src[j] = src;
    c.rb[j] = rb[i];
    c.dst_off[j] = L.off_payload[i];
    if (bulk_ok) {
      c.smem_off[j] = stage;
      stage += (uint32_t)rb[i];
    } else {
      c.vec[j] = vec_bytes(src, rank0 + L.off_payload[i], L.rank_stride, rb[i],
                           (uint32_t)h->copy_vec_bytes);
    }
  }
  if (bulk.np > 0) {
    bulk.tx_bytes = stage;
    bulk.stage_bytes = (uint32_t)align_up(stage, 128);
    // shared memory per CTA when `ctas` CTAs share an SM (1 KB per block is
    // reserved by the hardware; 2 KB covers the kernel's static arrays)
    const int ctas = h->copy_ctas_per_sm;
    const int64_t per_cta =
        std::min<int64_t>(h->max_smem_optin, (int64_t)228 * 1024 / ctas - 1024) - 2048;
    const bool staged = h->copy_path == 0;
    int64_t stages = h->copy_stages > 0 ? h->copy_stages : (staged ? 8 : 16);
    stages = std::min<int64_t>(stages, per_cta / bulk.stage_bytes);
    // the staged kernel holds a token's rows in its threads' registers
    const bool fits = !staged || (int64_t)(stage / 16) <=
                                     (int64_t)kStagedMaxVec * 32 * h->copy_consumer_warps;
    if (stages < 2 || !fits) {
      // rows too large to stage: move them with the vector copy instead
      for (int j = 0; j < bulk.np; ++j) {
        const int k = vec.np++;
        vec.src[k] = bulk.src[j];
        vec.rb[k] = bulk.rb[j];
        vec.dst_off[k] = bulk.dst_off[j];
        vec.vec[k] = vec_bytes(bulk.src[j], rank0 + bulk.dst_off[j], L.rank_stride, bulk.rb[j],
                               (uint32_t)h->copy_vec_bytes);
      }
      bulk.np = 0;
    } else {
      bulk.stages = (int)stages;
      const int grid =
          (int)std::max<int64_t>(1, std::min<int64_t>((int64_t)h->num_sms * ctas, ntok));
      if (staged) {
        slot = prof_begin(h, EP_A2A_KERNEL_COPY_STAGED, stream);
        e = launch_dispatch_staged(bulk, h->copy_consumer_warps, grid, stream, pdl);
      } else {
        slot = prof_begin(h, EP_A2A_KERNEL_COPY_BULK, stream);
        e = launch_dispatch_bulk(bulk, grid, stream, pdl);
      }
      prof_end(h, slot, stream);
      if (e != cudaSuccess) return cuda_fail(e, "bulk copy kernel launch");
    }
  }
  if (vec.np > 0 || fused) {
    const int64_t row_vectors = largest_row_vectors(vec);
    const int tpt = h->vec_threads_per_token > 0 ? h->vec_threads_per_token
                                                 : copy_threads_per_token(ntok, row_vectors);
    const int64_t groups_per_cta = 256 / tpt;
    // CTAs per SM and next-token prefetch: with at most 8 token slots per SM
    // and a 256-thread group per token, the four CTAs an SM holds loop over
    // the tokens and ask for each one's next token's rows to be brought into
    // L2 (decode step: 42.6 against 44.2-44.9 us per step; no gain on the
    // Zipf or wide-EP steps, where the default is 32 CTAs per SM requested and
    // no prefetch)
    const bool few = ntok <= (int64_t)8 * h->num_sms && tpt == 256;
    const int cps = h->vec_ctas_per_sm > 0 ? h->vec_ctas_per_sm : (few ? 4 : 32);
    vec.prefetch = h->copy_prefetch >= 0 ? h->copy_prefetch : (few ? 1 : 0);
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((ntok + groups_per_cta - 1) / groups_per_cta,
                             (int64_t)h->num_sms * cps));
    const int unroll = h->vec_unroll > 0 ? h->vec_unroll : copy_unroll(row_vectors, tpt);
    slot = prof_begin(h, EP_A2A_KERNEL_COPY_VEC, stream);
    e = launch_dispatch_vec(vec, grid, unroll, tpt, h->store_streaming != 0, stream, pdl);
    prof_end(h, slot, stream);
    if (e != cudaSuccess) return cuda_fail(e, "vector copy kernel launch");
  }

  std::memset(result, 0, sizeof(*result));
  result->tokens_per_rank = tpr;
  result->num_payloads = num_payloads;
  result->rank_stride_bytes = L.rank_stride;
  for (int i = 0; i < num_payloads; ++i) result->recv_payloads[i] = rank0 + L.off_payload[i];
  result->recv_topk_ids = reinterpret_cast<int32_t*>(rank0 + L.off_ids);
  result->recv_valid = rank0 + L.off_valid;
  result->eplb_gathered_stats =
      eplb_local_stats ? reinterpret_cast<int32_t*>(rank0 + L.off_eplb) : nullptr;
  result->send_counts = ra.send_counts;
  result->plan_num_dst = ra.plan_nd;
  result->plan_dst_ranks = ra.plan_dst;
  result->plan_stride = L.plan_stride;
  h->have_plan = true;
  h->last_tpr = tpr;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_combine(ep_a2a_handle h, const void* expert_output,
                                    ep_a2a_combine_dtype dtype, void* output, void* stream_v) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return fail(EP_A2A_ERR_NO_PLAN, "combine needs a preceding dispatch");
  if (!expert_output || !output)
    return fail(EP_A2A_ERR_INVALID_ARG, "expert_output / output is NULL");
  if (dtype != EP_A2A_COMBINE_BF16 && dtype != EP_A2A_COMBINE_FP8_E4M3)
    return fail(EP_A2A_ERR_INVALID_ARG, "unknown combine dtype %d", (int)dtype);
  const bool fp8 = dtype == EP_A2A_COMBINE_FP8_E4M3;
  CombineArgs a;
  a.plan_nd = h->ws + h->L.off_plan_nd;
  a.plan_dst = h->ws + h->L.off_plan_dst;
  a.x = static_cast<const uint8_t*>(expert_output);
  a.out = static_cast<uint16_t*>(output);
  a.ntok = (int64_t)h->p.ep_size * h->last_tpr;
  a.H = h->combine_hidden;
  a.plan_stride = h->L.plan_stride;
  a.ep = h->p.ep_size;
  a.err = reinterpret_cast<uint32_t*>(h->ws + h->L.off_err);
  const CombineLaunch c = combine_launch(h, fp8 ? kKindFp8 : kKindBf16, a.ntok);
  a.prefetch = c.prefetch;
  a.out32 = aligned(output, 32) ? 1 : 0;
  const int elems = fp8 ? 16 : 8;
  const bool vec = a.H % elems == 0 && aligned(expert_output, 16) && aligned(output, 16);
  const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE, (cudaStream_t)stream_v);
  cudaError_t e;
  if (vec && c.staged)
    e = launch_combine_staged(a, fp8 ? 1 : 0, nullptr, h->num_sms * c.staged_ctas_per_sm,
                              c.staged_ctas_per_sm, h->max_smem_optin, (cudaStream_t)stream_v,
                              h->pdl != 0);
  else
    e = launch_combine(a, fp8, vec, c.pipe, c.threads, c.grid, (cudaStream_t)stream_v,
                       h->pdl != 0, c.tight);
  prof_end(h, slot, (cudaStream_t)stream_v);
  if (e != cudaSuccess) return cuda_fail(e, "combine kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_combine_experts(ep_a2a_handle h, const float* topk_weights,
                                            const void* expert_output_per_slot, void* output,
                                            void* stream_v) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return fail(EP_A2A_ERR_NO_PLAN, "combine needs a preceding dispatch");
  if (!topk_weights || !expert_output_per_slot || !output)
    return fail(EP_A2A_ERR_INVALID_ARG, "topk_weights / expert output / output is NULL");
  CombineExpertsArgs a;
  a.plan_nd = h->ws + h->L.off_plan_nd;
  a.plan_dst = h->ws + h->L.off_plan_dst;
  a.recv_ids0 = h->ws + h->L.rank_base + h->L.off_ids;
  a.rank_stride = h->L.rank_stride;
  a.w = topk_weights;
  a.y = static_cast<const uint16_t*>(expert_output_per_slot);
  a.out = static_cast<uint16_t*>(output);
  a.ntok = (int64_t)h->p.ep_size * h->last_tpr;
  a.H = h->combine_hidden;
  a.k = h->p.top_k;
  a.E = h->p.num_experts;
  a.epr = h->p.num_experts / h->p.ep_size;
  a.plan_stride = h->L.plan_stride;
  a.ep = h->p.ep_size;
  a.err = reinterpret_cast<uint32_t*>(h->ws + h->L.off_err);
  const CombineLaunch c = combine_launch(h, kKindExperts, a.ntok);
  a.prefetch = c.prefetch;
  const bool vec = a.k <= 8 && a.H % 8 == 0 && aligned(expert_output_per_slot, 16) &&
                   aligned(output, 16);
  const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE_EXPERTS, (cudaStream_t)stream_v);
  cudaError_t e;
  if (vec && c.staged)
    e = launch_combine_experts_staged(a, h->num_sms * c.staged_ctas_per_sm, c.staged_ctas_per_sm,
                                      h->max_smem_optin, (cudaStream_t)stream_v, h->pdl != 0);
  else
    e = launch_combine_experts(a, vec, c.pipe, c.threads, c.grid, (cudaStream_t)stream_v,
                               h->pdl != 0);
  prof_end(h, slot, (cudaStream_t)stream_v);
  if (e != cudaSuccess) return cuda_fail(e, "expert combine kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_combine_experts_fp8(ep_a2a_handle h, const float* topk_weights,
                                                const void* expert_output_per_slot, void* output,
                                                void* stream_v) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return fail(EP_A2A_ERR_NO_PLAN, "combine needs a preceding dispatch");
  if (!topk_weights || !expert_output_per_slot || !output)
    return fail(EP_A2A_ERR_INVALID_ARG, "topk_weights / expert output / output is NULL");
  CombineExpertsArgs a;
  a.plan_nd = h->ws + h->L.off_plan_nd;
  a.plan_dst = h->ws + h->L.off_plan_dst;
  a.recv_ids0 = h->ws + h->L.rank_base + h->L.off_ids;
  a.rank_stride = h->L.rank_stride;
  a.w = topk_weights;
  a.y = static_cast<const uint16_t*>(expert_output_per_slot);
  a.out = static_cast<uint16_t*>(output);
  a.ntok = (int64_t)h->p.ep_size * h->last_tpr;
  a.H = h->combine_hidden;
  a.k = h->p.top_k;
  a.E = h->p.num_experts;
  a.epr = h->p.num_experts / h->p.ep_size;
  a.plan_stride = h->L.plan_stride;
  a.ep = h->p.ep_size;
  a.err = reinterpret_cast<uint32_t*>(h->ws + h->L.off_err);
  // the split kernel (below) prefetches a CTA's slice of the slot rows of the
  // token this many steps ahead: automatic 1 from 8192 token slots (prefill:
  // 1389 against 1426 us; Zipf 328 against 336 us), 0 below (slower by 4-5 %
  // on the decode and wide-EP steps)
  a.prefetch = h->combine_prefetch >= 0 ? h->combine_prefetch : (a.ntok >= 8192 ? 1 : 0);
  const bool vec8 = a.k <= 8 && a.H % 8 == 0 && aligned(expert_output_per_slot, 16) &&
                    aligned(output, 16);
  const int nvec = a.H / 8;
  const int rows = std::min(h->p.top_k, h->p.ep_size);
  if (vec8 && h->fp8_experts_kernel == 0) {
    // a cluster of C CTAs per token, each a slice of at most 512 column vectors
    // (two per thread) with its rows z_d in shared memory; C the fewest that
    // keep a slice's rows within 72 KB (three CTAs per SM)
    int C = 1;
    while (C < 8 && ((nvec + C - 1) / C > 512 ||
                     (int64_t)rows * ((nvec + C - 1) / C) * 16 > 72 * 1024))
      C *= 2;
    const int cvec = (nvec + C - 1) / C;
    if (cvec <= 512 && (int64_t)rows * cvec * 16 <= 72 * 1024) {
      const int threads = std::max(32, ((cvec + 1) / 2 + 31) / 32 * 32);
      const int cps = h->combine_ctas_per_sm > 0 ? h->combine_ctas_per_sm : 3;
      const int clusters = (int)std::max<int64_t>(
          1, std::min<int64_t>(a.ntok, std::max<int64_t>(1, (int64_t)h->num_sms * cps / C)));
      const size_t smem = (size_t)rows * cvec * 16;
      const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE_EXPERTS_FP8, (cudaStream_t)stream_v);
      cudaError_t e = launch_combine_experts_fp8_split(a, C, threads, cvec * 8, clusters, smem,
                                                       (cudaStream_t)stream_v, h->pdl != 0);
      prof_end(h, slot, (cudaStream_t)stream_v);
      if (e != cudaSuccess) return cuda_fail(e, "FP8 expert combine (split) kernel launch");
      return EP_A2A_OK;
    }
  }
  if (vec8 && h->fp8_experts_kernel == 1 && nvec <= 8 * 256) {
    // a cluster of C CTAs per token, one column vector per thread (the rows
    // z_d stay in registers); two CTAs per SM
    int C = 1;
    while (C * 256 < nvec) C *= 2;
    const int threads = ((nvec + C - 1) / C + 31) / 32 * 32;
    const int cps = h->combine_ctas_per_sm > 0 ? h->combine_ctas_per_sm : 2;
    const int clusters = (int)std::max<int64_t>(
        1, std::min<int64_t>(a.ntok, std::max<int64_t>(1, (int64_t)h->num_sms * cps / C)));
    const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE_EXPERTS_FP8, (cudaStream_t)stream_v);
    cudaError_t e = launch_combine_experts_fp8_cluster(a, C, threads, clusters,
                                                       (cudaStream_t)stream_v, h->pdl != 0);
    prof_end(h, slot, (cudaStream_t)stream_v);
    if (e != cudaSuccess) return cuda_fail(e, "FP8 expert combine (cluster) kernel launch");
    return EP_A2A_OK;
  }
  // The shared-memory kernel keeps a token's rows z_d (one per destination, at
  // most min(top_k, ep_size)) as bf16; two CTAs of at most 448 threads share an
  // SM when the rows take at most half of its shared memory.
  const size_t smem = (size_t)rows * a.H * 2;
  const bool smem_rows = a.k <= 8 && a.H % 8 == 0 && aligned(expert_output_per_slot, 16) &&
                         aligned(output, 16) && (int64_t)smem <= h->max_smem_optin - 2048;
  int threads, cps;
  if (smem_rows) {
    const int nvec = a.H / 8;
    threads = std::min(448, std::max(32, ((nvec + 1) / 2 + 31) / 32 * 32));
    cps = 2;
  } else {
    threads = 256;
    cps = 8;
  }
  if (h->combine_threads > 0) threads = std::min(h->combine_threads, smem_rows ? 448 : 256);
  if (h->combine_ctas_per_sm > 0) cps = h->combine_ctas_per_sm;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(a.ntok, (int64_t)h->num_sms * cps));
  const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE_EXPERTS_FP8, (cudaStream_t)stream_v);
  cudaError_t e = launch_combine_experts_fp8(a, smem_rows, threads, grid, smem_rows ? smem : 0,
                                             (cudaStream_t)stream_v, h->pdl != 0);
  prof_end(h, slot, (cudaStream_t)stream_v);
  if (e != cudaSuccess) return cuda_fail(e, "FP8 expert combine kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_combine_scaled(ep_a2a_handle h, const void* expert_output_e4m3,
                                           const float* row_scales, void* output,
                                           void* stream_v) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return fail(EP_A2A_ERR_NO_PLAN, "combine needs a preceding dispatch");
  if (!expert_output_e4m3 || !row_scales || !output)
    return fail(EP_A2A_ERR_INVALID_ARG, "expert_output / row_scales / output is NULL");
  CombineArgs a;
  a.plan_nd = h->ws + h->L.off_plan_nd;
  a.plan_dst = h->ws + h->L.off_plan_dst;
  a.x = static_cast<const uint8_t*>(expert_output_e4m3);
  a.out = static_cast<uint16_t*>(output);
  a.ntok = (int64_t)h->p.ep_size * h->last_tpr;
  a.H = h->combine_hidden;
  a.plan_stride = h->L.plan_stride;
  a.ep = h->p.ep_size;
  a.err = reinterpret_cast<uint32_t*>(h->ws + h->L.off_err);
  const CombineLaunch c = combine_launch(h, kKindFp8, a.ntok);
  a.prefetch = c.prefetch;
  a.out32 = aligned(output, 32) ? 1 : 0;
  const bool vec = a.H % 16 == 0 && aligned(expert_output_e4m3, 16) && aligned(output, 16);
  const int slot = prof_begin(h, EP_A2A_KERNEL_COMBINE, (cudaStream_t)stream_v);
  cudaError_t e;
  if (vec && c.staged)
    e = launch_combine_staged(a, 2, row_scales, h->num_sms * c.staged_ctas_per_sm,
                              c.staged_ctas_per_sm, h->max_smem_optin, (cudaStream_t)stream_v,
                              h->pdl != 0);
  else
    e = launch_combine_scaled(a, row_scales, vec, c.pipe, c.threads, c.grid,
                              (cudaStream_t)stream_v, h->pdl != 0);
  prof_end(h, slot, (cudaStream_t)stream_v);
  if (e != cudaSuccess) return cuda_fail(e, "scaled combine kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_quantize_e4m3_rows(const void* bf16_in, void* e4m3_out,
                                               float* row_scales, int64_t rows, int32_t hidden,
                                               void* stream) {
  if (rows < 0 || hidden < 1) return fail(EP_A2A_ERR_INVALID_ARG, "rows < 0 or hidden < 1");
  if (rows > 0 && (!bf16_in || !e4m3_out || !row_scales))
    return fail(EP_A2A_ERR_INVALID_ARG, "NULL buffer");
  cudaError_t e = launch_quantize_e4m3_rows(static_cast<const uint16_t*>(bf16_in),
                                            static_cast<uint8_t*>(e4m3_out), row_scales, rows,
                                            hidden, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "row quantize kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_quantize_e4m3(const void* bf16_in, void* e4m3_out, int64_t n,
                                          void* stream) {
  if (n < 0) return fail(EP_A2A_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && (!bf16_in || !e4m3_out)) return fail(EP_A2A_ERR_INVALID_ARG, "NULL buffer");
  cudaError_t e = launch_quantize_e4m3(static_cast<const uint16_t*>(bf16_in),
                                       static_cast<uint8_t*>(e4m3_out), n, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "quantize kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_get_status(ep_a2a_handle h, void* stream) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t word = 0;
  uint32_t* dev_word = reinterpret_cast<uint32_t*>(h->ws + h->L.off_err);
  e = cudaMemcpy(&word, dev_word, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word != 0) {
    e = cudaMemset(dev_word, 0, sizeof(word));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    if (word & kErrWaitTimeout)
      return fail(EP_A2A_ERR_DEVICE_TIMEOUT, "a bounded wait in a kernel ran out (word 0x%x)",
                  word);
    if (word & kErrBounds)
      return fail(EP_A2A_ERR_DEVICE_BOUNDS,
                  "a kernel found a plan entry out of range and skipped it (word 0x%x)", word);
  }
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_debug_wait_probe(ep_a2a_handle h, int64_t limit_ns, void* stream) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (limit_ns < 1 || limit_ns > 10000000000ll)
    return fail(EP_A2A_ERR_INVALID_ARG, "limit_ns must be in 1..1e10");
  cudaError_t e = launch_wait_timeout_probe(reinterpret_cast<uint32_t*>(h->ws + h->L.off_err),
                                            (unsigned long long)limit_ns, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "probe kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_profile_start(ep_a2a_handle h, int32_t max_launches) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (max_launches < 1 || max_launches > (1 << 20))
    return fail(EP_A2A_ERR_INVALID_ARG, "max_launches must be in 1..2^20");
  prof_free(h);
  h->prof_events.resize(2 * (size_t)max_launches);
  for (size_t i = 0; i < h->prof_events.size(); ++i) {
    cudaError_t e = cudaEventCreate(&h->prof_events[i]);
    if (e != cudaSuccess) {
      h->prof_events.resize(i);
      prof_free(h);
      return cuda_fail(e, "cudaEventCreate");
    }
  }
  h->prof_kernel.reserve(max_launches);
  h->prof_max = max_launches;
  h->profiling = true;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_profile_stop(ep_a2a_handle h, ep_a2a_kernel_times* times) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (!h->profiling) return fail(EP_A2A_ERR_INVALID_ARG, "profiling was not started");
  ep_a2a_kernel_times t;
  std::memset(&t, 0, sizeof(t));
  for (size_t i = 0; i < h->prof_kernel.size(); ++i) {
    cudaError_t e = cudaEventSynchronize(h->prof_events[2 * i + 1]);
    float ms = 0.f;
    if (e == cudaSuccess)
      e = cudaEventElapsedTime(&ms, h->prof_events[2 * i], h->prof_events[2 * i + 1]);
    if (e != cudaSuccess) {
      prof_free(h);
      return cuda_fail(e, "reading profiling events");
    }
    t.launches[h->prof_kernel[i]] += 1;
    t.total_ms[h->prof_kernel[i]] += ms;
  }
  prof_free(h);
  if (times) *times = t;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_grow_params(const ep_a2a_params* cur, const ep_a2a_params* req,
                                        ep_a2a_params* out, int32_t* grown) {
  ep_a2a_status st = check_params(cur);
  if (st != EP_A2A_OK) return st;
  if ((st = check_params(req)) != EP_A2A_OK) return st;
  if (!out || !grown) return fail(EP_A2A_ERR_INVALID_ARG, "out / grown is NULL");
  if (cur->ep_size != req->ep_size || cur->num_experts != req->num_experts ||
      cur->top_k != req->top_k)
    return fail(EP_A2A_ERR_INVALID_ARG,
                "ep_size / num_experts / top_k differ (%d/%d/%d vs %d/%d/%d): one handle "
                "serves one of each",
                cur->ep_size, cur->num_experts, cur->top_k, req->ep_size, req->num_experts,
                req->top_k);
  const int32_t inv_cur = cur->invalid_expert_id < 0 ? cur->num_experts : cur->invalid_expert_id;
  const int32_t inv_req = req->invalid_expert_id < 0 ? req->num_experts : req->invalid_expert_id;
  if (inv_cur != inv_req)
    return fail(EP_A2A_ERR_INVALID_ARG, "invalid_expert_id differs (%d vs %d)", inv_cur, inv_req);
  ep_a2a_params g = *cur;
  g.invalid_expert_id = inv_cur;
  g.max_tokens_per_rank = std::max(cur->max_tokens_per_rank, req->max_tokens_per_rank);
  g.hidden_size = std::max(cur->hidden_size, req->hidden_size);
  g.num_payloads = std::max(cur->num_payloads, req->num_payloads);
  for (int i = 0; i < kMaxPayloads; ++i) {
    const int64_t a = i < cur->num_payloads ? cur->payload_row_bytes[i] : 0;
    const int64_t b = i < req->num_payloads ? req->payload_row_bytes[i] : 0;
    g.payload_row_bytes[i] = i < g.num_payloads ? std::max(a, b) : 0;
  }
  g.eplb_stats_num_experts =
      (cur->eplb_stats_num_experts != 0 || req->eplb_stats_num_experts != 0) ? cur->num_experts
                                                                               : 0;
  g.enable_rank_mask = (cur->enable_rank_mask | req->enable_rank_mask) ? 1 : 0;
  if ((int64_t)g.ep_size * g.max_tokens_per_rank > (int64_t)1 << 30)
    return fail(EP_A2A_ERR_UNSUPPORTED, "grown ep_size * max_tokens_per_rank too large");
  bool differs = g.max_tokens_per_rank != cur->max_tokens_per_rank ||
                 g.hidden_size != cur->hidden_size || g.num_payloads != cur->num_payloads ||
                 g.eplb_stats_num_experts != cur->eplb_stats_num_experts ||
                 g.enable_rank_mask != cur->enable_rank_mask;
  for (int i = 0; i < g.num_payloads; ++i)
    differs |= g.payload_row_bytes[i] != cur->payload_row_bytes[i];
  *out = g;
  *grown = differs ? 1 : 0;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_set_combine_hidden(ep_a2a_handle h, int32_t hidden) {
  ep_a2a_status st = check_handle(h);
  if (st != EP_A2A_OK) return st;
  if (hidden < 1) return fail(EP_A2A_ERR_INVALID_ARG, "hidden %d must be >= 1", hidden);
  if (hidden > h->p.hidden_size)
    return fail(EP_A2A_ERR_CAPACITY, "hidden %d exceeds the handle's hidden_size %d", hidden,
                h->p.hidden_size);
  h->combine_hidden = hidden;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_destroy(ep_a2a_handle* hp) {
  if (!hp || !*hp) return EP_A2A_OK;
  ep_a2a_handle h = *hp;
  if (h->magic != kMagic) return fail(EP_A2A_ERR_NOT_INITIALIZED, "handle is not valid");
  prof_free(h);
  h->magic = 0;
  delete h;
  *hp = nullptr;
  return EP_A2A_OK;
}
