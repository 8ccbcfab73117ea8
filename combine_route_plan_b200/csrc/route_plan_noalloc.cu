// Routing plan for callers that cannot allocate device memory.
//
// ep_a2a_dispatch needs a workspace from ep_a2a_init, and part of that
// workspace is scratch for the routing kernel (per-(source, destination)
// send-count accumulators and one ticket per source rank).  Some callers
// cannot provide it: their device memory belongs to an outer allocator (for
// example a serving engine that reserves nearly all of HBM for its own pools
// when it starts, or a host application that does not let plug-in libraries
// call cudaMalloc), so they can hand a library the tensors of a step but
// cannot make it a new buffer.  ep_a2a_route_plan_noalloc runs the same
// routing-plan kernel with that scratch in a fixed device array compiled into
// this file; the caller passes only inputs and outputs.
//
// Limits and sharing: the array holds the scratch of at most
// EP_A2A_NOALLOC_MAX_RANKS ranks (16,640 bytes), and every GPU that loads the
// library keeps it until the process exits.  Its device address is looked up
// once per CUDA context (again after a device reset).  All calls share it: each call
// clears the part it uses on its stream before the kernel, so calls that
// follow one another in stream order are independent, but calls whose work
// overlaps on the GPU (different streams, or different host threads on the
// same device) race on the array.
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "ep_a2a_internal.cuh"

#define EP_API extern "C" __attribute__((visibility("default")))

// Scratch of the routing kernel: count accumulators [ep * ep] followed by
// tickets [ep], for ep <= EP_A2A_NOALLOC_MAX_RANKS.
static __device__ __align__(256)
    uint32_t g_route_scratch[EP_A2A_NOALLOC_MAX_RANKS * EP_A2A_NOALLOC_MAX_RANKS +
                             EP_A2A_NOALLOC_MAX_RANKS];

namespace ep_a2a {
namespace {

constexpr int kNoAllocMaxRanks = EP_A2A_NOALLOC_MAX_RANKS;
constexpr int kMaxDevices = 64;

// The array's device address is only valid in the CUDA context it was looked
// up in.  A device reset (or a primary context released and created again)
// gives the device a new context, where the array has a new address, so the
// cache holds the address together with the context's id (cuCtxGetId: unique
// for the life of the process) and looks it up again when the id changes.
struct ScratchEntry {
  unsigned long long ctx_id;   // 0 = not looked up yet
  void* addr;
};

std::mutex g_setup_mutex;
ScratchEntry g_scratch[kMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
CtxGetCurrentFn g_ctx_get_current = nullptr;
CtxGetIdFn g_ctx_get_id = nullptr;

ep_a2a_status noalloc_fail(ep_a2a_status st, const char* msg) {
  record_last_error(msg);
  return st;
}

// Id of the calling thread's current context (the runtime has made one
// current: callers run cudaGetDevice first, and the lookups below go through
// the driver entry points the runtime hands out, so no driver library is
// linked).
cudaError_t current_context_id(unsigned long long* id) {
  if (g_ctx_get_current == nullptr || g_ctx_get_id == nullptr) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    cudaError_t e = cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1);
    if (e != cudaSuccess) return e;
    e = cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2);
    if (e != cudaSuccess) return e;
    if (q1 != cudaDriverEntryPointSuccess || q2 != cudaDriverEntryPointSuccess || !f1 || !f2)
      return cudaErrorNotSupported;
    g_ctx_get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    g_ctx_get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (g_ctx_get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  if (g_ctx_get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  return cudaSuccess;
}

// Device address of the array on `dev` (the current device) in the current
// context.  The host-side symbol is only a stand-in, so the address is looked
// up (cudaGetSymbolAddress) with that device current, once per context, and
// cached with the context's id.
cudaError_t scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  unsigned long long ctx_id = 0;
  cudaError_t e = current_context_id(&ctx_id);
  if (e != cudaSuccess) return e;
  ScratchEntry& c = g_scratch[dev];
  if (c.ctx_id != ctx_id || c.addr == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    c.ctx_id = ctx_id;
    c.addr = p;
  }
  *out = c.addr;
  return cudaSuccess;
}

}  // namespace
}  // namespace ep_a2a

using namespace ep_a2a;

EP_API ep_a2a_status ep_a2a_route_plan_noalloc(
    int32_t ep_size, int32_t num_experts, int32_t top_k, int32_t tokens_per_rank,
    int32_t invalid_expert_id, const int32_t* token_selected_experts,
    const int32_t* local_num_tokens, const uint64_t* active_rank_mask, uint8_t* plan_num_dst,
    uint8_t* plan_dst_ranks, int32_t* send_counts, int32_t* recv_topk_ids, uint8_t* recv_valid,
    int64_t recv_rank_stride_bytes, void* stream_v) {
  if (ep_size < 1 || ep_size > kNoAllocMaxRanks)
    return noalloc_fail(EP_A2A_ERR_UNSUPPORTED,
                        "ep_size must be 1..64: the fixed scratch array holds 64 ranks");
  if (num_experts <= 0 || num_experts % 4 != 0 || num_experts % ep_size != 0)
    return noalloc_fail(EP_A2A_ERR_INVALID_ARG,
                        "num_experts must be a positive multiple of 4 and of ep_size");
  if (top_k < 1 || top_k > kMaxTopK)
    return noalloc_fail(EP_A2A_ERR_UNSUPPORTED, "top_k must be 1..32");
  if (tokens_per_rank < 1 || (int64_t)ep_size * tokens_per_rank > ((int64_t)1 << 30))
    return noalloc_fail(EP_A2A_ERR_INVALID_ARG, "tokens_per_rank out of range");
  if (!token_selected_experts || !local_num_tokens || !plan_num_dst || !plan_dst_ranks ||
      !send_counts || !recv_topk_ids || !recv_valid)
    return noalloc_fail(EP_A2A_ERR_INVALID_ARG, "NULL input or output pointer");
  if ((reinterpret_cast<uintptr_t>(recv_topk_ids) & 3u) != 0 || (recv_rank_stride_bytes & 3) != 0)
    return noalloc_fail(EP_A2A_ERR_INVALID_ARG,
                        "recv_topk_ids and recv_rank_stride_bytes must be 4-byte aligned");
  const int64_t slots = (int64_t)ep_size * tokens_per_rank;
  // Each rank's two receive arrays: ids [0, ids_bytes) and valid bytes
  // [off_valid, off_valid + slots), relative to its recv_topk_ids.  They must
  // not overlap, and with more than one rank both must fit inside one stride,
  // so that no rank's writes land on another array or another rank's.
  const int64_t ids_bytes = slots * top_k * 4;
  const int64_t off_valid =
      (int64_t)(reinterpret_cast<intptr_t>(recv_valid) - reinterpret_cast<intptr_t>(recv_topk_ids));
  if (off_valid < ids_bytes && off_valid + slots > 0)
    return noalloc_fail(EP_A2A_ERR_INVALID_ARG, "recv_valid overlaps recv_topk_ids");
  if (ep_size > 1) {
    const int64_t lo = off_valid < 0 ? off_valid : 0;
    const int64_t hi = off_valid + slots > ids_bytes ? off_valid + slots : ids_bytes;
    if (recv_rank_stride_bytes < hi - lo)
      return noalloc_fail(EP_A2A_ERR_INVALID_ARG,
                          "recv_rank_stride_bytes is smaller than one rank's recv_topk_ids and "
                          "recv_valid together");
  }

  RouteArgs ra;
  std::memset(&ra, 0, sizeof(ra));
  for (int w = 0; w < kMaskWords; ++w) ra.live[w] = ~0ull;
  if (active_rank_mask) {
    bool any = false;
    for (int w = 0; w < kMaskWords; ++w) ra.live[w] = active_rank_mask[w];
    for (int r = 0; r < ep_size; ++r) any |= ((ra.live[r >> 6] >> (r & 63)) & 1ull) != 0;
    if (!any) return noalloc_fail(EP_A2A_ERR_INVALID_ARG, "active_rank_mask has no active rank");
  }
  for (int r = 0; r < ep_size; ++r) {
    const int n = local_num_tokens[r];
    if (n < 0 || n > tokens_per_rank)
      return noalloc_fail(EP_A2A_ERR_INVALID_ARG, "local_num_tokens[r] outside 0..tokens_per_rank");
    ra.n[r] = ((ra.live[r >> 6] >> (r & 63)) & 1ull) ? n : 0;
  }

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(EP_A2A_ERR_CUDA, cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(EP_A2A_ERR_UNSUPPORTED, "device index");
  void* scratch = nullptr;
  e = scratch_address(dev, &scratch);
  if (e != cudaSuccess) return noalloc_fail(EP_A2A_ERR_CUDA, cudaGetErrorString(e));

  cudaStream_t stream = (cudaStream_t)stream_v;
  const size_t used = ((size_t)ep_size * ep_size + ep_size) * sizeof(uint32_t);
  e = cudaMemsetAsync(scratch, 0, used, stream);   // the kernel expects zeroed scratch
  if (e != cudaSuccess) return noalloc_fail(EP_A2A_ERR_CUDA, cudaGetErrorString(e));

  uint32_t* words = static_cast<uint32_t*>(scratch);
  ra.ids = token_selected_experts;
  ra.eplb_stats = nullptr;
  ra.plan_nd = plan_num_dst;
  ra.plan_dst = plan_dst_ranks;
  ra.count_acc = reinterpret_cast<int32_t*>(words);
  ra.count_ticket = words + (size_t)ep_size * ep_size;
  ra.send_counts = send_counts;
  ra.rank0 = reinterpret_cast<uint8_t*>(recv_topk_ids);
  ra.rank_stride = recv_rank_stride_bytes;
  ra.off_ids = 0;
  ra.off_valid = off_valid;
  ra.off_eplb = 0;
  ra.ep = ep_size;
  ra.E = num_experts;
  ra.k = top_k;
  ra.tpr = tokens_per_rank;
  ra.epr = num_experts / ep_size;
  ra.plan_stride = (int)align_up(top_k, 8);
  ra.eplb_n = 0;
  ra.invalid_id = invalid_expert_id < 0 ? num_experts : invalid_expert_id;
  e = launch_route_plan(ra, active_rank_mask != nullptr, stream);
  if (e != cudaSuccess) return noalloc_fail(EP_A2A_ERR_CUDA, cudaGetErrorString(e));
  return EP_A2A_OK;
}
