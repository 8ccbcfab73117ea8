// Expert-parallel dispatch and combine between real EP ranks: one process per
// rank, each owning a device "window" that its peers write into.
//
// What moves (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, dispatch() and
// combine(); the slot rule of flashinfer.moe_ep.NVLinkOneSidedConfig,
// `lamport` paragraph): rank r sends each of its tokens t, with every payload
// row and its routing ids, once to every live rank d that owns one of its
// top_k experts, landing at slot r * tpr + t of d's receive arrays; rank d
// returns one row per token it received, and rank r sums the rows of each of
// its tokens over its destination ranks in ascending rank order (fp32, one
// rounding to bf16).  The arithmetic and the layouts are those of the
// single-process library (ep_a2a_dispatch / ep_a2a_combine); only the
// transport differs.
//
// Transport.  Each rank's window is exported with a CUDA IPC handle and
// mapped by every other rank (cudaIpcOpenMemHandle).  Senders write rows into
// peer windows with plain stores; no rank loads from a peer's memory, and no
// bulk, TMA or multicast form is used anywhere.  After a kernel's last store
// to a peer, every CTA fences at system scope and takes a ticket; the last
// CTA writes one flag per (source, destination) pair into the destination's
// window with a release store: the step's epoch.  Receivers check the flags
// of every live source with acquire loads in a bounded wait (the pages'
// `timeout_sec`, flashinfer.moe_ep.NVLinkOneSidedConfig, traps the kernel on
// expiry; here the wait gives up after its limit, sets the handle's error
// word, and ep_mp_get_status returns EP_A2A_ERR_DEVICE_TIMEOUT).
//
// The library does no host communication.  The caller separates the send and
// receive phases with its own barrier (all ranks' send kernels complete before
// any rank starts a receive kernel), so no kernel ever waits for a kernel of
// another process to be scheduled; the flag check then confirms that every
// source's rows of this epoch have landed, and catches a rank that skipped
// its send.
#include <cuda.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <new>

#include "ep_a2a_internal.cuh"

#define EP_API extern "C" __attribute__((visibility("default")))

namespace ep_a2a {
namespace {

constexpr unsigned kFullMask = 0xFFFFFFFFu;
constexpr uint32_t kMpMagic = 0x45504d50u;   // "EPMP"
constexpr int64_t kMpAlign = 256;

ep_a2a_status mp_fail(ep_a2a_status st, const char* msg) {
  record_last_error(msg);
  return st;
}

ep_a2a_status mp_cuda_fail(cudaError_t e, const char* what) {
  static thread_local char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", what, cudaGetErrorString(e));
  record_last_error(buf);
  return EP_A2A_ERR_CUDA;
}

// Byte offsets inside one rank's window; the same on every rank.
struct MpLayout {
  // written by this rank only
  int64_t off_err, off_dticket, off_cticket, off_count_acc, off_counts, off_plan_nd,
      off_plan_dst;
  // written by peers
  int64_t off_dflag, off_cflag;          // [ep] u32 each: epoch of source / destination s
  int64_t off_payload[kMaxPayloads];     // [ep*cap, rb_i]
  int64_t off_ids, off_valid, off_eplb;  // [ep*cap, k] i32, [ep*cap] u8, [ep, E] i32
  int64_t off_landing;                   // [ep, cap, hidden] of 2-byte elements
  int64_t local_bytes;                   // [0, local_bytes) is this rank's own state
  int64_t total;
  int plan_stride;
};

MpLayout mp_layout(const ep_a2a_params& p) {
  MpLayout L{};
  const int64_t ep = p.ep_size, cap = p.max_tokens_per_rank, slots = ep * cap;
  L.plan_stride = (int)align_up(p.top_k, 8);
  int64_t c = 0;
  L.off_err = c;        c = align_up(c + 16, kMpAlign);
  L.off_dticket = c;    c = align_up(c + 16, kMpAlign);
  L.off_cticket = c;    c = align_up(c + 16, kMpAlign);
  L.off_count_acc = c;  c = align_up(c + ep * 4, kMpAlign);
  L.off_counts = c;     c = align_up(c + ep * 4, kMpAlign);
  L.off_plan_nd = c;    c = align_up(c + cap, kMpAlign);
  L.off_plan_dst = c;   c = align_up(c + cap * L.plan_stride, kMpAlign);
  L.local_bytes = c;
  L.off_dflag = c;      c = align_up(c + ep * 4, kMpAlign);
  L.off_cflag = c;      c = align_up(c + ep * 4, kMpAlign);
  for (int i = 0; i < kMaxPayloads; ++i) {
    L.off_payload[i] = c;
    if (i < p.num_payloads) c = align_up(c + slots * p.payload_row_bytes[i], kMpAlign);
  }
  L.off_ids = c;        c = align_up(c + slots * p.top_k * 4, kMpAlign);
  L.off_valid = c;      c = align_up(c + slots, kMpAlign);
  L.off_eplb = c;       c = align_up(c + ep * p.eplb_stats_num_experts * 4, kMpAlign);
  L.off_landing = c;    c = align_up(c + slots * (int64_t)p.hidden_size * 2, kMpAlign);
  L.total = c;
  return L;
}

// ---------------------------------------------------------------------------
// Device side
// ---------------------------------------------------------------------------

struct MpSendArgs {
  uint8_t* win[kMaxRanks];               // every rank's window (this rank's own included)
  const int32_t* ids;                    // [tpr, k] this rank's routing ids
  const uint8_t* src[kMaxPayloads];      // [tpr, rb] this rank's payload rows
  int64_t rb[kMaxPayloads];
  int64_t off_payload[kMaxPayloads];
  uint32_t vec[kMaxPayloads];            // bytes per access (16/8/4/2/1)
  int np;
  const int32_t* eplb_stats;             // [E] or nullptr
  int eplb_n;
  int rank, ep, E, k, epr, tpr, n_local, plan_stride, use_mask;
  int32_t invalid_id;
  uint64_t live[kMaskWords];
  int64_t off_ids, off_valid, off_eplb, off_dflag;
  uint8_t* plan_nd;                      // [tpr] this rank's plan (own window)
  uint8_t* plan_dst;                     // [tpr, plan_stride]
  int32_t* count_acc;                    // [ep] scratch; zero between calls
  int32_t* send_counts;                  // [ep] tokens this rank sent to each rank
  uint32_t* ticket;                      // scratch; zero between calls
  uint32_t epoch;
};

struct MpPushArgs {
  uint8_t* win[kMaxRanks];
  const uint8_t* x;                      // [ep*tpr, row] this rank's result per received slot
  const uint8_t* valid;                  // [ep*tpr] own window
  int64_t row;                           // bytes per row (hidden x element bytes)
  uint32_t vec;                          // bytes per access
  int rank, ep, tpr, use_mask;
  uint64_t live[kMaskWords];
  int64_t off_landing, off_cflag;
  uint32_t* ticket;
  uint32_t epoch;
};

__device__ __forceinline__ bool mp_live(const uint64_t* live, int use_mask, int r) {
  return !use_mask || ((live[r >> 6] >> (r & 63)) & 1ull);
}

__device__ __forceinline__ void store_release_sys(uint32_t* p, uint32_t v) {
  asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t load_acquire_sys(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One warp copies `bytes` bytes from s to d in T-sized accesses.
template <typename T>
__device__ __forceinline__ void warp_copy(uint8_t* d, const uint8_t* s, int64_t bytes, int lane) {
  const int64_t n = bytes / (int64_t)sizeof(T);
  const T* sp = reinterpret_cast<const T*>(s);
  T* dp = reinterpret_cast<T*>(d);
  for (int64_t i = lane; i < n; i += 32) dp[i] = sp[i];
}

__device__ __forceinline__ void warp_copy_any(uint8_t* d, const uint8_t* s, int64_t bytes,
                                              uint32_t vec, int lane) {
  switch (vec) {
    case 16: warp_copy<uint4>(d, s, bytes, lane); break;
    case 8: warp_copy<uint2>(d, s, bytes, lane); break;
    case 4: warp_copy<uint32_t>(d, s, bytes, lane); break;
    case 2: warp_copy<uint16_t>(d, s, bytes, lane); break;
    default: warp_copy<uint8_t>(d, s, bytes, lane); break;
  }
}

// The last CTA to finish writes `epoch` into the flag of every live rank (the
// flag at `off_flag + rank * 4` of its window), after every CTA's stores are
// fenced at system scope.  Returns in every thread; the ticket is reset.
__device__ __forceinline__ bool last_cta(uint32_t* ticket) {
  __shared__ bool s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence_system();
    s_last = atomicAdd(ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) __threadfence_system();
  return s_last;
}

// Warp per local token: route (the single-process rule), write the plan and the
// per-destination ids / valid byte into every live rank's window, copy the
// payload rows to the destinations; then dead sources' slots and the EPLB rows;
// then counts and flags.
__global__ void __launch_bounds__(256) mp_send_kernel(const MpSendArgs a) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int64_t gwarp = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * warps;
  for (int64_t t = gwarp; t < a.tpr; t += nwarps) {
    const bool exists = t < a.n_local;
    int32_t e = 0;
    int d = -1;
    if (exists && lane < a.k) {
      e = a.ids[t * a.k + lane];
      if (e >= 0 && e < a.E) {
        const int owner = e / a.epr;
        if (mp_live(a.live, a.use_mask, owner)) d = owner;
      }
    }
    const unsigned peers = __match_any_sync(kFullMask, d);
    const bool leader = d >= 0 && (__ffs(peers) - 1) == lane;
    const unsigned leaders = __ballot_sync(kFullMask, leader);
    const int nd = __popc(leaders);
    int pos = 0;
    uint32_t word = 0;                     // lane w: destination bits 32w..32w+31
    for (int i = 0; i < a.k; ++i) {
      const int other = __shfl_sync(kFullMask, d, i);
      pos += (((leaders >> i) & 1u) != 0u) && other < d;
      if (other >= 0 && (other >> 5) == lane) word |= 1u << (other & 31);
    }
    uint8_t* prow = a.plan_dst + t * a.plan_stride;
    if (lane == 0) a.plan_nd[t] = exists ? (uint8_t)nd : kNoToken;
    if (leader) {
      prow[pos] = (uint8_t)d;
      atomicAdd(&a.count_acc[d], 1);
    }
    if (lane < a.plan_stride && lane >= nd) prow[lane] = kPad;
    const int64_t slot = (int64_t)a.rank * a.tpr + t;
    // ids and valid byte of this slot in every live rank's window
    const int total = a.ep * a.k;
    for (int base = 0; base < total; base += 32) {
      const int idx = base + lane;
      const int dd = idx / a.k;
      const int j = idx - dd * a.k;
      const int32_t ej = __shfl_sync(kFullMask, e, j & 31);
      const uint32_t wd = __shfl_sync(kFullMask, word, (dd >> 5) & 7);
      if (idx < total && mp_live(a.live, a.use_mask, dd)) {
        int32_t* ids = reinterpret_cast<int32_t*>(a.win[dd] + a.off_ids);
        ids[slot * a.k + j] = ((wd >> (dd & 31)) & 1u) ? ej : a.invalid_id;
      }
    }
    for (int base = 0; base < a.ep; base += 32) {
      const int dd = base + lane;
      const uint32_t wd = __shfl_sync(kFullMask, word, (dd >> 5) & 7);
      if (dd < a.ep && mp_live(a.live, a.use_mask, dd))
        a.win[dd][a.off_valid + slot] = (uint8_t)((wd >> (dd & 31)) & 1u);
    }
    // payload rows to each destination (ascending ranks from the set bits)
    unsigned rest = leaders;
    while (rest) {
      const int l = __ffs(rest) - 1;
      rest &= rest - 1u;
      const int dd = __shfl_sync(kFullMask, d, l);
      for (int p = 0; p < a.np; ++p)
        warp_copy_any(a.win[dd] + a.off_payload[p] + slot * a.rb[p], a.src[p] + t * a.rb[p],
                      a.rb[p], a.vec[p], lane);
    }
  }
  // slots of dead sources in this rank's own window: nothing arrives there
  if (a.use_mask) {
    uint8_t* own = a.win[a.rank];
    const int64_t per = (int64_t)a.tpr * a.k;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)a.ep * per;
         i += (int64_t)gridDim.x * blockDim.x) {
      const int s = (int)(i / per);
      if (mp_live(a.live, 1, s)) continue;
      const int64_t rem = i - (int64_t)s * per;
      reinterpret_cast<int32_t*>(own + a.off_ids)[(int64_t)s * per + rem] = a.invalid_id;
      if (rem % a.k == 0) own[a.off_valid + (int64_t)s * a.tpr + rem / a.k] = 0;
    }
  }
  // EPLB: this rank's statistics row into row `rank` of every live rank's
  // gathered array; rows of dead sources in the own window are zero
  if (a.eplb_stats != nullptr) {
    const int64_t total = (int64_t)a.ep * a.eplb_n;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
      const int dd = (int)(i / a.eplb_n);
      const int c = (int)(i - (int64_t)dd * a.eplb_n);
      if (mp_live(a.live, a.use_mask, dd))
        reinterpret_cast<int32_t*>(a.win[dd] + a.off_eplb)[(int64_t)a.rank * a.eplb_n + c] =
            a.eplb_stats[c];
      if (!mp_live(a.live, a.use_mask, dd))     // dd as a dead source row of the own window
        reinterpret_cast<int32_t*>(a.win[a.rank] + a.off_eplb)[(int64_t)dd * a.eplb_n + c] = 0;
    }
  }
  if (last_cta(a.ticket)) {
    for (int i = threadIdx.x; i < a.ep; i += blockDim.x)
      a.send_counts[i] = atomicExch(&a.count_acc[i], 0);
    __threadfence_system();
    __syncthreads();
    for (int dd = threadIdx.x; dd < a.ep; dd += blockDim.x)
      if (mp_live(a.live, a.use_mask, dd))
        store_release_sys(reinterpret_cast<uint32_t*>(a.win[dd] + a.off_dflag) + a.rank, a.epoch);
    if (threadIdx.x == 0) atomicExch(a.ticket, 0u);
  }
}

// Warp per received slot: a valid slot s = src * tpr + t sends this rank's
// row for it to source src's landing rows at [this rank][t]; then flags.
__global__ void __launch_bounds__(256) mp_push_kernel(const MpPushArgs a) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int64_t gwarp = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * warps;
  const int64_t slots = (int64_t)a.ep * a.tpr;
  for (int64_t s = gwarp; s < slots; s += nwarps) {
    if (!a.valid[s]) continue;
    const int src = (int)(s / a.tpr);
    const int64_t t = s - (int64_t)src * a.tpr;
    uint8_t* dst = a.win[src] + a.off_landing + ((int64_t)a.rank * a.tpr + t) * a.row;
    warp_copy_any(dst, a.x + s * a.row, a.row, a.vec, lane);
  }
  if (last_cta(a.ticket)) {
    for (int dd = threadIdx.x; dd < a.ep; dd += blockDim.x)
      if (mp_live(a.live, a.use_mask, dd))
        store_release_sys(reinterpret_cast<uint32_t*>(a.win[dd] + a.off_cflag) + a.rank, a.epoch);
    if (threadIdx.x == 0) atomicExch(a.ticket, 0u);
  }
}

// One warp: wait until the flag of every live rank equals `epoch` (acquire
// loads), for at most limit_ns of %globaltimer in total; on expiry set the
// error word and return.
__global__ void mp_wait_kernel(const uint32_t* flags, int ep, int use_mask,
                               uint64_t live0, uint64_t live1, uint64_t live2, uint64_t live3,
                               uint32_t epoch, unsigned long long limit_ns, uint32_t* err) {
  const uint64_t live[kMaskWords] = {live0, live1, live2, live3};
  const unsigned long long t0 = global_timer_ns();
  bool ok = true;
  for (int r = threadIdx.x; r < ep && ok; r += blockDim.x) {
    if (!mp_live(live, use_mask, r)) continue;
    for (uint32_t it = 0;; ++it) {
      if (load_acquire_sys(flags + r) == epoch) break;
      if ((it & 63u) == 63u && global_timer_ns() - t0 > limit_ns) {
        ok = false;
        break;
      }
      __nanosleep(256);
    }
  }
  if (!ok) atomicOr(err, kErrWaitTimeout);
}

}  // namespace
}  // namespace ep_a2a

using namespace ep_a2a;

struct ep_mp_handle_s {
  uint32_t magic;
  ep_a2a_params p;
  MpLayout L;
  int rank;
  int device;
  int num_sms;
  uint8_t* win[kMaxRanks];               // own window and the mapped peer windows
  void* opened[kMaxRanks];               // bases returned by cudaIpcOpenMemHandle
  uint32_t dispatch_epoch, combine_epoch;
  bool have_plan;
  int last_tpr;
  int last_n;
  bool last_masked;
  uint64_t live[kMaskWords];
};

namespace {

ep_a2a_status mp_check(ep_mp_handle h) {
  if (!h || h->magic != kMpMagic)
    return mp_fail(EP_A2A_ERR_NOT_INITIALIZED, "multi-process handle is NULL or destroyed");
  return EP_A2A_OK;
}

using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

// Base of the allocation that holds `p` (cuMemGetAddressRange, through the
// driver entry point the runtime hands out).
cudaError_t allocation_base(const void* p, void** base) {
  static MemGetAddressRangeFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q);
    if (e != cudaSuccess) return e;
    if (q != cudaDriverEntryPointSuccess || f == nullptr) return cudaErrorNotSupported;
    fn = reinterpret_cast<MemGetAddressRangeFn>(f);
  }
  CUdeviceptr b = 0;
  size_t size = 0;
  if (fn(&b, &size, reinterpret_cast<CUdeviceptr>(p)) != CUDA_SUCCESS)
    return cudaErrorInvalidDevicePointer;
  *base = reinterpret_cast<void*>(b);
  return cudaSuccess;
}

uint32_t access_bytes(const void* a, const void* b, int64_t stride, int64_t rb) {
  for (uint32_t v : {16u, 8u, 4u, 2u}) {
    if (rb % v == 0 && reinterpret_cast<uintptr_t>(a) % v == 0 &&
        reinterpret_cast<uintptr_t>(b) % v == 0 && stride % v == 0)
      return v;
  }
  return 1u;
}

int mp_grid(int num_sms, int64_t warps_of_work) {
  const int64_t ctas = (warps_of_work + 7) / 8;
  return (int)std::max<int64_t>(1, std::min<int64_t>(ctas, (int64_t)num_sms * 8));
}

}  // namespace

EP_API ep_a2a_status ep_mp_window_size(const ep_a2a_params* params, size_t* bytes) {
  size_t ws = 0;
  ep_a2a_status st = ep_a2a_workspace_size(params, &ws);   // the same parameter rules
  if (st != EP_A2A_OK) return st;
  if (!bytes) return mp_fail(EP_A2A_ERR_INVALID_ARG, "bytes is NULL");
  *bytes = (size_t)mp_layout(*params).total;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_export(void* window, ep_mp_ipc_handle* out) {
  if (!window || !out) return mp_fail(EP_A2A_ERR_INVALID_ARG, "window / out is NULL");
  static_assert(sizeof(cudaIpcMemHandle_t) <= sizeof(out->handle), "IPC handle size");
  void* base = nullptr;
  cudaError_t e = allocation_base(window, &base);
  if (e != cudaSuccess) return mp_cuda_fail(e, "finding the window's allocation");
  cudaIpcMemHandle_t h;
  e = cudaIpcGetMemHandle(&h, base);
  if (e != cudaSuccess) return mp_cuda_fail(e, "cudaIpcGetMemHandle");
  std::memset(out, 0, sizeof(*out));
  std::memcpy(out->handle, &h, sizeof(h));
  out->offset = static_cast<uint8_t*>(window) - static_cast<uint8_t*>(base);
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_init(const ep_a2a_params* params, int32_t rank, void* window,
                                size_t window_bytes, const ep_mp_ipc_handle* peers, void* stream,
                                ep_mp_handle* out_handle) {
  size_t need = 0;
  ep_a2a_status st = ep_mp_window_size(params, &need);
  if (st != EP_A2A_OK) return st;
  if (!out_handle) return mp_fail(EP_A2A_ERR_INVALID_ARG, "out_handle is NULL");
  *out_handle = nullptr;
  if (rank < 0 || rank >= params->ep_size)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "rank out of range");
  if (!window || !peers) return mp_fail(EP_A2A_ERR_INVALID_ARG, "window / peers is NULL");
  if (reinterpret_cast<uintptr_t>(window) % kMpAlign != 0)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "window must be 256-byte aligned");
  if (window_bytes < need) return mp_fail(EP_A2A_ERR_INVALID_ARG, "window too small");
  const int ep = params->ep_size;
  for (int r = 0; r < ep; ++r)
    if (r != rank && (peers[r].offset < 0 || peers[r].offset % kMpAlign != 0))
      return mp_fail(EP_A2A_ERR_INVALID_ARG, "peer window offset must be a non-negative "
                                             "multiple of 256");
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return mp_cuda_fail(e, "cudaGetDevice");
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return mp_cuda_fail(e, "cudaDeviceGetAttribute");
  ep_mp_handle h = new (std::nothrow) ep_mp_handle_s();
  if (!h) return mp_fail(EP_A2A_ERR_INVALID_ARG, "out of host memory");
  h->p = *params;
  if (h->p.invalid_expert_id < 0) h->p.invalid_expert_id = h->p.num_experts;
  h->L = mp_layout(*params);
  h->rank = rank;
  h->device = dev;
  h->num_sms = sms;
  h->win[rank] = static_cast<uint8_t*>(window);
  for (int r = 0; r < ep; ++r) {
    if (r == rank) continue;
    cudaIpcMemHandle_t ih;
    std::memcpy(&ih, peers[r].handle, sizeof(ih));
    void* base = nullptr;
    e = cudaIpcOpenMemHandle(&base, ih, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
      for (int q = 0; q < r; ++q)
        if (h->opened[q]) cudaIpcCloseMemHandle(h->opened[q]);
      delete h;
      return mp_cuda_fail(e, "cudaIpcOpenMemHandle (a peer's window)");
    }
    h->opened[r] = base;
    h->win[r] = static_cast<uint8_t*>(base) + peers[r].offset;
  }
  // own state and flags start at zero; epochs start at 1
  e = cudaMemsetAsync(window, 0, (size_t)h->L.off_cflag + ep * 4, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) {
    for (int q = 0; q < ep; ++q)
      if (h->opened[q]) cudaIpcCloseMemHandle(h->opened[q]);
    delete h;
    return mp_cuda_fail(e, "clearing the window's control region");
  }
  h->magic = kMpMagic;
  *out_handle = h;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_dispatch(ep_mp_handle h, const int32_t* token_selected_experts,
                                    int32_t local_num_tokens, int32_t runtime_max_tokens_per_rank,
                                    const void* const* payloads, const int64_t* payload_row_bytes,
                                    int32_t num_payloads, const int32_t* eplb_local_stats,
                                    const uint64_t* active_rank_mask, void* stream_v,
                                    ep_a2a_dispatch_result* result) {
  ep_a2a_status st = mp_check(h);
  if (st != EP_A2A_OK) return st;
  const ep_a2a_params& p = h->p;
  const MpLayout& L = h->L;
  const int ep = p.ep_size;
  if (!token_selected_experts || !result)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "token_selected_experts / result is NULL");
  const int tpr = runtime_max_tokens_per_rank <= 0 ? p.max_tokens_per_rank
                                                   : runtime_max_tokens_per_rank;
  if (tpr > p.max_tokens_per_rank)
    return mp_fail(EP_A2A_ERR_CAPACITY, "runtime_max_tokens_per_rank exceeds the capacity");
  if (local_num_tokens < 0 || local_num_tokens > tpr)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "local_num_tokens outside 0..tpr");
  if (num_payloads < 0 || num_payloads > p.num_payloads)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "num_payloads outside 0..init num_payloads");
  if (num_payloads > 0 && !payloads) return mp_fail(EP_A2A_ERR_INVALID_ARG, "payloads is NULL");
  if (eplb_local_stats && p.eplb_stats_num_experts == 0)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "eplb_local_stats given but not enabled at init");
  if (active_rank_mask && !p.enable_rank_mask)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "active_rank_mask needs enable_rank_mask");
  MpSendArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int w = 0; w < kMaskWords; ++w) a.live[w] = active_rank_mask ? active_rank_mask[w] : ~0ull;
  if (!((a.live[h->rank >> 6] >> (h->rank & 63)) & 1ull))
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "this rank is masked off: it neither sends nor receives");
  for (int r = 0; r < ep; ++r) a.win[r] = h->win[r];
  uint8_t* own = h->win[h->rank];
  for (int i = 0; i < num_payloads; ++i) {
    const int64_t rb = payload_row_bytes ? payload_row_bytes[i] : p.payload_row_bytes[i];
    if (rb < 1 || rb > p.payload_row_bytes[i])
      return mp_fail(EP_A2A_ERR_CAPACITY, "payload row bytes outside 1..capacity");
    if (!payloads[i]) return mp_fail(EP_A2A_ERR_INVALID_ARG, "a payload is NULL");
    a.src[i] = static_cast<const uint8_t*>(payloads[i]);
    a.rb[i] = rb;
    a.off_payload[i] = L.off_payload[i];
    a.vec[i] = access_bytes(payloads[i], own + L.off_payload[i], 1 << 20, rb);
  }
  a.np = num_payloads;
  a.ids = token_selected_experts;
  a.eplb_stats = eplb_local_stats;
  a.eplb_n = p.eplb_stats_num_experts;
  a.rank = h->rank;
  a.ep = ep;
  a.E = p.num_experts;
  a.k = p.top_k;
  a.epr = p.num_experts / ep;
  a.tpr = tpr;
  a.n_local = local_num_tokens;
  a.plan_stride = L.plan_stride;
  a.use_mask = active_rank_mask != nullptr;
  a.invalid_id = p.invalid_expert_id;
  a.off_ids = L.off_ids;
  a.off_valid = L.off_valid;
  a.off_eplb = L.off_eplb;
  a.off_dflag = L.off_dflag;
  a.plan_nd = own + L.off_plan_nd;
  a.plan_dst = own + L.off_plan_dst;
  a.count_acc = reinterpret_cast<int32_t*>(own + L.off_count_acc);
  a.send_counts = reinterpret_cast<int32_t*>(own + L.off_counts);
  a.ticket = reinterpret_cast<uint32_t*>(own + L.off_dticket);
  a.epoch = h->dispatch_epoch + 1;
  const int grid = mp_grid(h->num_sms, std::max(tpr, 1));
  mp_send_kernel<<<grid, 256, 0, (cudaStream_t)stream_v>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return mp_cuda_fail(e, "multi-process send kernel launch");
  h->dispatch_epoch = a.epoch;
  h->have_plan = true;
  h->last_tpr = tpr;
  h->last_n = local_num_tokens;
  h->last_masked = active_rank_mask != nullptr;
  std::memcpy(h->live, a.live, sizeof(h->live));

  std::memset(result, 0, sizeof(*result));
  result->tokens_per_rank = tpr;
  result->num_payloads = num_payloads;
  for (int i = 0; i < num_payloads; ++i) result->recv_payloads[i] = own + L.off_payload[i];
  result->recv_topk_ids = reinterpret_cast<int32_t*>(own + L.off_ids);
  result->recv_valid = own + L.off_valid;
  result->eplb_gathered_stats =
      eplb_local_stats ? reinterpret_cast<int32_t*>(own + L.off_eplb) : nullptr;
  result->send_counts = a.send_counts;
  result->plan_num_dst = a.plan_nd;
  result->plan_dst_ranks = a.plan_dst;
  result->plan_stride = L.plan_stride;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_dispatch_wait(ep_mp_handle h, int64_t timeout_ns, void* stream) {
  ep_a2a_status st = mp_check(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return mp_fail(EP_A2A_ERR_NO_PLAN, "no dispatch on this handle");
  if (timeout_ns < 1 || timeout_ns > 10000000000ll)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "timeout_ns must be in 1..1e10");
  uint8_t* own = h->win[h->rank];
  mp_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
      reinterpret_cast<const uint32_t*>(own + h->L.off_dflag), h->p.ep_size, h->last_masked,
      h->live[0], h->live[1], h->live[2], h->live[3], h->dispatch_epoch,
      (unsigned long long)timeout_ns, reinterpret_cast<uint32_t*>(own + h->L.off_err));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return mp_cuda_fail(e, "wait kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_combine_send(ep_mp_handle h, const void* expert_output,
                                        ep_a2a_combine_dtype dtype, void* stream) {
  ep_a2a_status st = mp_check(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan) return mp_fail(EP_A2A_ERR_NO_PLAN, "combine needs a preceding dispatch");
  if (!expert_output) return mp_fail(EP_A2A_ERR_INVALID_ARG, "expert_output is NULL");
  if (dtype != EP_A2A_COMBINE_BF16 && dtype != EP_A2A_COMBINE_FP8_E4M3)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "unknown combine dtype");
  MpPushArgs a;
  std::memset(&a, 0, sizeof(a));
  for (int r = 0; r < h->p.ep_size; ++r) a.win[r] = h->win[r];
  uint8_t* own = h->win[h->rank];
  a.x = static_cast<const uint8_t*>(expert_output);
  a.valid = own + h->L.off_valid;
  a.row = (int64_t)h->p.hidden_size * (dtype == EP_A2A_COMBINE_BF16 ? 2 : 1);
  a.vec = access_bytes(expert_output, own + h->L.off_landing, a.row, a.row);
  a.rank = h->rank;
  a.ep = h->p.ep_size;
  a.tpr = h->last_tpr;
  a.use_mask = h->last_masked;
  std::memcpy(a.live, h->live, sizeof(a.live));
  a.off_landing = h->L.off_landing;
  a.off_cflag = h->L.off_cflag;
  a.ticket = reinterpret_cast<uint32_t*>(own + h->L.off_cticket);
  a.epoch = h->combine_epoch + 1;
  const int grid = mp_grid(h->num_sms, (int64_t)a.ep * a.tpr);
  mp_push_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return mp_cuda_fail(e, "combine push kernel launch");
  h->combine_epoch = a.epoch;
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_combine_finish(ep_mp_handle h, void* output, ep_a2a_combine_dtype dtype,
                                          int64_t timeout_ns, void* stream_v) {
  ep_a2a_status st = mp_check(h);
  if (st != EP_A2A_OK) return st;
  if (!h->have_plan || h->combine_epoch == 0)
    return mp_fail(EP_A2A_ERR_NO_PLAN, "combine_finish needs a preceding combine_send");
  if (!output) return mp_fail(EP_A2A_ERR_INVALID_ARG, "output is NULL");
  if (dtype != EP_A2A_COMBINE_BF16 && dtype != EP_A2A_COMBINE_FP8_E4M3)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "unknown combine dtype");
  if (timeout_ns < 1 || timeout_ns > 10000000000ll)
    return mp_fail(EP_A2A_ERR_INVALID_ARG, "timeout_ns must be in 1..1e10");
  cudaStream_t stream = (cudaStream_t)stream_v;
  uint8_t* own = h->win[h->rank];
  uint32_t* err = reinterpret_cast<uint32_t*>(own + h->L.off_err);
  mp_wait_kernel<<<1, 32, 0, stream>>>(
      reinterpret_cast<const uint32_t*>(own + h->L.off_cflag), h->p.ep_size, h->last_masked,
      h->live[0], h->live[1], h->live[2], h->live[3], h->combine_epoch,
      (unsigned long long)timeout_ns, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return mp_cuda_fail(e, "wait kernel launch");
  // The ordered sum over the landing rows [ep(d), tpr, H] with this rank's
  // plan: the single-process combine kernels with one source rank.
  const bool fp8 = dtype == EP_A2A_COMBINE_FP8_E4M3;
  CombineArgs c;
  c.plan_nd = own + h->L.off_plan_nd;
  c.plan_dst = own + h->L.off_plan_dst;
  c.x = own + h->L.off_landing;
  c.out = static_cast<uint16_t*>(output);
  c.ntok = h->last_tpr;
  c.H = h->p.hidden_size;
  c.plan_stride = h->L.plan_stride;
  c.prefetch = 0;
  c.ep = h->p.ep_size;
  c.err = err;
  c.out32 = reinterpret_cast<uintptr_t>(output) % 32 == 0;
  const int elems = fp8 ? 16 : 8;
  const bool vec = c.H % elems == 0 && reinterpret_cast<uintptr_t>(output) % 16 == 0;
  const bool pipe = vec && std::min(h->p.top_k, h->p.ep_size) <= 8;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(c.ntok, (int64_t)h->num_sms * 16));
  e = launch_combine(c, fp8, vec, pipe, vec ? 64 : 256, grid, stream, false);
  if (e != cudaSuccess) return mp_cuda_fail(e, "combine kernel launch");
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_get_status(ep_mp_handle h, void* stream) {
  ep_a2a_status st = mp_check(h);
  if (st != EP_A2A_OK) return st;
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return mp_cuda_fail(e, "cudaStreamSynchronize");
  uint32_t word = 0;
  uint32_t* dev_word = reinterpret_cast<uint32_t*>(h->win[h->rank] + h->L.off_err);
  e = cudaMemcpy(&word, dev_word, sizeof(word), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return mp_cuda_fail(e, "reading the error word");
  if (word != 0) {
    e = cudaMemset(dev_word, 0, sizeof(word));
    if (e != cudaSuccess) return mp_cuda_fail(e, "clearing the error word");
    if (word & kErrWaitTimeout)
      return mp_fail(EP_A2A_ERR_DEVICE_TIMEOUT,
                     "a peer's flag did not arrive within the wait limit");
    return mp_fail(EP_A2A_ERR_DEVICE_BOUNDS, "a kernel skipped an out-of-range plan entry");
  }
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_mp_destroy(ep_mp_handle* hp) {
  if (!hp || !*hp) return EP_A2A_OK;
  ep_mp_handle h = *hp;
  if (h->magic != kMpMagic) return mp_fail(EP_A2A_ERR_NOT_INITIALIZED, "handle is not valid");
  ep_a2a_status st = EP_A2A_OK;
  for (int r = 0; r < h->p.ep_size; ++r) {
    if (!h->opened[r]) continue;
    const cudaError_t e = cudaIpcCloseMemHandle(h->opened[r]);
    if (e != cudaSuccess && st == EP_A2A_OK) st = mp_cuda_fail(e, "cudaIpcCloseMemHandle");
  }
  h->magic = 0;
  delete h;
  *hp = nullptr;
  return st;
}
