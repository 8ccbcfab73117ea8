// Dispatch row copy: every payload row of a token is read from HBM once and
// written to the token's slot s = src * tpr + t in each destination rank's
// receive array (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, dispatch();
// flashinfer.moe_ep.NVLinkOneSidedConfig, `lamport` paragraph, for the slot).
// Bytes are moved verbatim, so every bit pattern arrives unchanged.
//
// Two kernels:
//   * dispatch_bulk_kernel — for payloads whose rows are 16-byte multiples at
//     16-byte-aligned addresses.  One warp per CTA; lane 0 drives a ring of
//     shared-memory stages: a bulk-async load (cp.async.bulk, completion on an
//     mbarrier) brings one token's rows of all such payloads into a stage, then
//     one bulk-async store per (destination, payload) writes the stage out.
//     Loads run `L = stages - Q` tokens ahead of the stores, and at most Q
//     tokens' store groups are still reading shared memory when a stage is
//     refilled.  The copy engine generates the addresses; the SM only issues.
//   * dispatch_vec_kernel — any row size and alignment.  One warp per token:
//     lanes load the row in the widest aligned vectors into registers once and
//     store them to each destination.
// Both read the plan (plan_nd / plan_dst) the routing kernel wrote just before.
#include "ep_a2a_internal.cuh"

namespace ep_a2a {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Warp-collective iterator over the tokens of [begin, end) that exist and have
// at least one destination.  All 32 lanes call next() together; the result is
// the same in every lane.
struct TokenStream {
  const uint8_t* plan_nd;
  const uint8_t* plan_dst;
  int plan_words;      // plan_stride / 8
  int64_t base, end;   // next batch starts at base
  int64_t batch;       // first token of the current batch
  unsigned pending;    // lanes of the current batch still to hand out
  int my_nd;
  uint64_t my_dst[kMaxTopK / 8];

  __device__ void init(const CopyArgs& a, int64_t b, int64_t e) {
    plan_nd = a.plan_nd;
    plan_dst = a.plan_dst;
    plan_words = a.plan_stride / 8;
    base = b;
    end = e;
    batch = b;
    pending = 0u;
  }

  // Returns the token index, or -1 when done; nd and dst words are broadcast.
  __device__ int64_t next(int lane, int& nd, uint64_t (&dst)[kMaxTopK / 8]) {
    while (pending == 0u) {
      if (base >= end) return -1;
      const int64_t tok = base + lane;
      int v = kNoToken;
      if (tok < end) {
        v = plan_nd[tok];
        const uint64_t* row = reinterpret_cast<const uint64_t*>(plan_dst + tok * plan_words * 8);
        if (v != kNoToken && v > 0) {
#pragma unroll
          for (int w = 0; w < kMaxTopK / 8; ++w)
            if (w < plan_words) my_dst[w] = row[w];
        }
      }
      my_nd = v;
      pending = __ballot_sync(kFull, v != kNoToken && v > 0);
      batch = base;
      base += 32;
    }
    const int src_lane = __ffs(pending) - 1;
    pending &= pending - 1u;
    nd = __shfl_sync(kFull, my_nd, src_lane);
#pragma unroll
    for (int w = 0; w < kMaxTopK / 8; ++w)
      if (w < plan_words) dst[w] = __shfl_sync(kFull, my_dst[w], src_lane);
    return batch + src_lane;
  }
};

// i-th destination rank of a packed plan row (byte i of words w0..w3); the
// words are chosen with selects so they stay in registers.
__device__ __forceinline__ int dst_rank(uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                        int i) {
  const uint64_t w = i < 8 ? w0 : (i < 16 ? w1 : (i < 24 ? w2 : w3));
  return (int)((w >> ((i & 7) * 8)) & 0xFFu);
}

template <int Q>
__global__ void __launch_bounds__(32) dispatch_bulk_kernel(const CopyArgs a) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t bars[kMaxStages];
  __shared__ int64_t st_tok[kMaxStages];
  __shared__ int st_nd[kMaxStages];
  __shared__ uint64_t st_dst[kMaxStages][kMaxTopK / 8];

  const int lane = threadIdx.x;
  const int S = a.stages;
  const int L = S - Q;                      // loads issued ahead of stores
  const int64_t chunk = (a.ntok + gridDim.x - 1) / gridDim.x;
  const int64_t begin = min(a.ntok, (int64_t)blockIdx.x * chunk);
  const int64_t end = min(a.ntok, begin + chunk);
  const uint32_t smem0 = smem_addr(stage_mem);
  const uint32_t bar0 = smem_addr(bars);

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  __syncwarp();

  TokenStream ts;
  ts.init(a, begin, end);
  int nd;
  uint64_t dst[kMaxTopK / 8];
  const int words = a.plan_stride / 8;

  auto issue_load = [&](int64_t tok, int s) {
    if (lane == 0) {
      st_tok[s] = tok;
      st_nd[s] = nd;
#pragma unroll
      for (int w = 0; w < kMaxTopK / 8; ++w)
        if (w < words) st_dst[s][w] = dst[w];
      const uint32_t bar = bar0 + 8 * s;
      mbar_arrive_expect_tx(bar, a.tx_bytes);
      const uint32_t stage = smem0 + (uint32_t)s * a.stage_bytes;
      for (int p = 0; p < a.np; ++p)
        bulk_load(stage + a.smem_off[p], a.src[p] + tok * a.rb[p], (uint32_t)a.rb[p], bar);
    }
  };

  int64_t issued = 0, done = 0;
  bool more = true;
  while (issued < L) {
    const int64_t tok = ts.next(lane, nd, dst);
    if (tok < 0) {
      more = false;
      break;
    }
    issue_load(tok, (int)(issued % S));
    ++issued;
  }

  bool timed_out = false;
  while (done < issued) {
    const int s = (int)(done % S);
    if (lane == 0) {
      const uint32_t parity = (uint32_t)((done / S) & 1);
      if (!mbar_wait_bounded(bar0 + 8 * s, parity, kWaitLimitNs)) {
        atomicOr(a.err, kErrWaitTimeout);
        timed_out = true;
      } else {
        fence_proxy_async_smem();
        const int64_t tok = st_tok[s];
        const int n = st_nd[s];
        const uint32_t stage = smem0 + (uint32_t)s * a.stage_bytes;
        for (int i = 0; i < n; ++i) {
          const int d = (int)((st_dst[s][i >> 3] >> ((i & 7) * 8)) & 0xFFu);
          uint8_t* rank = a.rank0 + (int64_t)d * a.rank_stride;
          for (int p = 0; p < a.np; ++p)
            bulk_store(rank + a.dst_off[p] + tok * a.rb[p], stage + a.smem_off[p],
                       (uint32_t)a.rb[p]);
        }
        bulk_commit();
      }
    }
    timed_out = __shfl_sync(kFull, timed_out, 0);
    if (timed_out) break;
    ++done;
    if (more) {
      const int64_t tok = ts.next(lane, nd, dst);
      if (tok < 0) {
        more = false;
      } else {
        if (lane == 0) bulk_wait_read<Q>();   // the stage's previous stores have read it
        issue_load(tok, (int)(issued % S));
        ++issued;
      }
    }
  }
  if (lane == 0) {
    bulk_wait_all();
    if (timed_out) {
      // Loads still in flight target this CTA's shared memory: give them a
      // bounded time to land before the CTA exits.
      for (int64_t i = done; i < issued; ++i)
        mbar_wait_bounded(bar0 + 8 * (int)(i % S), (uint32_t)((i / S) & 1), kWaitLimitNs);
    }
  }
}

template <typename T, int U>
__device__ __forceinline__ void copy_row(const uint8_t* __restrict__ src, int64_t rb,
                                         uint8_t* rank0, int64_t rank_stride, int64_t off,
                                         uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                         int nd, int lane) {
  const int64_t n = rb / (int64_t)sizeof(T);
  const T* s = reinterpret_cast<const T*>(src);
  for (int64_t i0 = lane; i0 < n; i0 += 32 * U) {
    T v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + (int64_t)u * 32;
      if (i < n) v[u] = s[i];
    }
    for (int q = 0; q < nd; ++q) {
      T* d = reinterpret_cast<T*>(rank0 + (int64_t)dst_rank(w0, w1, w2, w3, q) * rank_stride +
                                  off);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t i = i0 + (int64_t)u * 32;
        if (i < n) d[i] = v[u];
      }
    }
  }
}

constexpr int kVecThreads = 256;

__global__ void __launch_bounds__(kVecThreads) dispatch_vec_kernel(const CopyArgs a) {
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int words = a.plan_stride / 8;
  for (int64_t tok = (int64_t)blockIdx.x * (kVecThreads / 32) + warp; tok < a.ntok;
       tok += (int64_t)gridDim.x * (kVecThreads / 32)) {
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken || nd == 0) continue;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * words * 8);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    for (int p = 0; p < a.np; ++p) {
      const uint8_t* src = a.src[p] + tok * a.rb[p];
      const int64_t off = a.dst_off[p] + tok * a.rb[p];
      switch (a.vec[p]) {
        case 16:
          copy_row<uint4, 4>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd, lane);
          break;
        case 8:
          copy_row<uint2, 4>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd, lane);
          break;
        case 4:
          copy_row<uint32_t, 4>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                lane);
          break;
        case 2:
          copy_row<uint16_t, 4>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                lane);
          break;
        default:
          copy_row<uint8_t, 4>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                               lane);
          break;
      }
    }
  }
}

}  // namespace

int bulk_queue_depth(int stages) {
  // store groups allowed to be reading shared memory when a stage is refilled
  if (stages >= 16) return 8;
  if (stages >= 8) return 4;
  if (stages >= 4) return 2;
  return 1;
}

cudaError_t launch_dispatch_bulk(const CopyArgs& a, int grid, cudaStream_t stream) {
  const size_t smem = (size_t)a.stage_bytes * a.stages;
  const int q = bulk_queue_depth(a.stages);
  cudaError_t err = cudaSuccess;
  switch (q) {
    case 8:
      err = cudaFuncSetAttribute(dispatch_bulk_kernel<8>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err == cudaSuccess) dispatch_bulk_kernel<8><<<grid, 32, smem, stream>>>(a);
      break;
    case 4:
      err = cudaFuncSetAttribute(dispatch_bulk_kernel<4>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err == cudaSuccess) dispatch_bulk_kernel<4><<<grid, 32, smem, stream>>>(a);
      break;
    case 2:
      err = cudaFuncSetAttribute(dispatch_bulk_kernel<2>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err == cudaSuccess) dispatch_bulk_kernel<2><<<grid, 32, smem, stream>>>(a);
      break;
    default:
      err = cudaFuncSetAttribute(dispatch_bulk_kernel<1>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err == cudaSuccess) dispatch_bulk_kernel<1><<<grid, 32, smem, stream>>>(a);
      break;
  }
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_dispatch_vec(const CopyArgs& a, int grid, cudaStream_t stream) {
  dispatch_vec_kernel<<<grid, kVecThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace ep_a2a
