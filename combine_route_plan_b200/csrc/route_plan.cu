// Routing plan of rank-major MoE dispatch, for all virtual EP ranks at once,
// plus the EPLB statistics gather.
//
// What it computes (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, dispatch(); slot
// rule from flashinfer.moe_ep.NVLinkOneSidedConfig, `lamport` paragraph):
//   for a live source rank r and token t < n[r], the destination set is the set
//   of live ranks owning any of the token's top_k global expert ids (expert e is
//   owned by rank e / (E / ep)); ids outside [0, E) are owned by no rank.  The
//   token's row lands at slot s = r * tpr + t of every destination.
// Outputs:
//   plan_nd[s]            size of the set, or 0xFF if the token does not exist
//   plan_dst[s][0..k)     the set in ascending rank order, 0xFF padded
//   recv_valid[d][s]      1 if d received row s (every live d, every s)
//   recv_topk_ids[d][s]   the token's ids if valid, else invalid_expert_id
//                         (vllm.distributed.device_communicators.all2all,
//                         FlashInferNVLinkTwoSidedManager.get_communication)
//   send_counts[r][d]     tokens r sent to d
//   eplb_gathered[d][r]   rank r's eplb_local_stats (zeros for a masked-off r)
//                         (flashinfer.comm.moe_a2a_dispatch, Returns)
// Masked-off ranks (flashinfer.comm.moe_a2a_dispatch, active_rank_mask) neither
// send nor receive; their receive arrays are not written.
//
// Layout of the work: one warp handles 32 / G tokens, G = next power of two
// >= top_k lanes per token, lane j holding expert slot j.  Duplicate owners
// are removed with __match_any_sync (the lowest lane of each equal-owner group
// is the leader); a leader's position in the ascending list is the number of
// leaders of its token with a smaller rank.  Counts are reduced per block in
// shared memory; the last block of each source rank (ticket counter) writes the
// final row and resets the scratch to zero, so no memset is needed per call.
// The receive-side rows (ids and valid byte of each of the block's slots in
// every live destination) are written from the block's ids and destination
// sets, kept in shared memory by the first pass: one thread per (slot,
// destination) pair, consecutive threads on consecutive slots, so a warp
// stores contiguous rows.
#include <algorithm>

#include "ep_a2a_internal.cuh"

namespace ep_a2a {
namespace {

constexpr int kRouteThreads = 256;
constexpr int kRouteWarps = kRouteThreads / 32;
constexpr int kTokPerBlock = 32;

template <bool kMask>
__device__ __forceinline__ bool rank_live(const uint64_t* live, int r) {
  if (!kMask) return true;
  return (live[r >> 6] >> (r & 63)) & 1ull;
}

template <bool kMask>
__device__ void eplb_gather(const RouteArgs& a) {
  // gathered[d][r][:] = live(r) ? stats[r][:] : 0 for live d; E % 4 == 0, so
  // the rows move as int4.  Rank regions and offsets are 256-byte aligned.
  const int e4 = a.eplb_n / 4;
  const int64_t total = (int64_t)a.ep * a.ep * e4;
  const int4* src = reinterpret_cast<const int4*>(a.eplb_stats);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(i / ((int64_t)a.ep * e4));
    const int64_t rem = i - (int64_t)d * a.ep * e4;
    const int r = (int)(rem / e4);
    const int c = (int)(rem - (int64_t)r * e4);
    if (!rank_live<kMask>(a.live, d)) continue;
    int4 v = make_int4(0, 0, 0, 0);
    if (rank_live<kMask>(a.live, r)) v = src[(int64_t)r * e4 + c];
    int4* dst = reinterpret_cast<int4*>(a.rank0 + d * a.rank_stride + a.off_eplb);
    dst[(int64_t)r * e4 + c] = v;
  }
}

template <int G, bool kMask>
__global__ void __launch_bounds__(kRouteThreads) route_plan_kernel(const RouteArgs a) {
  pdl_wait();
  // The vector copy that follows routes its tokens itself and does not read
  // what this kernel writes, so it may run alongside; the combine after it
  // still waits for this grid (through the copy's final wait).
  pdl_launch_dependents();
  const int r = blockIdx.y;
  if (r == a.ep) {  // the extra row of blocks gathers EPLB statistics
    eplb_gather<kMask>(a);
    return;
  }
  __shared__ int s_cnt[kMaxRanks];
  __shared__ bool s_last;
  // the block's tokens' ids (rows padded by 4 words, so that the second pass's
  // 16-byte reads of consecutive tokens fall on different banks) and their
  // destination sets (bit d of 32-bit words)
  __shared__ __align__(16) int32_t s_ids[kTokPerBlock][kMaxTopK + 4];
  __shared__ uint32_t s_dst[kTokPerBlock][kMaxRanks / 32];
  for (int i = threadIdx.x; i < a.ep; i += kRouteThreads) s_cnt[i] = 0;
  for (int i = threadIdx.x; i < kTokPerBlock * (kMaxRanks / 32); i += kRouteThreads)
    (&s_dst[0][0])[i] = 0u;
  __syncthreads();

  constexpr int kTokPerWarp = 32 / G;
  constexpr unsigned kFull = 0xFFFFFFFFu;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int g = lane / G;        // token within the warp
  const int j = lane - g * G;    // expert slot within the token
  const unsigned gmask = (G == 32) ? kFull : (((1u << G) - 1u) << (g * G));
  const bool live_r = rank_live<kMask>(a.live, r);
  const int n_r = live_r ? a.n[r] : 0;
  const int t_begin = blockIdx.x * kTokPerBlock;
  const int t_end = min(a.tpr, t_begin + kTokPerBlock);

  // Expert slot j of token t: its global id e and owning live rank d (-1 if none).
  auto owner_of = [&](int t, int32_t& e, int& d, bool& in_range, bool& exists) {
    in_range = t < t_end;
    exists = in_range && t < n_r;
    e = 0;
    d = -1;
    if (exists && j < a.k) {
      e = a.ids[((int64_t)r * a.tpr + t) * a.k + j];
      if (e >= 0 && e < a.E) {
        const int owner = e / a.epr;
        if (rank_live<kMask>(a.live, owner)) d = owner;
      }
    }
  };

  // Pass 1: the plan (this rank's tokens) and the per-block send counts.
  for (int t0 = t_begin; t0 < t_end; t0 += kRouteWarps * kTokPerWarp) {
    const int t = t0 + warp * kTokPerWarp + g;
    int32_t e;
    int d;
    bool in_range, exists;
    owner_of(t, e, d, in_range, exists);
    const int64_t s = (int64_t)r * a.tpr + t;
    // de-duplicate owners within the token
    const unsigned key = ((unsigned)g << 9) | ((unsigned)d & 0x1FFu);
    const unsigned peers = __match_any_sync(kFull, key);
    const bool leader = d >= 0 && (__ffs(peers) - 1) == lane;
    const unsigned leaders = __ballot_sync(kFull, leader) & gmask;
    const int nd = __popc(leaders);
    int pos = 0;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const int other = __shfl_sync(kFull, d, g * G + i);
      pos += (((leaders >> (g * G + i)) & 1u) != 0u) && other < d;
    }
    if (in_range) {
      uint8_t* row = a.plan_dst + s * a.plan_stride;
      if (j == 0) a.plan_nd[s] = exists ? (uint8_t)nd : kNoToken;
      if (leader) {
        row[pos] = (uint8_t)d;
        atomicAdd(&s_cnt[d], 1);
        atomicOr(&s_dst[t - t_begin][d >> 5], 1u << (d & 31));
      }
      for (int c = j; c < a.plan_stride; c += G)
        if (c >= nd) row[c] = kPad;
      if (j < a.k) s_ids[t - t_begin][j] = e;
    }
  }

  // send_counts[r][:] = sum over this rank's blocks.  The block's totals go to
  // the accumulators; the last block to take a ticket writes the row and
  // resets the scratch.  Only plan writes precede the fence, so the ticket
  // chain stays short; the receive rows are written afterwards.
  __syncthreads();
  for (int i = threadIdx.x; i < a.ep; i += kRouteThreads) {
    const int v = s_cnt[i];
    if (v) atomicAdd(&a.count_acc[r * a.ep + i], v);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    const unsigned prev = atomicAdd(&a.count_ticket[r], 1u);
    s_last = (prev == gridDim.x - 1);
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    for (int i = threadIdx.x; i < a.ep; i += kRouteThreads)
      a.send_counts[r * a.ep + i] = atomicExch(&a.count_acc[r * a.ep + i], 0);
    if (threadIdx.x == 0) atomicExch(&a.count_ticket[r], 0u);
  }

  // Pass 2: receive-side rows of every slot in every live destination, one
  // (slot, destination) pair per thread (the first pass's shared arrays are
  // visible after the barriers above).
  const int nt = t_end - t_begin;
  for (int p = threadIdx.x; p < nt * a.ep; p += kRouteThreads) {
    const int dd = p / nt;
    const int tl = p - dd * nt;
    if (!rank_live<kMask>(a.live, dd)) continue;
    const bool got = (s_dst[tl][dd >> 5] >> (dd & 31)) & 1u;
    const int64_t s = (int64_t)r * a.tpr + t_begin + tl;
    uint8_t* base = a.rank0 + dd * a.rank_stride;
    int32_t* ids = reinterpret_cast<int32_t*>(base + a.off_ids) + s * a.k;
    if (a.vec_ids) {
      for (int q = 0; q < a.k; q += 4) {
        const int4 v = got ? *reinterpret_cast<const int4*>(&s_ids[tl][q])
                           : make_int4(a.invalid_id, a.invalid_id, a.invalid_id, a.invalid_id);
        *reinterpret_cast<int4*>(ids + q) = v;
      }
    } else {
      for (int q = 0; q < a.k; ++q) ids[q] = got ? s_ids[tl][q] : a.invalid_id;
    }
    base[a.off_valid + s] = got ? 1 : 0;
  }
}

template <int G>
cudaError_t launch_g(const RouteArgs& a, bool use_mask, dim3 grid, cudaStream_t stream, bool pdl) {
  if (use_mask)
    return launch_kernel(route_plan_kernel<G, true>, grid, dim3(kRouteThreads), 0, stream, pdl, a);
  return launch_kernel(route_plan_kernel<G, false>, grid, dim3(kRouteThreads), 0, stream, pdl, a);
}

}  // namespace

cudaError_t launch_route_plan(const RouteArgs& args, bool use_mask, cudaStream_t stream,
                              bool pdl) {
  RouteArgs a = args;
  // received ids as 16-byte stores when every slot's row allows it
  a.vec_ids = a.k % 4 == 0 && reinterpret_cast<uintptr_t>(a.rank0 + a.off_ids) % 16 == 0 &&
              a.rank_stride % 16 == 0;
  const int tok_blocks = (a.tpr + kTokPerBlock - 1) / kTokPerBlock;
  int gx = tok_blocks > 0 ? tok_blocks : 1;
  int gy = a.ep;
  if (a.eplb_stats != nullptr) {
    const int64_t total4 = (int64_t)a.ep * a.ep * (a.eplb_n / 4);
    const int64_t eb = (total4 + kRouteThreads - 1) / kRouteThreads;
    gx = (int)std::max<int64_t>(gx, std::min<int64_t>(eb, 1024));
    gy += 1;
  }
  const dim3 grid(gx, gy);
  int G = 1;
  while (G < a.k) G <<= 1;
  switch (G) {
    case 1: return launch_g<1>(a, use_mask, grid, stream, pdl);
    case 2: return launch_g<2>(a, use_mask, grid, stream, pdl);
    case 4: return launch_g<4>(a, use_mask, grid, stream, pdl);
    case 8: return launch_g<8>(a, use_mask, grid, stream, pdl);
    case 16: return launch_g<16>(a, use_mask, grid, stream, pdl);
    case 32: return launch_g<32>(a, use_mask, grid, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ep_a2a
