// Dispatch row copy: every payload row of a token is read from HBM once and
// written to the token's slot s = src * tpr + t in each destination rank's
// receive array (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll, dispatch();
// flashinfer.moe_ep.NVLinkOneSidedConfig, `lamport` paragraph, for the slot).
// Bytes are moved verbatim, so every bit pattern arrives unchanged.
//
// Three kernels:
//   * dispatch_vec_kernel (default) — any row size and alignment.  A group of
//     32..256 threads per token finds the token's destinations from its routing
//     ids (the routing kernel's rule, so it need not wait for the plan), loads
//     each row once in the widest aligned vectors (32 bytes with sm_100 256-bit
//     accesses, else 16 down to 1) into registers, and stores them to every
//     destination with evict-first stores.
//   * dispatch_staged_kernel — for payloads whose rows are 16-byte multiples at
//     16-byte-aligned addresses.  A producer warp streams each token's rows
//     from HBM into a ring of shared-memory stages with bulk-async loads
//     (completion counted on a "full" mbarrier per stage); consumer warps copy
//     the token from shared memory into registers, release the stage ("empty"
//     mbarrier), and write the rows to every destination with 16-byte vector
//     stores, all threads of the CTA sharing each token.  Loads run as far
//     ahead as the ring allows and cost no registers; the SM's threads only
//     issue stores.
//   * dispatch_bulk_kernel — the same staging, but the copy engine also does
//     the stores (one bulk-async store per destination and payload).  One warp
//     per CTA; lane 0 drives a ring of shared-memory stages: a bulk-async load
//     (cp.async.bulk, completion on an mbarrier) brings one token's rows of all
//     such payloads into a stage, then one bulk-async store per (destination,
//     payload) writes the stage out.  Loads run `L = stages - Q` tokens ahead of
//     the stores, and at most Q tokens' store groups are still reading shared
//     memory when a stage is refilled.  The copy engine generates the
//     addresses; the SM only issues.
// The two staged kernels read the plan (plan_nd / plan_dst) the routing kernel
// wrote just before them.
#include "ep_a2a_internal.cuh"

namespace ep_a2a {
namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

// Warp-collective iterator over the tokens begin, begin + stride, ... (< end)
// that exist and have at least one destination.  All 32 lanes call next()
// together; the result is the same in every lane.
struct TokenStream {
  const uint8_t* plan_nd;
  const uint8_t* plan_dst;
  int plan_words;      // plan_stride / 8
  int64_t base, end;   // next batch starts at base
  int64_t stride;      // distance between consecutive tokens of this stream
  int64_t batch;       // first token of the current batch
  unsigned pending;    // lanes of the current batch still to hand out
  int my_nd;
  uint64_t my_dst[kMaxTopK / 8];

  __device__ void init(const CopyArgs& a, int64_t b, int64_t e, int64_t st) {
    plan_nd = a.plan_nd;
    plan_dst = a.plan_dst;
    plan_words = a.plan_stride / 8;
    base = b;
    end = e;
    stride = st;
    batch = b;
    pending = 0u;
  }

  // Returns the token index, or -1 when done; nd and dst words are broadcast.
  __device__ int64_t next(int lane, int& nd, uint64_t (&dst)[kMaxTopK / 8]) {
    while (pending == 0u) {
      if (base >= end) return -1;
      const int64_t tok = base + lane * stride;
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
      base += 32 * stride;
    }
    const int src_lane = __ffs(pending) - 1;
    pending &= pending - 1u;
    nd = __shfl_sync(kFull, my_nd, src_lane);
#pragma unroll
    for (int w = 0; w < kMaxTopK / 8; ++w)
      if (w < plan_words) dst[w] = __shfl_sync(kFull, my_dst[w], src_lane);
    return batch + src_lane * stride;
  }
};

// This CTA's token stream: a contiguous chunk, or every gridDim.x-th token
// (interleaved, so that the CTAs of the grid work on neighbouring slots).
__device__ __forceinline__ void cta_tokens(const CopyArgs& a, int64_t& begin, int64_t& end,
                                           int64_t& stride) {
  if (a.interleave) {
    begin = blockIdx.x;
    end = a.ntok;
    stride = gridDim.x;
  } else {
    const int64_t chunk = (a.ntok + gridDim.x - 1) / gridDim.x;
    begin = min(a.ntok, (int64_t)blockIdx.x * chunk);
    end = min(a.ntok, begin + chunk);
    stride = 1;
  }
}

// i-th destination rank of a packed plan row (byte i of words w0..w3); the
// words are chosen with selects so they stay in registers.
__device__ __forceinline__ int dst_rank(uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                        int i) {
  const uint64_t w = i < 8 ? w0 : (i < 16 ? w1 : (i < 24 ? w2 : w3));
  return (int)((w >> ((i & 7) * 8)) & 0xFFu);
}

template <int Q>
__global__ void __launch_bounds__(32) dispatch_bulk_kernel(const CopyArgs a) {
  pdl_wait();
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t bars[kMaxStages];
  __shared__ int64_t st_tok[kMaxStages];
  __shared__ int st_nd[kMaxStages];
  __shared__ uint64_t st_dst[kMaxStages][kMaxTopK / 8];

  const int lane = threadIdx.x;
  const int S = a.stages;
  const int L = S - Q;                      // loads issued ahead of stores
  int64_t begin, end, stride;
  cta_tokens(a, begin, end, stride);
  const uint32_t smem0 = smem_addr(stage_mem);
  const uint32_t bar0 = smem_addr(bars);

  if (lane == 0) {
    for (int s = 0; s < S; ++s) mbar_init(bar0 + 8 * s, 1);
    mbar_init_fence();
  }
  __syncwarp();

  TokenStream ts;
  ts.init(a, begin, end, stride);
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

template <typename T>
__device__ __forceinline__ T load_src(const T* p) {
  return *p;
}
template <typename T>
__device__ __forceinline__ void store_dst(T* p, const T& v, bool) {
  *p = v;
}
// 16-byte accesses: the source is read once (no L1 allocation); with
// `streaming` the stores carry the evict-first (.cs) hint.
template <>
__device__ __forceinline__ uint4 load_src<uint4>(const uint4* p) {
  return ld_stream_v4(p);
}
template <>
__device__ __forceinline__ void store_dst<uint4>(uint4* p, const uint4& v, bool streaming) {
  if (streaming)
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
  else
    *p = v;
}

// 32-byte accesses (sm_100 256-bit loads and stores), the same hints.
struct alignas(32) Vec32 {
  uint32_t w[8];
};
template <>
__device__ __forceinline__ Vec32 load_src<Vec32>(const Vec32* p) {
  Vec32 v;
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(v.w[0]), "=r"(v.w[1]), "=r"(v.w[2]), "=r"(v.w[3]), "=r"(v.w[4]),
                 "=r"(v.w[5]), "=r"(v.w[6]), "=r"(v.w[7])
               : "l"(p));
  return v;
}
template <>
__device__ __forceinline__ void store_dst<Vec32>(Vec32* p, const Vec32& v, bool streaming) {
  if (streaming)
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
                 "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
  else
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p),
                 "r"(v.w[0]), "r"(v.w[1]), "r"(v.w[2]), "r"(v.w[3]), "r"(v.w[4]), "r"(v.w[5]),
                 "r"(v.w[6]), "r"(v.w[7])
                 : "memory");
}

// Copy one payload row of a token to its nd destinations: the TPT threads of a
// token group each take vectors gl, gl + TPT, ... (U of them in flight).
template <typename T, int U, int TPT>
__device__ __forceinline__ void copy_row(const uint8_t* __restrict__ src, int64_t rb,
                                         uint8_t* rank0, int64_t rank_stride, int64_t off,
                                         uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                         int nd, int gl, bool streaming) {
  const int64_t n = rb / (int64_t)sizeof(T);
  const T* s = reinterpret_cast<const T*>(src);
  for (int64_t i0 = gl; i0 < n; i0 += TPT * U) {
    T v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + (int64_t)u * TPT;
      if (i < n) v[u] = load_src<T>(s + i);
    }
    for (int q = 0; q < nd; ++q) {
      T* d = reinterpret_cast<T*>(rank0 + (int64_t)dst_rank(w0, w1, w2, w3, q) * rank_stride +
                                  off);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t i = i0 + (int64_t)u * TPT;
        if (i < n) store_dst<T>(d + i, v[u], streaming);
      }
    }
  }
}

constexpr int kVecThreads = 256;

__device__ __forceinline__ bool rank_is_live(const CopyArgs& a, int r) {
  return !a.use_mask || ((a.live[r >> 6] >> (r & 63)) & 1ull);
}

// Destinations of token `tok` (all lanes of the warp call it together): lanes
// j < k look at expert slot j, the owners are de-duplicated with a warp match,
// and the distinct live owners are packed as bytes into w0..w3.  The same rule
// as the routing kernel (owner = e / epr for e in [0, E), live ranks only);
// returns the number of destinations, or 0 for a token that does not exist.
__device__ __forceinline__ int token_destinations(const CopyArgs& a, int64_t tok, int lane,
                                                  uint64_t& w0, uint64_t& w1, uint64_t& w2,
                                                  uint64_t& w3) {
  const int r = (int)(tok / a.tpr);
  const int t = (int)(tok - (int64_t)r * a.tpr);
  w0 = w1 = w2 = w3 = 0;
  if (t >= a.n[r]) return 0;              // n[r] is 0 for masked-off ranks
  int d = -1;
  if (lane < a.k) {
    const int32_t e = a.ids[tok * a.k + lane];
    if (e >= 0 && e < a.E) {
      const int owner = e / a.epr;
      if (!a.use_mask || ((a.live[owner >> 6] >> (owner & 63)) & 1ull)) d = owner;
    }
  }
  const unsigned peers = __match_any_sync(kFull, d);
  const bool leader = d >= 0 && (__ffs(peers) - 1) == lane;
  unsigned leaders = __ballot_sync(kFull, leader);
  int nd = 0;
  while (leaders) {
    const int l = __ffs(leaders) - 1;
    leaders &= leaders - 1u;
    const uint64_t dd = (uint64_t)(__shfl_sync(kFull, d, l) & 0xFF);
    const int sh = (nd & 7) * 8;
    if (nd < 8) w0 |= dd << sh;
    else if (nd < 16) w1 |= dd << sh;
    else if (nd < 24) w2 |= dd << sh;
    else w3 |= dd << sh;
    ++nd;
  }
  return nd;
}

// Destinations of token slot `tok` (all lanes of the warp call it together),
// by the routing kernel's rule: lanes j < k look at expert slot j (owner =
// e / epr for e in [0, E), live ranks only), the owners are de-duplicated with
// a warp match, and the distinct owners are packed as bytes into w0..w3 (for
// the copy; lane order).  Returns their number, 0 for a token that does not
// exist.
//
// With a.route set, the same pass also writes the token's routing outputs,
// those of the routing kernel: plan_nd / plan_dst (destinations in ascending
// rank order), the send counts, and for every live rank d its valid byte and
// received ids (the token's ids if d is a destination, else invalid_id), for
// tokens that do not exist too.  Every warp of the token's group calls it;
// warp gw of nw writes the plan row and counts if gw == 0, and its share of the
// per-rank ids and valid bytes.  A leader's position in the ascending list is
// the number of leaders with a smaller rank; lane w < 8 holds bits
// 32w..32w+31 of the destination set, which the lanes writing rank d's row read
// by shuffle.  The ids are loaded once for both uses.
template <bool kRoute>
__device__ __forceinline__ int token_route(const CopyArgs& a, int64_t tok, int lane, int gw,
                                           int nw, uint64_t& w0, uint64_t& w1, uint64_t& w2,
                                           uint64_t& w3) {
  const int r = (int)(tok / a.tpr);
  const int t = (int)(tok - (int64_t)r * a.tpr);
  if (!kRoute) return token_destinations(a, tok, lane, w0, w1, w2, w3);
  const bool exists = t < a.n[r];          // n[r] is 0 for masked-off ranks
  w0 = w1 = w2 = w3 = 0;
  int32_t e = 0;
  int d = -1;
  if (exists && lane < a.k) {
    e = a.ids[tok * a.k + lane];
    if (e >= 0 && e < a.E) {
      const int owner = e / a.epr;
      if (rank_is_live(a, owner)) d = owner;
    }
  }
  const unsigned peers = __match_any_sync(kFull, d);
  const bool leader = d >= 0 && (__ffs(peers) - 1) == lane;
  const unsigned leaders = __ballot_sync(kFull, leader);
  const int nd = __popc(leaders);
  {
    unsigned rest = leaders;
    for (int q = 0; rest; ++q) {
      const int l = __ffs(rest) - 1;
      rest &= rest - 1u;
      const uint64_t dd = (uint64_t)(__shfl_sync(kFull, d, l) & 0xFF);
      const int sh = (q & 7) * 8;
      if (q < 8) w0 |= dd << sh;
      else if (q < 16) w1 |= dd << sh;
      else if (q < 24) w2 |= dd << sh;
      else w3 |= dd << sh;
    }
  }
  int pos = 0;
  uint32_t word = 0;                       // lane w: set bits 32w..32w+31
  for (int i = 0; i < a.k; ++i) {
    const int other = __shfl_sync(kFull, d, i);
    pos += (((leaders >> i) & 1u) != 0u) && other < d;
    if (other >= 0 && (other >> 5) == lane) word |= 1u << (other & 31);
  }
  if (gw == 0) {
    uint8_t* row = const_cast<uint8_t*>(a.plan_dst) + tok * a.plan_stride;
    if (lane == 0) const_cast<uint8_t*>(a.plan_nd)[tok] = exists ? (uint8_t)nd : kNoToken;
    if (leader) {
      row[pos] = (uint8_t)d;
      atomicAdd(&a.count_acc[r * a.ep + d], 1);
    }
    if (lane < a.plan_stride && lane >= nd) row[lane] = kPad;
  }
  // received ids of every live rank: lane handles (rank idx / k, slot idx % k)
  const int total = a.ep * a.k;
  for (int base = gw * 32; base < total; base += nw * 32) {
    const int idx = base + lane;
    const int dd = idx / a.k;
    const int j = idx - dd * a.k;
    const int32_t ej = __shfl_sync(kFull, e, j & 31);
    const uint32_t wd = __shfl_sync(kFull, word, (dd >> 5) & 7);
    if (idx < total && rank_is_live(a, dd)) {
      int32_t* ids = reinterpret_cast<int32_t*>(a.rank0 + (int64_t)dd * a.rank_stride + a.off_ids);
      ids[tok * a.k + j] = ((wd >> (dd & 31)) & 1u) ? ej : a.invalid_id;
    }
  }
  for (int base = gw * 32; base < a.ep; base += nw * 32) {
    const int dd = base + lane;
    const uint32_t wd = __shfl_sync(kFull, word, (dd >> 5) & 7);
    if (dd < a.ep && rank_is_live(a, dd))
      a.rank0[(int64_t)dd * a.rank_stride + a.off_valid + tok] = (uint8_t)((wd >> (dd & 31)) & 1u);
  }
  return exists ? nd : 0;
}

// EPLB gather: gathered[d][r][:] = live(r) ? stats[r][:] : 0 for live d, as
// int4 (E % 4 == 0; rank regions and offsets are 256-byte aligned).
__device__ __forceinline__ void eplb_gather_rows(const CopyArgs& a) {
  const int e4 = a.eplb_n / 4;
  const int64_t total = (int64_t)a.ep * a.ep * e4;
  const int4* src = reinterpret_cast<const int4*>(a.eplb_stats);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int d = (int)(i / ((int64_t)a.ep * e4));
    const int64_t rem = i - (int64_t)d * a.ep * e4;
    const int r = (int)(rem / e4);
    const int c = (int)(rem - (int64_t)r * e4);
    if (!rank_is_live(a, d)) continue;
    int4 v = make_int4(0, 0, 0, 0);
    if (rank_is_live(a, r)) v = src[(int64_t)r * e4 + c];
    reinterpret_cast<int4*>(a.rank0 + d * a.rank_stride + a.off_eplb)[(int64_t)r * e4 + c] = v;
  }
}

// send_counts = the accumulators, once every CTA has added its tokens: the
// last CTA to take a ticket copies them and resets the scratch to zero, so no
// clearing is needed per call.
__device__ __forceinline__ void finish_counts(const CopyArgs& a) {
  __shared__ bool s_last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(a.count_ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < a.ep * a.ep; i += blockDim.x)
    a.send_counts[i] = atomicExch(&a.count_acc[i], 0);
  if (threadIdx.x == 0) atomicExch(a.count_ticket, 0u);
}

// TPT threads per token (a warp for many tokens, up to the whole CTA for few,
// so that short steps still fill the GPU).  Each warp finds its token's
// destinations from the routing ids itself, so the kernel does not depend on
// the routing kernel's plan and may run alongside it (programmatic dependent
// launch); it waits for the preceding grid only before it exits, so that work
// after it sees the plan complete.  kAll = 16 or 32: every payload of the
// launch moves in vectors of that many bytes (one code path, fewer registers);
// kAll = 0: each payload picks its own vector width.
template <int U, int kAll, bool kStreaming, int TPT, bool kRoute>
__global__ void __launch_bounds__(kVecThreads) dispatch_vec_kernel(const CopyArgs a) {
  constexpr bool kUniform = kAll != 0;
  constexpr int kGroups = kVecThreads / TPT;
  const int gl = threadIdx.x % TPT;
  const int group = threadIdx.x / TPT;
  const int lane = threadIdx.x & 31;
  const int64_t tok_step = (int64_t)gridDim.x * kGroups;
  if (kRoute) {
    // this launch is the whole dispatch: it reads the caller's ids and rows and
    // rewrites the plan the previous combine read, so it waits for the
    // preceding grid first
    pdl_wait();
    if (a.eplb_stats != nullptr) eplb_gather_rows(a);
  }
  for (int64_t tok = (int64_t)blockIdx.x * kGroups + group; tok < a.ntok; tok += tok_step) {
    if (kUniform && a.prefetch && gl == 0 && tok + tok_step < a.ntok) {
      // the group's next token: its rows into L2 while this one is copied
      for (int p = 0; p < a.np; ++p)
        prefetch_l2(a.src[p] + (tok + tok_step) * a.rb[p], (uint32_t)a.rb[p]);
    }
    uint64_t w0, w1, w2, w3;
    const int nd = token_route<kRoute>(a, tok, lane, gl >> 5, TPT / 32, w0, w1, w2, w3);
    if (nd == 0) continue;
    for (int p = 0; p < a.np; ++p) {
      const uint8_t* src = a.src[p] + tok * a.rb[p];
      const int64_t off = a.dst_off[p] + tok * a.rb[p];
      if (kAll == 32) {
        copy_row<Vec32, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                gl, kStreaming);
        continue;
      }
      if (kAll == 16) {
        copy_row<uint4, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                gl, kStreaming);
        continue;
      }
      switch (a.vec[p]) {
        case 32:
          copy_row<Vec32, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                  gl, kStreaming);
          break;
        case 16:
          copy_row<uint4, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                  gl, kStreaming);
          break;
        case 8:
          copy_row<uint2, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3, nd,
                                  gl, false);
          break;
        case 4:
          copy_row<uint32_t, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3,
                                     nd, gl, false);
          break;
        case 2:
          copy_row<uint16_t, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3,
                                     nd, gl, false);
          break;
        default:
          copy_row<uint8_t, U, TPT>(src, a.rb[p], a.rank0, a.rank_stride, off, w0, w1, w2, w3,
                                    nd, gl, false);
          break;
      }
    }
  }
  if (kRoute)
    finish_counts(a);
  else
    pdl_wait();
}

template <int NCW, int MAXV>
__global__ void __launch_bounds__(32 * (NCW + 1)) dispatch_staged_kernel(const CopyArgs a) {
  pdl_wait();
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full_bar[kMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kMaxStages];
  __shared__ int64_t st_tok[kMaxStages];
  __shared__ int st_nd[kMaxStages];
  __shared__ uint64_t st_dst[kMaxStages][kMaxTopK / 8];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = a.stages;
  int64_t begin, end, stride;
  cta_tokens(a, begin, end, stride);
  const uint32_t smem0 = smem_addr(stage_mem);
  const uint32_t full0 = smem_addr(full_bar);
  const uint32_t empty0 = smem_addr(empty_bar);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, NCW);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == 0) {
    // producer: one token per stage, in order; the token after the last one is
    // a sentinel (index -1) that tells the consumers to stop
    TokenStream ts;
    ts.init(a, begin, end, stride);
    const int words = a.plan_stride / 8;
    for (int64_t i = 0;; ++i) {
      int nd = 0;
      uint64_t dst[kMaxTopK / 8];
      const int64_t tok = ts.next(lane, nd, dst);
      const int s = (int)(i % S);
      const uint32_t use = (uint32_t)(i / S);
      bool ok = true;
      if (lane == 0) {
        if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1u, kWaitLimitNs)) {
          atomicOr(a.err, kErrWaitTimeout);
          ok = false;
        } else {
          st_tok[s] = tok;
          st_nd[s] = nd;
#pragma unroll
          for (int w = 0; w < kMaxTopK / 8; ++w)
            if (w < words) st_dst[s][w] = dst[w];
          if (tok < 0) {
            mbar_arrive(full0 + 8 * s);
          } else {
            mbar_arrive_expect_tx(full0 + 8 * s, a.tx_bytes);
            const uint32_t stage = smem0 + (uint32_t)s * a.stage_bytes;
            for (int p = 0; p < a.np; ++p)
              bulk_load(stage + a.smem_off[p], a.src[p] + tok * a.rb[p], (uint32_t)a.rb[p],
                        full0 + 8 * s);
          }
        }
      }
      ok = __shfl_sync(kFull, ok, 0);
      if (tok < 0 || !ok) break;
    }
    return;
  }

  // consumers: thread c owns the stage's 16-byte vectors c, c + 32*NCW, ...
  // (at most MAXV of them); for each, the receive-array offset of its bytes
  // and the row length of its payload
  constexpr int kCons = 32 * NCW;
  const int c = threadIdx.x - 32;
  const int nvec_total = (int)(a.tx_bytes / 16);
  int64_t dbase[MAXV];
  uint32_t drow[MAXV];
#pragma unroll
  for (int j = 0; j < MAXV; ++j) {
    const int f = c + j * kCons;
    dbase[j] = 0;
    drow[j] = 0;
    if (f < nvec_total) {
      const uint32_t byte = (uint32_t)f * 16u;
      int p = 0;
      while (p + 1 < a.np && byte >= a.smem_off[p + 1]) ++p;
      dbase[j] = a.dst_off[p] + (int64_t)(byte - a.smem_off[p]);
      drow[j] = (uint32_t)a.rb[p];
    }
  }
  const int words = a.plan_stride / 8;
  for (int64_t i = 0;; ++i) {
    const int s = (int)(i % S);
    const uint32_t use = (uint32_t)(i / S);
    if (!mbar_wait_bounded(full0 + 8 * s, use & 1u, kWaitLimitNs)) {
      atomicOr(a.err, kErrWaitTimeout);
      break;
    }
    const int64_t tok = st_tok[s];
    if (tok < 0) break;
    const int nd = st_nd[s];
    const uint64_t w0 = st_dst[s][0];
    const uint64_t w1 = words > 1 ? st_dst[s][1] : 0;
    const uint64_t w2 = words > 2 ? st_dst[s][2] : 0;
    const uint64_t w3 = words > 3 ? st_dst[s][3] : 0;
    const uint8_t* stage = stage_mem + (size_t)s * a.stage_bytes;
    uint4 v[MAXV];
#pragma unroll
    for (int j = 0; j < MAXV; ++j)
      if (c + j * kCons < nvec_total)
        v[j] = *reinterpret_cast<const uint4*>(stage + (uint32_t)(c + j * kCons) * 16u);
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);      // this warp is done with the stage
    int64_t off[MAXV];
#pragma unroll
    for (int j = 0; j < MAXV; ++j) off[j] = dbase[j] + tok * (int64_t)drow[j];
    for (int q = 0; q < nd; ++q) {
      uint8_t* rank = a.rank0 + (int64_t)dst_rank(w0, w1, w2, w3, q) * a.rank_stride;
#pragma unroll
      for (int j = 0; j < MAXV; ++j)
        if (c + j * kCons < nvec_total) *reinterpret_cast<uint4*>(rank + off[j]) = v[j];
    }
  }
}

template <int NCW, int MAXV>
cudaError_t launch_staged(const CopyArgs& a, int grid, size_t smem, cudaStream_t stream,
                          bool pdl) {
  cudaError_t err = cudaFuncSetAttribute(dispatch_staged_kernel<NCW, MAXV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_kernel(dispatch_staged_kernel<NCW, MAXV>, dim3(grid), dim3(32 * (NCW + 1)), smem,
                       stream, pdl, a);
}

template <int NCW>
cudaError_t launch_staged_v(const CopyArgs& a, int grid, size_t smem, cudaStream_t stream,
                            bool pdl) {
  const int per_thread = (int)((a.tx_bytes / 16 + 32 * NCW - 1) / (32 * NCW));
  if (per_thread <= 1) return launch_staged<NCW, 1>(a, grid, smem, stream, pdl);
  if (per_thread <= 2) return launch_staged<NCW, 2>(a, grid, smem, stream, pdl);
  if (per_thread <= 4) return launch_staged<NCW, 4>(a, grid, smem, stream, pdl);
  if (per_thread <= 8) return launch_staged<NCW, 8>(a, grid, smem, stream, pdl);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_dispatch_staged(const CopyArgs& a, int consumer_warps, int grid,
                                   cudaStream_t stream, bool pdl) {
  const size_t smem = (size_t)a.stage_bytes * a.stages;
  switch (consumer_warps) {
    case 4: return launch_staged_v<4>(a, grid, smem, stream, pdl);
    case 8: return launch_staged_v<8>(a, grid, smem, stream, pdl);
    case 16: return launch_staged_v<16>(a, grid, smem, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

int bulk_queue_depth(int stages) {
  // store groups allowed to be reading shared memory when a stage is refilled
  if (stages >= 16) return 8;
  if (stages >= 8) return 4;
  if (stages >= 4) return 2;
  return 1;
}

template <int Q>
cudaError_t launch_bulk_q(const CopyArgs& a, int grid, size_t smem, cudaStream_t stream, bool pdl) {
  cudaError_t err = cudaFuncSetAttribute(dispatch_bulk_kernel<Q>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  return launch_kernel(dispatch_bulk_kernel<Q>, dim3(grid), dim3(32), smem, stream, pdl, a);
}

cudaError_t launch_dispatch_bulk(const CopyArgs& a, int grid, cudaStream_t stream, bool pdl) {
  const size_t smem = (size_t)a.stage_bytes * a.stages;
  switch (bulk_queue_depth(a.stages)) {
    case 8: return launch_bulk_q<8>(a, grid, smem, stream, pdl);
    case 4: return launch_bulk_q<4>(a, grid, smem, stream, pdl);
    case 2: return launch_bulk_q<2>(a, grid, smem, stream, pdl);
    default: return launch_bulk_q<1>(a, grid, smem, stream, pdl);
  }
}

template <int U, int TPT, bool kRoute>
cudaError_t launch_vec_utr(const CopyArgs& a, int grid, bool streaming, cudaStream_t stream,
                           bool pdl) {
  bool all16 = true, all32 = true;
  for (int p = 0; p < a.np; ++p) {
    all16 &= a.vec[p] == 16;
    all32 &= a.vec[p] == 32;
  }
  const dim3 g(grid), b(kVecThreads);
  if (all32) {
    if (streaming)
      return launch_kernel(dispatch_vec_kernel<U, 32, true, TPT, kRoute>, g, b, 0, stream, pdl,
                           a);
    return launch_kernel(dispatch_vec_kernel<U, 32, false, TPT, kRoute>, g, b, 0, stream, pdl, a);
  }
  if (all16) {
    if (streaming)
      return launch_kernel(dispatch_vec_kernel<U, 16, true, TPT, kRoute>, g, b, 0, stream, pdl,
                           a);
    return launch_kernel(dispatch_vec_kernel<U, 16, false, TPT, kRoute>, g, b, 0, stream, pdl, a);
  }
  if (streaming)
    return launch_kernel(dispatch_vec_kernel<U, 0, true, TPT, kRoute>, g, b, 0, stream, pdl, a);
  return launch_kernel(dispatch_vec_kernel<U, 0, false, TPT, kRoute>, g, b, 0, stream, pdl, a);
}

template <int U, int TPT>
cudaError_t launch_vec_ut(const CopyArgs& a, int grid, bool streaming, cudaStream_t stream,
                          bool pdl) {
  if (a.route) return launch_vec_utr<U, TPT, true>(a, grid, streaming, stream, pdl);
  return launch_vec_utr<U, TPT, false>(a, grid, streaming, stream, pdl);
}

template <int U>
cudaError_t launch_vec_u(const CopyArgs& a, int grid, int tpt, bool streaming,
                         cudaStream_t stream, bool pdl) {
  switch (tpt) {
    case 32: return launch_vec_ut<U, 32>(a, grid, streaming, stream, pdl);
    case 64: return launch_vec_ut<U, 64>(a, grid, streaming, stream, pdl);
    case 128: return launch_vec_ut<U, 128>(a, grid, streaming, stream, pdl);
    case 256: return launch_vec_ut<U, 256>(a, grid, streaming, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_dispatch_vec(const CopyArgs& a, int grid, int unroll, int threads_per_token,
                                bool streaming, cudaStream_t stream, bool pdl) {
  switch (unroll) {
    case 2: return launch_vec_u<2>(a, grid, threads_per_token, streaming, stream, pdl);
    case 4: return launch_vec_u<4>(a, grid, threads_per_token, streaming, stream, pdl);
    case 8: return launch_vec_u<8>(a, grid, threads_per_token, streaming, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ep_a2a
