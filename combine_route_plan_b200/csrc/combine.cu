// Combine of rank-major MoE dispatch (flashinfer.moe_ep.NVLinkTwoSidedAlltoAll,
// combine()): each existing token (src, t) gets the sum of the rows its
// destination ranks return, each row being that rank's experts' outputs for the
// token with the routing weights applied and summed.  The sum is an fp32
// accumulator that starts at +0.0f and adds the rows in ascending
// destination-rank order with round-to-nearest adds, then is
// rounded once to bf16 (nearest-even).  With the low-precision combine
// (flashinfer.moe_ep.NVLinkOneSidedConfig, use_low_precision_combine) the rows
// are E4M3, widened exactly to fp32 before the same sum.
//
// Memory plan: one CTA per token (grid-stride); each thread owns 16-byte column
// vectors of the row and issues the loads of all (up to 8 at a time)
// destination rows before the adds, so one thread keeps up to 128 bytes in
// flight.  Loads bypass L1 (each row is read exactly once).  The widening and
// the add are one sm_100 mixed-precision instruction per element
// (add.rn.f32.bf16 / add.rn.f32.f16).  The E4M3 combines and the combine of
// per-slot expert outputs do more arithmetic per loaded byte, so their
// kernels (combine_pipe_kernel, combine_experts_pipe_kernel) keep a second
// vector's loads in flight while they reduce the first.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>

#include "ep_a2a_internal.cuh"

namespace ep_a2a {
namespace {

__device__ __forceinline__ int dst_rank(uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                        int i) {
  const uint64_t w = i < 8 ? w0 : (i < 16 ? w1 : (i < 24 ? w2 : w3));
  return (int)((w >> ((i & 7) * 8)) & 0xFFu);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t bits16) {
  return __uint_as_float(bits16 << 16);
}

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// acc0 += widen(lo half of w), acc1 += widen(hi half of w), BF16 halves.  The
// mixed-precision add widens exactly and rounds once to nearest, so it equals
// __fadd_rn(acc, (float)bf16) with one instruction per element.
__device__ __forceinline__ void add_bf16x2(float& acc0, float& acc1, uint32_t w) {
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %2;\n\t"
      "add.rn.f32.bf16 %0, lo, %0;\n\t"
      "add.rn.f32.bf16 %1, hi, %1;\n\t}"
      : "+f"(acc0), "+f"(acc1)
      : "r"(w));
}

// The same for two FP16 values held as raw halves.
__device__ __forceinline__ void add_f16x2(float& acc0, float& acc1, uint16_t lo, uint16_t hi) {
  asm("add.rn.f32.f16 %0, %2, %0;\n\t"
      "add.rn.f32.f16 %1, %3, %1;"
      : "+f"(acc0), "+f"(acc1)
      : "h"(lo), "h"(hi));
}

// Add the 8 bf16 of a 16-byte vector into acc[0..8).
__device__ __forceinline__ void add_bf16x8(float* acc, const uint4& v) {
  add_bf16x2(acc[0], acc[1], v.x);
  add_bf16x2(acc[2], acc[3], v.y);
  add_bf16x2(acc[4], acc[5], v.z);
  add_bf16x2(acc[6], acc[7], v.w);
}

// Add the 16 E4M3 of a 16-byte vector into acc[0..16): each pair is widened
// exactly to FP16 (every E4M3 value is an FP16 normal or zero), then added in
// fp32 by the mixed-precision add.
__device__ __forceinline__ void add_e4m3x16(float* acc, const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w[i] >> (16 * h)) & 0xFFFFu);
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
      add_f16x2(acc[4 * i + 2 * h], acc[4 * i + 2 * h + 1], hr.x, hr.y);
    }
  }
}

// Two fp32 -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// Thread 0 asks for the rows of token `tok` (if it exists) to be brought into
// L2, so that this CTA's loads of it hit L2 when it gets there.  The combines
// call it for the token a.prefetch grid strides ahead of the current one.
template <int kElemBytes>
__device__ __forceinline__ void prefetch_token_rows(const CombineArgs& a, int64_t tok) {
  if (tok >= a.ntok) return;
  const int nd = a.plan_nd[tok];
  if (nd == kNoToken || nd == 0) return;
  const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
  const int words = a.plan_stride / 8;
  if (EP_A2A_CHECKS && !plan_row_ok(nd, row[0], words > 1 ? row[1] : 0, words > 2 ? row[2] : 0,
                                    words > 3 ? row[3] : 0, a.ep, a.plan_stride, nullptr))
    return;
  const uint32_t bytes = (uint32_t)a.H * kElemBytes;
  const int64_t rank_stride = a.ntok * (int64_t)a.H * kElemBytes;
  for (int q = 0; q < nd; ++q) {
    const uint64_t w = q < 8 ? row[0] : row[min(q >> 3, words - 1)];
    const int d = (int)((w >> ((q & 7) * 8)) & 0xFFu);
    prefetch_l2(a.x + (int64_t)d * rank_stride + tok * (int64_t)bytes, bytes);
  }
}

// kMaxThreads / kMinBlocks: launch bounds of the instance (the 128-thread
// BF16 instance is held to 72 registers, so that seven CTAs fit on an SM).
template <bool kFp8, int kMaxThreads = 512, int kMinBlocks = 0>
__global__ void __launch_bounds__(kMaxThreads, kMinBlocks) combine_vec_kernel(const CombineArgs a) {
  pdl_wait();
  constexpr int kElems = kFp8 ? 16 : 8;       // elements per 16-byte input vector
  constexpr int kElemBytes = kFp8 ? 1 : 2;
  const int nvec = a.H / kElems;
  const int words = a.plan_stride / 8;
  if (a.prefetch && threadIdx.x == 0)
    for (int p = 0; p < a.prefetch; ++p)
      prefetch_token_rows<kElemBytes>(a, blockIdx.x + (int64_t)p * gridDim.x);
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    if (a.prefetch && threadIdx.x == 0)
      prefetch_token_rows<kElemBytes>(a, tok + (int64_t)a.prefetch * gridDim.x);
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    const uint8_t* xt = a.x + tok * (int64_t)a.H * kElemBytes;           // rank 0's row
    const int64_t rank_stride = a.ntok * (int64_t)a.H * kElemBytes;      // bytes per rank
    uint16_t* out = a.out + tok * (int64_t)a.H;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float acc[kElems];
#pragma unroll
      for (int e = 0; e < kElems; ++e) acc[e] = 0.0f;
      for (int c0 = 0; c0 < nd; c0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (c0 + i < nd)
            raw[i] = ld_stream_v4(xt + (int64_t)dst_rank(w0, w1, w2, w3, c0 + i) * rank_stride +
                                  (int64_t)v * 16);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (c0 + i < nd) {
            if (kFp8)
              add_e4m3x16(acc, raw[i]);
            else
              add_bf16x8(acc, raw[i]);
          }
        }
      }
      uint4* o = reinterpret_cast<uint4*>(out + (int64_t)v * kElems);
#pragma unroll
      for (int q = 0; q < kElems / 8; ++q) {
        uint4 pk;
        pk.x = pack_bf16x2(acc[8 * q + 0], acc[8 * q + 1]);
        pk.y = pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]);
        pk.z = pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]);
        pk.w = pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]);
        o[q] = pk;
      }
    }
  }
}

enum CombineMode { kCombineBf16 = 0, kCombineFp8 = 1, kCombineFp8Scaled = 2 };

// acc[0..16) = fmaf(widen(code), scale, acc) for the 16 E4M3 codes of v.
__device__ __forceinline__ void fma_e4m3x16(float* acc, const uint4& v, float scale) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
          (__nv_fp8x2_storage_t)((w[q] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
      __half_raw lo, hi;
      lo.x = hr.x;
      hi.x = hr.y;
      float& a0 = acc[4 * q + 2 * h];
      float& a1 = acc[4 * q + 2 * h + 1];
      a0 = __fmaf_rn(__half2float(__half(lo)), scale, a0);
      a1 = __fmaf_rn(__half2float(__half(hi)), scale, a1);
    }
  }
}

// Loads of one 16-byte column vector (at byte offset `off`) of each of the
// token's first nd (<= 8) destination rows.
__device__ __forceinline__ void load_rows(uint4 (&r)[8], const uint8_t* const (&src)[8], int nd,
                                          int64_t off) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i < nd) r[i] = ld_stream_v4(src[i] + off);
}

// Sum one column vector over the rows in ascending destination order and store
// it as bf16 (the 32 output bytes of an E4M3 vector as one 256-bit store when
// `wide`, i.e. the output is 32-byte aligned).
template <int kMode>
__device__ __forceinline__ void reduce_store(const uint4 (&r)[8], const float (&sc)[8], int nd,
                                             uint16_t* o, bool wide) {
  constexpr int kElems = kMode == kCombineBf16 ? 8 : 16;
  float acc[kElems];
#pragma unroll
  for (int e = 0; e < kElems; ++e) acc[e] = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i < nd) {
      if (kMode == kCombineBf16)
        add_bf16x8(acc, r[i]);
      else if (kMode == kCombineFp8)
        add_e4m3x16(acc, r[i]);
      else
        fma_e4m3x16(acc, r[i], sc[i]);
    }
  }
  uint32_t pk[kElems / 2];
#pragma unroll
  for (int i = 0; i < kElems / 2; ++i) pk[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  if (kElems == 16 && wide) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(o),
                 "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3]), "r"(pk[kElems / 2 - 4]),
                 "r"(pk[kElems / 2 - 3]), "r"(pk[kElems / 2 - 2]), "r"(pk[kElems / 2 - 1])
                 : "memory");
    return;
  }
#pragma unroll
  for (int q = 0; q < kElems / 8; ++q)
    reinterpret_cast<uint4*>(o)[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                                                pk[4 * q + 3]);
}

// The combines for tokens with at most 8 destination ranks (top_k or ep_size
// <= 8), 16-byte vectors: the same sums as combine_vec_kernel and
// combine_scaled_kernel<true>, with each thread's loads pipelined two deep --
// the rows of its next column vector are in flight while it adds the current
// one, so a thread never waits on memory with its adds still to do.
template <int kMode>
__global__ void __launch_bounds__(512) combine_pipe_kernel(const CombineArgs a,
                                                           const float* __restrict__ scales) {
  pdl_wait();
  constexpr int kElems = kMode == kCombineBf16 ? 8 : 16;
  constexpr int kElemBytes = kMode == kCombineBf16 ? 2 : 1;
  const int nvec = a.H / kElems;
  const int64_t rank_stride = a.ntok * (int64_t)a.H * kElemBytes;
  const int64_t step = (int64_t)blockDim.x * 16;       // bytes between a thread's vectors
  if (a.prefetch && threadIdx.x == 0)
    for (int p = 0; p < a.prefetch; ++p)
      prefetch_token_rows<kElemBytes>(a, blockIdx.x + (int64_t)p * gridDim.x);
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    if (a.prefetch && threadIdx.x == 0)
      prefetch_token_rows<kElemBytes>(a, tok + (int64_t)a.prefetch * gridDim.x);
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken || (int)threadIdx.x >= nvec) continue;
    const uint64_t w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
    const uint8_t* xt = a.x + tok * (int64_t)a.H * kElemBytes + (int64_t)threadIdx.x * 16;
    const uint8_t* src[8];
    float sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int d = (int)((w0 >> (8 * i)) & 0xFFu);
      src[i] = xt + (int64_t)(i < nd ? d : 0) * rank_stride;
      sc[i] = 1.0f;
      if (kMode == kCombineFp8Scaled && i < nd) sc[i] = scales[(int64_t)d * a.ntok + tok];
    }
    uint16_t* o = a.out + tok * (int64_t)a.H + (int64_t)threadIdx.x * kElems;
    const int64_t ostep = (int64_t)blockDim.x * kElems;
    uint4 ra[8], rb[8];
    load_rows(ra, src, nd, 0);
    int64_t off = 0;
    for (int v = threadIdx.x;;) {
      const bool more_b = v + (int)blockDim.x < nvec;
      if (more_b) load_rows(rb, src, nd, off + step);
      reduce_store<kMode>(ra, sc, nd, o, a.out32 != 0);
      if (!more_b) break;
      v += blockDim.x;
      off += step;
      o += ostep;
      const bool more_a = v + (int)blockDim.x < nvec;
      if (more_a) load_rows(ra, src, nd, off + step);
      reduce_store<kMode>(rb, sc, nd, o, a.out32 != 0);
      if (!more_a) break;
      v += blockDim.x;
      off += step;
      o += ostep;
    }
  }
}

// The combines with their rows staged in shared memory by bulk-async copies
// (cp.async.bulk, completion counted on an mbarrier): a work item is one
// chunk of kChunk bytes of a token's row; the producer warp's lane 0 loads the
// chunk of every destination row of the item into a stage of a ring, and the
// consumer warps sum it in ascending rank order from shared memory, store the
// output and release the stage.  The loads cost no registers, so an SM keeps
// stages x destinations x kChunk bytes in flight whatever the token count.
// At most 8 destinations per token; rows of 16-byte multiples at 16-byte
// aligned addresses.
constexpr int kStageChunk = 4096;                 // bytes of one row per item
constexpr unsigned kFullMask32 = 0xFFFFFFFFu;
constexpr int kCombineMaxStages = 8;

template <int kMode, int NCW>
__global__ void __launch_bounds__(32 * (NCW + 1)) combine_staged_kernel(
    const CombineArgs a, const float* __restrict__ scales, int stages, int stage_rows) {
  pdl_wait();
  extern __shared__ __align__(128) uint8_t cs_mem[];
  __shared__ __align__(8) uint64_t full_bar[kCombineMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kCombineMaxStages];
  __shared__ int64_t st_item[kCombineMaxStages];
  __shared__ int st_nd[kCombineMaxStages];
  __shared__ uint64_t st_w0[kCombineMaxStages];
  constexpr int kElemBytes = kMode == kCombineBf16 ? 2 : 1;
  constexpr int kElems = 16 / kElemBytes;          // elements per 16-byte vector
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row_bytes = (int64_t)a.H * kElemBytes;
  const int chunks = (int)((row_bytes + kStageChunk - 1) / kStageChunk);
  const int64_t items = a.ntok * chunks;
  const int64_t rank_stride = a.ntok * row_bytes;
  const uint32_t stage_bytes = (uint32_t)stage_rows * kStageChunk;
  const uint32_t smem0 = smem_addr(cs_mem);
  const uint32_t full0 = smem_addr(full_bar);
  const uint32_t empty0 = smem_addr(empty_bar);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, NCW);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == 0) {
    // producer warp: items blockIdx.x, blockIdx.x + gridDim.x, ... in batches
    // of 32 (lane l reads the plan row of the batch's item l, one load round
    // per batch); for each item that exists, lane 0 takes a free stage and sets
    // the bytes to expect, then lanes q < nd each issue the load of row q.
    // After the last item a sentinel (item -1) tells the consumers to stop.
    int64_t n = 0;
    for (int64_t base = blockIdx.x;; base += 32 * (int64_t)gridDim.x) {
      const int64_t my_it = base + (int64_t)lane * gridDim.x;
      int my_nd = kNoToken;
      uint64_t my_w0 = 0;
      if (my_it < items) {
        const int64_t tok = my_it / chunks;
        my_nd = a.plan_nd[tok];
        if (my_nd != kNoToken) {
          my_w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
          if (!plan_row_ok(my_nd, my_w0, 0, 0, 0, a.ep, 8, a.err)) my_nd = kNoToken;
        }
      }
      const bool last_batch = base + 32 * (int64_t)gridDim.x >= items;   // no items after it
      unsigned todo = __ballot_sync(kFullMask32, my_nd != kNoToken);
      bool stop = false;
      while (!stop) {
        int64_t it;
        int nd;
        uint64_t w0;
        if (todo) {
          const int l = __ffs(todo) - 1;
          todo &= todo - 1u;
          it = base + (int64_t)l * gridDim.x;
          nd = __shfl_sync(kFullMask32, my_nd, l);
          w0 = __shfl_sync(kFullMask32, my_w0, l);
        } else if (last_batch) {
          it = -1;                                     // the sentinel
          nd = 0;
          w0 = 0;
          stop = true;
        } else {
          break;                                       // next batch
        }
        const int s = (int)(n % stages);
        const uint32_t use = (uint32_t)(n / stages);
        bool ok = true;
        if (lane == 0) {
          if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1u, kWaitLimitNs)) {
            atomicOr(a.err, kErrWaitTimeout);
            ok = false;
          } else {
            st_item[s] = it;
            st_nd[s] = nd;
            st_w0[s] = w0;
          }
        }
        if (!__shfl_sync(kFullMask32, ok, 0)) return;
        ++n;
        if (it < 0 || nd == 0) {
          if (lane == 0) mbar_arrive(full0 + 8 * s);
          continue;
        }
        const int64_t tok = it / chunks;
        const int c = (int)(it - tok * chunks);
        const int64_t off = (int64_t)c * kStageChunk;
        const int64_t left = row_bytes - off;
        const uint32_t cb = (uint32_t)(left < kStageChunk ? left : kStageChunk);
        if (lane == 0) mbar_arrive_expect_tx(full0 + 8 * s, cb * (uint32_t)nd);
        __syncwarp();
        if (lane < nd) {
          const int d = (int)((w0 >> (8 * lane)) & 0xFFu);
          bulk_load(smem0 + (uint32_t)s * stage_bytes + (uint32_t)lane * kStageChunk,
                    a.x + tok * row_bytes + off + (int64_t)d * rank_stride, cb, full0 + 8 * s);
        }
      }
      if (stop) return;
    }
  }

  // consumers: thread c sums the 16-byte column vectors c, c + 32*NCW, ...
  constexpr int kCons = 32 * NCW;
  const int ct = threadIdx.x - 32;
  for (int64_t n = 0;; ++n) {
    const int s = (int)(n % stages);
    if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((n / stages) & 1), kWaitLimitNs)) {
      atomicOr(a.err, kErrWaitTimeout);
      break;
    }
    const int64_t it = st_item[s];
    if (it < 0) break;
    const int nd = st_nd[s];
    const uint64_t w0 = st_w0[s];
    const int64_t tok = it / chunks;
    const int c = (int)(it - tok * chunks);
    const int64_t off = (int64_t)c * kStageChunk;
    const int64_t left = row_bytes - off;
    const int nvec = (int)((left < kStageChunk ? left : kStageChunk) / 16);
    float sc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      sc[q] = 1.0f;
      if (kMode == kCombineFp8Scaled && q < nd)
        sc[q] = scales[(int64_t)((w0 >> (8 * q)) & 0xFFu) * a.ntok + tok];
    }
    const uint8_t* stage = cs_mem + (size_t)s * stage_bytes;
    uint16_t* o = a.out + tok * (int64_t)a.H + off / kElemBytes;
    for (int v = ct; v < nvec; v += kCons) {
      uint4 r[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (q < nd)
          r[q] = *reinterpret_cast<const uint4*>(stage + q * kStageChunk + v * 16);
      reduce_store<kMode>(r, sc, nd, o + (int64_t)v * kElems, false);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);      // this warp is done with the stage
  }
}

// Any hidden size and alignment: one element per thread step.
template <bool kFp8>
__global__ void __launch_bounds__(512) combine_scalar_kernel(const CombineArgs a) {
  pdl_wait();
  const int words = a.plan_stride / 8;
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
      float acc = 0.0f;
      for (int i = 0; i < nd; ++i) {
        const int64_t idx = ((int64_t)dst_rank(w0, w1, w2, w3, i) * a.ntok + tok) * a.H + h;
        float x;
        if (kFp8) {
          const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)a.x[idx], __NV_E4M3);
          x = __half2float(__half(hr));
        } else {
          x = bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(a.x)[idx]);
        }
        acc = __fadd_rn(acc, x);
      }
      a.out[tok * (int64_t)a.H + h] = (uint16_t)f32_to_bf16_bits(acc);
    }
  }
}

// Round to bf16 (nearest even) and widen back: the value a bf16 combine row holds.
__device__ __forceinline__ float bf16_round(float z) {
  return __bfloat162float(__float2bfloat16_rn(z));
}

// Per-token routing seen by the expert combine: for each slot j, the owner rank
// of its expert if that rank is one of the token's destinations, else -1
// (ids outside [0, E) and masked-off owners are in no destination's sum).
template <int KMAX>
__device__ __forceinline__ void slot_owners(const CombineExpertsArgs& a, int64_t tok, int nd,
                                            uint64_t w0, uint64_t w1, uint64_t w2, uint64_t w3,
                                            int (&own)[KMAX], float (&wt)[KMAX]) {
  const int first = dst_rank(w0, w1, w2, w3, 0);
  const int32_t* ids =
      reinterpret_cast<const int32_t*>(a.recv_ids0 + (int64_t)first * a.rank_stride) + tok * a.k;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    own[j] = -1;
    wt[j] = 0.0f;
    if (j < a.k) {
      const int32_t e = ids[j];
      int o = (e >= 0 && e < a.E) ? e / a.epr : -1;
      bool in_set = false;
      for (int q = 0; q < nd; ++q) in_set |= dst_rank(w0, w1, w2, w3, q) == o;
      own[j] = in_set ? o : -1;
      wt[j] = a.w[tok * a.k + j];
    }
  }
}

// top_k <= 8, hidden a multiple of 8, 16-byte aligned rows: each thread owns
// 16-byte column vectors; the loads of all needed slots are issued first.
__global__ void __launch_bounds__(512) combine_experts_vec_kernel(const CombineExpertsArgs a) {
  pdl_wait();
  constexpr int KMAX = 8;
  const int nvec = a.H / 8;
  const int words = a.plan_stride / 8;
  // the k slot rows of a token are contiguous: one prefetch per token
  const uint32_t tok_bytes = (uint32_t)a.k * a.H * 2;
  if (a.prefetch && threadIdx.x == 0)
    for (int p = 0; p < a.prefetch; ++p) {
      const int64_t t = blockIdx.x + (int64_t)p * gridDim.x;
      if (t < a.ntok) prefetch_l2(a.y + t * a.k * a.H, tok_bytes);
    }
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    if (a.prefetch && threadIdx.x == 0) {
      const int64_t t = tok + (int64_t)a.prefetch * gridDim.x;
      if (t < a.ntok) prefetch_l2(a.y + t * a.k * a.H, tok_bytes);
    }
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (nd == 0) {           // every owner masked off: the sum is empty
      for (int v = threadIdx.x; v < nvec; v += blockDim.x)
        reinterpret_cast<uint4*>(out)[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    int own[KMAX];
    float wt[KMAX];
    slot_owners<KMAX>(a, tok, nd, w0, w1, w2, w3, own, wt);
    const uint16_t* yt = a.y + tok * (int64_t)a.k * a.H;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      uint4 raw[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        if (own[j] >= 0) raw[j] = ld_stream_v4(yt + (int64_t)j * a.H + (int64_t)v * 8);
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
      for (int q = 0; q < nd; ++q) {
        const int d = dst_rank(w0, w1, w2, w3, q);
        float z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = 0.0f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (own[j] != d) continue;
          const uint32_t wv[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            z[2 * i] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] & 0xFFFFu), z[2 * i]);
            z[2 * i + 1] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] >> 16), z[2 * i + 1]);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e)       // z_d to bf16 in pairs, then added exactly widened
          add_bf16x2(acc[2 * e], acc[2 * e + 1], pack_bf16x2(z[2 * e], z[2 * e + 1]));
      }
      uint4 pk;
      pk.x = pack_bf16x2(acc[0], acc[1]);
      pk.y = pack_bf16x2(acc[2], acc[3]);
      pk.z = pack_bf16x2(acc[4], acc[5]);
      pk.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out)[v] = pk;
    }
  }
}

// Loads of one 16-byte column vector of each slot row that takes part.
__device__ __forceinline__ void expert_rows_load(uint4 (&r)[8], const uint16_t* yv,
                                                 const int (&own)[8], int H) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (own[j] >= 0) r[j] = ld_stream_v4(yv + (int64_t)j * H);
}

// For each destination rank d in ascending order: z = fp32 fused multiply-add
// over the slots d owns (ascending), rounded to bf16, added to the sum; the sum
// is stored as bf16.
__device__ __forceinline__ void expert_rows_reduce_store(const uint4 (&raw)[8],
                                                         const int (&own)[8],
                                                         const float (&wt)[8], int nd,
                                                         uint64_t w0, uint16_t* o) {
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  for (int q = 0; q < nd; ++q) {
    const int d = (int)((w0 >> (8 * q)) & 0xFFu);
    float z[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) z[e] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (own[j] != d) continue;
      const uint32_t wv[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        z[2 * i] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] & 0xFFFFu), z[2 * i]);
        z[2 * i + 1] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] >> 16), z[2 * i + 1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e)           // z_d to bf16 in pairs, then added exactly widened
      add_bf16x2(acc[2 * e], acc[2 * e + 1], pack_bf16x2(z[2 * e], z[2 * e + 1]));
  }
  uint4 pk;
  pk.x = pack_bf16x2(acc[0], acc[1]);
  pk.y = pack_bf16x2(acc[2], acc[3]);
  pk.z = pack_bf16x2(acc[4], acc[5]);
  pk.w = pack_bf16x2(acc[6], acc[7]);
  *reinterpret_cast<uint4*>(o) = pk;
}

// combine_experts_vec_kernel with each thread's loads pipelined two deep: the
// slot rows of its next column vector are in flight while it reduces the
// current one.  top_k <= 8, so a token has at most 8 destinations.
__global__ void __launch_bounds__(512) combine_experts_pipe_kernel(const CombineExpertsArgs a) {
  pdl_wait();
  const int nvec = a.H / 8;
  const uint32_t tok_bytes = (uint32_t)a.k * a.H * 2;
  if (a.prefetch && threadIdx.x == 0)
    for (int p = 0; p < a.prefetch; ++p) {
      const int64_t t = blockIdx.x + (int64_t)p * gridDim.x;
      if (t < a.ntok) prefetch_l2(a.y + t * a.k * a.H, tok_bytes);
    }
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    if (a.prefetch && threadIdx.x == 0) {
      const int64_t t = tok + (int64_t)a.prefetch * gridDim.x;
      if (t < a.ntok) prefetch_l2(a.y + t * a.k * a.H, tok_bytes);
    }
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken || (int)threadIdx.x >= nvec) continue;
    uint16_t* o = a.out + tok * (int64_t)a.H + (int64_t)threadIdx.x * 8;
    const int64_t step = (int64_t)blockDim.x * 8;      // elements between a thread's vectors
    if (nd == 0) {           // every owner masked off: the sum is empty
      for (int v = threadIdx.x; v < nvec; v += blockDim.x, o += step)
        *reinterpret_cast<uint4*>(o) = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint64_t w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
    int own[8];
    float wt[8];
    slot_owners<8>(a, tok, nd, w0, 0, 0, 0, own, wt);
    const uint16_t* yv = a.y + tok * (int64_t)a.k * a.H + (int64_t)threadIdx.x * 8;
    uint4 ra[8], rb[8];
    expert_rows_load(ra, yv, own, a.H);
    for (int v = threadIdx.x;;) {
      const bool more_b = v + (int)blockDim.x < nvec;
      if (more_b) expert_rows_load(rb, yv + step, own, a.H);
      expert_rows_reduce_store(ra, own, wt, nd, w0, o);
      if (!more_b) break;
      v += blockDim.x;
      yv += step;
      o += step;
      const bool more_a = v + (int)blockDim.x < nvec;
      if (more_a) expert_rows_load(ra, yv + step, own, a.H);
      expert_rows_reduce_store(rb, own, wt, nd, w0, o);
      if (!more_a) break;
      v += blockDim.x;
      yv += step;
      o += step;
    }
  }
}

// ---------------------------------------------------------------------------
// Low-precision combine of per-expert outputs, quantised on the sending side
// (flashinfer.moe_ep.NVLinkOneSidedConfig, use_low_precision_combine, with the
// per-row scale convention of the scaled FP8 combine): for each destination d
// of a token, z_d = bf16(sum over d's slots of w_j * y_j) as in the expert
// combine; amax_d = max |z_d|, scale_d = amax_d / 448, inv_d = 448 / amax_d
// (fp32, rounded to nearest; 1 and 1 for a zero row); code = E4M3(z_d * inv_d)
// nearest-even, saturating; out = bf16(sum over d ascending of
// fmaf(decode(code), scale_d, acc)) from +0.0f.  Neither the rows z_d nor the
// codes and scales are written to memory.
// ---------------------------------------------------------------------------

// E4M3 round trip of 8 values scaled by inv: code = E4M3(z * inv) (product
// rounded to fp32, nearest-even, saturating), then acc = fmaf(decode, scale, acc).
__device__ __forceinline__ void fp8_roundtrip_acc(float* acc, const uint4& zb, float inv,
                                                  float scale) {
  const uint32_t w[4] = {zb.x, zb.y, zb.z, zb.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = make_float2(__fmul_rn(bf16_bits_to_f32(w[i] & 0xFFFFu), inv),
                                 __fmul_rn(bf16_bits_to_f32(w[i] >> 16), inv));
    const __nv_fp8x2_storage_t code = __nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(code, __NV_E4M3);
    __half_raw lo, hi;
    lo.x = hr.x;
    hi.x = hr.y;
    acc[2 * i] = __fmaf_rn(__half2float(__half(lo)), scale, acc[2 * i]);
    acc[2 * i + 1] = __fmaf_rn(__half2float(__half(hi)), scale, acc[2 * i + 1]);
  }
}

// The same for one value.
__device__ __forceinline__ float fp8_roundtrip(float z, float inv, float scale, float acc) {
  const __nv_fp8_storage_t code =
      __nv_cvt_float_to_fp8(__fmul_rn(z, inv), __NV_SATFINITE, __NV_E4M3);
  const __half_raw hr = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
  return __fmaf_rn(__half2float(__half(hr)), scale, acc);
}

// Per-destination scale and inverse from amax (the row quantiser's rule).
__device__ __forceinline__ void row_scale_of(float amax, float& scale, float& inv) {
  scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 1.0f;
}

constexpr int kFp8ExpertsMaxWarps = 32;

// top_k <= 8, hidden a multiple of 8, 16-byte aligned rows, and the token's
// rows z_d (at most min(top_k, ep) of them, bf16) fit in shared memory; at
// most 448 threads, so that two CTAs share an SM without spilling.  One
// token per CTA at a time: phase 1 loads each 16-byte column vector of every
// participating slot row once, forms every destination's z_d for it, stores
// it to shared memory and keeps a per-destination running max; the CTA
// reduces the maxima to the scales; phase 2 reads z_d back, takes each value
// through E4M3 and sums in ascending rank order.
__global__ void __launch_bounds__(448, 2) combine_experts_fp8_kernel(const CombineExpertsArgs a) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t z_mem[];       // [rows][H] bf16
  __shared__ float s_max[kFp8ExpertsMaxWarps][8];
  __shared__ float s_scale[8], s_inv[8];
  uint16_t* zs = reinterpret_cast<uint16_t*>(z_mem);
  const int nvec = a.H / 8;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (nd == 0) {           // every owner masked off: the sum is empty
      for (int v = threadIdx.x; v < nvec; v += blockDim.x)
        reinterpret_cast<uint4*>(out)[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint64_t w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
    int own[8];
    float wt[8];
    slot_owners<8>(a, tok, nd, w0, 0, 0, 0, own, wt);
    // phase 1: z rows into shared memory and the per-destination maxima
    float amax[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) amax[q] = 0.0f;
    const uint16_t* yt = a.y + tok * (int64_t)a.k * a.H;
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      uint4 raw[8];
      expert_rows_load(raw, yt + (int64_t)v * 8, own, a.H);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= nd) break;
        const int d = (int)((w0 >> (8 * q)) & 0xFFu);
        float z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (own[j] != d) continue;
          const uint32_t wv[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            z[2 * i] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] & 0xFFFFu), z[2 * i]);
            z[2 * i + 1] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] >> 16), z[2 * i + 1]);
          }
        }
        uint4 pk;
        pk.x = pack_bf16x2(z[0], z[1]);
        pk.y = pack_bf16x2(z[2], z[3]);
        pk.z = pack_bf16x2(z[4], z[5]);
        pk.w = pack_bf16x2(z[6], z[7]);
        const uint32_t pw[4] = {pk.x, pk.y, pk.z, pk.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          amax[q] = fmaxf(amax[q], fabsf(bf16_bits_to_f32(pw[i] & 0xFFFFu)));
          amax[q] = fmaxf(amax[q], fabsf(bf16_bits_to_f32(pw[i] >> 16)));
        }
        *reinterpret_cast<uint4*>(zs + (int64_t)q * a.H + (int64_t)v * 8) = pk;
      }
    }
    // the CTA's maxima -> scales
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        amax[q] = fmaxf(amax[q], __shfl_xor_sync(0xFFFFFFFFu, amax[q], o));
      if (lane == 0) s_max[warp][q] = amax[q];
    }
    __syncthreads();
    if (threadIdx.x < 8) {
      float m = 0.0f;
      for (int i = 0; i < nwarps; ++i) m = fmaxf(m, s_max[i][threadIdx.x]);
      row_scale_of(m, s_scale[threadIdx.x], s_inv[threadIdx.x]);
    }
    __syncthreads();
    // phase 2: through E4M3 and summed in ascending rank order
    for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= nd) break;
        const uint4 zb = *reinterpret_cast<const uint4*>(zs + (int64_t)q * a.H + (int64_t)v * 8);
        fp8_roundtrip_acc(acc, zb, s_inv[q], s_scale[q]);
      }
      uint4 pk;
      pk.x = pack_bf16x2(acc[0], acc[1]);
      pk.y = pack_bf16x2(acc[2], acc[3]);
      pk.z = pack_bf16x2(acc[4], acc[5]);
      pk.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out)[v] = pk;
    }
    __syncthreads();         // z rows and scales are rewritten for the next token
  }
}

// The same with a thread-block cluster of C CTAs per token, each CTA owning a
// slice of the row's 16-byte column vectors, one per thread, so that every
// z_d stays in registers: phase 1 loads the thread's vector of each
// participating slot row once and forms every destination's z_d (bf16) and
// its partial max; each CTA reduces its maxima, the cluster exchanges them
// through distributed shared memory (one cluster barrier per token; the
// exchange slots alternate between tokens so that one barrier suffices), and
// phase 2 takes each value through E4M3 and sums.  top_k <= 8, hidden a
// multiple of 8, 16-byte aligned rows, nvec <= C * blockDim.x.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// The float at the same shared-memory offset as `p` in CTA `rank` of the cluster.
__device__ __forceinline__ float ld_cluster_f32(const float* p, uint32_t rank) {
  uint32_t remote, local = smem_addr(p);
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
  return v;
}

// The u32 at the same shared-memory offset as `p` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t ld_cluster_u32(const uint32_t* p, uint32_t rank) {
  uint32_t remote, local = smem_addr(p), v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(local), "r"(rank));
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(remote) : "memory");
  return v;
}

template <int C>
__global__ void __launch_bounds__(256, 2) combine_experts_fp8_cluster_kernel(
    const CombineExpertsArgs a) {
  pdl_wait();
  __shared__ float s_max[8][8];            // [warp][destination]
  __shared__ float s_part[2][8];           // this CTA's maxima, by token parity
  __shared__ float s_scale[8], s_inv[8];
  const int nvec = a.H / 8;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  const uint32_t cr = cluster_cta_rank();
  const int v = (int)cr * blockDim.x + threadIdx.x;   // this thread's column vector
  const bool has_v = v < nvec;
  const int64_t clusters = gridDim.x / C;
  int parity = 0;
  for (int64_t tok = blockIdx.x / C; tok < a.ntok; tok += clusters) {
    const int nd = a.plan_nd[tok];                // the same in every CTA of the cluster
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (nd == 0) {           // every owner masked off: the sum is empty
      if (has_v) reinterpret_cast<uint4*>(out)[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint64_t w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
    int own[8];
    float wt[8];
    slot_owners<8>(a, tok, nd, w0, 0, 0, 0, own, wt);
    uint32_t zr[8][4];
    float amax[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) amax[q] = 0.0f;
    if (has_v) {
      uint4 raw[8];
      expert_rows_load(raw, a.y + tok * (int64_t)a.k * a.H + (int64_t)v * 8, own, a.H);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= nd) break;
        const int d = (int)((w0 >> (8 * q)) & 0xFFu);
        float z[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) z[e] = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (own[j] != d) continue;
          const uint32_t wv[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            z[2 * i] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] & 0xFFFFu), z[2 * i]);
            z[2 * i + 1] = __fmaf_rn(wt[j], bf16_bits_to_f32(wv[i] >> 16), z[2 * i + 1]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          zr[q][i] = pack_bf16x2(z[2 * i], z[2 * i + 1]);
          amax[q] = fmaxf(amax[q], fabsf(bf16_bits_to_f32(zr[q][i] & 0xFFFFu)));
          amax[q] = fmaxf(amax[q], fabsf(bf16_bits_to_f32(zr[q][i] >> 16)));
        }
      }
    }
    // the CTA's maxima, then the cluster's
#pragma unroll
    for (int q = 0; q < 8; ++q) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        amax[q] = fmaxf(amax[q], __shfl_xor_sync(0xFFFFFFFFu, amax[q], o));
      if (lane == 0) s_max[warp][q] = amax[q];
    }
    __syncthreads();
    if (threadIdx.x < 8) {
      float m = 0.0f;
      for (int i = 0; i < nwarps; ++i) m = fmaxf(m, s_max[i][threadIdx.x]);
      s_part[parity][threadIdx.x] = m;
    }
    cluster_sync_all();
    if (threadIdx.x < 8) {
      float m = 0.0f;
      for (uint32_t r = 0; r < (uint32_t)C; ++r)
        m = fmaxf(m, ld_cluster_f32(&s_part[parity][threadIdx.x], r));
      row_scale_of(m, s_scale[threadIdx.x], s_inv[threadIdx.x]);
    }
    __syncthreads();
    if (has_v) {
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= nd) break;
        fp8_roundtrip_acc(acc, make_uint4(zr[q][0], zr[q][1], zr[q][2], zr[q][3]), s_inv[q],
                          s_scale[q]);
      }
      uint4 pk;
      pk.x = pack_bf16x2(acc[0], acc[1]);
      pk.y = pack_bf16x2(acc[2], acc[3]);
      pk.z = pack_bf16x2(acc[4], acc[5]);
      pk.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out)[v] = pk;
    }
    parity ^= 1;
  }
  cluster_sync_all();        // no CTA leaves while a partner may still read its maxima
}

// The sender-side FP8 expert combine, split over a cluster of C CTAs per
// token (each CTA a slice of the row's 16-byte column vectors, two per thread)
// with the rows z_d of its slice in shared memory.  Per token, warp 0 orders
// the participating slots destination-major (ascending slot within each
// destination, destinations in ascending rank), so phase 1 is one run of
// fused multiply-adds over the slots with a uniform branch where a
// destination's slots end; there z_d is rounded to bf16, stored, and its
// maximum |z_d| taken on the packed bf16 bits (non-negative bf16 values order
// like their bit patterns): a packed 16-bit max per pair, a warp max
// reduction (redux) and a shared atomic max per warp.  The CTAs of the cluster
// exchange their maxima through distributed shared memory (one cluster
// barrier per token; the slots alternate between tokens), then phase 2 takes
// the values through E4M3 and sums in ascending rank order.  top_k <= 8,
// hidden a multiple of 8, 16-byte aligned rows, hidden / 8 <= C * 2 * blockDim.x.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

template <int C>
__global__ void __launch_bounds__(256, 3) combine_experts_fp8_split_kernel(
    const CombineExpertsArgs a, int cols) {
  pdl_wait();
  extern __shared__ __align__(16) uint8_t zsplit_mem[];    // [8][cols] bf16
  __shared__ int s_slot[8];          // slot of position p (destination-major order)
  __shared__ float s_wt[8];
  __shared__ uint32_t s_end;         // 4 bits per destination: its slots end before this position
  __shared__ int s_ns;               // participating slots
  __shared__ uint32_t s_amax[2][8];  // per destination, by token parity: max |z| as bf16 bits
  __shared__ float s_scale[8], s_inv[8];
  uint16_t* zs = reinterpret_cast<uint16_t*>(zsplit_mem);
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const uint32_t cr = C > 1 ? cluster_cta_rank() : 0u;
  const int nvec = a.H / 8;
  const int cvec = cols / 8;                       // vectors of this CTA's slice
  const int vbase = (int)cr * cvec;
  const int64_t clusters = gridDim.x / C;
  const int pf_bytes = (min(cvec, nvec - vbase) > 0 ? min(cvec, nvec - vbase) : 0) * 16;
  int parity = 0;
  for (int64_t tok = blockIdx.x / C; tok < a.ntok; tok += clusters) {
    if (a.prefetch && (int)threadIdx.x < a.k && pf_bytes > 0) {
      // this CTA's slice of each slot row of the token a.prefetch steps ahead
      // into L2 while this one is summed
      const int64_t nt = tok + (int64_t)a.prefetch * clusters;
      if (nt < a.ntok)
        prefetch_l2(a.y + (nt * a.k + threadIdx.x) * (int64_t)a.H + (int64_t)vbase * 8,
                    (uint32_t)pf_bytes);
    }
    const int nd = a.plan_nd[tok];                 // the same in every CTA of the cluster
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (nd == 0) {           // every owner masked off: the sum is empty
      for (int i = threadIdx.x; i < cvec; i += blockDim.x)
        if (vbase + i < nvec) reinterpret_cast<uint4*>(out)[vbase + i] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint64_t w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
    if (warp == 0) {
      // lane j < k: slot j's destination index q (its owner's position in the
      // plan row) and weight; its position in the destination-major order
      int q = -1;
      float wj = 0.0f;
      if (lane < a.k) {
        const int first = (int)(w0 & 0xFFu);
        const int32_t e = reinterpret_cast<const int32_t*>(
            a.recv_ids0 + (int64_t)first * a.rank_stride)[tok * a.k + lane];
        const int o = (e >= 0 && e < a.E) ? e / a.epr : -1;
        for (int i = 0; i < nd; ++i)
          if ((int)((w0 >> (8 * i)) & 0xFFu) == o) q = i;
        wj = a.w[tok * a.k + lane];
      }
      const unsigned part = __ballot_sync(0xFFFFFFFFu, q >= 0);
      int pos = 0, cnt = 0;
      for (int i = 0; i < 8; ++i) {
        const int qi = __shfl_sync(0xFFFFFFFFu, q, i);
        if (q >= 0 && qi >= 0 && (qi < q || (qi == q && i < lane))) ++pos;
        if (lane < 8 && qi >= 0 && qi <= lane) ++cnt;   // slots of destinations 0..lane
      }
      if (q >= 0) {
        s_slot[pos] = lane;
        s_wt[pos] = wj;
      }
      uint32_t endw = (lane < 8 && lane < nd) ? ((uint32_t)cnt << (4 * lane)) : 0u;
      endw = __reduce_or_sync(0xFFFFFFFFu, endw);
      if (lane == 0) {
        s_end = endw;
        s_ns = __popc(part);
      }
      if (lane < 8) s_amax[parity][lane] = 0u;
    }
    __syncthreads();
    int slot[8];
    float wt[8];
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      slot[p] = s_slot[p];
      wt[p] = s_wt[p];
    }
    const int ns = s_ns;
    const uint32_t endw = s_end;
    const uint16_t* yt = a.y + tok * (int64_t)a.k * a.H;
    // phase 1: this thread's vectors i = threadIdx.x, threadIdx.x + blockDim.x
    for (int i = threadIdx.x; i < 2 * (int)blockDim.x; i += blockDim.x) {
      const int v = vbase + i;
      const bool has = i < cvec && v < nvec;       // warp-uniform except at the edge
      uint4 raw[8];
#pragma unroll
      for (int p = 0; p < 8; ++p)
        if (p < ns && has) raw[p] = ld_stream_v4(yt + (int64_t)slot[p] * a.H + (int64_t)v * 8);
      float z[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = 0.0f;
      int q = 0;
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        if (p >= ns) break;
        if (has) {
          const uint32_t wv[4] = {raw[p].x, raw[p].y, raw[p].z, raw[p].w};
#pragma unroll
          for (int k2 = 0; k2 < 4; ++k2) {
            z[2 * k2] = __fmaf_rn(wt[p], bf16_bits_to_f32(wv[k2] & 0xFFFFu), z[2 * k2]);
            z[2 * k2 + 1] = __fmaf_rn(wt[p], bf16_bits_to_f32(wv[k2] >> 16), z[2 * k2 + 1]);
          }
        }
        if ((int)((endw >> (4 * q)) & 0xFu) == p + 1) {   // destination q's slots end here
          uint32_t m = 0u;
          if (has) {
            const uint32_t pk0 = pack_bf16x2(z[0], z[1]), pk1 = pack_bf16x2(z[2], z[3]);
            const uint32_t pk2 = pack_bf16x2(z[4], z[5]), pk3 = pack_bf16x2(z[6], z[7]);
            *reinterpret_cast<uint4*>(zs + (int64_t)q * cols + (int64_t)i * 8) =
                make_uint4(pk0, pk1, pk2, pk3);
            const uint32_t mm = max_u16x2(max_u16x2(pk0 & 0x7FFF7FFFu, pk1 & 0x7FFF7FFFu),
                                          max_u16x2(pk2 & 0x7FFF7FFFu, pk3 & 0x7FFF7FFFu));
            m = max(mm & 0xFFFFu, mm >> 16);
          }
          m = __reduce_max_sync(0xFFFFFFFFu, m);
          if (lane == 0) atomicMax(&s_amax[parity][q], m);
#pragma unroll
          for (int e = 0; e < 8; ++e) z[e] = 0.0f;
          ++q;
        }
      }
    }
    __syncthreads();
    if (C > 1) cluster_sync_all();
    if (threadIdx.x < nd) {
      uint32_t m = 0u;
      for (uint32_t r = 0; r < (uint32_t)C; ++r)
        m = max(m, C > 1 ? ld_cluster_u32(&s_amax[parity][threadIdx.x], r)
                         : s_amax[parity][threadIdx.x]);
      row_scale_of(__uint_as_float(m << 16), s_scale[threadIdx.x], s_inv[threadIdx.x]);
    }
    __syncthreads();
    // phase 2
    for (int i = threadIdx.x; i < cvec; i += blockDim.x) {
      const int v = vbase + i;
      if (v >= nvec) break;
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (q >= nd) break;
        const uint4 zb = *reinterpret_cast<const uint4*>(zs + (int64_t)q * cols + (int64_t)i * 8);
        fp8_roundtrip_acc(acc, zb, s_inv[q], s_scale[q]);
      }
      uint4 pk;
      pk.x = pack_bf16x2(acc[0], acc[1]);
      pk.y = pack_bf16x2(acc[2], acc[3]);
      pk.z = pack_bf16x2(acc[4], acc[5]);
      pk.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out)[v] = pk;
    }
    parity ^= 1;
  }
  if (C > 1) cluster_sync_all();   // no CTA leaves while a partner may still read its maxima
}

// Any top_k (<= 32) and hidden size, no shared-memory rows: for each
// destination a first pass recomputes z_d over the row to find its maximum;
// a second pass recomputes z_d, takes it through E4M3 and sums.
__global__ void __launch_bounds__(256) combine_experts_fp8_any_kernel(const CombineExpertsArgs a) {
  pdl_wait();
  constexpr int KMAX = kMaxTopK;
  __shared__ float s_max[8];
  __shared__ float s_scale[KMAX], s_inv[KMAX];
  const int words = a.plan_stride / 8;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    int own[KMAX];
    float wt[KMAX];
    if (nd > 0) slot_owners<KMAX>(a, tok, nd, w0, w1, w2, w3, own, wt);
    const uint16_t* yt = a.y + tok * (int64_t)a.k * a.H;
    auto z_of = [&](int d, int h) {
      float z = 0.0f;
      for (int j = 0; j < a.k; ++j)
        if (own[j] == d) z = __fmaf_rn(wt[j], bf16_bits_to_f32(yt[(int64_t)j * a.H + h]), z);
      return bf16_round(z);
    };
    for (int q = 0; q < nd; ++q) {
      const int d = dst_rank(w0, w1, w2, w3, q);
      float m = 0.0f;
      for (int h = threadIdx.x; h < a.H; h += blockDim.x) m = fmaxf(m, fabsf(z_of(d, h)));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (lane == 0) s_max[warp] = m;
      __syncthreads();
      if (threadIdx.x == 0) {
        float mm = 0.0f;
        for (int i = 0; i < nwarps; ++i) mm = fmaxf(mm, s_max[i]);
        row_scale_of(mm, s_scale[q], s_inv[q]);
      }
      __syncthreads();
    }
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
      float acc = 0.0f;
      for (int q = 0; q < nd; ++q)
        acc = fp8_roundtrip(z_of(dst_rank(w0, w1, w2, w3, q), h), s_inv[q], s_scale[q], acc);
      out[h] = (uint16_t)f32_to_bf16_bits(acc);
    }
    __syncthreads();         // scales are rewritten for the next token
  }
}

// combine_experts_pipe_kernel with the slot rows staged in shared memory by
// bulk-async copies, as combine_staged_kernel does for the per-rank rows: a
// work item is one kStageChunk-byte chunk of a token's slot rows; the
// producer lane finds the slots' owners and weights, loads the chunk of every
// participating slot row into a stage, and the consumer warps form each
// destination's z_d and the ordered sum from shared memory.  top_k <= 8,
// hidden a multiple of 8, 16-byte aligned rows.
template <int NCW>
__global__ void __launch_bounds__(32 * (NCW + 1)) combine_experts_staged_kernel(
    const CombineExpertsArgs a, int stages) {
  pdl_wait();
  extern __shared__ __align__(128) uint8_t es_mem[];
  __shared__ __align__(8) uint64_t full_bar[kCombineMaxStages];
  __shared__ __align__(8) uint64_t empty_bar[kCombineMaxStages];
  __shared__ int64_t st_item[kCombineMaxStages];
  __shared__ int st_nd[kCombineMaxStages];
  __shared__ uint64_t st_w0[kCombineMaxStages];
  __shared__ int st_own[kCombineMaxStages][8];
  __shared__ float st_wt[kCombineMaxStages][8];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t row_bytes = (int64_t)a.H * 2;
  const int chunks = (int)((row_bytes + kStageChunk - 1) / kStageChunk);
  const int64_t items = a.ntok * chunks;
  const uint32_t stage_bytes = 8u * kStageChunk;
  const uint32_t smem0 = smem_addr(es_mem);
  const uint32_t full0 = smem_addr(full_bar);
  const uint32_t empty0 = smem_addr(empty_bar);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, NCW);
    }
    mbar_init_fence();
  }
  __syncthreads();

  if (warp == 0) {
    if (lane != 0) return;
    int64_t n = 0;
    for (int64_t it = blockIdx.x;; it += gridDim.x) {
      int nd = 0;
      uint64_t w0 = 0;
      int own[8];
      float wt[8];
      const int64_t tok = it < items ? it / chunks : 0;
      if (it < items) {
        nd = a.plan_nd[tok];
        if (nd == kNoToken) continue;
        w0 = *reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
        if (!plan_row_ok(nd, w0, 0, 0, 0, a.ep, 8, a.err)) continue;
        if (nd > 0) slot_owners<8>(a, tok, nd, w0, 0, 0, 0, own, wt);
      }
      const int s = (int)(n % stages);
      const uint32_t use = (uint32_t)(n / stages);
      if (use > 0 && !mbar_wait_bounded(empty0 + 8 * s, (use - 1) & 1u, kWaitLimitNs)) {
        atomicOr(a.err, kErrWaitTimeout);
        return;
      }
      ++n;
      st_item[s] = it < items ? it : -1;
      st_nd[s] = nd;
      st_w0[s] = w0;
      if (it >= items || nd == 0) {
        mbar_arrive(full0 + 8 * s);
        if (it >= items) return;
        continue;
      }
      const int c = (int)(it - tok * chunks);
      const int64_t off = (int64_t)c * kStageChunk;
      const int64_t left = row_bytes - off;
      const uint32_t cb = (uint32_t)(left < kStageChunk ? left : kStageChunk);
      uint32_t tx = 0;
      for (int j = 0; j < 8; ++j) {
        st_own[s][j] = own[j];
        st_wt[s][j] = wt[j];
        if (own[j] >= 0) tx += cb;
      }
      mbar_arrive_expect_tx(full0 + 8 * s, tx);
      const uint8_t* yt = reinterpret_cast<const uint8_t*>(a.y) + tok * a.k * row_bytes + off;
      for (int j = 0; j < 8; ++j)
        if (own[j] >= 0)
          bulk_load(smem0 + (uint32_t)s * stage_bytes + (uint32_t)j * kStageChunk,
                    yt + (int64_t)j * row_bytes, cb, full0 + 8 * s);
    }
  }

  constexpr int kCons = 32 * NCW;
  const int ct = threadIdx.x - 32;
  for (int64_t n = 0;; ++n) {
    const int s = (int)(n % stages);
    if (!mbar_wait_bounded(full0 + 8 * s, (uint32_t)((n / stages) & 1), kWaitLimitNs)) {
      atomicOr(a.err, kErrWaitTimeout);
      break;
    }
    const int64_t it = st_item[s];
    if (it < 0) break;
    const int nd = st_nd[s];
    const uint64_t w0 = st_w0[s];
    const int64_t tok = it / chunks;
    const int c = (int)(it - tok * chunks);
    const int64_t off = (int64_t)c * kStageChunk;
    const int64_t left = row_bytes - off;
    const int nvec = (int)((left < kStageChunk ? left : kStageChunk) / 16);
    uint16_t* o = a.out + tok * (int64_t)a.H + off / 2;
    if (nd == 0) {
      for (int v = ct; v < nvec; v += kCons)
        reinterpret_cast<uint4*>(o)[v] = make_uint4(0u, 0u, 0u, 0u);
    } else {
      int own[8];
      float wt[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        own[j] = st_own[s][j];
        wt[j] = st_wt[s][j];
      }
      const uint8_t* stage = es_mem + (size_t)s * stage_bytes;
      for (int v = ct; v < nvec; v += kCons) {
        uint4 r[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (own[j] >= 0) r[j] = *reinterpret_cast<const uint4*>(stage + j * kStageChunk + v * 16);
        expert_rows_reduce_store(r, own, wt, nd, w0, o + (int64_t)v * 8);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
}

// Any top_k (<= 32) and hidden size: one element per thread step.
__global__ void __launch_bounds__(512) combine_experts_any_kernel(const CombineExpertsArgs a) {
  pdl_wait();
  constexpr int KMAX = kMaxTopK;
  const int words = a.plan_stride / 8;
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    int own[KMAX];
    float wt[KMAX];
    if (nd > 0) slot_owners<KMAX>(a, tok, nd, w0, w1, w2, w3, own, wt);
    const uint16_t* yt = a.y + tok * (int64_t)a.k * a.H;
    for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
      float acc = 0.0f;
      for (int q = 0; q < nd; ++q) {
        const int d = dst_rank(w0, w1, w2, w3, q);
        float z = 0.0f;
        for (int j = 0; j < a.k; ++j)
          if (own[j] == d) z = __fmaf_rn(wt[j], bf16_bits_to_f32(yt[(int64_t)j * a.H + h]), z);
        acc = __fadd_rn(acc, bf16_round(z));
      }
      out[h] = (uint16_t)f32_to_bf16_bits(acc);
    }
  }
}

// FP8 combine with one fp32 scale per row: acc = fmaf(decode(q), scale_d, acc)
// over the token's destination ranks in ascending order.
template <bool kVec>
__global__ void __launch_bounds__(512) combine_scaled_kernel(const CombineArgs a,
                                                             const float* __restrict__ scales) {
  pdl_wait();
  const int words = a.plan_stride / 8;
  const int nvec = kVec ? a.H / 16 : 0;
  if (kVec && a.prefetch && threadIdx.x == 0)
    for (int p = 0; p < a.prefetch; ++p)
      prefetch_token_rows<1>(a, blockIdx.x + (int64_t)p * gridDim.x);
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    if (kVec && a.prefetch && threadIdx.x == 0)
      prefetch_token_rows<1>(a, tok + (int64_t)a.prefetch * gridDim.x);
    const int nd = a.plan_nd[tok];
    if (nd == kNoToken) continue;
    const uint64_t* row = reinterpret_cast<const uint64_t*>(a.plan_dst + tok * a.plan_stride);
    const uint64_t w0 = row[0];
    const uint64_t w1 = words > 1 ? row[1] : 0;
    const uint64_t w2 = words > 2 ? row[2] : 0;
    const uint64_t w3 = words > 3 ? row[3] : 0;
    if (!plan_row_ok(nd, w0, w1, w2, w3, a.ep, a.plan_stride, a.err)) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (kVec) {
      const uint8_t* xt = a.x + tok * (int64_t)a.H;
      const int64_t rank_stride = a.ntok * (int64_t)a.H;
      for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
        for (int c0 = 0; c0 < nd; c0 += 8) {
          uint4 raw[8];
          float sc[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (c0 + i < nd) {
              const int d = dst_rank(w0, w1, w2, w3, c0 + i);
              raw[i] = ld_stream_v4(xt + (int64_t)d * rank_stride + (int64_t)v * 16);
              sc[i] = scales[(int64_t)d * a.ntok + tok];
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (c0 + i >= nd) continue;
            const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(
                    (__nv_fp8x2_storage_t)((w[q] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
                __half_raw lo, hi;
                lo.x = hr.x;
                hi.x = hr.y;
                float& a0 = acc[4 * q + 2 * h];
                float& a1 = acc[4 * q + 2 * h + 1];
                a0 = __fmaf_rn(__half2float(__half(lo)), sc[i], a0);
                a1 = __fmaf_rn(__half2float(__half(hi)), sc[i], a1);
              }
            }
          }
        }
        uint4* o = reinterpret_cast<uint4*>(out + (int64_t)v * 16);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint4 pk;
          pk.x = pack_bf16x2(acc[8 * q + 0], acc[8 * q + 1]);
          pk.y = pack_bf16x2(acc[8 * q + 2], acc[8 * q + 3]);
          pk.z = pack_bf16x2(acc[8 * q + 4], acc[8 * q + 5]);
          pk.w = pack_bf16x2(acc[8 * q + 6], acc[8 * q + 7]);
          o[q] = pk;
        }
      }
    } else {
      for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
        float acc = 0.0f;
        for (int i = 0; i < nd; ++i) {
          const int d = dst_rank(w0, w1, w2, w3, i);
          const int64_t r = (int64_t)d * a.ntok + tok;
          const __half_raw hr =
              __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)a.x[r * a.H + h], __NV_E4M3);
          acc = __fmaf_rn(__half2float(__half(hr)), scales[r], acc);
        }
        out[h] = (uint16_t)f32_to_bf16_bits(acc);
      }
    }
  }
}

// One scale per row: amax = max |x|, scale = amax / 448, inv = 448 / amax
// (each rounded to nearest; 1 and 1 for a zero row), code = E4M3(x * inv),
// nearest even, saturating.  One CTA per row; the row stays in registers
// between the amax pass and the encode pass when it fits (kVec), else it is
// read twice.
template <bool kVec>
__global__ void __launch_bounds__(256) quantize_e4m3_rows_kernel(const uint16_t* __restrict__ in,
                                                                 uint8_t* __restrict__ out,
                                                                 float* __restrict__ scales,
                                                                 int64_t rows, int hidden) {
  constexpr int kMaxV = 4;            // 16-byte vectors per thread held in registers
  __shared__ float s_amax[8];
  __shared__ float s_scale, s_inv;
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const uint16_t* x = in + r * hidden;
    float amax = 0.0f;
    uint4 v[kMaxV];
    if (kVec) {
#pragma unroll
      for (int i = 0; i < kMaxV; ++i) {
        const int c = threadIdx.x + i * 256;
        if (c * 8 < hidden) {
          v[i] = reinterpret_cast<const uint4*>(x)[c];
          const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[q] & 0xFFFFu)));
            amax = fmaxf(amax, fabsf(bf16_bits_to_f32(w[q] >> 16)));
          }
        }
      }
    } else {
      for (int h = threadIdx.x; h < hidden; h += 256)
        amax = fmaxf(amax, fabsf(bf16_bits_to_f32(x[h])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) s_amax[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = 0.0f;
      for (int i = 0; i < 8; ++i) m = fmaxf(m, s_amax[i]);
      s_scale = m > 0.0f ? __fdiv_rn(m, 448.0f) : 1.0f;
      s_inv = m > 0.0f ? __fdiv_rn(448.0f, m) : 1.0f;
      scales[r] = s_scale;
    }
    __syncthreads();
    const float inv = s_inv;
    uint8_t* o = out + r * hidden;
    if (kVec) {
#pragma unroll
      for (int i = 0; i < kMaxV; ++i) {
        const int c = threadIdx.x + i * 256;
        if (c * 8 < hidden) {
          const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
          uint32_t pk[2] = {0u, 0u};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = make_float2(__fmul_rn(bf16_bits_to_f32(w[q] & 0xFFFFu), inv),
                                         __fmul_rn(bf16_bits_to_f32(w[q] >> 16), inv));
            const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
            pk[q >> 1] |= pair << (16 * (q & 1));
          }
          reinterpret_cast<uint2*>(o)[c] = make_uint2(pk[0], pk[1]);
        }
      }
    } else {
      for (int h = threadIdx.x; h < hidden; h += 256)
        o[h] = (uint8_t)__nv_cvt_float_to_fp8(__fmul_rn(bf16_bits_to_f32(x[h]), inv),
                                              __NV_SATFINITE, __NV_E4M3);
    }
    __syncthreads();   // s_amax / s_inv are rewritten for the next row
  }
}

// bf16 -> E4M3, round to nearest even, saturating (satfinite).
__global__ void quantize_e4m3_kernel(const uint16_t* __restrict__ in, uint8_t* __restrict__ out,
                                     int64_t n, bool vec) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  int64_t n_vec = 0;
  if (vec) {
    n_vec = n / 8;
    for (int64_t i = tid; i < n_vec; i += stride) {
      const uint4 v = reinterpret_cast<const uint4*>(in)[i];
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[2] = {0u, 0u};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = make_float2(bf16_bits_to_f32(w[q] & 0xFFFFu), bf16_bits_to_f32(w[q] >> 16));
        const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);
        o[q >> 1] |= pair << (16 * (q & 1));
      }
      reinterpret_cast<uint2*>(out)[i] = make_uint2(o[0], o[1]);
    }
    n_vec *= 8;
  }
  for (int64_t i = n_vec + tid; i < n; i += stride)
    out[i] = (uint8_t)__nv_cvt_float_to_fp8(bf16_bits_to_f32(in[i]), __NV_SATFINITE, __NV_E4M3);
}

// Failure-detection probe: waits on a barrier whose byte count never arrives,
// with a bounded wait; on expiry it sets the error word and returns.
__global__ void wait_timeout_probe_kernel(uint32_t* err, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_addr(&bar);
  mbar_init(b, 1);
  mbar_init_fence();
  mbar_arrive_expect_tx(b, 16);   // no copy will ever complete these 16 bytes
  if (!mbar_wait_bounded(b, 0, limit_ns)) atomicOr(err, kErrWaitTimeout);
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, bool fp8, bool vec, bool pipe, int threads,
                           int grid, cudaStream_t stream, bool pdl, bool tight) {
  const dim3 g(grid), b(threads);
  const float* no_scales = nullptr;
  if (vec && pipe) {
    if (fp8) return launch_kernel(combine_pipe_kernel<kCombineFp8>, g, b, 0, stream, pdl, a,
                                  no_scales);
    return launch_kernel(combine_pipe_kernel<kCombineBf16>, g, b, 0, stream, pdl, a, no_scales);
  }
  if (vec) {
    if (fp8) return launch_kernel(combine_vec_kernel<true>, g, b, 0, stream, pdl, a);
    if (tight && threads == 128)
      return launch_kernel(combine_vec_kernel<false, 128, 7>, g, b, 0, stream, pdl, a);
    return launch_kernel(combine_vec_kernel<false>, g, b, 0, stream, pdl, a);
  }
  if (fp8) return launch_kernel(combine_scalar_kernel<true>, g, b, 0, stream, pdl, a);
  return launch_kernel(combine_scalar_kernel<false>, g, b, 0, stream, pdl, a);
}

cudaError_t launch_combine_staged(const CombineArgs& a, int mode, const float* scales,
                                  int grid, int ctas_per_sm, int max_smem, cudaStream_t stream,
                                  bool pdl) {
  constexpr int NCW = 8;
  const int rows = 8;
  const int stage_bytes = rows * kStageChunk;
  // shared memory per CTA when `ctas_per_sm` share an SM (1 KB per CTA is
  // reserved; 1 KB covers the static arrays)
  const int per_cta = std::min(max_smem, 228 * 1024 / std::max(1, ctas_per_sm) - 1024) - 1024;
  const int stages = std::min(kCombineMaxStages, per_cta / stage_bytes);
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = (size_t)stages * stage_bytes;
  const dim3 g(grid), b(32 * (NCW + 1));
  cudaError_t e;
  switch (mode) {
    case kCombineBf16:
      e = cudaFuncSetAttribute(combine_staged_kernel<kCombineBf16, NCW>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      return launch_kernel(combine_staged_kernel<kCombineBf16, NCW>, g, b, smem, stream, pdl, a,
                           scales, stages, rows);
    case kCombineFp8:
      e = cudaFuncSetAttribute(combine_staged_kernel<kCombineFp8, NCW>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      return launch_kernel(combine_staged_kernel<kCombineFp8, NCW>, g, b, smem, stream, pdl, a,
                           scales, stages, rows);
    default:
      e = cudaFuncSetAttribute(combine_staged_kernel<kCombineFp8Scaled, NCW>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      return launch_kernel(combine_staged_kernel<kCombineFp8Scaled, NCW>, g, b, smem, stream, pdl,
                           a, scales, stages, rows);
  }
}

cudaError_t launch_combine_scaled(const CombineArgs& a, const float* scales, bool vec, bool pipe,
                                  int threads, int grid, cudaStream_t stream, bool pdl) {
  const dim3 g(grid), b(threads);
  if (vec && pipe)
    return launch_kernel(combine_pipe_kernel<kCombineFp8Scaled>, g, b, 0, stream, pdl, a, scales);
  if (vec) return launch_kernel(combine_scaled_kernel<true>, g, b, 0, stream, pdl, a, scales);
  return launch_kernel(combine_scaled_kernel<false>, g, b, 0, stream, pdl, a, scales);
}

cudaError_t launch_quantize_e4m3_rows(const uint16_t* in, uint8_t* out, float* scales,
                                      int64_t rows, int hidden, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const bool vec = hidden % 8 == 0 && hidden <= 4 * 256 * 8 &&
                   reinterpret_cast<uintptr_t>(in) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out) % 8 == 0;
  const int grid = (int)std::min<int64_t>(rows, 148 * 8);
  if (vec)
    quantize_e4m3_rows_kernel<true><<<grid, 256, 0, stream>>>(in, out, scales, rows, hidden);
  else
    quantize_e4m3_rows_kernel<false><<<grid, 256, 0, stream>>>(in, out, scales, rows, hidden);
  return cudaGetLastError();
}

cudaError_t launch_combine_experts(const CombineExpertsArgs& a, bool vec, bool pipe, int threads,
                                   int grid, cudaStream_t stream, bool pdl) {
  const dim3 g(grid), b(threads);
  if (vec && pipe) return launch_kernel(combine_experts_pipe_kernel, g, b, 0, stream, pdl, a);
  if (vec) return launch_kernel(combine_experts_vec_kernel, g, b, 0, stream, pdl, a);
  return launch_kernel(combine_experts_any_kernel, g, b, 0, stream, pdl, a);
}

cudaError_t launch_combine_experts_staged(const CombineExpertsArgs& a, int grid, int ctas_per_sm,
                                          int max_smem, cudaStream_t stream, bool pdl) {
  constexpr int NCW = 8;
  const int stage_bytes = 8 * kStageChunk;
  const int per_cta = std::min(max_smem, 228 * 1024 / std::max(1, ctas_per_sm) - 1024) - 1024;
  const int stages = std::min(kCombineMaxStages, per_cta / stage_bytes);
  if (stages < 2) return cudaErrorInvalidValue;
  const size_t smem = (size_t)stages * stage_bytes;
  cudaError_t e = cudaFuncSetAttribute(combine_experts_staged_kernel<NCW>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(combine_experts_staged_kernel<NCW>, dim3(grid), dim3(32 * (NCW + 1)), smem,
                       stream, pdl, a, stages);
}

template <int C>
cudaError_t launch_fp8_cluster(const CombineExpertsArgs& a, int clusters, int threads,
                               cudaStream_t stream, bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * C);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, combine_experts_fp8_cluster_kernel<C>, a);
}

cudaError_t launch_combine_experts_fp8_cluster(const CombineExpertsArgs& a, int cluster,
                                               int threads, int clusters, cudaStream_t stream,
                                               bool pdl) {
  switch (cluster) {
    case 1: return launch_fp8_cluster<1>(a, clusters, threads, stream, pdl);
    case 2: return launch_fp8_cluster<2>(a, clusters, threads, stream, pdl);
    case 4: return launch_fp8_cluster<4>(a, clusters, threads, stream, pdl);
    case 8: return launch_fp8_cluster<8>(a, clusters, threads, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

template <int C>
cudaError_t launch_fp8_split(const CombineExpertsArgs& a, int clusters, int threads, int cols,
                             size_t smem, cudaStream_t stream, bool pdl) {
  cudaError_t e = cudaFuncSetAttribute(combine_experts_fp8_split_kernel<C>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(clusters * C);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  if (C > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = C;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, combine_experts_fp8_split_kernel<C>, a, cols);
}

cudaError_t launch_combine_experts_fp8_split(const CombineExpertsArgs& a, int cluster, int threads,
                                             int cols, int clusters, size_t smem,
                                             cudaStream_t stream, bool pdl) {
  switch (cluster) {
    case 1: return launch_fp8_split<1>(a, clusters, threads, cols, smem, stream, pdl);
    case 2: return launch_fp8_split<2>(a, clusters, threads, cols, smem, stream, pdl);
    case 4: return launch_fp8_split<4>(a, clusters, threads, cols, smem, stream, pdl);
    case 8: return launch_fp8_split<8>(a, clusters, threads, cols, smem, stream, pdl);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_combine_experts_fp8(const CombineExpertsArgs& a, bool smem_rows, int threads,
                                       int grid, size_t smem, cudaStream_t stream, bool pdl) {
  const dim3 g(grid), b(threads);
  if (smem_rows) {
    cudaError_t e = cudaFuncSetAttribute(combine_experts_fp8_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_kernel(combine_experts_fp8_kernel, g, b, smem, stream, pdl, a);
  }
  return launch_kernel(combine_experts_fp8_any_kernel, g, b, 0, stream, pdl, a);
}

cudaError_t launch_quantize_e4m3(const uint16_t* in, uint8_t* out, int64_t n,
                                 cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  const bool vec = (reinterpret_cast<uintptr_t>(in) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) % 8 == 0);
  const int threads = 256;
  const int64_t work = vec ? (n / 8 + 1) : n;
  const int grid = (int)std::min<int64_t>((work + threads - 1) / threads, 148 * 16);
  quantize_e4m3_kernel<<<grid, threads, 0, stream>>>(in, out, n, vec);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_probe(uint32_t* err, unsigned long long limit_ns,
                                      cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(err, limit_ns);
  return cudaGetLastError();
}

}  // namespace ep_a2a
