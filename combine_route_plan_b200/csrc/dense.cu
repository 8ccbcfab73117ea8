// Dense variant of dispatch / combine (vllm.distributed.device_communicators.
// all2all, AgRsAll2AllManager): dispatch as an all-gather (every live rank
// receives every token of every live rank), combine as a reduce-scatter (each
// token's row summed over all live ranks, fp32 in ascending rank order, one
// bf16 rounding).  It keeps the rank-major slot layout src * tpr + t, so both
// variants run on the same arrays and can be compared byte for byte; it needs
// no routing plan.
#include <cuda_bf16.h>

#include <algorithm>
#include <cstring>

#include "ep_a2a_internal.cuh"

#define EP_API extern "C" __attribute__((visibility("default")))

namespace ep_a2a {
namespace {

struct DenseArgs {
  int ep, tpr;
  int64_t ntok;
  int32_t n[kMaxRanks];          // 0 for masked-off ranks
  uint64_t live[kMaskWords];
  // all-gather
  int np;
  const uint8_t* src[kMaxPayloads];
  int64_t rb[kMaxPayloads];
  uint8_t* dst0[kMaxPayloads];   // rank 0's receive array of each payload
  int64_t rank_stride;
  uint32_t vec[kMaxPayloads];
  // reduce-scatter
  const uint16_t* x;             // [ep, ep*tpr, H]
  uint16_t* out;                 // [ep, tpr, H]
  int H;
};

__device__ __forceinline__ bool live_rank(const DenseArgs& a, int r) {
  return (a.live[r >> 6] >> (r & 63)) & 1ull;
}

template <typename T>
__device__ __forceinline__ void gather_row(const DenseArgs& a, int p, int64_t tok, int lane) {
  constexpr int U = 4;
  const int64_t n = a.rb[p] / (int64_t)sizeof(T);
  const T* s = reinterpret_cast<const T*>(a.src[p] + tok * a.rb[p]);
  for (int64_t i0 = lane; i0 < n; i0 += 32 * U) {
    T v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (i0 + u * 32 < n) v[u] = s[i0 + u * 32];
    for (int d = 0; d < a.ep; ++d) {
      if (!live_rank(a, d)) continue;
      T* o = reinterpret_cast<T*>(a.dst0[p] + (int64_t)d * a.rank_stride + tok * a.rb[p]);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + u * 32 < n) o[i0 + u * 32] = v[u];
    }
  }
}

// A warp per token: each payload row is read once and stored to every live rank.
__global__ void __launch_bounds__(256) allgather_kernel(const DenseArgs a) {
  const int lane = threadIdx.x & 31;
  for (int64_t tok = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); tok < a.ntok;
       tok += (int64_t)gridDim.x * 8) {
    const int r = (int)(tok / a.tpr);
    if (tok - (int64_t)r * a.tpr >= a.n[r]) continue;
    for (int p = 0; p < a.np; ++p) {
      switch (a.vec[p]) {
        case 16: gather_row<uint4>(a, p, tok, lane); break;
        case 8: gather_row<uint2>(a, p, tok, lane); break;
        case 4: gather_row<uint32_t>(a, p, tok, lane); break;
        case 2: gather_row<uint16_t>(a, p, tok, lane); break;
        default: gather_row<uint8_t>(a, p, tok, lane); break;
      }
    }
  }
}

// A CTA per token; each thread a 16-byte column vector (kVec) or one element,
// summing the rows of all live ranks (8 loads in flight at a time) in
// ascending rank order.
template <bool kVec>
__global__ void __launch_bounds__(512) reduce_scatter_kernel(const DenseArgs a) {
  const int64_t slots = a.ntok;
  for (int64_t tok = blockIdx.x; tok < a.ntok; tok += gridDim.x) {
    const int r = (int)(tok / a.tpr);
    if (tok - (int64_t)r * a.tpr >= a.n[r]) continue;
    uint16_t* out = a.out + tok * (int64_t)a.H;
    if (kVec) {
      const int nvec = a.H / 8;
      for (int v = threadIdx.x; v < nvec; v += blockDim.x) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
        for (int d0 = 0; d0 < a.ep; d0 += 8) {
          uint4 raw[8];
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (d0 + i < a.ep && live_rank(a, d0 + i))
              raw[i] = ld_stream_v4(a.x + ((int64_t)(d0 + i) * slots + tok) * a.H + (int64_t)v * 8);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (d0 + i >= a.ep || !live_rank(a, d0 + i)) continue;
            const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              acc[2 * q] = __fadd_rn(acc[2 * q], __uint_as_float((w[q] & 0xFFFFu) << 16));
              acc[2 * q + 1] = __fadd_rn(acc[2 * q + 1], __uint_as_float(w[q] & 0xFFFF0000u));
            }
          }
        }
        uint32_t pw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
          pw[q] = *reinterpret_cast<const uint32_t*>(&b);
        }
        reinterpret_cast<uint4*>(out)[v] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
      }
    } else {
      for (int h = threadIdx.x; h < a.H; h += blockDim.x) {
        float acc = 0.0f;
        for (int d = 0; d < a.ep; ++d)
          if (live_rank(a, d))
            acc = __fadd_rn(acc, __uint_as_float((uint32_t)a.x[((int64_t)d * slots + tok) * a.H + h]
                                                 << 16));
        out[h] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
      }
    }
  }
}

bool aligned_to(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

ep_a2a_status fill_ranks(DenseArgs& a, int32_t ep_size, int32_t tpr,
                         const int32_t* local_num_tokens, const uint64_t* active_rank_mask) {
  if (ep_size < 1 || ep_size > kMaxRanks) {
    record_last_error("ep_size outside 1..256");
    return EP_A2A_ERR_UNSUPPORTED;
  }
  if (tpr < 1 || (int64_t)ep_size * tpr > ((int64_t)1 << 30) || !local_num_tokens) {
    record_last_error("tokens_per_rank out of range or local_num_tokens is NULL");
    return EP_A2A_ERR_INVALID_ARG;
  }
  a.ep = ep_size;
  a.tpr = tpr;
  a.ntok = (int64_t)ep_size * tpr;
  for (int w = 0; w < kMaskWords; ++w) a.live[w] = active_rank_mask ? active_rank_mask[w] : ~0ull;
  bool any = false;
  for (int r = 0; r < ep_size; ++r) {
    const bool live = ((a.live[r >> 6] >> (r & 63)) & 1ull) != 0;
    any |= live;
    if (local_num_tokens[r] < 0 || local_num_tokens[r] > tpr) {
      record_last_error("local_num_tokens[r] outside 0..tokens_per_rank");
      return EP_A2A_ERR_INVALID_ARG;
    }
    a.n[r] = live ? local_num_tokens[r] : 0;
  }
  if (!any) {
    record_last_error("active_rank_mask has no active rank");
    return EP_A2A_ERR_INVALID_ARG;
  }
  return EP_A2A_OK;
}

}  // namespace
}  // namespace ep_a2a

using namespace ep_a2a;

EP_API ep_a2a_status ep_a2a_allgather(int32_t ep_size, int32_t tokens_per_rank,
                                      const int32_t* local_num_tokens,
                                      const uint64_t* active_rank_mask,
                                      const void* const* payloads,
                                      const int64_t* payload_row_bytes, int32_t num_payloads,
                                      void* const* recv_payloads, int64_t recv_rank_stride_bytes,
                                      void* stream) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  ep_a2a_status st = fill_ranks(a, ep_size, tokens_per_rank, local_num_tokens, active_rank_mask);
  if (st != EP_A2A_OK) return st;
  if (num_payloads < 0 || num_payloads > kMaxPayloads ||
      (num_payloads > 0 && (!payloads || !payload_row_bytes || !recv_payloads))) {
    record_last_error("payload list is invalid");
    return EP_A2A_ERR_INVALID_ARG;
  }
  a.np = num_payloads;
  a.rank_stride = recv_rank_stride_bytes;
  for (int p = 0; p < num_payloads; ++p) {
    const int64_t rb = payload_row_bytes[p];
    if (rb < 1 || !payloads[p] || !recv_payloads[p] ||
        (ep_size > 1 && recv_rank_stride_bytes < a.ntok * rb)) {
      record_last_error("payload row bytes, pointer or receive stride is invalid");
      return EP_A2A_ERR_INVALID_ARG;
    }
    a.src[p] = static_cast<const uint8_t*>(payloads[p]);
    a.rb[p] = rb;
    a.dst0[p] = static_cast<uint8_t*>(recv_payloads[p]);
    uint32_t v = 1;
    for (uint32_t c : {16u, 8u, 4u, 2u})
      if (rb % c == 0 && aligned_to(a.src[p], c) && aligned_to(a.dst0[p], c) &&
          recv_rank_stride_bytes % c == 0) {
        v = c;
        break;
      }
    a.vec[p] = v;
  }
  if (num_payloads == 0) return EP_A2A_OK;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((a.ntok + 7) / 8, 148 * 32));
  allgather_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_last_error(cudaGetErrorString(e));
    return EP_A2A_ERR_CUDA;
  }
  return EP_A2A_OK;
}

EP_API ep_a2a_status ep_a2a_reduce_scatter(int32_t ep_size, int32_t tokens_per_rank,
                                           int32_t hidden, const int32_t* local_num_tokens,
                                           const uint64_t* active_rank_mask, const void* x,
                                           void* out, void* stream) {
  DenseArgs a;
  std::memset(&a, 0, sizeof(a));
  ep_a2a_status st = fill_ranks(a, ep_size, tokens_per_rank, local_num_tokens, active_rank_mask);
  if (st != EP_A2A_OK) return st;
  if (hidden < 1 || !x || !out) {
    record_last_error("hidden < 1 or NULL buffer");
    return EP_A2A_ERR_INVALID_ARG;
  }
  a.x = static_cast<const uint16_t*>(x);
  a.out = static_cast<uint16_t*>(out);
  a.H = hidden;
  const bool vec = hidden % 8 == 0 && aligned_to(x, 16) && aligned_to(out, 16);
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(a.ntok, 148 * 128));
  if (vec)
    reduce_scatter_kernel<true><<<grid, 64, 0, (cudaStream_t)stream>>>(a);
  else
    reduce_scatter_kernel<false><<<grid, 64, 0, (cudaStream_t)stream>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    record_last_error(cudaGetErrorString(e));
    return EP_A2A_ERR_CUDA;
  }
  return EP_A2A_OK;
}
