// Router: logits (router linear) and score / top-k / gates.
//
// GPT-4 "2%" article §4.1 (router code: logits = router_proj(h), softmax,
// topk), §2.3 (softmax then top-k); ThunderEP PCIe blog §1.1 (top-1 / top-2
// routing), §2.1 (top-k indices and gates drive the combine).
//
// Both kernels are bandwidth / latency bound: the router linear streams X
// once (T*d*2 bytes) and the top-k reads T*E*4 bytes of logits.
#include <cfloat>

#include "common.cuh"
#include "launch.h"

namespace moe {

// ---------------------------------------------------------------------------
// router linear: L[t, e] = sum_c X[t, c] * Wr[e, c]   (fp32 accumulate)
//
// One warp handles kTokPerWarp consecutive tokens and experts in groups of 8:
// each lane owns 8 consecutive bf16 of the row per step (16-byte loads), keeps
// kTokPerWarp x 8 fp32 partial sums, and the warp reduces them at the end.
// Router weights are small (E*d*2 bytes) and stay in L1/L2.
// ---------------------------------------------------------------------------
constexpr int kTokPerWarp = 4;
constexpr int kRouterWarps = 8;

__device__ __forceinline__ float dot8(const uint4& a, const uint4& b, float acc) {
  acc = fmaf(bf16_lo(a.x), bf16_lo(b.x), acc);
  acc = fmaf(bf16_hi(a.x), bf16_hi(b.x), acc);
  acc = fmaf(bf16_lo(a.y), bf16_lo(b.y), acc);
  acc = fmaf(bf16_hi(a.y), bf16_hi(b.y), acc);
  acc = fmaf(bf16_lo(a.z), bf16_lo(b.z), acc);
  acc = fmaf(bf16_hi(a.z), bf16_hi(b.z), acc);
  acc = fmaf(bf16_lo(a.w), bf16_lo(b.w), acc);
  acc = fmaf(bf16_hi(a.w), bf16_hi(b.w), acc);
  return acc;
}

__global__ void __launch_bounds__(kRouterWarps * 32)
    router_logits_kernel(const uint4* __restrict__ X, const uint4* __restrict__ Wr, int T,
                         int row_vecs, int E, float* __restrict__ L) {
  const int warp = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int t0 = warp * kTokPerWarp;
  if (t0 >= T) return;
  const int ntok = min(kTokPerWarp, T - t0);
  for (int e0 = 0; e0 < E; e0 += 8) {
    const int ne = min(8, E - e0);
    float acc[kTokPerWarp][8];
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int c = lane; c < row_vecs; c += 32) {
      uint4 xv[kTokPerWarp];
#pragma unroll
      for (int i = 0; i < kTokPerWarp; ++i)
        xv[i] = (i < ntok) ? ld_stream_v4(X + (size_t)(t0 + i) * row_vecs + c) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < ne) {
          const uint4 wv = __ldg(Wr + (size_t)(e0 + j) * row_vecs + c);
#pragma unroll
          for (int i = 0; i < kTokPerWarp; ++i) acc[i][j] = dot8(xv[i], wv, acc[i][j]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float v = acc[i][j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        acc[i][j] = v;
      }
    if (lane == 0) {
      for (int i = 0; i < ntok; ++i)
        for (int j = 0; j < ne; ++j) L[(size_t)(t0 + i) * E + e0 + j] = acc[i][j];
    }
  }
}

cudaError_t launch_router_logits(const void* X, const void* Wr, int T, int d, int E, float* L,
                                 cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int warps = (T + kTokPerWarp - 1) / kTokPerWarp;
  const int blocks = (warps + kRouterWarps - 1) / kRouterWarps;
  router_logits_kernel<<<blocks, kRouterWarps * 32, 0, stream>>>(
      static_cast<const uint4*>(X), static_cast<const uint4*>(Wr), T, d / 8, E, L);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// top-k + gates: one warp per token.
//
// Lane l holds logits of experts l, l+32, l+64, ... (kEPL of them).  k rounds
// of a warp-wide argmax pick the experts in descending order; the comparison
// (value greater, or equal value and lower id) breaks ties toward the lower
// expert id, and -0 == +0 counts as a tie.  The chosen expert is marked taken
// in its owner lane.  Gates are computed in fp32 from the chosen logits.
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 8;

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <int kEPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float* __restrict__ L, int T, int E, int k, int score, int renorm,
                      int32_t* __restrict__ idx, float* __restrict__ gates) {
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const float* row = L + (size_t)t * E;
  float v[kEPL];
#pragma unroll
  for (int i = 0; i < kEPL; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(row + e) : -FLT_MAX;
  }
  uint32_t taken = 0;
  float selv[kMaxTopK];
  int sele[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    selv[j] = 0.f;
    sele[j] = 0;
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k) {
      float bv = -FLT_MAX;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kEPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !((taken >> i) & 1u) && better(v[i], e, bv, be)) {
          bv = v[i];
          be = e;
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (better(ov, oe, bv, be)) {
          bv = ov;
          be = oe;
        }
      }
      selv[j] = bv;
      sele[j] = be;
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
    }
  }
  // gates
  const float m = selv[0];
  float denom = 0.f;
  if (score == MOE_SCORE_SOFTMAX) {
    if (renorm) {
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j)
        if (j < k) denom += expf(selv[j] - m);
    } else {
      float part = 0.f;
#pragma unroll
      for (int i = 0; i < kEPL; ++i)
        if (lane + 32 * i < E) part += expf(v[i] - m);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      denom = part;
    }
  } else {
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < k) denom += 1.f / (1.f + expf(-selv[j]));
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k && lane == j) {
      float g;
      if (score == MOE_SCORE_SOFTMAX) {
        g = expf(selv[j] - m) / denom;
      } else {
        const float s = 1.f / (1.f + expf(-selv[j]));
        g = renorm ? s / denom : s;
      }
      idx[(size_t)t * k + j] = sele[j];
      gates[(size_t)t * k + j] = g;
    }
  }
}

cudaError_t launch_route(const float* L, int T, int E, int k, int score, int renormalize,
                         int32_t* idx, float* gates, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kRouteWarps - 1) / kRouteWarps;
  const int epl = (E + 31) / 32;
#define MOE_ROUTE_CASE(N)                                                                    \
  case N:                                                                                    \
    route_topk_kernel<N><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score,         \
                                                                  renormalize, idx, gates); \
    break;
  switch (epl) {
    MOE_ROUTE_CASE(1)
    MOE_ROUTE_CASE(2)
    MOE_ROUTE_CASE(4)
    MOE_ROUTE_CASE(8)
    MOE_ROUTE_CASE(16)
    MOE_ROUTE_CASE(32)
    default:
      if (epl <= 4) {
        route_topk_kernel<4><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score,
                                                                      renormalize, idx, gates);
      } else if (epl <= 8) {
        route_topk_kernel<8><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score,
                                                                      renormalize, idx, gates);
      } else if (epl <= 16) {
        route_topk_kernel<16><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score,
                                                                       renormalize, idx, gates);
      } else {
        route_topk_kernel<32><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score,
                                                                       renormalize, idx, gates);
      }
  }
#undef MOE_ROUTE_CASE
  return cudaGetLastError();
}

}  // namespace moe
