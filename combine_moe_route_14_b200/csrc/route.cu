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
// HBM-bound on X (T*d*2 bytes).  A CTA of 8 warps takes 16 tokens, two per
// warp; each lane owns 16-byte slices (8 bf16) of the row and keeps
// kUnroll slices of both tokens in flight before the FMAs.  Router weights
// (E*d*2 bytes) are staged once per CTA in shared memory when they fit,
// else read through L1.  Experts are processed in groups of 8 (one partial
// sum per token and expert per lane), then reduced across the warp.
// ---------------------------------------------------------------------------
constexpr int kRouterWarps = 8;
constexpr int kTokPerWarp = 2;
constexpr int kRouterUnroll = 4;
constexpr int kRouterSmemMax = 96 * 1024;

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

template <bool kSmemW>
__global__ void __launch_bounds__(kRouterWarps * 32)
    router_logits_kernel(const uint4* __restrict__ X, const uint4* __restrict__ Wr, int T,
                         int row_vecs, int E, float* __restrict__ L) {
  extern __shared__ uint4 s_w[];
  if (kSmemW) {
    const int n = E * row_vecs;
    for (int i = threadIdx.x; i < n; i += blockDim.x) s_w[i] = __ldg(Wr + i);
    __syncthreads();
  }
  const uint4* W = kSmemW ? s_w : Wr;
  const int lane = threadIdx.x & 31;
  const int t0 = (blockIdx.x * kRouterWarps + (threadIdx.x >> 5)) * kTokPerWarp;
  if (t0 >= T) return;
  const bool two = t0 + 1 < T;
  const uint4* x0 = X + (size_t)t0 * row_vecs;
  const uint4* x1 = X + (size_t)(two ? t0 + 1 : t0) * row_vecs;
  for (int e0 = 0; e0 < E; e0 += 8) {
    const int ne = min(8, E - e0);
    float acc0[8], acc1[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) acc0[j] = acc1[j] = 0.f;
    for (int c0 = lane; c0 < row_vecs; c0 += 32 * kRouterUnroll) {
      uint4 a[kRouterUnroll], b[kRouterUnroll];
#pragma unroll
      for (int u = 0; u < kRouterUnroll; ++u) {
        const int c = c0 + u * 32;
        if (c < row_vecs) {
          a[u] = ld_stream_v4(x0 + c);
          b[u] = ld_stream_v4(x1 + c);
        }
      }
#pragma unroll
      for (int u = 0; u < kRouterUnroll; ++u) {
        const int c = c0 + u * 32;
        if (c < row_vecs) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (j < ne) {
              const uint4 w = kSmemW ? W[(size_t)(e0 + j) * row_vecs + c]
                                     : __ldg(W + (size_t)(e0 + j) * row_vecs + c);
              acc0[j] = dot8(a[u], w, acc0[j]);
              acc1[j] = dot8(b[u], w, acc1[j]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        acc0[j] += __shfl_xor_sync(0xffffffffu, acc0[j], off);
        acc1[j] += __shfl_xor_sync(0xffffffffu, acc1[j], off);
      }
    }
    // lane j < ne writes expert e0+j of token t0, lane 8+j of token t0+1
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (lane == j && j < ne) L[(size_t)t0 * E + e0 + j] = acc0[j];
      if (two && lane == 8 + j && j < ne) L[(size_t)(t0 + 1) * E + e0 + j] = acc1[j];
    }
  }
}

cudaError_t launch_router_logits(const void* X, const void* Wr, int T, int d, int E, float* L,
                                 cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int per_cta = kRouterWarps * kTokPerWarp;
  const int blocks = (T + per_cta - 1) / per_cta;
  const size_t wbytes = (size_t)E * d * 2;
  const uint4* x = static_cast<const uint4*>(X);
  const uint4* w = static_cast<const uint4*>(Wr);
  if (wbytes <= (size_t)kRouterSmemMax) {
    if (wbytes > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(router_logits_kernel<true>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           kRouterSmemMax);
      if (e != cudaSuccess) return e;
    }
    router_logits_kernel<true><<<blocks, kRouterWarps * 32, wbytes, stream>>>(x, w, T, d / 8, E, L);
  } else {
    router_logits_kernel<false><<<blocks, kRouterWarps * 32, 0, stream>>>(x, w, T, d / 8, E, L);
  }
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
