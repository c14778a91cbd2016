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
constexpr int kRouterUnroll = 8;
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
  if (kSmemW) {  // stage the weights: 8 loads in flight per thread before the stores
    const int n = E * row_vecs;
    constexpr int kBatch = 8;
    for (int i0 = threadIdx.x; i0 < n; i0 += blockDim.x * kBatch) {
      uint4 w[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n) w[u] = __ldg(Wr + i);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int i = i0 + u * blockDim.x;
        if (i < n) s_w[i] = w[u];
      }
    }
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
// in its owner lane, and lane j keeps slot j.  Gates are computed in fp32
// from logit / temperature ([GPT] §2.3, §4.1); with a threshold, a slot whose
// probability is not above it is dropped (index -1, gate 0) and renormalised
// gates divide by the kept slots' sum.
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 8;

__device__ __forceinline__ bool better(float v, int e, float bv, int be) {
  return v > bv || (v == bv && e < be);
}

template <int kEPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float* __restrict__ L, int T, int E, int k, int score, int renorm,
                      float inv_temp, float min_prob, int32_t* __restrict__ idx,
                      float* __restrict__ gates) {
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
  float my_v = 0.f;  // lane j < k: logit of slot j
  int my_e = 0;      // lane j < k: expert of slot j
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
      if (lane == j) {
        my_v = bv;
        my_e = be;
      }
      if ((be & 31) == lane) taken |= 1u << (be >> 5);
    }
  }
  // Gates.  z = logit / temperature; the largest chosen logit is lane 0's.
  const bool slot = lane < k;
  const bool thr = min_prob > 0.f;
  const float m = __shfl_sync(0xffffffffu, my_v, 0);
  float q;  // unnormalised score of this lane's slot
  if (score == MOE_SCORE_SOFTMAX) {
    q = slot ? expf((my_v - m) * inv_temp) : 0.f;
  } else {
    q = slot ? 1.f / (1.f + expf(-my_v * inv_temp)) : 0.f;
  }
  float prob = q;  // softmax: q / sum over all E; sigmoid: q
  if (score == MOE_SCORE_SOFTMAX && (thr || !renorm)) {
    float part = 0.f;
#pragma unroll
    for (int i = 0; i < kEPL; ++i)
      if (lane + 32 * i < E) part += expf((v[i] - m) * inv_temp);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    prob = q / part;
  }
  const bool keep = slot && (!thr || prob > min_prob);
  float g;
  if (renorm) {
    // softmax: prob_j / sum_kept prob = q_j / sum_kept q; sigmoid: s_j / sum_kept s
    float den = keep ? q : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
    g = (keep && den > 0.f) ? q / den : 0.f;
  } else {
    g = keep ? prob : 0.f;
  }
  if (slot) {
    idx[(size_t)t * k + lane] = keep ? my_e : -1;
    gates[(size_t)t * k + lane] = g;
  }
}

cudaError_t launch_route(const float* L, int T, int E, int k, int score, int renormalize,
                         float temperature, float min_prob, int32_t* idx, float* gates,
                         cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kRouteWarps - 1) / kRouteWarps;
  const int epl = (E + 31) / 32;
  const float inv_temp = 1.0f / temperature;
#define MOE_ROUTE_LAUNCH(N)                                                                    \
  route_topk_kernel<N><<<blocks, kRouteWarps * 32, 0, stream>>>(L, T, E, k, score, renormalize, \
                                                                inv_temp, min_prob, idx, gates)
  if (epl <= 1) MOE_ROUTE_LAUNCH(1);
  else if (epl <= 2) MOE_ROUTE_LAUNCH(2);
  else if (epl <= 4) MOE_ROUTE_LAUNCH(4);
  else if (epl <= 8) MOE_ROUTE_LAUNCH(8);
  else if (epl <= 16) MOE_ROUTE_LAUNCH(16);
  else MOE_ROUTE_LAUNCH(32);
#undef MOE_ROUTE_LAUNCH
  return cudaGetLastError();
}

}  // namespace moe
