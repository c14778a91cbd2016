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
// A GEMM with N = E (8 for the Mixtral shape): tensor-core mma.sync tiles of
// 16 tokens x 8 experts x 16 K (bf16 in, fp32 accumulate) fit it exactly,
// and it is bound by streaming X (T*d*2 bytes) from HBM.  A CTA of 8 warps
// takes 16 tokens; the warps split K into 64-column chunks (warp w takes
// chunks w, w+8, ...) and their partial 16 x E tiles are summed in shared
// memory in warp order (deterministic).
//
// Operand loads use a K permutation shared by both operands: in a 64-column
// chunk, the thread with q = lane % 4 loads columns [16q, 16q+16) of its two
// token rows (lane / 4 and lane / 4 + 8) and of expert row lane / 4, as two
// 16-byte vectors each (the four threads of a row read 128 contiguous
// bytes).  MMA m of the chunk takes words 2m, 2m+1 of each: logical k-pair
// (2q, 2q+1) is column 16q + 4m + {0, 1} and (2q+8, 2q+9) is 16q + 4m + {2, 3}
// for A and B alike, so the 4 MMAs cover the chunk's 64 columns exactly once.
// More than 64 experts are processed in groups of 8 n-tiles, re-reading X.
// The X vectors of a warp's next chunk are loaded while the current chunk's
// MMAs run (a warp walks nchunks / 8 chunks; for a handful of tokens, e.g.
// decode, those loads would otherwise be serial round trips).
// ---------------------------------------------------------------------------
constexpr int kRouterWarps = 8;
constexpr int kRouterTok = 16;     // tokens per CTA (the MMA's M)
constexpr int kRouterGroup = 8;    // n-tiles of 8 experts per pass

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 16 bytes at p (8 bf16) when the 8 values at column `col` exist, else zeros
__device__ __forceinline__ uint4 ld_row_v4(const uint4* p, bool ok) {
  return ok ? ld_stream_v4(p) : make_uint4(0u, 0u, 0u, 0u);
}

__global__ void __launch_bounds__(kRouterWarps * 32)
    router_logits_kernel(const uint4* __restrict__ X, const uint4* __restrict__ Wr, int T,
                         int row_vecs, int E, float* __restrict__ L) {
  __shared__ float s_part[kRouterWarps][kRouterGroup][kRouterTok * 8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = lane >> 2, q = lane & 3;
  const int t0 = blockIdx.x * kRouterTok;
  const bool okA0 = t0 + r0 < T, okA1 = t0 + r0 + 8 < T;
  const uint4* xa0 = X + (size_t)(okA0 ? t0 + r0 : 0) * row_vecs;
  const uint4* xa1 = X + (size_t)(okA1 ? t0 + r0 + 8 : 0) * row_vecs;
  const int nchunks = (row_vecs + 7) / 8;  // 64 columns = 8 vectors per chunk
  const int ntiles = (E + 7) / 8;
  for (int g0 = 0; g0 < ntiles; g0 += kRouterGroup) {
    const int G = min(kRouterGroup, ntiles - g0);
    float acc[kRouterGroup][4];
#pragma unroll
    for (int j = 0; j < kRouterGroup; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
    uint4 n00, n01, n10, n11;  // the next chunk's X vectors
    {
      const int v = warp * 8 + 2 * q;
      const bool ok0 = warp < nchunks && v < row_vecs, ok1 = warp < nchunks && v + 1 < row_vecs;
      n00 = ld_row_v4(xa0 + v, okA0 && ok0);
      n01 = ld_row_v4(xa0 + v + 1, okA0 && ok1);
      n10 = ld_row_v4(xa1 + v, okA1 && ok0);
      n11 = ld_row_v4(xa1 + v + 1, okA1 && ok1);
    }
    for (int c = warp; c < nchunks; c += kRouterWarps) {
      const int v = c * 8 + 2 * q;  // this thread's first vector of the chunk
      const bool ok0 = v < row_vecs, ok1 = v + 1 < row_vecs;
      const uint4 x00 = n00, x01 = n01, x10 = n10, x11 = n11;
      {
        const int cn = c + kRouterWarps, vn = cn * 8 + 2 * q;
        const bool m0 = cn < nchunks && vn < row_vecs, m1 = cn < nchunks && vn + 1 < row_vecs;
        n00 = ld_row_v4(xa0 + vn, okA0 && m0);
        n01 = ld_row_v4(xa0 + vn + 1, okA0 && m1);
        n10 = ld_row_v4(xa1 + vn, okA1 && m0);
        n11 = ld_row_v4(xa1 + vn + 1, okA1 && m1);
      }
      const uint32_t A0[8] = {x00.x, x00.y, x00.z, x00.w, x01.x, x01.y, x01.z, x01.w};
      const uint32_t A1[8] = {x10.x, x10.y, x10.z, x10.w, x11.x, x11.y, x11.z, x11.w};
#pragma unroll
      for (int j = 0; j < kRouterGroup; ++j) {
        if (j < G) {
          const int e = (g0 + j) * 8 + r0;
          const bool okB = e < E;
          const uint4* wr = Wr + (size_t)(okB ? e : 0) * row_vecs;
          const uint4 w0 = okB && ok0 ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
          const uint4 w1 = okB && ok1 ? __ldg(wr + v + 1) : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t B[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int m = 0; m < 4; ++m)
            mma_bf16_16816(acc[j], A0[2 * m], A1[2 * m], A0[2 * m + 1], A1[2 * m + 1], B[2 * m],
                           B[2 * m + 1]);
        }
      }
    }
    // partial tile of this warp: c0,c1 = (row r0, experts 2q, 2q+1), c2,c3 = row r0 + 8
#pragma unroll
    for (int j = 0; j < kRouterGroup; ++j) {
      if (j < G) {
        float* p = s_part[warp][j];
        p[r0 * 8 + 2 * q] = acc[j][0];
        p[r0 * 8 + 2 * q + 1] = acc[j][1];
        p[(r0 + 8) * 8 + 2 * q] = acc[j][2];
        p[(r0 + 8) * 8 + 2 * q + 1] = acc[j][3];
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * kRouterTok * 8; i += blockDim.x) {
      const int j = i / (kRouterTok * 8), rc = i % (kRouterTok * 8);
      const int r = rc / 8, e = (g0 + j) * 8 + rc % 8;
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kRouterWarps; ++w) sum += s_part[w][j][rc];
      if (t0 + r < T && e < E) L[(size_t)(t0 + r) * E + e] = sum;
    }
    __syncthreads();
  }
}

cudaError_t launch_router_logits(const void* X, const void* Wr, int T, int d, int E, float* L,
                                 cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kRouterTok - 1) / kRouterTok;
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
