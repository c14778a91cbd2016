// FP8 (E4M3) quantisation: per-tensor dynamic scales, the quantising
// dispatch, and the one-time per-expert weight quantisation.
//
// ThunderEP PCIe blog §3.3 and §5.2: the activations a dispatch moves are
// cast to FP8 with one dynamic per-tensor scale before the transfer and
// cast back after it, halving the bytes; hardware with FP8 tensor cores
// computes on them directly.  Here the dispatched token rows are written as
// E4M3 codes (one byte per value instead of two) and GEMM-1 consumes them.
//
// Arithmetic (identical on every path, so the codes are reproducible):
//   amax  = max |x| over the tensor (exact: a maximum of bf16 magnitudes),
//   inv   = 448 / amax          (fp32, round to nearest; 1 when amax == 0),
//   code  = E4M3(x * inv)       (fp32 product, round to nearest even,
//                                magnitudes past 448 saturate to 448),
//   scale = amax / 448          (fp32; 1 when amax == 0), so x ~= scale * code.
// Inputs must be finite.
//
// All kernels are HBM streams: 16-byte bf16 loads, 8-byte code stores, grids
// a multiple of the SM count.
#include "common.cuh"
#include "launch.h"

namespace moe {

constexpr int kQThreads = 256;
constexpr int kQUnroll = 4;  // 16-byte loads in flight per thread
constexpr float kE4M3Max = 448.0f;

__device__ __forceinline__ float inv_scale_of(float amax) {
  return amax > 0.f ? __fdiv_rn(kE4M3Max, amax) : 1.0f;
}
__device__ __forceinline__ float scale_of(float amax) {
  return amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.0f;
}

// 8 bf16 values -> 8 E4M3 codes (value j in byte j).
__device__ __forceinline__ uint2 quant8(uint4 v, float inv) {
  uint2 o;
  o.x = cvt_e4m3x2(__fmul_rn(bf16_lo(v.x), inv), __fmul_rn(bf16_hi(v.x), inv)) |
        (cvt_e4m3x2(__fmul_rn(bf16_lo(v.y), inv), __fmul_rn(bf16_hi(v.y), inv)) << 16);
  o.y = cvt_e4m3x2(__fmul_rn(bf16_lo(v.z), inv), __fmul_rn(bf16_hi(v.z), inv)) |
        (cvt_e4m3x2(__fmul_rn(bf16_lo(v.w), inv), __fmul_rn(bf16_hi(v.w), inv)) << 16);
  return o;
}

// Per-group absolute maximum of bf16 values.  Group g is the `vecs` 16-byte
// vectors starting at X + g * vecs (blockIdx.y = g).  Magnitudes are compared
// as bf16 bit patterns with the sign cleared (the order of non-negative
// floats), two at a time; the block's maximum is merged into amax[g] (which
// the launcher zeroes) with an integer atomicMax on its fp32 bits.
__global__ void __launch_bounds__(kQThreads)
    amax_kernel(const uint4* __restrict__ X, size_t vecs, uint32_t* amax_bits) {
  pdl_wait_and_release();
  const uint4* p = X + (size_t)blockIdx.y * vecs;
  uint32_t m2 = 0;  // two 16-bit magnitudes
  const size_t stride = (size_t)gridDim.x * kQThreads;
  size_t i = (size_t)blockIdx.x * kQThreads + threadIdx.x;
  for (; i + (kQUnroll - 1) * stride < vecs; i += kQUnroll * stride) {
    uint4 v[kQUnroll];
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) v[u] = ld_stream_v4(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) {
      m2 = __vmaxu2(m2, v[u].x & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].y & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].z & 0x7FFF7FFFu);
      m2 = __vmaxu2(m2, v[u].w & 0x7FFF7FFFu);
    }
  }
  for (; i < vecs; i += stride) {
    const uint4 v = ld_stream_v4(p + i);
    m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.w & 0x7FFF7FFFu);
  }
  uint32_t m = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  __shared__ uint32_t s_m[kQThreads / 32];
  if ((threadIdx.x & 31) == 0) s_m[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kQThreads / 32 ? s_m[threadIdx.x] : 0u;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (threadIdx.x == 0 && m != 0u) atomicMax(amax_bits + blockIdx.y, m << 16);  // bf16 -> fp32 bits
  }
}

// Wq[g] = E4M3(W[g] * inv(amax[g])) for each group g = blockIdx.y; when
// scale_out is given (not aliasing amax), CTA (0, g) writes its scale there.
__global__ void __launch_bounds__(kQThreads)
    quantize_kernel(const uint4* __restrict__ W, size_t vecs, const float* __restrict__ amax,
                    uint2* __restrict__ Wq, float* scale_out) {
  pdl_wait_and_release();
  const float inv = inv_scale_of(amax[blockIdx.y]);
  if (scale_out && blockIdx.x == 0 && threadIdx.x == 0)
    scale_out[blockIdx.y] = scale_of(amax[blockIdx.y]);
  const uint4* p = W + (size_t)blockIdx.y * vecs;
  uint2* q = Wq + (size_t)blockIdx.y * vecs;
  const size_t stride = (size_t)gridDim.x * kQThreads;
  size_t i = (size_t)blockIdx.x * kQThreads + threadIdx.x;
  for (; i + (kQUnroll - 1) * stride < vecs; i += kQUnroll * stride) {
    uint4 v[kQUnroll];
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) v[u] = ld_stream_v4(p + i + u * stride);
#pragma unroll
    for (int u = 0; u < kQUnroll; ++u) q[i + u * stride] = quant8(v[u], inv);
  }
  for (; i < vecs; i += stride) q[i] = quant8(ld_stream_v4(p + i), inv);
}

// amax -> dequantisation scale, in place.
__global__ void scale_finalize_kernel(float* s, int n) {
  pdl_wait_and_release();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) s[i] = scale_of(s[i]);
}

constexpr int kDispWarps = 8;
constexpr int kDispUnroll = 8;

// Xeq[r, :] = E4M3(X[src_of[r] / k, :] * inv(amax)), amax = x_scale[1] (set by
// amax_kernel before this launch); CTA 0 writes the scale to x_scale[0].
// src_of == -1 marks an unused row (dropped slots) and is skipped.
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_fp8_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ src_of, int R,
                        int k, int row_vecs, float* x_scale, uint2* __restrict__ Xeq,
                        uint32_t* status) {
  pdl_wait_and_release();
  const float amax = x_scale[1];
  const float inv = inv_scale_of(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) x_scale[0] = scale_of(amax);
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kDispWarps;
  for (int r = blockIdx.x * kDispWarps + (threadIdx.x >> 5); r < R; r += nwarps) {
    const int s = __ldg(src_of + r);
    if (s < 0 || s >= R) {
      if (s != -1 && lane == 0) flag_error(status, MOE_DEV_BAD_ROW);
      continue;
    }
    const uint4* src = X + (size_t)(s / k) * row_vecs;
    uint2* dst = Xeq + (size_t)r * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kDispUnroll) {
      uint4 v[kDispUnroll];
#pragma unroll
      for (int u = 0; u < kDispUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) v[u] = ld_stream_v4(src + c);
      }
#pragma unroll
      for (int u = 0; u < kDispUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) dst[c] = quant8(v[u], inv);
      }
    }
  }
}

// Token-ordered form: Xeq[row_of[t*k + j], :] = E4M3(X[t, :] * inv(amax)) for
// each kept slot j (each token read and quantised once, written k times).
__global__ void __launch_bounds__(kDispWarps * 32)
    dispatch_fp8_rows_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ row_of,
                             int T, int k, int row_vecs, float* x_scale, uint2* __restrict__ Xeq,
                             uint32_t* status) {
  pdl_wait_and_release();
  const float amax = x_scale[1];
  const float inv = inv_scale_of(amax);
  if (blockIdx.x == 0 && threadIdx.x == 0) x_scale[0] = scale_of(amax);
  const int R = T * k;
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kDispWarps;
  for (int t = blockIdx.x * kDispWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    int my_row = -1;
    if (lane < k) {
      my_row = __ldg(row_of + (size_t)t * k + lane);
      if (my_row < -1 || my_row >= R) {
        flag_error(status, MOE_DEV_BAD_ROW);
        my_row = -1;
      }
    }
    const uint32_t live = __ballot_sync(0xffffffffu, lane < k && my_row >= 0);
    if (!live) continue;
    const uint4* src = X + (size_t)t * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kDispUnroll) {
      uint2 q[kDispUnroll];
#pragma unroll
      for (int u = 0; u < kDispUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) q[u] = quant8(ld_stream_v4(src + c), inv);
      }
      for (uint32_t m = live; m; m &= m - 1) {
        const int r = __shfl_sync(0xffffffffu, my_row, __ffs(m) - 1);
        uint2* dst = Xeq + (size_t)r * row_vecs;
#pragma unroll
        for (int u = 0; u < kDispUnroll; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < row_vecs) dst[c] = q[u];
        }
      }
    }
  }
}

static int stream_grid(size_t vecs, int groups, const DeviceInfo& dev) {
  const size_t need = (vecs + (size_t)kQThreads * kQUnroll - 1) / ((size_t)kQThreads * kQUnroll);
  const int cap = (dev.sm_count * 8 + groups - 1) / groups;  // ~8 CTAs of 256 threads per SM
  const size_t g = need < (size_t)cap ? need : (size_t)cap;
  return g < 1 ? 1 : (int)g;
}

static cudaError_t launch_amax(const void* X, size_t vecs, int groups, float* amax,
                               const DeviceInfo& dev, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(amax, 0, (size_t)groups * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  if (vecs == 0) return cudaSuccess;
  launch_kernel(amax_kernel, dim3(stream_grid(vecs, groups, dev), groups), dim3(kQThreads), 0, stream,
      static_cast<const uint4*>(X), vecs, reinterpret_cast<uint32_t*>(amax));
  return cudaGetLastError();
}

cudaError_t launch_quantize_experts(const void* W, int E, int64_t per_expert, void* Wq,
                                    float* scales, const DeviceInfo& dev, cudaStream_t stream) {
  const size_t vecs = (size_t)per_expert / 8;
  cudaError_t e = launch_amax(W, vecs, E, scales, dev, stream);
  if (e != cudaSuccess) return e;
  if (vecs > 0) {
    launch_kernel(quantize_kernel, dim3(stream_grid(vecs, E, dev), E), dim3(kQThreads), 0, stream,
      static_cast<const uint4*>(W), vecs, scales, static_cast<uint2*>(Wq), nullptr);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  launch_kernel(scale_finalize_kernel, dim3((E + 255) / 256), dim3(256), 0, stream,
      scales, E);
  return cudaGetLastError();
}

cudaError_t launch_quantize_tensor(const void* X, int64_t n, void* Xq, float* x_scale,
                                   const DeviceInfo& dev, cudaStream_t stream) {
  const size_t vecs = (size_t)n / 8;
  cudaError_t e = launch_amax(X, vecs, 1, x_scale + 1, dev, stream);
  if (e != cudaSuccess) return e;
  // n == 0 still runs one CTA so that x_scale[0] is written
  launch_kernel(quantize_kernel, dim3(stream_grid(vecs, 1, dev)), dim3(kQThreads), 0, stream,
      static_cast<const uint4*>(X), vecs, x_scale + 1, static_cast<uint2*>(Xq), x_scale);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8(const void* X, const int32_t* src_of, int T, int d, int k,
                                void* Xeq, float* x_scale, const DeviceInfo& dev,
                                cudaStream_t stream) {
  cudaError_t e = launch_amax(X, (size_t)T * d / 8, 1, x_scale + 1, dev, stream);
  if (e != cudaSuccess) return e;
  const int R = T * k;
  const int need = (R + kDispWarps - 1) / kDispWarps;
  const int cap = dev.sm_count * 8;
  const int grid = need < 1 ? 1 : (need < cap ? need : cap);
  // R == 0 still runs one CTA so that x_scale[0] is written
  launch_kernel(dispatch_fp8_kernel, dim3(grid), dim3(kDispWarps * 32), 0, stream,
      static_cast<const uint4*>(X), src_of, R, k, d / 8, x_scale, static_cast<uint2*>(Xeq),
      dev.status);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_fp8_rows(const void* X, const int32_t* row_of, int T, int d, int k,
                                     void* Xeq, float* x_scale, const DeviceInfo& dev,
                                     cudaStream_t stream) {
  cudaError_t e = launch_amax(X, (size_t)T * d / 8, 1, x_scale + 1, dev, stream);
  if (e != cudaSuccess) return e;
  const int need = (T + kDispWarps - 1) / kDispWarps;
  const int cap = dev.sm_count * 8;
  const int grid = need < 1 ? 1 : (need < cap ? need : cap);
  // T == 0 still runs one CTA so that x_scale[0] is written
  launch_kernel(dispatch_fp8_rows_kernel, dim3(grid), dim3(kDispWarps * 32), 0, stream,
      static_cast<const uint4*>(X), row_of, T, k, d / 8, x_scale, static_cast<uint2*>(Xeq),
      dev.status);
  return cudaGetLastError();
}

int fp8_dispatch_kernel_count(int64_t T) { return T > 0 ? 2 : 1; }

}  // namespace moe
