// Dispatch (token -> its k expert rows) and combine (gate-weighted sum of a
// token's k expert rows).
//
// DySHARP review (marsggbo) §1: dispatch sends the same token data to each of
// its k experts; combine reduces the k results into one.  ThunderEP PCIe
// blog §1.1 and §2.1: the gate values weight the combine sum.
//
// Both are pure HBM streams of bf16 rows (d*2 bytes each): one warp moves one
// row (dispatch) or produces one row (combine) with 16-byte vector accesses,
// several loads in flight per lane before the dependent stores.  Grids are
// sized to a multiple of the SM count and walk rows grid-stride.
#include "common.cuh"
#include "launch.h"

namespace moe {

constexpr int kGatherWarps = 8;  // warps per CTA
constexpr int kCopyUnroll = 8;   // 16-byte vectors in flight per lane

// Xe[r, :] = X[src_of[r] / k, :]
__global__ void __launch_bounds__(kGatherWarps * 32)
    dispatch_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ src_of, int R,
                    int k, int row_vecs, uint4* __restrict__ Xe, uint32_t* status) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kGatherWarps;
  for (int r = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); r < R; r += nwarps) {
    const int s = __ldg(src_of + r);
    if (s < 0 || s >= R) {
      // -1: a row past the kept slots (dropped slots leave it unused)
      if (s != -1 && lane == 0) flag_error(status, MOE_DEV_BAD_ROW);
      continue;
    }
    const uint4* src = X + (size_t)(s / k) * row_vecs;
    uint4* dst = Xe + (size_t)r * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kCopyUnroll) {
      uint4 v[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) v[u] = ld_stream_v4(src + c);
      }
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) dst[c] = v[u];
      }
    }
  }
}

// Token-ordered dispatch: Xe[row_of[t*k + j], :] = X[t, :] for each kept slot j.
// Each token row is read from HBM once and written to its k rows; the
// row-ordered form above reads X[t] once per slot, which goes back to HBM
// k times when X does not stay in L2 (8192 x 7168 bf16 tokens with k = 8:
// 117 MB read 8 times beside a 940 MB write stream).
__global__ void __launch_bounds__(kGatherWarps * 32)
    dispatch_rows_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ row_of, int T,
                         int k, int R, int row_vecs, uint4* __restrict__ Xe, uint32_t* status) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kGatherWarps;
  for (int t = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    int my_row = -1;  // lane j < k: the row of slot j (-1: dropped)
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
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kCopyUnroll) {
      uint4 v[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) v[u] = ld_stream_v4(src + c);
      }
      for (uint32_t m = live; m; m &= m - 1) {
        const int r = __shfl_sync(0xffffffffu, my_row, __ffs(m) - 1);
        uint4* dst = Xe + (size_t)r * row_vecs;
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < row_vecs) dst[c] = v[u];
        }
      }
    }
  }
}

// Token-ordered dispatch that also finishes the layout: slot i = t*k + j of
// expert e_i = idx[i] with stable rank rank_i (row_of[i] on entry, from the
// routing's ranking) takes row offsets[e_i] + rank_i.  Writes that row into
// row_of[i] (in place), src_of[row] = i, and the token row into Xe[row];
// rows past offsets[E] get src_of = -1.
__global__ void __launch_bounds__(kGatherWarps * 32)
    dispatch_scatter_kernel(const uint4* __restrict__ X, const int32_t* __restrict__ idx,
                            int32_t* __restrict__ row_of, const int32_t* __restrict__ offsets,
                            int T, int k, int R, int E, int row_vecs, uint4* __restrict__ Xe,
                            int32_t* __restrict__ src_of, uint32_t* status) {
  pdl_wait_and_release();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kGatherWarps;
  const int kept = min(max(__ldg(offsets + E), 0), R);
  for (int r = kept + blockIdx.x * blockDim.x + threadIdx.x; r < R; r += gridDim.x * blockDim.x)
    src_of[r] = -1;
  for (int t = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    int my_row = -1;  // lane j < k: the row of slot j (-1: dropped)
    if (lane < k) {
      const int i = t * k + lane;
      const int e = __ldg(idx + i);
      if (e >= 0 && e < E) {
        my_row = __ldg(offsets + e) + row_of[i];
        if (my_row < 0 || my_row >= R) {
          flag_error(status, MOE_DEV_BAD_ROW);
          my_row = -1;
        }
      }
      row_of[i] = my_row;
      if (my_row >= 0) src_of[my_row] = i;
    }
    const uint32_t live = __ballot_sync(0xffffffffu, lane < k && my_row >= 0);
    if (!live || X == nullptr) continue;  // X null: the rows only (moe_route_layout)
    const uint4* src = X + (size_t)t * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kCopyUnroll) {
      uint4 v[kCopyUnroll];
#pragma unroll
      for (int u = 0; u < kCopyUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c < row_vecs) v[u] = ld_stream_v4(src + c);
      }
      for (uint32_t m = live; m; m &= m - 1) {
        const int r = __shfl_sync(0xffffffffu, my_row, __ffs(m) - 1);
        uint4* dst = Xe + (size_t)r * row_vecs;
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
          const int c = c0 + u * 32 + lane;
          if (c < row_vecs) dst[c] = v[u];
        }
      }
    }
  }
}

// Y[t, :] = bf16( sum_{j<k} gates[t, j] * Ye[row_of[t*k + j], :] ), fp32 sum in slot order;
// a dropped slot (row_of -1) contributes nothing.
// kK > 0: k known at compile time; kK == 0: runtime k (<= kMaxTopK).
template <int kK>
__global__ void __launch_bounds__(kGatherWarps * 32)
    combine_kernel(const uint4* __restrict__ Ye, const int32_t* __restrict__ row_of,
                   const float* __restrict__ gates, int T, int R, int k_rt, int row_vecs,
                   uint4* __restrict__ Y, uint32_t* status) {
  pdl_wait_and_release();
  constexpr int kSlots = kK > 0 ? kK : kMaxTopK;
  constexpr int kUnroll = kK > 0 ? (kK >= 4 ? 2 : 4) : 1;
  const int k = kK > 0 ? kK : k_rt;
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * kGatherWarps;
  for (int t = blockIdx.x * kGatherWarps + (threadIdx.x >> 5); t < T; t += nwarps) {
    // lanes j < k fetch slot j's row and gate; broadcast below
    int my_row = -1;
    float my_gate = 0.f;
    if (lane < k) {
      my_row = __ldg(row_of + (size_t)t * k + lane);
      my_gate = __ldg(gates + (size_t)t * k + lane);
      if (my_row < -1 || my_row >= R) {  // -1 is a dropped slot
        flag_error(status, MOE_DEV_BAD_ROW);
        my_row = -2;
      }
    }
    const bool bad = __any_sync(0xffffffffu, lane < k && my_row == -2);
    if (bad) continue;
    const uint32_t live = __ballot_sync(0xffffffffu, lane < k && my_row >= 0);  // kept slots
    const uint4* src[kSlots];
    float g[kSlots];
#pragma unroll
    for (int j = 0; j < kSlots; ++j) {
      const int rj = __shfl_sync(0xffffffffu, my_row, j);
      g[j] = __shfl_sync(0xffffffffu, my_gate, j);
      src[j] = Ye + (size_t)(rj < 0 ? 0 : rj) * row_vecs;
    }
    uint4* dst = Y + (size_t)t * row_vecs;
    for (int c0 = 0; c0 < row_vecs; c0 += 32 * kUnroll) {
      uint4 v[kUnroll][kSlots];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
#pragma unroll
        for (int j = 0; j < kSlots; ++j)
          if (j < k && ((live >> j) & 1u) && c < row_vecs) v[u][j] = ld_stream_v4(src[j] + c);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int c = c0 + u * 32 + lane;
        if (c >= row_vecs) continue;
        float acc[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
        for (int j = 0; j < kSlots; ++j) {
          if (j < k && ((live >> j) & 1u)) {
            const uint4 w = v[u][j];
            acc[0] = fmaf(g[j], bf16_lo(w.x), acc[0]);
            acc[1] = fmaf(g[j], bf16_hi(w.x), acc[1]);
            acc[2] = fmaf(g[j], bf16_lo(w.y), acc[2]);
            acc[3] = fmaf(g[j], bf16_hi(w.y), acc[3]);
            acc[4] = fmaf(g[j], bf16_lo(w.z), acc[4]);
            acc[5] = fmaf(g[j], bf16_hi(w.z), acc[5]);
            acc[6] = fmaf(g[j], bf16_lo(w.w), acc[6]);
            acc[7] = fmaf(g[j], bf16_hi(w.w), acc[7]);
          }
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        dst[c] = o;
      }
    }
  }
}

static int gather_grid(int rows, const DeviceInfo& dev) {
  // up to 8 resident CTAs of 8 warps per SM; never more CTAs than rows need
  const int need = (rows + kGatherWarps - 1) / kGatherWarps;
  const int cap = dev.sm_count * 8;
  return need < cap ? need : cap;
}

cudaError_t launch_dispatch(const void* X, const int32_t* src_of, int T, int d, int k, void* Xe,
                            const DeviceInfo& dev, cudaStream_t stream) {
  const int R = T * k;
  if (R == 0) return cudaSuccess;
  launch_kernel(dispatch_kernel, dim3(gather_grid(R, dev)), dim3(kGatherWarps * 32), 0, stream,
                static_cast<const uint4*>(X), src_of, R, k, d / 8, static_cast<uint4*>(Xe),
                dev.status);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_rows(const void* X, const int32_t* row_of, int T, int d, int k,
                                 void* Xe, const DeviceInfo& dev, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  launch_kernel(dispatch_rows_kernel, dim3(gather_grid(T, dev)), dim3(kGatherWarps * 32), 0,
                stream, static_cast<const uint4*>(X), row_of, T, k, T * k, d / 8,
                static_cast<uint4*>(Xe), dev.status);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scatter(const void* X, const int32_t* idx, int32_t* row_of,
                                    const int32_t* offsets, int T, int d, int k, int E, void* Xe,
                                    int32_t* src_of, const DeviceInfo& dev, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  launch_kernel(dispatch_scatter_kernel, dim3(gather_grid(T, dev)), dim3(kGatherWarps * 32), 0,
                stream, static_cast<const uint4*>(X), idx, row_of, offsets, T, k, T * k, E,
                d / 8, static_cast<uint4*>(Xe), src_of, dev.status);
  return cudaGetLastError();
}

cudaError_t launch_combine(const void* Ye, const int32_t* row_of, const float* gates, int T,
                           int d, int k, void* Y, const DeviceInfo& dev, cudaStream_t stream) {
  if (T == 0) return cudaSuccess;
  const int grid = gather_grid(T, dev);
  const uint4* ye = static_cast<const uint4*>(Ye);
  uint4* y = static_cast<uint4*>(Y);
  const int R = T * k;
  switch (k) {
    case 1:
      launch_kernel(combine_kernel<1>, dim3(grid), dim3(kGatherWarps * 32), 0, stream, ye,
                    row_of, gates, T, R, k, d / 8, y, dev.status);
      break;
    case 2:
      launch_kernel(combine_kernel<2>, dim3(grid), dim3(kGatherWarps * 32), 0, stream, ye,
                    row_of, gates, T, R, k, d / 8, y, dev.status);
      break;
    case 4:
      launch_kernel(combine_kernel<4>, dim3(grid), dim3(kGatherWarps * 32), 0, stream, ye,
                    row_of, gates, T, R, k, d / 8, y, dev.status);
      break;
    case 8:
      launch_kernel(combine_kernel<8>, dim3(grid), dim3(kGatherWarps * 32), 0, stream, ye,
                    row_of, gates, T, R, k, d / 8, y, dev.status);
      break;
    default:
      launch_kernel(combine_kernel<0>, dim3(grid), dim3(kGatherWarps * 32), 0, stream, ye,
                    row_of, gates, T, R, k, d / 8, y, dev.status);
  }
  return cudaGetLastError();
}

}  // namespace moe
