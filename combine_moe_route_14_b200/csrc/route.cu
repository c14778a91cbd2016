// Router: logits (router linear) and score / top-k / gates.
//
// GPT-4 "2%" article §4.1 (router code: logits = router_proj(h), softmax,
// topk), §2.3 (softmax then top-k); ThunderEP PCIe blog §1.1 (top-1 / top-2
// routing), §2.1 (top-k indices and gates drive the combine).
//
// Both kernels are bandwidth / latency bound: the router linear streams X
// once (T*d*2 bytes) and the top-k reads T*E*4 bytes of logits.
#include <cfloat>
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

// ---------------------------------------------------------------------------
// router linear: L[t, e] = sum_c X[t, c] * Wr[e, c]   (fp32 accumulate)
//
// A GEMM with N = E (8 for the Mixtral shape): tensor-core mma.sync tiles of
// 16 tokens x 8 experts x 16 K (bf16 in, fp32 accumulate) fit it exactly,
// and it is bound by streaming X (T*d*2 bytes) from HBM once.
//
// Streaming.  A CTA takes tiles of 16 tokens (CTA i: tiles i, i + grid, ...)
// and walks each tile's rows in slices of kRouterSlice columns.  A producer
// warp copies a slice (16 row pieces of up to 2 KB) into a ring of
// kRouterStages shared-memory stages with 1-D bulk copies, one row per lane
// (requests from one thread are issued one after another, so a single
// issuing thread would cap the rate), all signalled on the stage's mbarrier;
// up to three slices per CTA are in flight while the MMA warps work on
// earlier ones.  The grid is at most what is co-resident, so every CTA keeps
// its ring busy from start to end; with a handful of tokens (decode) one CTA
// still has most of its tile in flight at once.
//
// MMA warps.  8 warps split a slice into 64-column chunks (warp w takes
// chunks w, w+8, ...), accumulate their 16 x 8 tiles over all slices of the
// token tile in registers, and the partial tiles are summed in shared memory
// in warp order (deterministic).  Operands use a K permutation shared by
// both: in a 64-column chunk the thread with q = lane % 4 reads columns
// [16q, 16q+16) of its two token rows (lane / 4 and lane / 4 + 8) and of
// expert row lane / 4, as two 16-byte vectors each; MMA m of the chunk takes
// words 2m, 2m+1 of each, so logical k-pair (2q, 2q+1) is column 16q + 4m +
// {0, 1} and (2q+8, 2q+9) is 16q + 4m + {2, 3} for A and B alike, and the 4
// MMAs cover the chunk's 64 columns exactly once.  Shared-memory rows are
// padded by 16 bytes, so the 8 rows a quarter-warp reads fall in distinct
// banks.  X comes from shared memory.  Wr (E x d) is re-read by every tile:
// with at most 8 experts (one n-tile) and d up to kRouterWsMaxD the producer
// copies it into shared memory once per CTA, next to the ring; otherwise it
// is read through the read-only cache.  More than 64 experts are processed
// in groups of 8 n-tiles, streaming the tile's X once per group.
// ---------------------------------------------------------------------------
constexpr int kRouterWarps = 8;                            // MMA warps; warp 8 copies
constexpr int kRouterThreads = (kRouterWarps + 1) * 32;
constexpr int kRouterTok = 16;                             // tokens per tile (the MMA's M)
constexpr int kRouterGroup = 8;                            // n-tiles of 8 experts per pass
constexpr int kRouterSlice = 1024;                         // columns per ring stage
constexpr int kRouterStages = 3;
constexpr int kRouterPitch = kRouterSlice * 2 + 16;        // bytes per staged row
constexpr int kRouterStageBytes = kRouterTok * kRouterPitch;
constexpr int kRouterRingBytes = kRouterStages * kRouterStageBytes;

// Dynamic shared memory: ring | full[S] | empty[S] | Wr barrier | abort flag
// | partial tiles | (staged Wr: 8 rows of d*2 + 16 bytes).
__host__ __device__ constexpr size_t router_part_offset() {
  return (size_t)kRouterRingBytes + (2 * kRouterStages + 1) * 8 + 8;
}
__host__ __device__ constexpr size_t router_smem_bytes(int groups_in_pass) {
  return router_part_offset() + (size_t)kRouterWarps * groups_in_pass * kRouterTok * 8 * 4;
}
__host__ __device__ constexpr int router_w_pitch(int d) { return d * 2 + 16; }
constexpr size_t kRouterSmemMax = 232448;  // opt-in shared memory per block
// The largest d whose 8 staged Wr rows fit beside the ring (one n-tile per pass).
constexpr int kRouterWsMaxD =
    (int)(((kRouterSmemMax - router_smem_bytes(1)) / 8 - 16) / 2) / 8 * 8;

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Barrier `id` over the first `threads` threads of the CTA (the MMA warps).
__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

__device__ __forceinline__ uint4 lds_v4(const uint8_t* p, bool ok) {
  return ok ? *reinterpret_cast<const uint4*>(p) : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ bool router_warp_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                                 volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

// kG: n-tiles per pass at most (1 when E <= 8: fewer registers).  kWs: Wr
// staged in shared memory (kG == 1 only).
template <int kG, bool kWs>
__global__ void __launch_bounds__(kRouterThreads, kG == 1 ? 2 : 1)
    router_logits_kernel(const uint8_t* __restrict__ X, const uint4* __restrict__ Wr, int T,
                         int d, int E, float* __restrict__ L, uint32_t* status,
                         uint32_t* __restrict__ zero_words, int n_zero_words) {
  pdl_wait_and_release();
  // side job: clear the next kernel's counter words (saves a memset launch)
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero_words; i += gridDim.x * blockDim.x)
    zero_words[i] = 0u;
  static_assert(!kWs || kG == 1, "Wr is staged for one n-tile only");
  extern __shared__ __align__(128) uint8_t smem_r[];
  uint8_t* ring = smem_r;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_r + kRouterRingBytes);
  uint64_t* empty = full + kRouterStages;
  uint64_t* wbar = empty + kRouterStages;  // staged Wr landed
  volatile int* s_abort = reinterpret_cast<volatile int*>(wbar + 1);
  float* s_part = reinterpret_cast<float*>(smem_r + router_part_offset());
  uint8_t* s_w = smem_r + router_smem_bytes(kG);  // staged Wr (kWs)
  const int wpitch = router_w_pitch(d);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntok_tiles = (T + kRouterTok - 1) / kRouterTok;
  const int ntiles = (E + 7) / 8;  // n-tiles of 8 experts
  const int ngroups = (ntiles + kG - 1) / kG;
  const int nslices = (d + kRouterSlice - 1) / kRouterSlice;
  const int row_vecs = d / 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouterStages; ++s) {
      mbar_init(&full[s], 1);              // the producer's expect_tx arrive
      mbar_init(&empty[s], kRouterWarps);  // one arrive per MMA warp
    }
    mbar_init(wbar, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  __syncthreads();

  if (warp == kRouterWarps) {
    // ------------------------------------------------------------ producer warp
    // Lane 0 posts a stage's byte count; then lane r issues row r's copy.
    int s = 0;
    uint32_t ph = 0;
    uint32_t pending = 0;  // bit s: a copy into stage s may still be in flight
    uint32_t pend_ph = 0;  // bit s: the parity that copy completes
    bool ok = true;
    if (kWs) {  // Wr once per CTA: E rows of d*2 bytes, padded pitch
      const uint32_t wbytes = (uint32_t)d * 2u;
      if (lane == 0) mbar_arrive_expect_tx(wbar, wbytes * (uint32_t)E);
      __syncwarp();
      for (int e = lane; e < E; e += 32)
        bulk_load_g2s(s_w + e * wpitch, reinterpret_cast<const uint8_t*>(Wr) + (size_t)e * wbytes,
                      wbytes, wbar);
    }
    for (int tt = blockIdx.x; ok && tt < ntok_tiles; tt += gridDim.x) {
      const int t0 = tt * kRouterTok;
      const int nrows = min(kRouterTok, T - t0);
      for (int g = 0; ok && g < ngroups; ++g) {
        for (int sl = 0; sl < nslices; ++sl) {
          if (!router_warp_wait(&empty[s], ph ^ 1u, status, s_abort)) {
            ok = false;
            break;
          }
          const int c0 = sl * kRouterSlice;
          const uint32_t bytes = (uint32_t)min(kRouterSlice, d - c0) * 2u;
          if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes * (uint32_t)nrows);
          __syncwarp();
          if (lane < nrows)
            bulk_load_g2s(ring + s * kRouterStageBytes + lane * kRouterPitch,
                          X + ((size_t)(t0 + lane) * d + c0) * 2, bytes, &full[s]);
          pending |= 1u << s;
          pend_ph = (pend_ph & ~(1u << s)) | (ph << s);
          if (++s == kRouterStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
    }
    if (!ok && lane == 0) {  // an MMA warp gave up: let issued copies land before the CTA leaves
      int dummy = 0;
      if (kWs) mbar_wait(wbar, 0, nullptr, (volatile int*)&dummy, 20ull * 1000ull * 1000ull);
      for (int q = 0; q < kRouterStages; ++q)
        if ((pending >> q) & 1u)
          mbar_wait(&full[q], (pend_ph >> q) & 1u, nullptr, (volatile int*)&dummy,
                    20ull * 1000ull * 1000ull);
    }
    return;
  }

  // -------------------------------------------------------------- MMA warps
  const int r0 = lane >> 2, q = lane & 3;
  if (kWs && !router_warp_wait(wbar, 0, status, s_abort)) return;
  int s = 0;
  uint32_t ph = 0;
  for (int tt = blockIdx.x; tt < ntok_tiles; tt += gridDim.x) {
    const int t0 = tt * kRouterTok;
    for (int g = 0; g < ngroups; ++g) {
      const int G = min(kG, ntiles - g * kG);
      float acc[kG][4];
#pragma unroll
      for (int j = 0; j < kG; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
      for (int sl = 0; sl < nslices; ++sl) {
        if (!router_warp_wait(&full[s], ph, status, s_abort)) return;
        const uint8_t* st = ring + s * kRouterStageBytes;
        const int c0 = sl * kRouterSlice;
        const int w = min(kRouterSlice, d - c0);  // valid columns of this slice
        const int nch = (w + 63) / 64;
        for (int c = warp; c < nch; c += kRouterWarps) {
          const int col = c * 64 + 16 * q;  // this thread's first column in the slice
          const bool ok0 = col < w, ok1 = col + 8 < w;
          const uint8_t* ra = st + r0 * kRouterPitch + col * 2;
          const uint8_t* rb = ra + 8 * kRouterPitch;
          const uint4 x00 = lds_v4(ra, ok0), x01 = lds_v4(ra + 16, ok1);
          const uint4 x10 = lds_v4(rb, ok0), x11 = lds_v4(rb + 16, ok1);
          const uint32_t A0[8] = {x00.x, x00.y, x00.z, x00.w, x01.x, x01.y, x01.z, x01.w};
          const uint32_t A1[8] = {x10.x, x10.y, x10.z, x10.w, x11.x, x11.y, x11.z, x11.w};
          const int v = (c0 + col) / 8;  // vector index of the column in a row of Wr
#pragma unroll
          for (int j = 0; j < kG; ++j) {
            if (j < G) {
              const int e = (g * kG + j) * 8 + r0;
              const bool okB = e < E;
              uint4 w0, w1;
              if (kWs) {
                const uint8_t* ws = s_w + (okB ? e : 0) * wpitch + (size_t)v * 16;
                w0 = lds_v4(ws, okB && ok0);
                w1 = lds_v4(ws + 16, okB && ok1);
              } else {
                const uint4* wr = Wr + (size_t)(okB ? e : 0) * row_vecs;
                w0 = okB && ok0 ? __ldg(wr + v) : make_uint4(0u, 0u, 0u, 0u);
                w1 = okB && ok1 ? __ldg(wr + v + 1) : make_uint4(0u, 0u, 0u, 0u);
              }
              const uint32_t B[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
              for (int m = 0; m < 4; ++m)
                mma_bf16_16816(acc[j], A0[2 * m], A1[2 * m], A0[2 * m + 1], A1[2 * m + 1],
                               B[2 * m], B[2 * m + 1]);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp is done with the stage
        if (++s == kRouterStages) {
          s = 0;
          ph ^= 1u;
        }
      }
      // partial tile of this warp: c0,c1 = (row r0, experts 2q, 2q+1), c2,c3 = row r0 + 8
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        if (j < G) {
          float* p = s_part + (size_t)(warp * G + j) * (kRouterTok * 8);
          p[r0 * 8 + 2 * q] = acc[j][0];
          p[r0 * 8 + 2 * q + 1] = acc[j][1];
          p[(r0 + 8) * 8 + 2 * q] = acc[j][2];
          p[(r0 + 8) * 8 + 2 * q + 1] = acc[j][3];
        }
      }
      named_barrier_sync(1, kRouterWarps * 32);
      for (int i = threadIdx.x; i < G * kRouterTok * 8; i += kRouterWarps * 32) {
        const int j = i / (kRouterTok * 8), rc = i % (kRouterTok * 8);
        const int r = rc / 8, e = (g * kG + j) * 8 + rc % 8;
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < kRouterWarps; ++ww)
          sum += s_part[(size_t)(ww * G + j) * (kRouterTok * 8) + rc];
        if (t0 + r < T && e < E) L[(size_t)(t0 + r) * E + e] = sum;
      }
      named_barrier_sync(1, kRouterWarps * 32);
    }
  }
}

struct RouterSlot {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
};
static RouterSlot g_router[64];

cudaError_t launch_router_logits(const void* X, const void* Wr, int T, int d, int E, float* L,
                                 const DeviceInfo& dev, cudaStream_t stream, uint32_t* zero_words,
                                 int n_zero_words) {
  if (T == 0) return cudaSuccess;
  const int ntiles = (E + 7) / 8;
  const int gmax = ntiles < kRouterGroup ? ntiles : kRouterGroup;  // n-tiles per pass
  RouterSlot& rs = g_router[dev.device & 63];
  std::call_once(rs.once, [&] {
    rs.err = cudaFuncSetAttribute(router_logits_kernel<1, true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRouterSmemMax);
    if (rs.err == cudaSuccess)
      rs.err = cudaFuncSetAttribute(router_logits_kernel<1, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kRouterSmemMax);
    if (rs.err == cudaSuccess)
      rs.err = cudaFuncSetAttribute(router_logits_kernel<kRouterGroup, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)kRouterSmemMax);
  });
  if (rs.err != cudaSuccess) return rs.err;
  const bool ws = gmax == 1 && d <= kRouterWsMaxD;
  const size_t smem = router_smem_bytes(gmax) + (ws ? (size_t)8 * router_w_pitch(d) : 0);
  // CTAs co-resident on an SM: by registers two with one n-tile per pass (72
  // per thread), one with eight (128); by shared memory, 228 KB per SM with
  // 1 KB reserved per CTA.  A larger grid would only run in waves.
  int per_sm = gmax > 1 ? 1 : 2;
  const int by_smem = (int)(233472 / (smem + 1024));
  if (by_smem < per_sm) per_sm = by_smem > 0 ? by_smem : 1;
  const int tiles = (T + kRouterTok - 1) / kRouterTok;
  const int resident = per_sm * dev.sm_count;
  const int blocks = tiles < resident ? tiles : resident;
  const uint8_t* x = static_cast<const uint8_t*>(X);
  const uint4* w = static_cast<const uint4*>(Wr);
  if (ws)
    launch_kernel(router_logits_kernel<1, true>, dim3(blocks), dim3(kRouterThreads), smem, stream,
                  x, w, T, d, E, L, dev.status, zero_words, n_zero_words);
  else if (gmax == 1)
    launch_kernel(router_logits_kernel<1, false>, dim3(blocks), dim3(kRouterThreads), smem,
                  stream, x, w, T, d, E, L, dev.status, zero_words, n_zero_words);
  else
    launch_kernel(router_logits_kernel<kRouterGroup, false>, dim3(blocks), dim3(kRouterThreads),
                  smem, stream, x, w, T, d, E, L, dev.status, zero_words, n_zero_words);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Split router for small batches (T <= kSplitMaxT, E <= 32): the router
// linear over column slices of kSplitCols, one CTA per slice, each writing
// its partial logits P[s][t][e]; the routing kernel adds the partials of a
// logit in slice order (deterministic).  With a handful of tokens the whole
// router is one CTA streaming X and Wr (two DRAM round trips and a reduction
// in one SM); split, every slice's bytes arrive at once.  The sums are fp32
// in a different order from router_logits_kernel, so the logits may differ
// in the last bits.
//   A CTA stages the slice of X (T rows, zero-padded to 64) and of Wr (E rows,
// zero-padded to 32) in shared memory, rows padded by 16 bytes so that a
// quarter-warp's 8 rows fall in distinct banks, and 8 warps take the
// (16-token, 8-expert) tiles with mma.sync m16n8k16 over the slice.
// ---------------------------------------------------------------------------
constexpr int kSplitCols = 256;                       // bf16 columns per slice
constexpr int kSplitWords = kSplitCols / 2 + 4;       // 32-bit words per staged row (+16 B)
constexpr int kSplitRowsX = kSplitMaxT;               // 64
constexpr int kSplitRowsW = 32;
constexpr size_t kSplitSmem = (size_t)(kSplitRowsX + kSplitRowsW) * kSplitWords * 4;

__global__ void __launch_bounds__(256)
    router_split_kernel(const uint4* __restrict__ X, const uint4* __restrict__ Wr, int T, int d,
                        int E, float* __restrict__ P, uint32_t* __restrict__ zero_words,
                        int n_zero_words) {
  pdl_wait_and_release();
  extern __shared__ uint32_t sw[];
  uint32_t* xs = sw;                                // [64][kSplitWords]
  uint32_t* ws = sw + kSplitRowsX * kSplitWords;    // [32][kSplitWords]
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero_words; i += gridDim.x * blockDim.x)
    zero_words[i] = 0u;
  const int s = blockIdx.x;
  const int c0 = s * kSplitCols;
  const int nvec = min(kSplitCols, d - c0) / 8;     // 16-byte vectors of a row in this slice
  const int row_vecs = d / 8;
  constexpr int kVecs = kSplitCols / 8;             // 32
  for (int i = threadIdx.x; i < (kSplitRowsX + kSplitRowsW) * kVecs; i += blockDim.x) {
    const int r = i / kVecs, v = i - r * kVecs;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < kSplitRowsX) {
      if (r < T && v < nvec) val = __ldg(X + (size_t)r * row_vecs + c0 / 8 + v);
      *reinterpret_cast<uint4*>(xs + r * kSplitWords + v * 4) = val;
    } else {
      const int e = r - kSplitRowsX;
      if (e < E && v < nvec) val = __ldg(Wr + (size_t)e * row_vecs + c0 / 8 + v);
      *reinterpret_cast<uint4*>(ws + e * kSplitWords + v * 4) = val;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntt = (T + 15) / 16, nte = (E + 7) / 8;
  for (int tile = warp; tile < ntt * nte; tile += 8) {
    const int tt = tile / nte, te = tile - tt * nte;
    const int ra = tt * 16 + (lane >> 2), rb = te * 8 + (lane >> 2);
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int kk = 0; kk < kSplitCols / 16; ++kk) {
      // A (16 x 16, row-major): rows ra and ra + 8, k pairs (lane%4)*2 and +8;
      // B (16 x 8, column-major = Wr rows): expert rb, the same k pairs
      const int w0 = kk * 8 + (lane & 3);
      const uint32_t a0 = xs[ra * kSplitWords + w0], a1 = xs[(ra + 8) * kSplitWords + w0];
      const uint32_t a2 = xs[ra * kSplitWords + w0 + 4], a3 = xs[(ra + 8) * kSplitWords + w0 + 4];
      const uint32_t b0 = ws[rb * kSplitWords + w0], b1 = ws[rb * kSplitWords + w0 + 4];
      mma_bf16_16816(c, a0, a1, a2, a3, b0, b1);
    }
    // c[0], c[1]: token ra, experts te*8 + (lane%4)*2 + {0, 1}; c[2], c[3]: token ra + 8
    const int e0 = te * 8 + (lane & 3) * 2;
    float* out = P + (size_t)s * T * E;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int t = ra + 8 * h;
      if (t < T) {
        if (e0 < E) out[(size_t)t * E + e0] = c[2 * h];
        if (e0 + 1 < E) out[(size_t)t * E + e0 + 1] = c[2 * h + 1];
      }
    }
  }
}

int router_split_count(int d) { return (d + kSplitCols - 1) / kSplitCols; }

static RouterSlot g_router_split[64];

cudaError_t launch_router_split(const void* X, const void* Wr, int T, int d, int E, float* P,
                                const DeviceInfo& dev, cudaStream_t stream,
                                uint32_t* zero_words, int n_zero_words) {
  if (T == 0) return cudaSuccess;
  RouterSlot& rs = g_router_split[dev.device & 63];
  std::call_once(rs.once, [&] {
    rs.err = cudaFuncSetAttribute(router_split_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSplitSmem);
  });
  if (rs.err != cudaSuccess) return rs.err;
  launch_kernel(router_split_kernel, dim3(router_split_count(d)), dim3(256), kSplitSmem, stream,
                static_cast<const uint4*>(X), static_cast<const uint4*>(Wr), T, d, E, P,
                zero_words, n_zero_words);
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
// gates divide by the kept slots' sum.  A -inf or NaN logit is never chosen
// (it is not above the -FLT_MAX start value); a slot left with no candidate
// is dropped like a thresholded one, so every index written is in [0, E) or -1.
// ---------------------------------------------------------------------------
constexpr int kRouteWarps = 8;
constexpr int kNoPick = 0x7fffffff;  // larger than every expert id

// Order-preserving key of a logit for the warp-wide maximum: a larger logit
// has a larger key, and +0 and -0 share one (they tie, as floats do).  -inf
// and NaN, which are never chosen, have key 0, below every candidate
// (-FLT_MAX has key 0x00800000).
__device__ __forceinline__ uint32_t logit_key(float x) {
  if (!(x >= -FLT_MAX)) return 0u;  // -inf or NaN
  if (x == 0.f) x = 0.f;            // -0 -> +0
  const uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_logit(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// One token's routing by one warp: lanes j < k get slot j's expert (or -1
// when the slot is dropped) and its gate.  Every lane must call it.
template <int kEPL>
// The token's logits are row[e], or with nsplit > 1 the sum over s in order
// of the partial logits row[s * split_stride + e] (the split router's).
__device__ __forceinline__ void route_token(const float* __restrict__ row, int E, int k, int score,
                                            int renorm, float inv_temp, float min_prob,
                                            int lane, int& e_out, float& g_out, int nsplit = 1,
                                            size_t split_stride = 0) {
  float v[kEPL];
  uint32_t key[kEPL];  // 0: not a candidate (past E, -inf, NaN, or taken)
#pragma unroll
  for (int i = 0; i < kEPL; ++i) {
    const int e = lane + 32 * i;
    float x = -FLT_MAX;
    if (e < E) {
      x = __ldg(row + e);
      // partials 1 .. nsplit-1, eight loads in flight, added in slice order
      for (int s0 = 1; s0 < nsplit; s0 += 8) {
        float p[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          p[u] = s0 + u < nsplit ? __ldg(row + (size_t)(s0 + u) * split_stride + e) : 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (s0 + u < nsplit) x += p[u];
      }
    }
    v[i] = x;
    key[i] = (e < E) ? logit_key(v[i]) : 0u;
  }
  float my_v = 0.f;  // lane j < k: logit of slot j
  int my_e = 0;      // lane j < k: expert of slot j
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    if (j < k) {
      // this lane's best: the largest key, the lowest expert id among equals
      // (ids grow with i, so a strictly larger key replaces)
      uint32_t bk = 0u;
      int be = kNoPick;
#pragma unroll
      for (int i = 0; i < kEPL; ++i)
        if (key[i] > bk) {
          bk = key[i];
          be = lane + 32 * i;
        }
      // the warp's largest key, then the lowest id holding it (ties -> lower id)
      const uint32_t gk = __reduce_max_sync(0xffffffffu, bk);
      const uint32_t ge = __reduce_min_sync(0xffffffffu,
                                            (gk != 0u && bk == gk) ? (uint32_t)be : 0xffffffffu);
      // no candidate left (every remaining logit is -inf or NaN): the slot
      // keeps kNoPick and is dropped below
      const int pick = gk != 0u ? (int)ge : kNoPick;
      if (lane == j) {
        my_v = gk != 0u ? key_logit(gk) : -FLT_MAX;
        my_e = pick;
      }
#pragma unroll
      for (int i = 0; i < kEPL; ++i)  // taken (unrolled: key[] stays in registers)
        if (pick == lane + 32 * i) key[i] = 0u;
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
  const bool keep = slot && my_e != kNoPick && (!thr || prob > min_prob);
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
  e_out = keep ? my_e : -1;
  g_out = g;
}

// A token with no kept slot gets no expert row, so no later stage writes
// its output; when asked, its output row is zeroed here.
__device__ __forceinline__ void zero_row_if_dropped(int e_lane, int k, int lane, uint4* zero_rows,
                                                    int zero_vecs, int t) {
  if (zero_rows && __ballot_sync(0xffffffffu, lane < k && e_lane >= 0) == 0u) {
    uint4* row = zero_rows + (size_t)t * zero_vecs;
    for (int c = lane; c < zero_vecs; c += 32) row[c] = make_uint4(0u, 0u, 0u, 0u);
  }
}

template <int kEPL>
__global__ void __launch_bounds__(kRouteWarps * 32)
    route_topk_kernel(const float* __restrict__ L, int T, int E, int k, int score, int renorm,
                      float inv_temp, float min_prob, int32_t* __restrict__ idx,
                      float* __restrict__ gates, uint4* __restrict__ zero_rows, int zero_vecs,
                      uint32_t* __restrict__ zero_words, int n_zero_words, int nsplit) {
  pdl_wait_and_release();
  // side job: clear the caller's counter words (grid-stride; the layer's
  // later kernels run after this one on the same stream)
  if (zero_words) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero_words;
         i += gridDim.x * blockDim.x)
      zero_words[i] = 0u;
  }
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  int e;
  float g;
  route_token<kEPL>(L + (size_t)t * E, E, k, score, renorm, inv_temp, min_prob, lane, e, g, nsplit,
                    (size_t)T * E);
  if (lane < k) {
    idx[(size_t)t * k + lane] = e;
    gates[(size_t)t * k + lane] = g;
  }
  zero_row_if_dropped(e, k, lane, zero_rows, zero_vecs, t);
}

// ---------------------------------------------------------------------------
// Routing fused with the layout's ranking (the layer's path): each CTA
// routes a tile of tokens, taken in ticket order, and also gives every kept
// slot i its stable rank among the slots of its expert:
//   rank[i] = #{i' < i : e_i' = e_i}            (DySHARP review §3.1 item 3:
// layout blocks allocated incrementally, in logical order), written into
// row_of[i].  Within the tile the ranks come from warp match / popcount over
// the slots in order; across tiles each CTA adds, per expert, the count of
// all earlier tiles, found with a decoupled look-back (Merrill & Garland,
// "Single-pass Parallel Prefix Scan with Decoupled Look-back", 2016) over
// per-tile status words.  The CTA with the last ticket holds the totals and
// writes counts and offsets.  The token-walking dispatch then turns ranks
// into rows (row_of[i] = offsets[e_i] + rank[i], src_of[row] = i) while it
// copies the token rows, so no separate layout launch runs.
// ---------------------------------------------------------------------------
// Warps (= tokens) per CTA: 32, or 16 when a lane holds 32 logits (E > 512),
// which needs more registers than 1024 threads leave.
__host__ __device__ constexpr int rank_warps(int epl) { return epl >= 32 ? 16 : 32; }
constexpr uint32_t kLbAggregate = 1u << 30;
constexpr uint32_t kLbInclusive = 2u << 30;
constexpr uint32_t kLbValue = (1u << 30) - 1u;

static int rank_tile(int E) { return rank_warps((E + 31) / 32 > 16 ? 32 : 1); }
int route_rank_tiles(int T, int E) { return (T + rank_tile(E) - 1) / rank_tile(E); }
size_t route_rank_lookback_words(int T, int E) { return 1 + (size_t)route_rank_tiles(T, E) * E; }

template <int kEPL>
__global__ void __launch_bounds__(rank_warps(kEPL) * 32)
    route_rank_kernel(const float* __restrict__ L, int T, int E, int k, int score, int renorm,
                      float inv_temp, float min_prob, int32_t* __restrict__ idx,
                      float* __restrict__ gates, int32_t* __restrict__ rank,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      uint32_t* __restrict__ lookback, uint4* __restrict__ zero_rows,
                      int zero_vecs, uint32_t* __restrict__ zero_words, int n_zero_words,
                      uint32_t* status, int nsplit) {
  pdl_wait_and_release();
  constexpr int kRankWarps = rank_warps(kEPL);
  constexpr int kRankTile = kRankWarps;  // one token per warp
  // shared: keys[kRankTile * k] | run[E] | tile id
  extern __shared__ int sm[];
  const int nslot = kRankTile * k;
  int* keys = sm;
  int* run = keys + nslot;
  int* s_tile = run + E;
  uint32_t* ticket = lookback;          // word 0
  uint32_t* words = lookback + 1;       // [tiles][E] status words
  if (zero_words) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n_zero_words;
         i += gridDim.x * blockDim.x)
      zero_words[i] = 0u;
  }
  if (threadIdx.x == 0) *s_tile = (int)atomicAdd(ticket, 1u);
  for (int e = threadIdx.x; e < E; e += blockDim.x) run[e] = 0;
  __syncthreads();
  const int tile = *s_tile;
  const int tiles = (int)gridDim.x;
  const int t0 = tile * kRankTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // ---- route this tile's tokens, one warp per token
  {
    const int t = t0 + warp;
    int e = -1;
    float g = 0.f;
    if (t < T) {
      route_token<kEPL>(L + (size_t)t * E, E, k, score, renorm, inv_temp, min_prob, lane, e, g,
                        nsplit, (size_t)T * E);
      if (lane < k) {
        idx[(size_t)t * k + lane] = e;
        gates[(size_t)t * k + lane] = g;
      }
      zero_row_if_dropped(e, k, lane, zero_rows, zero_vecs, t);
    }
    if (lane < k) keys[warp * k + lane] = t < T ? e : -1;
  }
  __syncthreads();
  // ---- ranks within the tile: warp 0 walks the slots in order, 32 at a time
  if (warp == 0) {
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int c = 0; c < nslot; c += 32) {
      const int key = c + lane < nslot ? keys[c + lane] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, key);
      const int r = key >= 0 ? run[key] + __popc(peers & lt_mask) : -1;
      __syncwarp();
      if (key >= 0 && lane == __ffs(peers) - 1) run[key] += __popc(peers);
      if (c + lane < nslot) keys[c + lane] = key >= 0 ? (key << 20) | r : -1;  // e, local rank
      __syncwarp();
    }
  }
  __syncthreads();
  // ---- per expert: this tile's base among all earlier tiles, by a
  // warp-wide look-back (one warp per expert; lane l reads tile p - l, so 32
  // predecessors' status words are in flight at once)
  for (int e = warp; e < E; e += kRankWarps) {
    uint32_t* my = words + (size_t)tile * E + e;
    const uint32_t a = (uint32_t)run[e];
    uint32_t excl = 0;
    if (tile == 0) {
      if (lane == 0) st_release_gpu(my, kLbInclusive | a);
    } else {
      if (lane == 0) st_release_gpu(my, kLbAggregate | a);
      int p = tile - 1;
      uint64_t tstart = 0;
      uint32_t spins = 0;
      bool timed_out = false;
      while (true) {
        const int pred = p - lane;
        // before tile 0: an inclusive prefix of 0
        const uint32_t sw = pred >= 0 ? ld_acquire_gpu(words + (size_t)pred * E + e) : kLbInclusive;
        const uint32_t flag = sw & ~kLbValue;
        const uint32_t inc = __ballot_sync(0xffffffffu, flag == kLbInclusive);
        const uint32_t pub = __ballot_sync(0xffffffffu, flag != 0u);
        const int first = inc ? __ffs(inc) - 1 : 31;   // nearest inclusive prefix (or all 32)
        const uint32_t need = first == 31 ? 0xffffffffu : ((2u << first) - 1u);
        if ((pub & need) != need) {
          // a predecessor has not published: its CTA took its ticket earlier,
          // so it is running; wait, but not forever
          if (spins == 0) tstart = globaltimer_ns();
          if ((++spins & 63u) == 0 && globaltimer_ns() - tstart > kWaitLimitNs) {
            timed_out = true;
            break;
          }
          __nanosleep(32);
          continue;
        }
        uint32_t v = lane <= first ? (sw & kLbValue) : 0u;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        excl += v;
        if (inc) break;
        p -= 32;
      }
      if (timed_out && lane == 0) flag_error(status, MOE_DEV_TIMEOUT);
      if (lane == 0) st_release_gpu(my, kLbInclusive | ((excl + a) & kLbValue));
    }
    if (lane == 0) {
      if (tile == tiles - 1) counts[e] = (int)(excl + a);  // the last tile sees every slot
      run[e] = (int)excl;
    }
  }
  __syncthreads();
// ---- ranks out (into row_of)
  for (int i = threadIdx.x; i < nslot; i += blockDim.x) {
    const int t = t0 + i / k;
    if (t >= T) continue;
    const int kv = keys[i];
    rank[(size_t)t0 * k + i] = kv < 0 ? -1 : run[kv >> 20] + (kv & 0xFFFFF);
  }
  // ---- the last tile: offsets = exclusive scan of the counts
  if (tile == tiles - 1) {
    __threadfence_block();
    if (warp == 0) {
      int base = 0;
      for (int e0 = 0; e0 < E; e0 += 32) {
        const int e = e0 + lane;
        const int c = e < E ? counts[e] : 0;
        int incl = c;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        if (e < E) offsets[e] = base + incl - c;
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) offsets[E] = base;
    }
  }
}

cudaError_t launch_route(const float* L, int T, int E, int k, int score, int renormalize,
                         float temperature, float min_prob, int32_t* idx, float* gates,
                         cudaStream_t stream, void* zero_rows, int zero_d, uint32_t* zero_words,
                         int n_zero_words, int nsplit) {
  if (T == 0) return cudaSuccess;
  const int blocks = (T + kRouteWarps - 1) / kRouteWarps;
  const int epl = (E + 31) / 32;
  const float inv_temp = 1.0f / temperature;
#define MOE_ROUTE_LAUNCH(N)                                                                    \
  launch_kernel(route_topk_kernel<N>, dim3(blocks), dim3(kRouteWarps * 32), 0, stream, L, T, E,  \
                k, score, renormalize, inv_temp, min_prob, idx, gates,                           \
                static_cast<uint4*>(zero_rows), zero_d / 8, zero_words, n_zero_words, nsplit)
  if (epl <= 1) MOE_ROUTE_LAUNCH(1);
  else if (epl <= 2) MOE_ROUTE_LAUNCH(2);
  else if (epl <= 4) MOE_ROUTE_LAUNCH(4);
  else if (epl <= 8) MOE_ROUTE_LAUNCH(8);
  else if (epl <= 16) MOE_ROUTE_LAUNCH(16);
  else MOE_ROUTE_LAUNCH(32);
#undef MOE_ROUTE_LAUNCH
  return cudaGetLastError();
}

cudaError_t launch_route_rank(const float* L, int T, int E, int k, int score, int renormalize,
                              float temperature, float min_prob, int32_t* idx, float* gates,
                              int32_t* rank, int32_t* counts, int32_t* offsets, uint32_t* lookback,
                              const DeviceInfo& dev, cudaStream_t stream, void* zero_rows,
                              int zero_d, uint32_t* zero_words, int n_zero_words, int nsplit) {
  if (T == 0) return cudaSuccess;
  const int blocks = route_rank_tiles(T, E);
  const int epl = (E + 31) / 32;
  const float inv_temp = 1.0f / temperature;
  const size_t smem = (size_t)(rank_tile(E) * k + E + 1) * sizeof(int);
#define MOE_RANK_LAUNCH(N)                                                                     \
  launch_kernel(route_rank_kernel<N>, dim3(blocks), dim3(rank_warps(N) * 32), smem, stream, L, T, \
                E, k, score, renormalize, inv_temp, min_prob, idx, gates, rank, counts, offsets, \
                lookback, static_cast<uint4*>(zero_rows), zero_d / 8, zero_words, n_zero_words,  \
                dev.status, nsplit)
  if (epl <= 1) MOE_RANK_LAUNCH(1);
  else if (epl <= 2) MOE_RANK_LAUNCH(2);
  else if (epl <= 4) MOE_RANK_LAUNCH(4);
  else if (epl <= 8) MOE_RANK_LAUNCH(8);
  else if (epl <= 16) MOE_RANK_LAUNCH(16);
  else MOE_RANK_LAUNCH(32);
#undef MOE_RANK_LAUNCH
  return cudaGetLastError();
}

}  // namespace moe
