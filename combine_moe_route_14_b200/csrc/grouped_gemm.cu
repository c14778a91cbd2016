// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// GPT-4 "2%" article §3.1 table: each expert is Linear -> GELU -> Linear;
// DySHARP review (marsggbo) §3.2: GEMM-1 then GEMM-2 per expert, over the
// dense per-expert row blocks that the layout built (§3.1 item 3).
//
//   out[r, n] = act( sum_c A[r, c] * W[e, n, c] )   for r in expert e's block
//
// Design (one persistent CTA per SM, 10 warps):
//   * Operand roles are swapped with respect to the usual token-major GEMM:
//     128 weight rows (output features) form the MMA's M side, and up to 256
//     token rows of one expert form its N side.  N is chosen per tile at run
//     time (a multiple of 16), so a ragged expert block of c rows costs
//     ceil(c/16)*16 columns of MMA work instead of a full 128-row tile.
//   * warp 0 (one lane) streams K-blocks of 64 through a 4-stage ring with
//     TMA (128-byte swizzle), warp 1 (one lane) issues tcgen05.mma into one
//     of two TMEM accumulators (2 x 256 fp32 columns), warps 2-9 drain the
//     other accumulator (tcgen05.ld), apply GELU, round to bf16, transpose
//     through shared memory and store token rows.  Each epilogue warp owns
//     one TMEM lane quarter (32 features) and one half of the tile's tokens,
//     so every SM sub-partition runs two of them.  Mainloop and epilogue of
//     consecutive tiles overlap.
//   * The tile list comes from the per-expert offsets in device memory: no
//     host synchronisation.  Tiles are ordered (expert, feature block, token
//     block) with the token block fastest, so CTAs running at the same time
//     share one weight block through L2.
//   * Every wait is bounded (see mbar_wait); on a timeout the CTA raises a
//     status bit, drains what it issued and frees its TMEM.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

namespace gg {
constexpr int BM = 128;                      // weight rows per tile (UMMA M)
constexpr int BN = 256;                      // token rows per tile, at most (UMMA N)
constexpr int BK = 64;                       // K per stage: one 128-byte swizzled bf16 row
constexpr int UMMA_K = 16;                   // K per tcgen05.mma (kind::f16)
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;         // 16 KB
constexpr int B_STAGE = BN * BK * 2;         // 32 KB
constexpr int B_BOX_ROWS = 32;
constexpr int B_BOX = B_BOX_ROWS * BK * 2;   // 4 KB
constexpr int EPI_WARPS = 8;                 // two per SM sub-partition
constexpr int THREADS = 64 + EPI_WARPS * 32; // producer, MMA, 8 epilogue warps
constexpr uint32_t TMEM_COLS = 2 * BN;       // two accumulators
constexpr int XPOSE = EPI_WARPS * 32 * 32 * 2;  // per-warp 32x32 bf16 transpose tile
constexpr int NUM_BARS = 2 * STAGES + 4 + 1;
constexpr uint64_t kDrainLimitNs = 20ull * 1000ull * 1000ull;  // 20 ms

__host__ __device__ constexpr size_t smem_bytes(int E) {
  return 1024 /* alignment slack */ + (size_t)STAGES * (A_STAGE + B_STAGE) + XPOSE +
         NUM_BARS * 8 + 16 + (size_t)3 * (E + 1) * sizeof(int);
}

struct Args {
  const int32_t* offsets;  // [E+1]
  uint16_t* out;           // [R, N] bf16
  uint32_t* status;
  int E, R, N, K;
  int n_fblocks;           // ceil(N / BM)
  int num_kb;              // ceil(K / BK)
};

struct Tile {
  int e, fb, row0, ntok;
};

__device__ __forceinline__ Tile decode(int tile, const int* s_start, const int* s_lo,
                                       const int* s_hi, int E) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // last expert whose first tile is <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (s_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.e = lo;
  const int local = tile - s_start[lo];
  const int ntb = (s_hi[lo] - s_lo[lo] + BN - 1) / BN;
  t.fb = local / ntb;
  const int tb = local - t.fb * ntb;
  t.row0 = s_lo[lo] + tb * BN;
  t.ntok = min(BN, s_hi[lo] - t.row0);
  return t;
}

// Warp-uniform bounded wait: every lane polls, the outcome is agreed by vote.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          volatile int* abort_flag,
                                          uint64_t limit = kWaitLimitNs) {
  const bool ok = mbar_wait(bar, parity, status, abort_flag, limit);
  return __all_sync(0xffffffffu, ok);
}

// GELU(x) = x * Phi(x), Phi the standard normal CDF (the exact, erf-based
// GELU).  With z = |x| / sqrt(2), Phi(-|x|) = erfc(z) / 2, and erfc is
// evaluated with the rational approximation of Abramowitz & Stegun,
// "Handbook of Mathematical Functions", eq. 7.1.26 (Hastings):
//   erfc(z) ~= (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) exp(-z^2),
//   t = 1 / (1 + p z),  |error| <= 1.5e-7 for z >= 0.
// Then Phi(x) = 1 - Phi(-|x|) for x >= 0.  The result is within a few 1e-7
// of the exact GELU relative to |x|, far below one bf16 ulp of the output.
__device__ __forceinline__ float gelu_erf(float x) {
  const float z = fabsf(x) * 0.70710678118654752440f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
  float p = fmaf(1.061405429f, t, -1.453152027f);
  p = fmaf(p, t, 1.421413741f);
  p = fmaf(p, t, -0.284496736f);
  p = fmaf(p, t, 0.254829592f);
  const float q = 0.5f * p * t * __expf(-z * z);  // Phi(-|x|)
  return x * (x >= 0.f ? 1.0f - q : q);
}

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

template <bool kGelu>
__global__ void __launch_bounds__(THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x, const Args args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_STAGE;
  uint16_t* sX = reinterpret_cast<uint16_t*>(sB + STAGES * B_STAGE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(sX) + XPOSE);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + NUM_BARS);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  const int E = args.E;
  int* s_lo = reinterpret_cast<int*>(s_tmem + 4);
  int* s_hi = s_lo + (E + 1);
  int* s_start = s_hi + (E + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EPI_WARPS);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  // Expert row ranges, clamped into [0, R) so that malformed offsets can
  // only produce wrong numbers, never out-of-range stores.
  bool bad_offsets = false;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int a = __ldg(args.offsets + e), b = __ldg(args.offsets + e + 1);
    if (a < 0 || b < a || b > args.R) bad_offsets = true;
    const int lo = min(max(a, 0), args.R);
    s_lo[e] = lo;
    s_hi[e] = min(max(b, lo), args.R);
  }
  if (bad_offsets && blockIdx.x == 0) flag_error(args.status, MOE_DEV_BAD_ROW);
  __syncthreads();
  if (warp == 0) {  // exclusive scan of per-expert tile counts
    const int per = (E + 31) / 32;
    const int e0 = min(E, lane * per), e1 = min(E, e0 + per);
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += ((s_hi[e] - s_lo[e] + BN - 1) / BN) * args.n_fblocks;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
      s_start[e] = run;
      run += ((s_hi[e] - s_lo[e] + BN - 1) / BN) * args.n_fblocks;
    }
    if (lane == 31) s_start[E] = incl;
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const int total_tiles = s_start[E];

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const uint64_t pol_tokens = l2_policy_evict_last();   // re-read by every feature block
    const uint64_t pol_weights = l2_policy_evict_normal(); // shared by the CTAs of one feature block
    int s = 0;
    uint32_t ph = 0;
    uint32_t issued = 0;  // bit s: stage s has a load in flight or landed
    uint32_t last_ph = 0; // bit s: parity of the last load issued on stage s
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x) {
      const Tile t = decode(tile, s_start, s_lo, s_hi, E);
      const int nbox = (t.ntok + B_BOX_ROWS - 1) / B_BOX_ROWS;
      const uint32_t bytes = A_STAGE + nbox * B_BOX;
      const int wy = t.e * args.N + t.fb * BM;
      for (int kb = 0; kb < args.num_kb; ++kb) {
        ok = warp_wait(&empty[s], ph ^ 1u, args.status, s_abort);
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&full[s], bytes);
          tma_load_2d(sA + s * A_STAGE, &tm_w, kb * BK, wy, &full[s], pol_weights);
          for (int j = 0; j < nbox; ++j)
            tma_load_2d(sB + s * B_STAGE + j * B_BOX, &tm_x, kb * BK, t.row0 + j * B_BOX_ROWS,
                        &full[s], pol_tokens);
        }
        __syncwarp();
        issued |= 1u << s;
        last_ph = (last_ph & ~(1u << s)) | (ph << s);
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok) {  // let issued copies land before the CTA leaves
      int dummy = 0;
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u)
          mbar_wait(&full[q], (last_ph >> q) & 1u, nullptr, (volatile int*)&dummy, kDrainLimitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int s = 0;
    uint32_t ph = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < total_tiles; tile += gridDim.x, ++it) {
      const Tile t = decode(tile, s_start, s_lo, s_hi, E);
      const uint32_t nmma = (uint32_t)((t.ntok + 15) & ~15);
      const uint32_t idesc = idesc_bf16_f32(BM, nmma);
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      ok = warp_wait(&tempty[acc], aph ^ 1u, args.status, s_abort);
      if (!ok) break;
      tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
      for (int kb = 0; kb < args.num_kb; ++kb) {
        ok = warp_wait(&full[s], ph, args.status, s_abort);
        if (!ok) break;
        tc_fence_after_sync();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + s * A_STAGE);
          const uint32_t b0 = smem_u32(sB + s * B_STAGE);
#pragma unroll
          for (int kk = 0; kk < BK / UMMA_K; ++kk)
            tc_mma_bf16(d_tmem, smem_desc_k128(a0 + kk * UMMA_K * 2),
                        smem_desc_k128(b0 + kk * UMMA_K * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);  // the stage is free once these MMAs have read it
        }
        __syncwarp();
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(&tfull[acc]);  // accumulator complete
      __syncwarp();
    }
    if (!ok) {  // wait for every MMA already issued before TMEM is freed
      if (lane == 0) tc_commit(drain);
      __syncwarp();
      int dummy = 0;
      mbar_wait(drain, 0, nullptr, (volatile int*)&dummy, kDrainLimitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;    // which 128 of the tile's 256 token columns
    uint16_t* xp = sX + (warp - 2) * 32 * 32;
    uint16_t* out = args.out;
    const int N = args.N;
    int it = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++it) {
      const Tile t = decode(tile, s_start, s_lo, s_hi, E);
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      if (!warp_wait(&tfull[acc], aph, args.status, s_abort)) break;
      tc_fence_after_sync();
      const int fbase = t.fb * BM + q * 32;  // this warp's 32 output features
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int c_end = min(t.ntok, half * (BN / 2) + BN / 2);
      for (int c0 = half * (BN / 2); c0 < c_end; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + (uint32_t)c0, v);
        tmem_wait_ld();
        // v[j] = accumulator of feature (fbase + lane), token (c0 + j)
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          float x = __uint_as_float(v[j]);
          if (kGelu) x = gelu_erf(x);
          xp[j * 32 + lane] = to_bf16_bits(x);
        }
        __syncwarp();
#pragma unroll
        for (int pass = 0; pass < 4; ++pass) {
          const int j = pass * 8 + (lane >> 2);
          const int f0 = fbase + (lane & 3) * 8;
          const int tok = c0 + j;
          if (tok < t.ntok && f0 < N) {
            const uint4 val = *reinterpret_cast<const uint4*>(xp + j * 32 + (lane & 3) * 8);
            *reinterpret_cast<uint4*>(out + (size_t)(t.row0 + tok) * N + f0) = val;
          }
        }
        __syncwarp();
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gg

// ---------------------------------------------------------------------------
// host side: TMA descriptors and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over a row-major [rows, cols] matrix, box = box_rows x 64
// columns, 128-byte swizzle (the layout the MMA descriptors expect).
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows, std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled is unavailable from the driver";
    return false;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {(cuuint32_t)gg::BK, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return false;
  }
  return true;
}

static std::once_flag g_attr_once[64][2];

cudaError_t launch_grouped_gemm(const void* A, const int32_t* offsets, const void* W, int E,
                                int R, int N, int K, bool gelu, void* out,
                                const DeviceInfo& dev, cudaStream_t stream, std::string* err) {
  if (R == 0 || N == 0) return cudaSuccess;
  CUtensorMap tm_w, tm_x;
  if (!make_map(&tm_w, W, (uint64_t)E * (uint64_t)N, (uint64_t)K, gg::BM, err) ||
      !make_map(&tm_x, A, (uint64_t)R, (uint64_t)K, gg::B_BOX_ROWS, err))
    return cudaErrorInvalidValue;
  gg::Args args;
  args.offsets = offsets;
  args.out = static_cast<uint16_t*>(out);
  args.status = dev.status;
  args.E = E;
  args.R = R;
  args.N = N;
  args.K = K;
  args.n_fblocks = (N + gg::BM - 1) / gg::BM;
  args.num_kb = (K + gg::BK - 1) / gg::BK;
  const size_t smem = gg::smem_bytes(kMaxExperts);  // one attribute value for every E
  cudaError_t e = cudaSuccess;
  auto kern = gelu ? gg::grouped_gemm_kernel<true> : gg::grouped_gemm_kernel<false>;
  if (dev.device >= 0 && dev.device < 64) {
    std::call_once(g_attr_once[dev.device][gelu ? 1 : 0], [&] {
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    });
  } else {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  }
  if (e != cudaSuccess) return e;
  // an upper bound on the tile count: every expert adds at most one partial token block
  const long long max_tiles =
      ((long long)(R + gg::BN - 1) / gg::BN + E) * (long long)args.n_fblocks;
  const int grid = (int)(max_tiles < dev.sm_count ? max_tiles : dev.sm_count);
  kern<<<grid, gg::THREADS, gg::smem_bytes(E), stream>>>(tm_w, tm_x, args);
  return cudaGetLastError();
}

}  // namespace moe
