// Layout: per-expert histogram, exclusive scan and the logical -> layout table.
//
// DySHARP review (marsggbo) §3.1 item 3: the destination keeps an AL table
// from the logical i-th token to its position in a dense per-expert tensor,
// allocating layout blocks incrementally, and combine reads rows back through
// the same table.  ThunderEP PCIe blog §2.2: tokens for the same expert are
// grouped into one contiguous block.
//
// With R = T*k slots, slot i = t*k + j bound for expert e_i:
//   counts[e]  = #{i : e_i = e},  offsets = exclusive scan of counts,
//   row_of[i]  = offsets[e_i] + #{i' < i : e_i' = e_i},  src_of[row_of[i]] = i.
// A dropped slot (e_i = -1) takes no row: row_of[i] = -1, and the rows past
// offsets[E] get src_of = -1.
// This is a stable counting sort of the slots by expert id.  It is
// deterministic: ranks come from warp match/popc over items in order, never
// from the order in which atomics land.
//
// Two paths:
//  * small R (single_path): one CTA does everything (one launch; decode sizes).
//  * larger R: tiles of kTile slots.  Kernel 1 builds a block-level histogram
//    per tile and adds it into counts.  Kernel 2 takes tiles in launch order
//    (an atomic ticket), finds each tile's per-expert base with a decoupled
//    look-back over the preceding tiles (Merrill & Garland, "Single-pass
//    Parallel Prefix Scan with Decoupled Look-back", 2016), and scatters.
#include "common.cuh"
#include "launch.h"

namespace moe {

constexpr int kLayoutThreads = 512;                 // 16 warps
constexpr int kLayoutWarps = kLayoutThreads / 32;
// Slots per tile of the multi-CTA path.  Measured on a B200 (moe_layout,
// 20 calls back to back): 2048-slot tiles against 8192, 18.9 vs 33.2 us for
// 65536 slots over 256 experts, 16.2 vs 22.9 us for 60000 over 8, 23.7 vs
// 37.3 us for 65536 over 1024, 41.5 vs 78.4 us for 1M over 128: more CTAs on
// the histogram and the scatter, and look-back chains that stay short.
constexpr int kTile = 2048;
// Slots handled by the one-CTA path: up to 8192 with at most 32 experts (one
// ballot per expert ranks a warp's slots), 4096 otherwise.  Measured against
// the two-kernel path with 2048-slot tiles (us): 16384 slots over 8 experts
// 22.0 one CTA vs 14.2; 8192 over 64, 18.7 vs 14.8; 8192 over 8, 12.3 vs 13.3.
constexpr int kSingleMaxSmallE = 8192;
constexpr int kSingleMax = 4096;
static bool single_path(int64_t R, int E) {
  return R <= (E <= 32 ? kSingleMaxSmallE : kSingleMax);
}

// Look-back status word: bits 31-30 = flag, bits 29-0 = count (R < 2^30).
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1u;

// Copies the expert ids of slots [begin, end) into shared memory (one
// coalesced pass, all loads in flight together).  -1 marks a dropped slot
// (no row); any other id outside [0, E) is flagged and treated as dropped.
__device__ __forceinline__ void stage_keys(const int32_t* idx, int begin, int end, int E,
                                           int* keys, uint32_t* status) {
  constexpr int kBatch = 8;  // loads in flight per thread before the stores
  for (int i0 = begin + threadIdx.x; i0 < end; i0 += blockDim.x * kBatch) {
    int e[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * blockDim.x;
      e[u] = i < end ? __ldg(idx + i) : -1;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u * blockDim.x;
      if (i < end) {
        int v = e[u];
        if (v < -1 || v >= E) {
          if (status) flag_error(status, MOE_DEV_BAD_EXPERT_ID);
          v = -1;
        }
        keys[i - begin] = v;
      }
    }
  }
}

// Rows past the last kept slot hold no token: src_of[total..R) = -1.
__device__ __forceinline__ void mark_unused_rows(int32_t* src_of, int total, int R) {
  for (int r = total + threadIdx.x; r < R; r += blockDim.x) src_of[r] = -1;
}

// Per-warp histogram of the staged slots [begin, end) (indices into `keys`)
// owned by this warp, walked in 32-slot chunks.  warp_hist is this warp's
// row of E counters.
__device__ __forceinline__ void warp_histogram(const int* keys, int begin, int end,
                                               int* warp_hist) {
  const int lane = threadIdx.x & 31;
  for (int c = begin; c < end; c += 32) {
    const int key = c + lane < end ? keys[c + lane] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, key);
    const int leader = __ffs(peers) - 1;
    if (key >= 0 && lane == leader) warp_hist[key] += __popc(peers);
    __syncwarp();
  }
}

// Second walk over the same slots: stable rank within the warp's running
// counts, then row = base[key] + warp_run[key] + rank-in-chunk.  `first` is
// the global slot number of keys[0].
__device__ __forceinline__ void warp_scatter(const int* keys, int first, int begin, int end,
                                             int* warp_run, const int* base, int32_t* row_of,
                                             int32_t* src_of) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int c = begin; c < end; c += 32) {
    const int li = c + lane;
    const int key = li < end ? keys[li] : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, key);
    int row = 0;
    if (key >= 0) row = base[key] + warp_run[key] + __popc(peers & lt_mask);
    __syncwarp();
    const int leader = __ffs(peers) - 1;
    if (key >= 0 && lane == leader) warp_run[key] += __popc(peers);
    if (key >= 0) {
      row_of[first + li] = row;
      src_of[row] = first + li;
    } else if (li < end) {
      row_of[first + li] = -1;  // a dropped slot (or a bad expert id) has no row
    }
    __syncwarp();
  }
}

// The same two walks for E <= 32 without shared-memory updates: per 32-slot
// chunk one ballot per expert; lane e keeps expert e's running count in a
// register, and a slot's rank is the popcount of its expert's ballot below
// its lane (fetched from lane `key` with one shuffle).
__device__ __forceinline__ void warp_histogram_small(const int* keys, int begin, int end, int E,
                                                     int* warp_hist) {
  const int lane = threadIdx.x & 31;
  int count = 0;  // lane e: slots of expert e seen so far
  for (int c = begin; c < end; c += 32) {
    const int key = c + lane < end ? keys[c + lane] : -1;
    for (int e = 0; e < E; ++e) {
      const uint32_t m = __ballot_sync(0xffffffffu, key == e);
      if (lane == e) count += __popc(m);
    }
  }
  if (lane < E) warp_hist[lane] = count;
}

__device__ __forceinline__ void warp_scatter_small(const int* keys, int first, int begin, int end,
                                                   int E, const int* warp_base, const int* base,
                                                   int32_t* row_of, int32_t* src_of) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int run = lane < E ? warp_base[lane] : 0;  // lane e: slots of expert e before this chunk
  for (int c = begin; c < end; c += 32) {
    const int li = c + lane;
    const int key = li < end ? keys[li] : -1;
    uint32_t mine = 0;  // lane e: ballot of expert e in this chunk
    for (int e = 0; e < E; ++e) {
      const uint32_t m = __ballot_sync(0xffffffffu, key == e);
      if (lane == e) mine = m;
    }
    const uint32_t mk = __shfl_sync(0xffffffffu, mine, key < 0 ? 0 : key);
    const int rk = __shfl_sync(0xffffffffu, run, key < 0 ? 0 : key);
    if (key >= 0) {
      const int row = base[key] + rk + __popc(mk & lt_mask);
      row_of[first + li] = row;
      src_of[row] = first + li;
    } else if (li < end) {
      row_of[first + li] = -1;  // a dropped slot (or a bad expert id) has no row
    }
    run += __popc(mine);
  }
}

// In-place exclusive scan of s[0..n) by the whole CTA (n <= 2 * blockDim).
// Returns the total.  Uses `tmp` (>= kLayoutWarps ints) as scratch.
__device__ int block_exclusive_scan(int* s, int n, int* tmp) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (n + blockDim.x - 1) / blockDim.x;  // <= 2
  const int b = tid * per;
  int local = 0;
  for (int q = 0; q < per; ++q)
    if (b + q < n) local += s[b + q];
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = lane < (int)(blockDim.x >> 5) ? tmp[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += y;
    }
    if (lane < (int)(blockDim.x >> 5)) tmp[lane] = wi - w;  // exclusive warp base
    if (lane == 31) tmp[32] = wi;                            // total
  }
  __syncthreads();
  int run = tmp[warp] + incl - local;
  for (int q = 0; q < per; ++q)
    if (b + q < n) {
      const int v = s[b + q];
      s[b + q] = run;
      run += v;
    }
  const int total = tmp[32];
  __syncthreads();
  return total;
}

// Per-expert exclusive scan across the warps of the CTA: hist[w][e] becomes
// the count of expert e in warps < w; returns through agg[e] the CTA total.
__device__ void scan_over_warps(int* hist, int E, int* agg) {
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    for (int w = 0; w < kLayoutWarps; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    agg[e] = run;
  }
}

// ---------------------------------------------------------------------------
// one-CTA path
// smem: keys[R] | hist[kLayoutWarps][E] | base[E+1] | tmp[33]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads)
    layout_single_kernel(const int32_t* __restrict__ idx, int R, int E, int32_t* counts,
                         int32_t* offsets, int32_t* row_of, int32_t* src_of, uint32_t* status) {
  pdl_wait_and_release();
  extern __shared__ int smem_i[];
  int* keys = smem_i;
  int* hist = keys + R;
  int* base = hist + kLayoutWarps * E;
  int* tmp = base + E + 1;
  stage_keys(idx, 0, R, E, keys, status);
  for (int i = threadIdx.x; i < kLayoutWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int per_warp = ((R + kLayoutWarps * 32 - 1) / (kLayoutWarps * 32)) * 32;
  const int begin = min(R, warp * per_warp), end = min(R, begin + per_warp);
  if (E <= 32) warp_histogram_small(keys, begin, end, E, hist + warp * E);
  else warp_histogram(keys, begin, end, hist + warp * E);
  __syncthreads();
  scan_over_warps(hist, E, base);
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) counts[e] = base[e];
  __syncthreads();
  const int total = block_exclusive_scan(base, E, tmp);
  for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = base[e];
  if (threadIdx.x == 0) offsets[E] = total;
  mark_unused_rows(src_of, total, R);
  if (E <= 32) warp_scatter_small(keys, 0, begin, end, E, hist + warp * E, base, row_of, src_of);
  else warp_scatter(keys, 0, begin, end, hist + warp * E, base, row_of, src_of);
}

// ---------------------------------------------------------------------------
// multi-CTA path, kernel 1: block histogram of one tile, added into counts
// (counts zeroed by the host before).  Also clears this tile's look-back
// status row and, in tile 0, the ticket counter for kernel 2.
// smem: hist[E]
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads)
    layout_hist_kernel(const int32_t* __restrict__ idx, int R, int E, int32_t* counts,
                       uint32_t* lookback, uint32_t* ticket, uint32_t* status) {
  pdl_wait_and_release();
  extern __shared__ int smem_i[];
  int* hist = smem_i;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    hist[e] = 0;
    lookback[(size_t)blockIdx.x * E + e] = 0u;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *ticket = 0u;
  __syncthreads();
  const int tile_begin = blockIdx.x * kTile;
  const int tile_end = min(R, tile_begin + kTile);
  for (int i = tile_begin + threadIdx.x; i < tile_end; i += blockDim.x) {
    const int e = __ldg(idx + i);
    if (e >= 0 && e < E) atomicAdd(&hist[e], 1);  // order of adds does not matter for a count
    else if (e != -1) flag_error(status, MOE_DEV_BAD_EXPERT_ID);  // -1: a dropped slot
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    if (hist[e]) atomicAdd(counts + e, hist[e]);
}

// ---------------------------------------------------------------------------
// multi-CTA path, kernel 2: per-tile stable ranks + decoupled look-back.
// smem: keys[kTile] | hist[kLayoutWarps][E] | agg[E] | base[E+1] | tmp[33] | tile id
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLayoutThreads)
    layout_scatter_kernel(const int32_t* __restrict__ idx, int R, int E,
                          const int32_t* __restrict__ counts, int32_t* offsets, int32_t* row_of,
                          int32_t* src_of, uint32_t* lookback, uint32_t* ticket,
                          uint32_t* status) {
  pdl_wait_and_release();
  extern __shared__ int smem_i[];
  int* keys = smem_i;
  int* hist = keys + kTile;
  int* agg = hist + kLayoutWarps * E;
  int* base = agg + E;
  int* tmp = base + E + 1;
  int* s_tile = tmp + 33;
  if (threadIdx.x == 0) *s_tile = (int)atomicAdd(ticket, 1u);
  for (int i = threadIdx.x; i < kLayoutWarps * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int tile = *s_tile;
  const int tile_begin = tile * kTile;
  const int tile_end = min(R, tile_begin + kTile);
  const int n = tile_end - tile_begin;
  stage_keys(idx, tile_begin, tile_end, E, keys, nullptr);  // kernel 1 flagged bad ids
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const int per_warp = ((n + kLayoutWarps * 32 - 1) / (kLayoutWarps * 32)) * 32;
  const int begin = min(n, warp * per_warp);
  const int end = min(n, begin + per_warp);
  if (E <= 32) warp_histogram_small(keys, begin, end, E, hist + warp * E);
  else warp_histogram(keys, begin, end, hist + warp * E);
  __syncthreads();
  scan_over_warps(hist, E, agg);
  __syncthreads();

  // Decoupled look-back, one thread per expert: publish this tile's
  // aggregate, sum predecessors until an inclusive prefix is found, publish
  // the inclusive prefix.  Waits are bounded.
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    uint32_t* my = lookback + (size_t)tile * E + e;
    const uint32_t a = (uint32_t)agg[e];
    if (tile == 0) {
      st_release_gpu(my, kFlagInclusive | a);
      agg[e] = 0;  // exclusive prefix of tile 0
      continue;
    }
    st_release_gpu(my, kFlagAggregate | a);
    uint32_t excl = 0;
    int pred = tile - 1;
    uint64_t t0 = 0;
    uint32_t spins = 0;
    while (pred >= 0) {
      const uint32_t s = ld_acquire_gpu(lookback + (size_t)pred * E + e);
      const uint32_t flag = s & ~kValueMask;
      if (flag == kFlagInclusive) {
        excl += s & kValueMask;
        break;
      }
      if (flag == kFlagAggregate) {
        excl += s & kValueMask;
        --pred;
        continue;
      }
      // predecessor not published yet: it started earlier (ticket order), so
      // it is running; wait, but not forever
      if (spins == 0) t0 = globaltimer_ns();
      if ((++spins & 255u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs) {
        flag_error(status, MOE_DEV_TIMEOUT);
        break;
      }
      __nanosleep(32);
    }
    st_release_gpu(my, kFlagInclusive | ((excl + a) & kValueMask));
    agg[e] = (int)excl;  // this tile's per-expert base among earlier tiles
  }
  // offsets from the complete counts (kernel 1 finished before this launch)
  for (int e = threadIdx.x; e < E; e += blockDim.x) base[e] = counts[e];
  __syncthreads();
  const int total = block_exclusive_scan(base, E, tmp);
  if (tile == 0) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) offsets[e] = base[e];
    if (threadIdx.x == 0) offsets[E] = total;
    mark_unused_rows(src_of, total, R);
  }
  for (int e = threadIdx.x; e < E; e += blockDim.x) base[e] += agg[e];
  __syncthreads();
  if (E <= 32)
    warp_scatter_small(keys, tile_begin, begin, end, E, hist + warp * E, base, row_of, src_of);
  else
    warp_scatter(keys, tile_begin, begin, end, hist + warp * E, base, row_of, src_of);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int num_tiles(int64_t R) { return (int)((R + kTile - 1) / kTile); }

int layout_kernel_count(int64_t R, int E) { return single_path(R, E) ? 1 : 2; }

size_t layout_workspace_bytes(int64_t R, int E) {
  if (single_path(R, E)) return 0;
  return 256 + (size_t)num_tiles(R) * (size_t)E * sizeof(uint32_t);
}

cudaError_t launch_layout(const int32_t* idx, int R, int E, int32_t* counts, int32_t* offsets,
                          int32_t* row_of, int32_t* src_of, void* ws, const DeviceInfo& dev,
                          cudaStream_t stream) {
  if (single_path(R, E)) {
    const size_t smem = (size_t)(R + kLayoutWarps * E + E + 1 + 33) * sizeof(int);
    if (smem > 48 * 1024) {
      cudaError_t err = cudaFuncSetAttribute(layout_single_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (err != cudaSuccess) return err;
    }
    launch_kernel(layout_single_kernel, dim3(1), dim3(kLayoutThreads), smem, stream, idx, R, E,
                  counts, offsets, row_of, src_of, dev.status);
    return cudaGetLastError();
  }
  uint32_t* ticket = static_cast<uint32_t*>(ws);
  uint32_t* lookback = reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + 256);
  const int tiles = num_tiles(R);
  cudaError_t err = cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), stream);
  if (err != cudaSuccess) return err;
  launch_kernel(layout_hist_kernel, dim3(tiles), dim3(kLayoutThreads), (size_t)E * sizeof(int),
                stream, idx, R, E, counts, lookback, ticket, dev.status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = (size_t)(kTile + kLayoutWarps * E + E + E + 1 + 33 + 1) * sizeof(int);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(layout_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
    if (err != cudaSuccess) return err;
  }
  launch_kernel(layout_scatter_kernel, dim3(tiles), dim3(kLayoutThreads), smem, stream,
      idx, R, E, counts, offsets, row_of, src_of, lookback, ticket, dev.status);
  return cudaGetLastError();
}

}  // namespace moe
