// Grouped expert GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// GPT-4 "2%" article §3.1 table: each expert is Linear -> GELU -> Linear;
// DySHARP review (marsggbo) §3.2: GEMM-1 then GEMM-2 per expert, over the
// dense per-expert row blocks that the layout built (§3.1 item 3).
//
//   out[r, n] = act( sum_c A[r, c] * W[e, n, c] )   for r in expert e's block
//
// Operands are bf16, or E4M3 FP8 codes with per-tensor scales (ThunderEP PCIe
// blog §3.3 and §5.2: activations cast to FP8 with a per-tensor dynamic scale;
// FP8-capable tensor cores compute on them directly):
//   out[r, n] = act( a_scale * w_scale[e] * sum_c Aq[r, c] * Wq[e, n, c] ).
// A stage holds 128 bytes of K per row in both cases (64 bf16 or 128 E4M3
// values), so the ring, the swizzle and the descriptors are shared; the FP8
// form issues kind::f8f6f4 MMAs (K = 32) and scales in the epilogue.
//
// Gather-on-load form (DySHARP review §3.2: dispatch fused into the expert
// GEMM): A's rows are fetched straight from the token matrix through the
// layout table, A[r] = X[src_of[r] / k], with TMA gather4 loads (four rows
// per request), so no dispatched copy of the tokens is ever written.
//
// Design (one persistent CTA per SM, 11 warps):
//   * Operand roles are swapped with respect to the usual token-major GEMM:
//     128 weight rows (output features) form the MMA's M side, and up to 256
//     token rows of one expert form its N side.  N is chosen per tile at run
//     time (a multiple of 16), so a ragged expert block of c rows costs
//     ceil(c/16)*16 columns of MMA work instead of a full 128-row tile.
//   * warps 0 and 1 (one lane each) stream 128-byte K-blocks of the weight and
//     the token operand with TMA (128-byte swizzle) through a ring of 3
//     slots of KPS = 2 K-blocks each (paired CTAs; as many as shared memory
//     holds; one K-block per slot in 4 slots with a single CTA): one
//     barrier round trip and one MMA commit per two K-blocks (each commit
//     costs MMA issue throughput; measured 8% faster than one K-block per
//     slot in 7 slots, despite one K-block less in flight),
//     warp 2 (one lane) issues tcgen05.mma into one of two TMEM
//     accumulators (2 x 256 fp32 columns), warps 3-10 drain the
//     other accumulator (tcgen05.ld), apply GELU, round to bf16 and store
//     token rows (a warp writes 32 consecutive features of a row per store
//     instruction).  Each epilogue warp owns
//     one TMEM lane quarter (32 features) and one half of the tile's tokens,
//     so every SM sub-partition runs two of them.  Mainloop and epilogue of
//     consecutive tiles overlap.
//   * The tile list comes from the per-expert offsets in device memory: no
//     host synchronisation.  Tiles are ordered (expert, feature block, token
//     block) with the token block fastest, so CTAs running at the same time
//     share one weight block through L2.
//   * Fused FFN form (kFused): GEMM-1 and GEMM-2 in one persistent launch
//     (the GEMM half of the token-centric pipeline of the DySHARP review
//     §3.2).  The tile list is GEMM-1's tiles followed by GEMM-2's; a GEMM-2
//     tile of token block b starts once every GEMM-1 tile of b has stored
//     its part of H: each GEMM-1 epilogue warp publishes its stores (fence,
//     then an atomic add on b's counter) and GEMM-2's token producer waits,
//     bounded, for the count (acquire), then fences the async proxy before
//     its TMA reads of H.  GEMM-1 tiles wait on nothing and every CTA is
//     resident, so the waits always end; the GEMM-1 tail, the second launch
//     and its prologue disappear.
//   * Every wait is bounded (see mbar_wait); on a timeout the CTA raises a
//     status bit, drains what it issued and frees its TMEM.
#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace moe {

namespace gg {
constexpr int BM = 128;                      // weight rows per CTA (UMMA M per CTA)
constexpr int BN = 256;                      // token rows per tile, at most (UMMA N)
constexpr int BK = 64;                       // K per stage: one 128-byte swizzled bf16 row
constexpr int BK_FP8 = 128;                  // the same 128 bytes as E4M3 values
constexpr int UMMA_K = 16;                   // K per tcgen05.mma (kind::f16); 32 for kind::f8f6f4
constexpr int UMMA_K_BYTES = UMMA_K * 2;     // 32 bytes of a row per MMA in both kinds
constexpr int A_STAGE = BM * BK * 2;         // 16 KB of weight rows per CTA and stage
constexpr int B_BOX_ROWS = 32;
constexpr int B_BOX = B_BOX_ROWS * BK * 2;   // 4 KB
// Token rows a CTA stages for a tile (up to 128 per CTA with a pair, up to 256
// with one CTA) are loaded in 128-row boxes of 16 KB instead of 4 KB ones,
// since TMA throughput grows with the request size; a half-tile of at least
// kWideMin rows takes ceil(rows / 128) such boxes (over-fetching at most 32
// rows past the last one, inside the stage buffer).
constexpr int B_WIDE_ROWS = 128;
constexpr int kWideMin = 96;
constexpr int EPI_WARPS = 8;                 // two per SM sub-partition
#ifndef MOE_GATHER_WARPS
#define MOE_GATHER_WARPS 8
#endif
// Gather form: gather4 requests are issued one lane at a time, about one per
// ~90 cycles per issuing warp, so the token rows are fetched by several warps.
constexpr int kGatherWarps = MOE_GATHER_WARPS;
// Warp roles: warp 0 streams weights, the next NTOK warps token rows, warp
// MMA issues the MMAs (leader CTA), warp SCHED (leader CTA, dynamic
// schedule) publishes the work items, warps EPI0.. drain the accumulators.
template <bool kGather, int kPair> struct Roles {
  static constexpr int NW = 1;
  static constexpr int NTOK = kGather ? kGatherWarps : 1;
  static constexpr int NPROD = NW + NTOK;
  static constexpr int MMA = NPROD;
  static constexpr int SCHED = MMA + 1;
  static constexpr int EPI0 = SCHED + 1;
  static constexpr int THREADS = (EPI0 + EPI_WARPS) * 32;
  // arrivals on a stage's full barrier (leader CTA): one per issuing warp,
  // one for all the gather warps together
  static constexpr int FULL_ARRIVALS = NW + (kGather ? 1 : NTOK);
};
constexpr uint32_t TMEM_COLS = 2 * BN;       // two accumulators
// Merged last token block (paired CTAs, plain two-launch forms): an expert
// whose last token block would hold at most kMergeRows rows gives them to
// the block before it, which then spans up to BN_MAX rows in one tile.  A
// tile's pace is set by streaming its weight rows, whatever its token count,
// so a 16-row tail tile costs about as much as a full one; merged, the
// expert's weight block streams through the ring once instead of twice.  The
// merged tile issues two MMAs per K step (N = 256 and N = the tail) into
// BN_MAX accumulator columns.  Accumulators then no longer sit in two fixed
// halves of TMEM: tiles alternate between a low placement (from column 0)
// and a high one (ending at column 512), and where two consecutive tiles'
// columns overlap, the next tile's MMAs wait until the epilogue has drained
// the shared columns, which it drains first.
constexpr int kMergeRows = 64;
// Merging is used when the mean rows per expert is above kMergeMinMeanRows
// (below it hardly any expert reaches 257 rows, and the variant costs ~1 % on
// the decode shapes for nothing) and at most kMergeMaxMeanRows.  With few
// rows per expert the GEMM is bound by streaming each tile's weights and a
// tail tile doubles that stream.  With many (the Mixtral shape, ~1024 per
// expert) the GEMM runs near its tensor rate, the tail tile's weights come
// from L2 beside the full tiles, and a merged tile costs more than the tail
// tile it replaces: its second, narrow MMA per K step reads the weight stage
// again, neighbouring tiles whose columns overlap cannot overlap their MMAs
// with its epilogue, and the static schedule gives the wider tiles to some
// clusters only.  Measured on a B200: the fine-grained shape (256 rows per
// expert) -10 % per GEMM, 1040 rows per expert +27 %.
constexpr int kMergeMinMeanRows = 128;
constexpr int kMergeMaxMeanRows = 384;
constexpr int BN_MAX = BN + kMergeRows;      // 320 accumulator columns at most
constexpr int kHighMin = 2 * BN - BN_MAX;    // 192: the lowest column a high tile starts at
// A merged tile's tail rows (up to 32 per CTA) go into a ring of their own,
// one 4 KB box per K-block beside each slot, so that the ordinary stage
// layout and its address arithmetic stay as they are.
constexpr int MAX_STAGES = 8;                // barrier slots; the ring uses Args::stages of them
constexpr size_t kSmemBudget = 232448;       // B200 opt-in shared memory per block
constexpr uint64_t kDrainLimitNs = 20ull * 1000ull * 1000ull;  // 20 ms
// Work items reach every role of a cluster through a queue of this depth in
// shared memory, filled by the leader CTA's weight producer (the role that
// runs furthest ahead); a slot is reused once every other role has read it.
constexpr int kQueue = 4;
// Dispatch items of the fused FFN: layout rows per item, and 16-byte vectors
// in flight per lane while copying them.
constexpr int kDispRows = 64;
// Weight K-blocks prefetched into L2 ahead of their TMA loads by the weight
// producer's idle lanes, for launches whose expert blocks are small (few
// rows per expert: the weight stream is the whole cost and DRAM latency
// bounds it).  Measured on a B200: decode-sized layers -5 %; with 256 or
// more rows per expert it costs 4-6 %, so it is off there.
constexpr int kWPrefetchSmall = 4;
#ifndef MOE_W_EVICT_FIRST
#define MOE_W_EVICT_FIRST 0  // L2 policy of the weight stream: evict_first instead of normal
#endif
#ifndef MOE_KPS_PAIR
#define MOE_KPS_PAIR 2       // K-blocks per ring slot with paired CTAs
#endif
constexpr int kWPrefetchMaxRows = 64;  // mean rows per expert at or below which it is on
constexpr int kDispUnroll = 8;

// kPair = 1: one CTA computes a 128-feature x N-token tile (cta_group::1).
// kPair = 2: a cluster of two CTAs computes a 256-feature x N-token tile with
//   the paired MMA (cta_group::2, M = 256): each CTA stages its own 128
//   weight rows and half of the token rows, so per-SM shared-memory traffic
//   and L2 reads per FLOP are a third lower, and 6 stages fit.
template <int kPair> struct Cfg {
  static constexpr int B_STAGE = (BN / kPair) * BK * 2;  // token rows this CTA stages
  // K-blocks per ring slot: two with paired CTAs (3 slots of 64 KB), one with
  // a single CTA (its 48 KB K-block already leaves only 4 slots)
  static constexpr int KPS = kPair == 2 ? MOE_KPS_PAIR : 1;
  static constexpr int NUM_BARS = 2 * MAX_STAGES + 4 + 1 + 2 * kQueue + 1 + 2;
  static constexpr int FEAT = BM * kPair;                // output features per tile
};

// Shared memory: the stage ring, barriers, and the per-expert tile table.
template <int kPair>
__host__ __device__ constexpr size_t fixed_smem(int E) {
  return 1024 /* alignment slack */ + Cfg<kPair>::NUM_BARS * 8 + 16 + kQueue * sizeof(int) +
         (size_t)4 * (E + 1) * sizeof(int);
}
// merge: each slot also holds KPS tail boxes (merged last token blocks)
template <int kPair>
__host__ __device__ constexpr size_t slot_bytes(bool merge) {
  return (size_t)Cfg<kPair>::KPS * (size_t)(A_STAGE + Cfg<kPair>::B_STAGE + (merge ? B_BOX : 0));
}
template <int kPair>
__host__ __device__ constexpr size_t smem_bytes(int E, int stages, bool merge) {
  return fixed_smem<kPair>(E) + (size_t)stages * slot_bytes<kPair>(merge);
}
// As many stages as fit (more bytes in flight hide more load latency).
template <int kPair>
inline int stages_for(int E, bool merge = false) {
  const size_t avail = kSmemBudget - fixed_smem<kPair>(E);
  const int n = (int)(avail / slot_bytes<kPair>(merge));
  return n < MAX_STAGES ? n : MAX_STAGES;
}

struct Args {
  const int32_t* offsets;  // [E+1]
  uint16_t* out;           // [R, N] bf16
  uint32_t* status;
  const float* a_scale;    // FP8 form: dequantisation scale of A (device scalar)
  const float* w_scale;    // FP8 form: [E] dequantisation scales of W
  const int32_t* gather_src;  // gather form: src_of [R]; A row r is token src_of[r] / gather_k
  int gather_k;
  int a_rows;              // gather form: rows of the token matrix (T)
  int E, R, N, K;
  int n_fblocks;           // ceil(N / features per tile)
  int num_kb;              // ceil(K / K-values per stage)
  int stages;              // ring slots of KPS K-blocks (<= MAX_STAGES)
  // fused FFN form: phase 1 = GEMM-2 over phase 0's output (A = out)
  uint16_t* out2;          // [R, N2] bf16
  int N2, n_fblocks2, num_kb2;
  uint32_t* ready;         // [token blocks]: GEMM-1 epilogue warps done, per token block
  uint32_t ready_target;   // arrivals that complete a token block
  const uint8_t* w_ptr;    // W as bytes (phase 0), row pitch w_pitch; W2 for phase 1
  const uint8_t* w2_ptr;
  int w_pitch, w2_pitch;
  int w_prefetch;          // weight K-blocks prefetched into L2 ahead (0: none)
  bool fb_fastest, fb_fastest2;  // tile order of phase 0 / phase 1 (see decode)
  // Dynamic schedule: non-null -> clusters take items from this counter, in
  // item order (zeroed before the launch); null -> static round-robin.
  uint32_t* ticket;
  // Dispatch items (fused form with a ticket): the epilogue warps gather the
  // token operand's rows A[r] = disp_X[disp_src[r] / disp_k] in chunks of
  // kDispRows rows; GEMM-1 tiles wait for the chunks under their rows.
  const uint4* disp_X;     // [disp_T, K] bf16 (null: no dispatch items)
  uint4* disp_A;           // the token operand A [R, K], written here
  const int32_t* disp_src; // src_of [R]
  int disp_k, disp_T, disp_vecs;  // disp_vecs = K / 8
  uint32_t* dready;        // [ceil(R / kDispRows)] arrivals per chunk
  // Combine in the epilogue of the GEMM without GELU (GEMM-2), k <= 2:
  // Y[t] = bf16(sum_j gates[t, j] * acc(row_of[t*k + j])).  A token with one
  // kept slot is written at once; with two, the first slot to arrive stores
  // its gate-weighted fp32 row in comb_part and raises a flag, and the second
  // adds it to its own and writes Y.  Rows of `out` are not stored.
  uint16_t* comb_Y;            // [comb_T, N] bf16 (null: store `out` as usual)
  const int32_t* comb_src;     // src_of [R]
  const int32_t* comb_row_of;  // row_of [comb_T * comb_k]
  const float* comb_gates;     // [comb_T, comb_k]
  float* comb_part;            // [comb_T, N] fp32
  uint32_t* comb_cnt;          // [comb_T * ceil(N / 32)] arrival words, zeroed before the launch
  int comb_k, comb_T;
};

struct Tile {
  int e, fb, row0, ntok;
};

// Token blocks of an expert with c rows: ceil(c / 256) blocks of 256 rows,
// the last one ragged; with `merge`, a last block of at most kMergeRows rows
// joins the one before it.  (Splitting c evenly across the blocks was
// measured slower: the kernel is bound by operand loads, and even blocks
// cost more load requests than one ragged block.)
__device__ __forceinline__ int token_blocks(int c, bool merge) {
  int nb = (c + BN - 1) / BN;
  if (merge && nb >= 2 && c - (nb - 1) * BN <= kMergeRows) --nb;
  return nb;
}

// First TMEM column of a tile's accumulator: buffer 0 (even tiles) at 0,
// buffer 1 at 256, or with merged blocks ending at column 512 (its width
// rounded up to 32 columns, the epilogue's chunk), so that consecutive
// tiles overlap only when their widths add up to more than 512.
__device__ __forceinline__ int acc_base(int buf, int width, bool merge) {
  return buf == 0 ? 0 : merge ? 2 * BN - ((width + 31) & ~31) : BN;
}

// fb_fastest = false: an expert's tiles go token block fastest (the CTAs
// running at once share each weight block through L2); true: feature block
// fastest (they share each token block instead: every feature-block tile of a
// token block runs at about the same time, so the token rows are read from
// DRAM once even when a long K leaves no room in L2 to keep them).
__device__ __forceinline__ Tile decode(int tile, const int* s_start, const int* s_lo,
                                       const int* s_hi, int E, bool fb_fastest, int n_fb,
                                       bool merge) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {  // last expert whose first tile is <= tile
    const int mid = (lo + hi + 1) >> 1;
    if (s_start[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  Tile t;
  t.e = lo;
  const int local = tile - s_start[lo];
  const int c = s_hi[lo] - s_lo[lo];
  const int ntb = token_blocks(c, merge);
  int tb;
  if (fb_fastest) {
    tb = local / n_fb;
    t.fb = local - tb * n_fb;
  } else {
    t.fb = local / ntb;
    tb = local - t.fb * ntb;
  }
  t.row0 = s_lo[lo] + tb * BN;
  t.ntok = tb == ntb - 1 ? c - tb * BN : BN;  // up to BN_MAX when merged
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
// Then Phi(x) = 1 - Phi(-|x|) for x >= 0.  The result is within 0.75e-7 * |x|
// of the exact GELU, far below one bf16 ulp of the output.
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

// kMerge: merged last token blocks (paired CTAs, plain forms only)
template <bool kGelu, int kPair, bool kFp8, bool kGather, bool kFused, bool kMerge>
__global__ void __launch_bounds__(Roles<kGather, kPair>::THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_xw,
                        const __grid_constant__ CUtensorMap tm_w2,
                        const __grid_constant__ CUtensorMap tm_x2,
                        const __grid_constant__ CUtensorMap tm_xw2, const Args args) {
  using C = Cfg<kPair>;
  using Ro = Roles<kGather, kPair>;
  constexpr int KPS = C::KPS;
  constexpr int KB = kFp8 ? BK_FP8 : BK;  // K values per stage (128 bytes of a row)
  const int STAGES = args.stages;
  constexpr int B_STAGE = C::B_STAGE;
  static_assert(!kMerge || (kPair == 2 && !kGather && !kFused),
                "merged blocks: paired CTAs, neither gathered nor fused");
  constexpr bool merge = kMerge;
  // queue readers: the producers and epilogue warps of both CTAs and the
  // leader's MMA warp
  constexpr uint32_t kQReaders = kPair * Ro::NPROD + 1 + kPair * EPI_WARPS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * KPS * A_STAGE;  // slot s, K-block h: sA + (s*KPS + h)*A_STAGE
  uint8_t* sT = sB + STAGES * KPS * B_STAGE;  // merged tails: slot s, K-block h at (s*KPS + h)*B_BOX
  uint64_t* bars = reinterpret_cast<uint64_t*>(sT + (merge ? STAGES * KPS * B_BOX : 0));
  uint64_t* full = bars;                   // used in the leader CTA: both CTAs' bytes land here
  uint64_t* empty = bars + MAX_STAGES;     // per CTA: the MMAs have read this stage
  uint64_t* tfull = bars + 2 * MAX_STAGES; // per CTA: accumulator ready
  uint64_t* tempty = tfull + 2;        // leader CTA: both CTAs' epilogues drained it
  uint64_t* drain = tempty + 2;
  uint64_t* qfull = drain + 1;         // per CTA: queue slot holds the next item
  uint64_t* qempty = qfull + kQueue;   // leader CTA: every reader has taken the slot
  uint64_t* qprod = qempty + kQueue;   // leader CTA: its weight producer has taken an item
  uint64_t* tearly = qprod + 1;        // leader CTA: both CTAs' epilogues drained the columns
                                       // the next tile may share (drained first)
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(bars + C::NUM_BARS);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);
  volatile int* s_queue = reinterpret_cast<volatile int*>(s_tmem + 4);
  const int E = args.E;
  int* s_lo = reinterpret_cast<int*>(s_tmem + 4 + kQueue);
  int* s_hi = s_lo + (E + 1);
  int* s_start = s_hi + (E + 1);
  int* s_start2 = s_start + (E + 1);  // fused form: GEMM-2's per-expert first tile

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair == 2 ? cluster_ctarank() : 0u;  // 0 = MMA leader
  const int cid = blockIdx.x / kPair;                          // tile-scheduling unit
  const int ncl_launched = gridDim.x / kPair;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], Ro::FULL_ARRIVALS);  // the issuing warps of the leader CTA
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kPair * EPI_WARPS);
      mbar_init(&tearly[a], kPair * EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(&qfull[q], 1);
      mbar_init(&qempty[q], kQReaders);
    }
    mbar_init(qprod, 1);
    *s_abort = 0;
    fence_mbarrier_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_xw);
    if (kFused) {
      tma_prefetch_desc(&tm_w2);
      tma_prefetch_desc(&tm_x2);
      tma_prefetch_desc(&tm_xw2);
    }
  }
  if (warp == Ro::MMA) {
    tmem_alloc<kPair>(s_tmem, TMEM_COLS);
    tmem_relinquish<kPair>();
  }
  // The set-up above touches no global memory; from here on the kernel reads
  // its stream predecessors' results.  The GEMM releases its dependents only
  // at its end: their blocks would otherwise wait beside its warps for the
  // whole launch (measured on the fine-grained shape: +3 % per layer).
  pdl_wait();
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
    for (int e = e0; e < e1; ++e) sum += token_blocks(s_hi[e] - s_lo[e], merge) * args.n_fblocks;
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
      s_start[e] = run;
      run += token_blocks(s_hi[e] - s_lo[e], merge) * args.n_fblocks;
    }
    if (lane == 31) s_start[E] = incl;
    if (kFused) {  // GEMM-2's tiles: same token blocks, n_fblocks2 feature blocks each
      run = (incl - sum) / args.n_fblocks * args.n_fblocks2;
      for (int e = e0; e < e1; ++e) {
        s_start2[e] = run;
        run += token_blocks(s_hi[e] - s_lo[e], merge) * args.n_fblocks2;
      }
      if (lane == 31) s_start2[E] = incl / args.n_fblocks * args.n_fblocks2;
    }
  }
  tc_fence_before_sync();
  if (kPair == 2) cluster_sync();  // the peer's barriers are initialised before any remote use
  else __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  const int tiles0 = s_start[E];
  // Items, in the order clusters take them: dispatch chunks (fused form with
  // dispatch), then GEMM-1's tiles, then (fused form) GEMM-2's.  An item only
  // ever waits on items before it, so with tickets taken in this order every
  // wait ends, however many clusters are resident.
  const int kept = s_hi[E - 1];  // rows of kept slots: offsets[E], clamped
  const bool disp = kFused && !kGather && args.disp_X != nullptr && args.ticket != nullptr;
  const int n_disp = disp ? (kept + kDispRows - 1) / kDispRows : 0;
  const int total_items = n_disp + tiles0 + (kFused ? s_start2[E] : 0);
  // Static schedule (no ticket): balanced grid, the fewest clusters that
  // still need the same number of rounds (the tile count is known only here,
  // from the routing).  A last round with a few busy clusters would otherwise
  // set the kernel's time while most SMs idle; e.g. 448 tiles over 74
  // clusters run 6 full rounds and a seventh of 4 tiles, over 64 clusters 7
  // full rounds.  Surplus clusters take no tile.
  const int rounds = (total_items + ncl_launched - 1) / max(ncl_launched, 1);
  const int ncl = rounds > 0 ? (total_items + rounds - 1) / rounds : ncl_launched;
  // item -> (tile, phase); phase -1: dispatch chunk `chunk`; 1: GEMM-2 of the fused form
  auto item_at = [&](int x, int& phase, int& chunk) -> Tile {
    chunk = -1;
    if (x < n_disp) {
      phase = -1;
      chunk = x;
      return Tile{0, 0, 0, 0};
    }
    x -= n_disp;
    if (kFused && x >= tiles0) {
      phase = 1;
      return decode(x - tiles0, s_start2, s_lo, s_hi, E, args.fb_fastest2, args.n_fblocks2,
                    merge);
    }
    phase = 0;
    return decode(x, s_start, s_lo, s_hi, E, args.fb_fastest, args.n_fblocks, merge);
  };
  // fused form: index of the token block holding a tile's rows
  auto block_of = [&](const Tile& t) -> int {
    return s_start[t.e] / args.n_fblocks + (t.row0 - s_lo[t.e]) / BN;
  };
  // the leader's barriers as cluster addresses (the CTA's own when kPair == 1)
  const uint32_t full_lead = kPair == 2 ? cluster_map(smem_u32(full), 0) : smem_u32(full);
  const uint32_t tempty_lead = kPair == 2 ? cluster_map(smem_u32(tempty), 0) : smem_u32(tempty);
  const uint32_t tearly_lead = kPair == 2 ? cluster_map(smem_u32(tearly), 0) : smem_u32(tearly);
  const uint32_t qempty_lead = kPair == 2 ? cluster_map(smem_u32(qempty), 0) : smem_u32(qempty);

  // Static schedule: every role computes this cluster's i-th item itself.
  // Dynamic schedule (a ticket): queue slot i % kQueue carries this
  // cluster's i-th item (-1: no more).  fill(): the leader's scheduler warp
  // takes the next ticket and publishes the item in both CTAs; take(): every
  // role reads it.  Both are called by a whole warp; false = aborted.  The
  // scheduler claims item i + 1 once the weight producer has taken item i:
  // one item ahead, so the ticket's round trip to L2 is hidden behind a
  // tile, and a cluster never holds tiles it has not started while others
  // run dry at the end (claiming further ahead measured slower on uniform
  // tiles: up to a whole extra round).  kQueue slots cover the lag of the
  // slowest role (the epilogue).
  auto fill = [&](int i, int& item) -> bool {
    const int q = i % kQueue;
    const uint32_t ph = (uint32_t)(i / kQueue) & 1u;
    int v = -1;
    bool ok = true;
    if (lane == 0) {
      ok = mbar_wait_cluster(&qempty[q], ph ^ 1u, args.status, s_abort);
      if (ok) {
        if (args.ticket) {
          const uint32_t x = atomicAdd(args.ticket, 1u);
          v = x < (uint32_t)total_items ? (int)x : -1;
        } else {
          const long long x = (long long)cid + (long long)i * ncl;
          v = (cid < ncl && x < total_items) ? (int)x : -1;
        }
        s_queue[q] = v;
        if (kPair == 2) {
          st_shared_cluster_u32(cluster_map(smem_u32((const void*)(s_queue + q)), 1), (uint32_t)v);
          mbar_arrive_cluster(cluster_map(smem_u32(&qfull[q]), 1));
        }
        mbar_arrive(&qfull[q]);
      }
    }
    item = __shfl_sync(0xffffffffu, v, 0);
    return __shfl_sync(0xffffffffu, ok, 0);
  };
  const bool dyn = args.ticket != nullptr;
  auto static_item = [&](int i) -> int {
    const long long x = (long long)cid + (long long)i * ncl;
    return (cid < ncl && x < total_items) ? (int)x : -1;
  };
  auto take = [&](int i, int& item) -> bool {
    const int q = i % kQueue;
    const uint32_t ph = (uint32_t)(i / kQueue) & 1u;
    const bool got = mbar_wait_cluster(&qfull[q], ph, args.status, s_abort);
    if (!__all_sync(0xffffffffu, got)) {
      item = -1;
      return false;
    }
    item = s_queue[q];
    __syncwarp();
    if (lane == 0) mbar_arrive_cluster(qempty_lead + (uint32_t)q * 8u);
    return true;
  };
  auto next_item = [&](int i, int& item) -> bool {
    if (!dyn) {
      item = static_item(i);
      return true;
    }
    return take(i, item);
  };
  // The counters that gate a tile's token rows: GEMM-2 tiles wait for their
  // token block's H (GEMM-1 epilogue arrivals), GEMM-1 tiles of the fused
  // form with dispatch items for the chunks under their rows.
  auto gate = [&](const Tile& tt, bool ph1, const uint32_t*& cp, int& cn, uint32_t& tgt) {
    if (ph1) {
      cp = args.ready + block_of(tt);
      cn = 1;
      tgt = args.ready_target;
    } else {
      const int c0 = tt.row0 / kDispRows;
      cp = args.dready + c0;
      cn = (tt.row0 + tt.ntok - 1) / kDispRows - c0 + 1;  // <= BN / kDispRows + 1
      tgt = (uint32_t)(kPair * EPI_WARPS);
    }
  };
  constexpr int kMaxGate = BN / kDispRows + 1;

  if (warp < Ro::NPROD) {
    // ------------------------------------------------------------ producers (both CTAs)
    // Warp 0 streams the weight rows, warp 1 (and in the gather form warps
    // 2..NTOK) the token rows, each into the same ring of stages: separate
    // issuing threads keep more TMA requests in flight than one.  In the
    // leader CTA warps 0 and 1 arm the stage's barrier with the bytes of
    // their operand in both CTAs of the pair.
    const bool is_w = warp < Ro::NW;
    const int tw = warp - Ro::NW;  // token warp index
    const uint64_t pol = is_w ? (MOE_W_EVICT_FIRST ? l2_policy_evict_first() : l2_policy_evict_normal())
                              : l2_policy_evict_last();   // re-read by every feature block
    int s = 0;
    uint32_t ph = 0;
    uint32_t issued = 0;  // bit s: stage s has a load in flight or landed
    uint32_t last_ph = 0; // bit s: parity of the last load issued on stage s
    bool ok = true;
    // token producers, dynamic schedule: the gate counters of the next item,
    // loaded while this item's loads are issued (counts only grow, so a
    // complete count seen early stays complete)
    int peek_x = -1, peek_n = 0;
    uint32_t peek_v[kMaxGate], peek_tgt = 0;
    for (int qi = 0; ok; ++qi) {
      int x;
      ok = next_item(qi, x);
      if (!ok || x < 0) break;
      if (dyn && warp == 0 && rank == 0 && lane == 0) mbar_arrive(qprod);  // claim the next
      int phase, chunk;
      const Tile t = item_at(x, phase, chunk);
      if (phase < 0) continue;  // a dispatch chunk: the epilogue warps copy it
      const bool p1 = kFused && phase == 1;
      const CUtensorMap* map_w = p1 ? &tm_w2 : &tm_w;
      const CUtensorMap* map_x = p1 ? &tm_x2 : &tm_x;
      const CUtensorMap* map_xw = p1 ? &tm_xw2 : &tm_xw;
      const int kbv = (kFp8 && !p1) ? BK_FP8 : BK;  // K values per stage in this phase
      const int nkb = p1 ? args.num_kb2 : args.num_kb;
      const int Np = p1 ? args.N2 : args.N;
      if (!is_w && (p1 || disp)) {
        // Token rows written by other CTAs in this launch: GEMM-2 reads H rows
        // that GEMM-1 tiles store, GEMM-1 (with dispatch items) reads rows
        // that dispatch chunks copy.  Wait (bounded) for their counts, acquire,
        // then order those generic-proxy stores before our TMA reads.
        bool rdy = true;
        if (lane == 0) {
          const uint32_t* cp;
          int cn;
          uint32_t tgt;
          gate(t, p1, cp, cn, tgt);
          bool early = x == peek_x;  // counts read one item ahead, all complete?
#pragma unroll
          for (int i = 0; i < kMaxGate; ++i)
            if (i < peek_n) early &= peek_v[i] >= peek_tgt;
          if (early) fence_acq_rel_gpu();
          else rdy = wait_counts_geq(cp, cn, tgt, args.status, s_abort);
          if (rdy) fence_proxy_async_global();
        }
        if (!__shfl_sync(0xffffffffu, rdy, 0)) {
          ok = false;
          break;
        }
      }
      const int nmma = (t.ntok + 15) & ~15;
      // a merged tile's first 256 rows, then its tail (a second MMA)
      const int nmain = (kMerge && nmma > BN) ? BN : nmma;
      const int half = nmain / kPair;  // token rows staged by this CTA (a multiple of 8)
      const bool wide = half >= kWideMin;
      const int nbox = (half + B_BOX_ROWS - 1) / B_BOX_ROWS;
      // wide boxes of 128 rows: one with paired CTAs (half <= 128), up to two
      // with a single CTA (half <= 256); the stage holds BN / kPair rows
      const int nwide = (half + B_WIDE_ROWS - 1) / B_WIDE_ROWS;
      // merged tile: this CTA's half of the tail (8..32 rows), one 32-row box
      // in the tail ring (a merged tile's first half-tile is 128 rows: wide)
      const int half2 = (nmma - nmain) / kPair;
      const int nbox2 = (kMerge && half2 > 0) ? 1 : 0;
      const uint32_t bytes = is_w ? (uint32_t)(kPair * A_STAGE)
                                  : (uint32_t)kPair * ((wide ? nwide * B_WIDE_ROWS * BK * 2
                                                             : nbox * B_BOX) +
                                                       nbox2 * B_BOX);
      const int wy = t.e * Np + t.fb * C::FEAT + (int)rank * BM;
      // weight prefetch: this CTA's 128 weight rows, 4 per lane
      const uint8_t* wrow = (p1 ? args.w2_ptr : args.w_ptr) +
                            (size_t)(wy + lane) * (size_t)(p1 ? args.w2_pitch : args.w_pitch);
      const size_t wstep = (size_t)32 * (size_t)(p1 ? args.w2_pitch : args.w_pitch);
      const int wpf = args.w_prefetch;
      if (wpf > 0 && is_w) {
        const int nrow = min(BM, Np - (wy - t.e * Np));
        for (int kb = 0; kb < min(wpf, nkb); ++kb)
#pragma unroll
          for (int r4 = 0; r4 < 4; ++r4)
            if (lane + 32 * r4 < nrow) prefetch_l2(wrow + r4 * wstep + (size_t)kb * 128);
      }
      const int by = t.row0 + (int)rank * half;
      // gather form: request q (4 rows) of this CTA's half-tile is issued
      // by token warp q % NTOK, lane q / NTOK % 32 (up to 64 requests: 256
      // rows with a single CTA); the token ids are read once per tile.  Rows
      // past the expert's block (the MMA's padding to a multiple of 16) read
      // token 0 and are never stored.
      const int nreq = half / 4;
      int g[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
      if (kGather && !is_w) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int q = (lane + 32 * h) * Ro::NTOK + tw;
          if (q >= nreq) continue;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int local = (int)rank * half + q * 4 + i;
            int row = 0;
            if (local < t.ntok) {
              const int src = __ldg(args.gather_src + t.row0 + local);
              if (src >= 0 && src < args.a_rows * args.gather_k) row = src / args.gather_k;
              else flag_error(args.status, MOE_DEV_BAD_ROW);
            }
            g[h][i] = row;
          }
        }
      }
      const uint32_t gbytes = (uint32_t)(kPair * half * 128);
      // dynamic schedule: look for the next item while this one streams (it
      // is published about one ticket round trip after this one was taken)
      bool peeking = dyn && !is_w && lane == 0;
      if (peeking) {
        peek_x = -1;
        peek_n = 0;
      }
      for (int ks = 0; ks * KPS < nkb; ++ks) {  // ring slot of K-blocks ks*KPS ..
        const int nsub = min(KPS, nkb - ks * KPS);
        if (peeking) {
          const int q1 = (qi + 1) % kQueue;
          if (mbar_try_wait_cluster(&qfull[q1], (uint32_t)((qi + 1) / kQueue) & 1u)) {
            peeking = false;
            const int xn = s_queue[q1];
            int phn = -1, chn;
            const Tile tn = xn >= 0 ? item_at(xn, phn, chn) : Tile{0, 0, 0, 0};
            const bool p1n = kFused && phn == 1;
            if (phn >= 0 && (p1n || disp)) {  // its gate counts, loaded while we stream
              const uint32_t* cpn;
              gate(tn, p1n, cpn, peek_n, peek_tgt);
#pragma unroll
              for (int i = 0; i < kMaxGate; ++i)
                if (i < peek_n) peek_v[i] = ld_relaxed_gpu(cpn + i);
              peek_x = xn;
            }
          }
        }
        ok = warp_wait(&empty[s], ph ^ 1u, args.status, s_abort);
        if (!ok) break;
        if (wpf > 0 && is_w) {  // K-blocks wpf ahead
          const int nrow = min(BM, Np - (wy - t.e * Np));
          for (int hh = 0; hh < nsub; ++hh) {
            const int kb = ks * KPS + hh + wpf;
            if (kb < nkb) {
#pragma unroll
              for (int r4 = 0; r4 < 4; ++r4)
                if (lane + 32 * r4 < nrow) prefetch_l2(wrow + r4 * wstep + (size_t)kb * 128);
            }
          }
        }
        if (kGather && !is_w) {
          const uint32_t fb_addr = full_lead + (uint32_t)s * 8u;
          if (tw == 0 && lane == 0 && rank == 0)
            mbar_arrive_expect_tx(&full[s], gbytes * (uint32_t)nsub);
          for (int hh = 0; hh < nsub; ++hh) {
            const int kb = ks * KPS + hh;
            uint8_t* dst = sB + (s * KPS + hh) * B_STAGE;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int q = (lane + 32 * h) * Ro::NTOK + tw;
              if (q < nreq)
                tma_gather4_cg<kPair>(dst + q * 512, &tm_x, kb * KB, g[h][0], g[h][1], g[h][2],
                                      g[h][3], fb_addr, pol);
            }
          }
        } else if (lane == 0) {
          const uint32_t fb_addr = full_lead + (uint32_t)s * 8u;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], bytes * (uint32_t)nsub);
          for (int hh = 0; hh < nsub; ++hh) {  // one request per operand and K-block
            const int kb = ks * KPS + hh;
            if (is_w) {
              tma_load_2d_cg<kPair>(sA + (s * KPS + hh) * A_STAGE, map_w, kb * kbv, wy, fb_addr,
                                    pol);
            } else if (wide) {  // (nearly) full 128-row boxes: large requests
              for (int j = 0; j < nwide; ++j)
                tma_load_2d_cg<kPair>(sB + (s * KPS + hh) * B_STAGE + j * B_WIDE_ROWS * 128,
                                      map_xw, kb * kbv, by + j * B_WIDE_ROWS, fb_addr, pol);
              if (kMerge && nbox2)  // a merged tile's tail rows, into the tail ring
                tma_load_2d_cg<kPair>(sT + (s * KPS + hh) * B_BOX, map_x, kb * kbv,
                                      t.row0 + BN + (int)rank * half2, fb_addr, pol);
            } else {
              for (int j = 0; j < nbox; ++j)
                tma_load_2d_cg<kPair>(sB + (s * KPS + hh) * B_STAGE + j * B_BOX, map_x, kb * kbv,
                                      by + j * B_BOX_ROWS, fb_addr, pol);
            }
          }
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
    if (!ok && rank == 0 && warp == 0) {  // let issued copies land before the CTA leaves
      int dummy = 0;
      for (int q = 0; q < STAGES; ++q)
        if ((issued >> q) & 1u)
          mbar_wait(&full[q], (last_ph >> q) & 1u, nullptr, (volatile int*)&dummy, kDrainLimitNs);
    }
  } else if (warp == Ro::SCHED) {
    // ------------------------------------------------------------ scheduler (leader, tickets)
    if (rank == 0 && dyn) {
      for (int qi = 0;; ++qi) {
        // item qi - 1 taken by the weight producer (bounded wait)
        if (qi > 0 && !warp_wait(qprod, (uint32_t)(qi - 1) & 1u, args.status, s_abort)) break;
        int x;
        if (!fill(qi, x) || x < 0) break;
      }
    }
  } else if (warp == Ro::MMA) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0) {
      int s = 0;
      uint32_t ph = 0;
      int it = 0;  // GEMM tiles so far (selects the accumulator)
      int prev_lo = 0, prev_hi = 0;  // TMEM columns of the previous tile's accumulator
      bool ok = true;
      for (int qi = 0; ok; ++qi) {
        int x;
        ok = next_item(qi, x);
        if (!ok || x < 0) break;
        int phase, chunk;
        const Tile t = item_at(x, phase, chunk);
        if (phase < 0) continue;
        const bool p1 = kFused && phase == 1;
        const bool f8 = kFp8 && !p1;  // GEMM-2 of the fused form is bf16
        const int nkb = p1 ? args.num_kb2 : args.num_kb;
        const uint32_t nmma = (uint32_t)((t.ntok + 15) & ~15);
        // a merged tile (nmma > 256): N = 256, then N = the tail at column +256
        const uint32_t n1 = (kMerge && nmma > (uint32_t)BN) ? (uint32_t)BN : nmma;
        const uint32_t n2 = kMerge ? nmma - n1 : 0u;
        const uint32_t idesc = f8 ? idesc_e4m3_f32((uint32_t)C::FEAT, n1)
                                  : idesc_bf16_f32((uint32_t)C::FEAT, n1);
        const uint32_t idesc2 = n2 == 0 ? 0u
                                : f8 ? idesc_e4m3_f32((uint32_t)C::FEAT, n2)
                                     : idesc_bf16_f32((uint32_t)C::FEAT, n2);
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)((it >> 1) & 1);
        const int base = acc_base(acc, (int)nmma, merge);
        // the tile before this one used the other buffer: if their columns
        // overlap, wait until its epilogue has drained the shared ones
        const bool shares = kMerge && it > 0 && prev_lo < base + (int)nmma && base < prev_hi;
        const uint32_t pph = (uint32_t)(((it - 1) >> 1) & 1);
        prev_lo = base;
        prev_hi = base + (int)nmma;
        ++it;
        ok = warp_wait(&tempty[acc], aph ^ 1u, args.status, s_abort);
        if (ok && shares) ok = warp_wait(&tearly[acc ^ 1], pph, args.status, s_abort);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem_base + (uint32_t)base;
        for (int ks = 0; ks * KPS < nkb; ++ks) {
          const int nsub = min(KPS, nkb - ks * KPS);
          ok = warp_wait(&full[s], ph, args.status, s_abort);
          if (!ok) break;
          tc_fence_after_sync();
          if (lane == 0) {
            if (!kMerge || n2 == 0) {
              for (int hh = 0; hh < nsub; ++hh) {
                const int kb = ks * KPS + hh;
                const uint32_t a0 = smem_u32(sA + (s * KPS + hh) * A_STAGE);
                const uint32_t b0 = smem_u32(sB + (s * KPS + hh) * B_STAGE);
#pragma unroll
                for (int kk = 0; kk < 128 / UMMA_K_BYTES; ++kk) {
                  const uint64_t ad = smem_desc_k128(a0 + kk * UMMA_K_BYTES);
                  const uint64_t bd = smem_desc_k128(b0 + kk * UMMA_K_BYTES);
                  if (f8)
                    tc_mma_e4m3<kPair>(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                  else
                    tc_mma_bf16<kPair>(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                }
              }
            } else {  // merged tile: N = 256, then the tail from the tail ring
              for (int hh = 0; hh < nsub; ++hh) {
                const int kb = ks * KPS + hh;
                const uint32_t a0 = smem_u32(sA + (s * KPS + hh) * A_STAGE);
                const uint32_t b0 = smem_u32(sB + (s * KPS + hh) * B_STAGE);
                const uint32_t t0 = smem_u32(sT + (s * KPS + hh) * B_BOX);
#pragma unroll
                for (int kk = 0; kk < 128 / UMMA_K_BYTES; ++kk) {
                  const uint64_t ad = smem_desc_k128(a0 + kk * UMMA_K_BYTES);
                  const uint64_t bd = smem_desc_k128(b0 + kk * UMMA_K_BYTES);
                  const uint64_t td = smem_desc_k128(t0 + kk * UMMA_K_BYTES);
                  const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
                  if (f8) {
                    tc_mma_e4m3<kPair>(d_tmem, ad, bd, idesc, accum);
                    tc_mma_e4m3<kPair>(d_tmem + (uint32_t)BN, ad, td, idesc2, accum);
                  } else {
                    tc_mma_bf16<kPair>(d_tmem, ad, bd, idesc, accum);
                    tc_mma_bf16<kPair>(d_tmem + (uint32_t)BN, ad, td, idesc2, accum);
                  }
                }
              }
            }
            // the stage is free (in both CTAs) once these MMAs have read it
            if (kPair == 2) tc_commit_pair(smem_u32(&empty[s]));
            else tc_commit<kPair>(smem_u32(&empty[s]));
          }
          __syncwarp();
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) {  // accumulator complete, in both CTAs
          if (kPair == 2) tc_commit_pair(smem_u32(&tfull[acc]));
          else tc_commit<kPair>(smem_u32(&tfull[acc]));
        }
        __syncwarp();
      }
      if (!ok) {  // wait for every MMA already issued before TMEM is freed
        if (lane == 0) tc_commit<kPair>(smem_u32(drain));
        __syncwarp();
        int dummy = 0;
        mbar_wait(drain, 0, nullptr, (volatile int*)&dummy, kDrainLimitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    // the tile's 32-column chunks are dealt out round robin over NSPAN warps
    // per lane quarter: this warp takes chunks hsel, hsel + NSPAN, ...
    constexpr int NSPAN = EPI_WARPS / 4;
    const int hsel = (warp - Ro::EPI0) >> 2;
    int it = 0;  // GEMM tiles so far
    for (int qi = 0;; ++qi) {
      int x;
      if (!next_item(qi, x) || x < 0) break;
      int phase, chunk;
      const Tile t = item_at(x, phase, chunk);
      if (phase < 0) {
        // ---- dispatch chunk: A[r] = X[src_of[r] / k] for rows [r0, r1), by
        // the epilogue warps of both CTAs, then one arrival per warp
        const int w = (int)rank * EPI_WARPS + (warp - Ro::EPI0);
        const int r0 = chunk * kDispRows, r1 = min(r0 + kDispRows, kept);
        const int vecs = args.disp_vecs;
        const int nslots = args.disp_T * args.disp_k;
        for (int r = r0 + w; r < r1; r += kPair * EPI_WARPS) {
          const int src = __ldg(args.disp_src + r);
          if (src < 0 || src >= nslots) {
            if (lane == 0) flag_error(args.status, MOE_DEV_BAD_ROW);
            continue;
          }
          const uint4* from = args.disp_X + (size_t)(src / args.disp_k) * vecs;
          uint4* to = args.disp_A + (size_t)r * vecs;
          for (int c0 = 0; c0 < vecs; c0 += 32 * kDispUnroll) {
            uint4 v[kDispUnroll];
#pragma unroll
            for (int u = 0; u < kDispUnroll; ++u) {
              const int c = c0 + u * 32 + lane;
              if (c < vecs) v[u] = ld_stream_v4(from + c);
            }
#pragma unroll
            for (int u = 0; u < kDispUnroll; ++u) {
              const int c = c0 + u * 32 + lane;
              if (c < vecs) to[c] = v[u];
            }
          }
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(args.dready + chunk, 1u);
        continue;
      }
      const bool p1 = kFused && phase == 1;
      const bool f8 = kFp8 && !p1;
      const bool gelu = kGelu && !p1;  // the fused form's GEMM-2 has no activation
      // gate-weighted combine in this epilogue (GEMM-2: no activation)
      const bool comb = args.comb_Y != nullptr && !gelu;
      uint16_t* out = p1 ? args.out2 : args.out;
      const int N = p1 ? args.N2 : args.N;
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)((it >> 1) & 1);
      ++it;
      const int nmma = (t.ntok + 15) & ~15;
      const int base = acc_base(acc, nmma, merge);
      // Columns of this accumulator (relative to base) that the next tile may
      // reuse, drained first: a low tile's from column 192 on (a high tile
      // starts there at the earliest), a high tile's below column 320 (where
      // a low tile ends at the latest).  None without merged blocks.
      const int ov0 = acc == 0 ? kHighMin : 0;
      const int ov1 = !merge ? 0 : acc == 0 ? nmma : BN_MAX - base;
      if (!warp_wait(&tfull[acc], aph, args.status, s_abort)) break;
      tc_fence_after_sync();
      // this lane's output feature; the warp covers 32 consecutive features
      const int f0 = t.fb * C::FEAT + (int)rank * BM + q * 32;
      const int f = f0 + lane;
      const float sc = f8 ? __ldg(args.a_scale) * __ldg(args.w_scale + t.e) : 1.0f;
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)base;
      const int nch = (t.ntok + 31) >> 5;
      // one 32-column chunk of the accumulator: tokens c0 .. c0 + 31
      auto drain_chunk = [&](const int c0) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + (uint32_t)c0, v);
        tmem_wait_ld();
        // v[j] = accumulator of feature f, token (c0 + j).  For a fixed j the
        // warp writes 32 consecutive features of one token row: 64 contiguous
        // bytes per store instruction, no shared-memory transpose needed.
        const int jmax = min(32, t.ntok - c0);
        if (!comb) {
          uint16_t* col = out + (size_t)(t.row0 + c0) * N + f;
          if (f < N) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              float x = __uint_as_float(v[j]);
              if (f8) x *= sc;
              if (gelu) x = gelu_erf(x);
              if (j < jmax) col[(size_t)j * N] = to_bf16_bits(x);
            }
          }
          return;
        }
        // ---- combine: lane j describes token column j of this chunk.  A warp
        // whose 32 features all lie past N (last feature block) has nothing
        // to write, and its counter index would name the next token's word.
        if (f0 >= N) return;
        int tok = 0, mode = 0;  // mode 1: the token's only kept slot; 2: one of two
        float g = 0.f;
        if (lane < jmax) {
          const int sl = __ldg(args.comb_src + t.row0 + c0 + lane);
          if (sl >= 0 && sl < args.comb_T * args.comb_k) {
            tok = sl / args.comb_k;
            g = __ldg(args.comb_gates + sl);
            // k == 2: the token's slots are 2t and 2t + 1
            mode = (args.comb_k == 2 && __ldg(args.comb_row_of + (sl ^ 1)) >= 0) ? 2 : 1;
          } else {
            flag_error(args.status, MOE_DEV_BAD_ROW);
          }
        }
        uint32_t* cw = args.comb_cnt + (size_t)tok * (uint32_t)((N + 31) >> 5) + (f0 >> 5);
        const uint32_t old = mode == 2 ? atomicAdd(cw, 1u) : 0u;
        const uint32_t sole = __ballot_sync(0xffffffffu, mode == 1);
        const uint32_t first = __ballot_sync(0xffffffffu, mode == 2 && old == 0u);
        const uint32_t second = __ballot_sync(0xffffffffu, mode == 2 && old != 0u);
        // Products and the sum are rounded explicitly (no fused multiply-add),
        // so a token's two results give the same bits whichever arrives second.
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int tj = __shfl_sync(0xffffffffu, tok, j);
          const float gj = __shfl_sync(0xffffffffu, g, j);
          const float y = __fmul_rn(gj, __uint_as_float(v[j]));
          if (f < N) {
            if ((sole >> j) & 1u) args.comb_Y[(size_t)tj * N + f] = to_bf16_bits(y);
            else if ((first >> j) & 1u) args.comb_part[(size_t)tj * N + f] = y;
          }
        }
        if (first) {  // publish the partials, then one flag per token
          __threadfence();
          __syncwarp();
          if ((first >> lane) & 1u) atomicOr(cw, 0x100u);
        }
        if (second) {  // the partner slot's flag, then its partial
          bool got = true;
          if ((second >> lane) & 1u) got = wait_bits_set(cw, 0x100u, args.status, s_abort);
          if (!__all_sync(0xffffffffu, got)) return;
          __threadfence();
          // the partners' partial rows, 8 loads in flight at a time
#pragma unroll
          for (int j0 = 0; j0 < 32; j0 += 8) {
            float p[8];
#pragma unroll
            for (int j = j0; j < j0 + 8; ++j) {
              const int tj = __shfl_sync(0xffffffffu, tok, j);
              p[j - j0] = (((second >> j) & 1u) && f < N)
                              ? __ldcg(args.comb_part + (size_t)tj * N + f) : 0.f;
            }
#pragma unroll
            for (int j = j0; j < j0 + 8; ++j) {
              const int tj = __shfl_sync(0xffffffffu, tok, j);
              const float gj = __shfl_sync(0xffffffffu, g, j);
              if (((second >> j) & 1u) && f < N) {
                const float y = __fmul_rn(gj, __uint_as_float(v[j]));
                args.comb_Y[(size_t)tj * N + f] = to_bf16_bits(__fadd_rn(p[j - j0], y));
              }
            }
          }
        }
      };
      if constexpr (!kMerge) {  // each warp a contiguous span of the tile's columns
        constexpr int SPAN = BN / NSPAN;
        const int c_end = min(t.ntok, hsel * SPAN + SPAN);
        for (int c0 = hsel * SPAN; c0 < c_end; c0 += 32) drain_chunk(c0);
      } else {
        // chunks dealt out round robin; first those the next tile may reuse,
        // then a tearly arrival, then the others
        for (int ch = hsel; ch < nch; ch += NSPAN)
          if (ch * 32 + 32 > ov0 && ch * 32 < ov1) drain_chunk(ch * 32);
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tearly_lead + (uint32_t)acc * 8u);
        for (int ch = hsel; ch < nch; ch += NSPAN)
          if (!(ch * 32 + 32 > ov0 && ch * 32 < ov1)) drain_chunk(ch * 32);
      }
      if (kFused && !p1) {  // publish this warp's part of H for GEMM-2's tiles
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicAdd(args.ready + block_of(t), 1u);
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_lead + (uint32_t)acc * 8u);
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  pdl_release();
  if (kPair == 2) cluster_sync();  // no CTA leaves while its peer may still signal it
  if (warp == Ro::MMA) {
    tc_fence_after_sync();
    tmem_dealloc<kPair>(tmem_base, TMEM_COLS);
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

// 2-D map over a row-major [rows, cols] matrix of bf16 (fp8 = false) or
// 1-byte E4M3 codes (fp8 = true); box = box_rows x 128 bytes of columns,
// 128-byte swizzle (the layout the MMA descriptors expect).
static bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows, bool fp8, std::string* err) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) {
    *err = "cuTensorMapEncodeTiled is unavailable from the driver";
    return false;
  }
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * (fp8 ? 1 : 2)};
  const cuuint32_t box[2] = {(cuuint32_t)(fp8 ? gg::BK_FP8 : gg::BK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    *err = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return false;
  }
  return true;
}

struct KernelSlot {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int max_clusters = 0;  // co-resident clusters (pairs) or CTAs of this kernel
};
static KernelSlot g_slots[64][64];

template <bool kGelu, int kPair, bool kFp8, bool kGather, bool kFused = false, bool kMerge = false>
static cudaError_t launch_variant(const CUtensorMap& tm_w, const CUtensorMap& tm_x,
                                  const CUtensorMap& tm_xw, const gg::Args& args, long long max_tiles, const DeviceInfo& dev,
                                  cudaStream_t stream, const CUtensorMap* tm2 = nullptr) {
  auto kern = gg::grouped_gemm_kernel<kGelu, kPair, kFp8, kGather, kFused, kMerge>;
  const size_t smem_max = gg::kSmemBudget;  // one attribute for every E
  const int slot =
      (kGelu ? 1 : 0) + (kPair == 2 ? 2 : 0) + (kFp8 ? 4 : 0) + (kGather ? 8 : 0) + (kFused ? 16 : 0) +
      (kMerge ? 32 : 0);
  KernelSlot& ks = g_slots[dev.device & 63][slot];
  std::call_once(ks.once, [&] {
    ks.err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
    if (ks.err != cudaSuccess) return;
    if (kPair == 2) {
      cudaLaunchConfig_t cfg = {};
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.gridDim = dim3(2 * dev.sm_count, 1, 1);
      cfg.blockDim = dim3(gg::Roles<kGather, kPair>::THREADS, 1, 1);
      cfg.dynamicSmemBytes = smem_max;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      ks.err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      ks.max_clusters = n;
    } else {
      ks.max_clusters = dev.sm_count;
    }
  });
  if (ks.err != cudaSuccess) return ks.err;
  if (ks.max_clusters < 1) return cudaErrorInvalidConfiguration;
  const long long units = max_tiles < ks.max_clusters ? max_tiles : ks.max_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kPair;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((unsigned)(units * kPair), 1, 1);
  cfg.blockDim = dim3(gg::Roles<kGather, kPair>::THREADS, 1, 1);
  cfg.dynamicSmemBytes = gg::smem_bytes<kPair>(args.E, args.stages, kMerge);
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  // the fused form's GEMM-2 maps; the other forms pass copies they never read
  const CUtensorMap& w2 = tm2 ? tm2[0] : tm_w;
  const CUtensorMap& x2 = tm2 ? tm2[1] : tm_x;
  const CUtensorMap& xw2 = tm2 ? tm2[2] : tm_xw;
  return cudaLaunchKernelEx(&cfg, kern, tm_w, tm_x, tm_xw, w2, x2, xw2, args);
}

int combine_counter_words(int T, int N) { return T * ((N + 31) / 32); }
int dispatch_counter_words(int R) { return (R + gg::kDispRows - 1) / gg::kDispRows; }

// Copies the optional parts of a launch into the kernel arguments.
static void apply_extras(gg::Args& args, const GemmExtras* ex) {
  if (!ex) return;
  args.ticket = ex->ticket;
  args.comb_Y = static_cast<uint16_t*>(ex->comb_Y);
  args.comb_src = ex->comb_src;
  args.comb_row_of = ex->comb_row_of;
  args.comb_gates = ex->comb_gates;
  args.comb_part = ex->comb_part;
  args.comb_cnt = ex->comb_cnt;
  args.comb_k = ex->comb_k;
  args.comb_T = ex->comb_T;
}

// Gather form: A is the token matrix [a_rows, K] and row r of the GEMM reads
// A[gather_src[r] / gather_k]; otherwise A is [R, K] and gather_src is null.
template <bool kFp8>
static cudaError_t launch_gemm(const void* A, const float* a_scale, const int32_t* gather_src,
                               int gather_k, int a_rows, const int32_t* offsets, const void* W,
                               const float* w_scale, int E, int R, int N, int K, bool gelu,
                               void* out, const DeviceInfo& dev, cudaStream_t stream,
                               std::string* err, const GemmExtras* ex = nullptr) {
  if (R == 0 || N == 0) return cudaSuccess;
  const bool gather = gather_src != nullptr;
  // Paired CTAs (256 features per tile) unless the layer is too narrow to fill them.
  const int pair = N > gg::BM ? 2 : 1;
  CUtensorMap tm_w, tm_x, tm_xw;
  if (!make_map(&tm_w, W, (uint64_t)E * (uint64_t)N, (uint64_t)K, gg::BM, kFp8, err))
    return cudaErrorInvalidValue;
  if (gather) {  // one-row boxes for gather4; the wide map is unused
    if (!make_map(&tm_x, A, (uint64_t)a_rows, (uint64_t)K, 1, kFp8, err))
      return cudaErrorInvalidValue;
    tm_xw = tm_x;
  } else if (!make_map(&tm_x, A, (uint64_t)R, (uint64_t)K, gg::B_BOX_ROWS, kFp8, err) ||
             !make_map(&tm_xw, A, (uint64_t)R, (uint64_t)K, gg::B_WIDE_ROWS, kFp8, err)) {
    return cudaErrorInvalidValue;
  }
  gg::Args args = {};
  args.offsets = offsets;
  args.out = static_cast<uint16_t*>(out);
  args.status = dev.status;
  args.a_scale = a_scale;
  args.w_scale = w_scale;
  args.w_ptr = static_cast<const uint8_t*>(W);
  args.w_pitch = K * (kFp8 ? 1 : 2);
  args.w_prefetch = R <= gg::kWPrefetchMaxRows * E ? gg::kWPrefetchSmall : 0;
  args.gather_src = gather_src;
  args.gather_k = gather_k;
  args.a_rows = a_rows;
  args.E = E;
  args.R = R;
  args.N = N;
  args.K = K;
  args.n_fblocks = (N + gg::BM * pair - 1) / (gg::BM * pair);
  const int kb = kFp8 ? gg::BK_FP8 : gg::BK;
  args.num_kb = (K + kb - 1) / kb;
  args.stages = pair == 2 ? gg::stages_for<2>(E) : gg::stages_for<1>(E);
#ifndef MOE_MERGE_TAILS
#define MOE_MERGE_TAILS 1
#endif
  // Merged last token blocks (paired CTAs, tokens by rows, few rows per
  // expert): each slot also holds 4 KB tail boxes, which costs no ring slot
  // as long as as many slots still fit (E up to ~600).
  bool merge = false;
  if (MOE_MERGE_TAILS && pair == 2 && !gather && (long long)R > (long long)gg::kMergeMinMeanRows * E &&
      (long long)R <= (long long)gg::kMergeMaxMeanRows * E) {
    const int st = gg::stages_for<2>(E, true);
    if (st >= args.stages) {
      merge = true;
      args.stages = st;
    }
  }
  apply_extras(args, ex);
  if (gelu) args.comb_Y = nullptr;  // the combine belongs to the GEMM without activation
#ifndef MOE_GEMM2_FB_FASTEST
#define MOE_GEMM2_FB_FASTEST 0
#endif
  // Token block fastest for both GEMMs.  Feature block fastest for GEMM-2
  // (each block of H shared by its feature-block tiles at once) measured
  // more DRAM reads on the Mixtral shape (1.66 vs 1.41 GB, the W2 blocks
  // then being read again) at the same time; it stays a build option.
  args.fb_fastest = !gelu && MOE_GEMM2_FB_FASTEST;
  // an upper bound on the tile count: every expert adds at most one partial token block
  const long long max_tiles =
      ((long long)(R + gg::BN - 1) / gg::BN + E) * (long long)args.n_fblocks;
#define MOE_GG_LAUNCH(G, P, GA) \
  launch_variant<G, P, kFp8, GA>(tm_w, tm_x, tm_xw, args, max_tiles, dev, stream)
  if (merge)
    return gelu ? launch_variant<true, 2, kFp8, false, false, true>(tm_w, tm_x, tm_xw, args,
                                                                     max_tiles, dev, stream)
                : launch_variant<false, 2, kFp8, false, false, true>(tm_w, tm_x, tm_xw, args,
                                                                      max_tiles, dev, stream);
  if (gather) {
    if (pair == 2) return gelu ? MOE_GG_LAUNCH(true, 2, true) : MOE_GG_LAUNCH(false, 2, true);
    return gelu ? MOE_GG_LAUNCH(true, 1, true) : MOE_GG_LAUNCH(false, 1, true);
  }
  if (pair == 2) return gelu ? MOE_GG_LAUNCH(true, 2, false) : MOE_GG_LAUNCH(false, 2, false);
  return gelu ? MOE_GG_LAUNCH(true, 1, false) : MOE_GG_LAUNCH(false, 1, false);
#undef MOE_GG_LAUNCH
}

cudaError_t launch_grouped_gemm(const void* A, const int32_t* offsets, const void* W, int E,
                                int R, int N, int K, bool gelu, void* out,
                                const DeviceInfo& dev, cudaStream_t stream, std::string* err,
                                const GemmExtras* ex) {
  return launch_gemm<false>(A, nullptr, nullptr, 1, R, offsets, W, nullptr, E, R, N, K, gelu,
                            out, dev, stream, err, ex);
}

cudaError_t launch_grouped_gemm_fp8(const void* Aq, const float* a_scale, const int32_t* offsets,
                                    const void* Wq, const float* w_scale, int E, int R, int N,
                                    int K, bool gelu, void* out, const DeviceInfo& dev,
                                    cudaStream_t stream, std::string* err, const GemmExtras* ex) {
  return launch_gemm<true>(Aq, a_scale, nullptr, 1, R, offsets, Wq, w_scale, E, R, N, K, gelu,
                           out, dev, stream, err, ex);
}

// Fused FFN: H = act(A W1[e]^T) (A = Xe, bf16 or E4M3 codes), then
// Ye = H W2[e]^T, in one persistent launch.  `ctr` holds the ticket (word 0)
// and one readiness counter per token block (ffn_ready_count).
int ffn_ready_count(int R, int E) { return (R + gg::BN - 1) / gg::BN + E; }
int ffn_counter_words(int R, int E) { return 1 + ffn_ready_count(R, E); }

cudaError_t launch_fused_ffn(const void* A, const float* a_scale, const int32_t* offsets,
                             const void* W1, const float* w1_scale, const void* W2, int E, int R,
                             int d, int f, bool fp8, void* H, void* Ye, uint32_t* ctr,
                             bool zeroed, const DeviceInfo& dev, cudaStream_t stream,
                             std::string* err, const GemmExtras* ex) {
  if (R == 0) return cudaSuccess;
  if (!zeroed) {
    cudaError_t e = cudaMemsetAsync(ctr, 0, (size_t)ffn_counter_words(R, E) * sizeof(uint32_t),
                                    stream);
    if (e != cudaSuccess) return e;
  }
  // one pair setting for both phases: paired CTAs when both GEMMs are wide enough
  const int pair = (f > gg::BM && d > gg::BM) ? 2 : 1;
  CUtensorMap tm_w, tm_x, tm_xw, tm2[3];
  if (!make_map(&tm_w, W1, (uint64_t)E * (uint64_t)f, (uint64_t)d, gg::BM, fp8, err) ||
      !make_map(&tm_x, A, (uint64_t)R, (uint64_t)d, gg::B_BOX_ROWS, fp8, err) ||
      !make_map(&tm_xw, A, (uint64_t)R, (uint64_t)d, gg::B_WIDE_ROWS, fp8, err) ||
      !make_map(&tm2[0], W2, (uint64_t)E * (uint64_t)d, (uint64_t)f, gg::BM, false, err) ||
      !make_map(&tm2[1], H, (uint64_t)R, (uint64_t)f, gg::B_BOX_ROWS, false, err) ||
      !make_map(&tm2[2], H, (uint64_t)R, (uint64_t)f, gg::B_WIDE_ROWS, false, err))
    return cudaErrorInvalidValue;
  gg::Args args = {};
  args.offsets = offsets;
  args.out = static_cast<uint16_t*>(H);
  args.status = dev.status;
  args.a_scale = a_scale;
  args.w_scale = w1_scale;
  args.w_ptr = static_cast<const uint8_t*>(W1);
  args.w_pitch = d * (fp8 ? 1 : 2);
  args.w2_ptr = static_cast<const uint8_t*>(W2);
  args.w2_pitch = f * 2;
  args.w_prefetch = R <= gg::kWPrefetchMaxRows * E ? gg::kWPrefetchSmall : 0;
  args.gather_k = 1;
  args.a_rows = R;
  args.E = E;
  args.R = R;
  args.N = f;
  args.K = d;
  args.n_fblocks = (f + gg::BM * pair - 1) / (gg::BM * pair);
  const int kb1 = fp8 ? gg::BK_FP8 : gg::BK;
  args.num_kb = (d + kb1 - 1) / kb1;
  args.out2 = static_cast<uint16_t*>(Ye);
  args.N2 = d;
  args.n_fblocks2 = (d + gg::BM * pair - 1) / (gg::BM * pair);
  args.num_kb2 = (f + gg::BK - 1) / gg::BK;
  args.fb_fastest2 = MOE_GEMM2_FB_FASTEST;
  apply_extras(args, ex);
  // Always the dynamic schedule: tickets are taken in item order, so a tile
  // only ever waits on tiles that running clusters hold (any residency).
  args.ticket = ctr;
  args.ready = ctr + 1;
  args.ready_target = (uint32_t)(args.n_fblocks * pair * gg::EPI_WARPS);
  long long items = 0;
  if (ex && ex->disp_X && !fp8) {
    args.disp_X = static_cast<const uint4*>(ex->disp_X);
    args.disp_A = static_cast<uint4*>(const_cast<void*>(A));
    args.disp_src = ex->disp_src;
    args.disp_k = ex->disp_k;
    args.disp_T = ex->disp_T;
    args.disp_vecs = d / 8;
    args.dready = ex->dready;
    items = dispatch_counter_words(R);
  }
  args.stages = pair == 2 ? gg::stages_for<2>(E) : gg::stages_for<1>(E);
  const long long max_tiles = items + ((long long)(R + gg::BN - 1) / gg::BN + E) *
                                          (long long)(args.n_fblocks + args.n_fblocks2);
  if (fp8)
    return pair == 2 ? launch_variant<true, 2, true, false, true>(tm_w, tm_x, tm_xw, args, max_tiles,
                                                                  dev, stream, tm2)
                     : launch_variant<true, 1, true, false, true>(tm_w, tm_x, tm_xw, args, max_tiles,
                                                                  dev, stream, tm2);
  return pair == 2 ? launch_variant<true, 2, false, false, true>(tm_w, tm_x, tm_xw, args, max_tiles,
                                                                 dev, stream, tm2)
                   : launch_variant<true, 1, false, false, true>(tm_w, tm_x, tm_xw, args, max_tiles,
                                                                 dev, stream, tm2);
}

cudaError_t launch_grouped_gemm_gather(const void* X, const float* x_scale, const int32_t* src_of,
                                       int T, int k, const int32_t* offsets, const void* W,
                                       const float* w_scale, int E, int N, int K, bool gelu,
                                       bool fp8, void* out, const DeviceInfo& dev,
                                       cudaStream_t stream, std::string* err) {
  const int R = T * k;
  if (fp8)
    return launch_gemm<true>(X, x_scale, src_of, k, T, offsets, W, w_scale, E, R, N, K, gelu, out,
                             dev, stream, err);
  return launch_gemm<false>(X, nullptr, src_of, k, T, offsets, W, nullptr, E, R, N, K, gelu, out,
                            dev, stream, err);
}

}  // namespace moe
