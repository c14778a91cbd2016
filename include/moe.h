/*
 * moe.h -- C ABI of libmoe.so: one Mixture-of-Experts layer on one B200 (sm_100a).
 *
 * The layer, as the source pages describe it (DySHARP review, marsggbo, §1 and
 * §3.1-3.2; "ThunderEP" PCIe blog, dpshk.com, §1.1 and §2.1-2.2; GPT-4 "2%"
 * article, CSDN, §2.3, §3.1 table and §4.1):
 *
 *   route     a router scores each token, picks its top-k experts and a gate
 *             value per chosen expert;
 *   layout    tokens bound for the same expert are grouped into one dense,
 *             contiguous block: a table maps the logical i-th (token, slot) to
 *             its layout row (DySHARP §3.1 item 3, the AL table);
 *   dispatch  the same token row is copied to each of its k experts;
 *   expert    each expert applies Linear(d->f), GELU, Linear(f->d);
 *   combine   the k expert outputs of a token are reduced into one row,
 *             weighted by the gates.
 *
 * Conventions for every entry point
 *   - Tensor arguments are DEVICE pointers owned by the caller, row-major and
 *     contiguous, 16-byte aligned.  bf16 data is passed as void* holding
 *     IEEE bfloat16 (the __nv_bfloat16 layout); indices are int32, gates and
 *     logits fp32.
 *   - Every call is asynchronous and stream-ordered on `stream` (a
 *     cudaStream_t, passed as void*; NULL = the legacy default stream).  No
 *     call synchronises the host or copies data to it (only
 *     moe_device_status does, on request), so sequences of calls can be
 *     captured in a CUDA graph.  Sizes that depend on the routing (per-expert
 *     counts, offsets) stay in device memory.
 *   - The library never allocates device memory.  Scratch space is a caller
 *     workspace of at least the size the matching *_workspace_size returns.
 *   - Arguments are validated on the host before any launch.  A rejected call
 *     launches nothing and returns MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED;
 *     moe_last_error_string() then describes the problem.
 *   - Kernels that meet bad data (an expert id outside [0, E)) or a wait that
 *     runs past its time limit set a sticky bit in a per-device status word
 *     instead of trapping; read it with moe_device_status().
 *   - Limits: 1 <= E <= 1024, 1 <= k <= min(E, 16), d % 8 == 0, f % 8 == 0,
 *     T*k < 2^30.  T == 0 is a valid no-op.
 *   - Threads may call the library concurrently; calls on streams that run at
 *     the same time must not share output buffers or workspaces.
 *   - Kernels are launched as programmatic dependents of their stream
 *     predecessor (cudaLaunchAttributeProgrammaticStreamSerialization): a
 *     kernel's blocks may be scheduled before the previous kernel on the
 *     stream has finished, and wait (griddepcontrol.wait) before their first
 *     global memory access, so stream order holds for every access.  The
 *     environment variable MOE_PDL=0, read once per process, launches them
 *     without the attribute.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, negative size, k > E, short workspace, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2, /* valid, but outside the limits above (d % 8 != 0, E > 1024, ...) */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_DEVICE = 4       /* moe_device_status found a bit set by a kernel */
} moe_status;

typedef enum moe_score {
  MOE_SCORE_SOFTMAX = 0, /* p_e = softmax over the E logits */
  MOE_SCORE_SIGMOID = 1  /* s_e = 1 / (1 + exp(-logit_e)) */
} moe_score;

/* Bits of the per-device status word (moe_device_status). */
#define MOE_DEV_BAD_EXPERT_ID 0x1u /* an expert id outside [0, E) reached layout / dispatch */
#define MOE_DEV_TIMEOUT       0x2u /* a bounded device-side wait gave up; outputs are invalid */
#define MOE_DEV_BAD_ROW       0x4u /* a row index outside [0, T*k) reached dispatch / combine */

/* moe_layer_desc.flags */
#define MOE_LAYER_GATHER_ON_LOAD 0x1 /* GEMM-1 reads token rows through src_of (TMA gather4)
                                        instead of a dispatched copy; see
                                        moe_expert_gemm_gather.  Same results, bit for bit. */
#define MOE_LAYER_FUSED_FFN 0x2      /* GEMM-1 and GEMM-2 in one persistent launch; see
                                        moe_expert_ffn_fused.  Same results, bit for bit.
                                        Not combinable with MOE_LAYER_GATHER_ON_LOAD. */
#define MOE_LAYER_FUSED_COMBINE 0x4  /* k <= 2: the gate-weighted combine runs in GEMM-2's
                                        epilogue (DySHARP review §3.2, kernel fusion): no Ye
                                        rows and no combine kernel.  A token's k slot results
                                        are weighted in fp32 from the unrounded accumulators
                                        and summed once (a + b, so the order of the two
                                        arrivals does not matter: deterministic).  Within the
                                        float tolerance of the default path, not bitwise.
                                        Ignored for k > 2 (the combine kernel runs). */
#define MOE_LAYER_FUSED_DISPATCH 0x8 /* with MOE_LAYER_FUSED_FFN (bf16 only): the dispatch
                                        copies run as work items of the fused FFN kernel, in
                                        chunks of 64 expert rows, and each GEMM-1 tile starts
                                        once the chunks under its rows are copied.  Same
                                        results as the default path, bit for bit. */
/* The token-centric pipeline of the DySHARP review §3.2 as one persistent kernel
 * after the routing: dispatch chunks, GEMM-1 + GELU and GEMM-2 tiles with the
 * combine in its epilogue, each item starting as soon as its inputs are ready. */
#define MOE_LAYER_PIPELINE (MOE_LAYER_FUSED_FFN | MOE_LAYER_FUSED_COMBINE | MOE_LAYER_FUSED_DISPATCH)

/* Shape and routing recipe of one layer. */
typedef struct moe_layer_desc {
  int32_t T;           /* tokens */
  int32_t d;           /* model dim */
  int32_t E;           /* experts */
  int32_t k;           /* experts per token */
  int32_t f;           /* FFN hidden dim */
  int32_t score;       /* moe_score */
  int32_t renormalize; /* 1: gates renormalised over the chosen k; 0: plain probability */
  int32_t flags;       /* MOE_LAYER_* bits; 0 = the default path */
  float temperature;   /* router temperature (see moe_route_ex); 0 reads as 1 */
  float min_prob;      /* drop chosen slots whose probability is <= min_prob; <= 0 keeps all */
} moe_layer_desc;

/* ---------------------------------------------------------------------------
 * moe_router_logits -- the router linear layer (GPT-4 "2%" article §4.1:
 * logits = router_proj(h); §3.1 table: the router maps a token to one logit
 * per expert).
 *   logits[t, e] = sum_c X[t, c] * Wr[e, c], accumulated in fp32.
 *   X [T, d] bf16, Wr [E, d] bf16 (nn.Linear [out, in] layout), logits [T, E] fp32.
 * ------------------------------------------------------------------------- */
moe_status moe_router_logits(const void* X, const void* Wr, int32_t T, int32_t d, int32_t E,
                             float* logits, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route -- scores, top-k and gates (GPT-4 "2%" article §2.3 and §4.1:
 * softmax over the logits, then top-k; ThunderEP blog §1.1: top-1 / top-2
 * routing, §2.1: top-k indices and gate values drive the combine).
 *   Per token t: the k experts with the largest logit, in descending order,
 *   ties broken toward the lower expert id (selection on the fp32 logit equals
 *   selection on the score, which is strictly increasing in it).
 *   Gates, for chosen logits L_0 >= ... >= L_{k-1}:
 *     SOFTMAX, renormalize=1: exp(L_j - L_0) / sum_{i<k} exp(L_i - L_0)
 *     SOFTMAX, renormalize=0: exp(L_j - L_0) / sum_{e<E} exp(L_e - L_0)
 *     SIGMOID, renormalize=1: s_j / sum_{i<k} s_i,  s = 1/(1+exp(-L))
 *     SIGMOID, renormalize=0: s_j
 *   logits [T, E] fp32, finite for the results above.  A -inf or NaN logit
 *   is never chosen; a slot with no candidate left (fewer than k logits that
 *   are finite or +inf) is dropped: topk_idx = -1, gate 0, as for
 *   moe_route_ex's threshold.  Gates of a token with a NaN logit are
 *   unspecified; its indices are still in [0, E) or -1.
 *   topk_idx [T, k] int32, gates [T, k] fp32.
 * ------------------------------------------------------------------------- */
moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                     int32_t renormalize, int32_t* topk_idx, float* gates, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_ex -- moe_route with a router temperature and a minimum-probability
 * threshold (GPT-4 "2%" article §2.3: a temperature scales the logits before
 * the softmax, and chosen experts whose probability falls under a minimum
 * activation threshold are dropped; §4.1: probabilities not above the
 * threshold give index -1).
 *   Scores use z = logit / temperature (temperature > 0; the top-k order is
 *   the same for every temperature).  A chosen slot's probability is its
 *   softmax over all E experts, or its sigmoid.  When min_prob > 0, a slot
 *   whose probability is <= min_prob is dropped: topk_idx = -1, gate 0.
 *   Gates of kept slots: renormalize=1 divides by the kept slots' sum (the
 *   softmax case equals exp(z_j - z_0) / sum_kept exp(z_i - z_0));
 *   renormalize=0 keeps the probability.  A token with every slot dropped has
 *   all gates 0 (its layer output is 0).  moe_route(...) ==
 *   moe_route_ex(..., temperature = 1, min_prob = 0, ...).
 * ------------------------------------------------------------------------- */
moe_status moe_route_ex(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                        int32_t renormalize, float temperature, float min_prob,
                        int32_t* topk_idx, float* gates, void* stream);

/* ---------------------------------------------------------------------------
 * moe_layout -- per-expert histogram, exclusive scan and the logical->layout
 * table (DySHARP §3.1 item 3: an AL table translates the logical i-th token to
 * its position in a dense per-expert tensor, layout blocks being allocated
 * incrementally; combine reuses the same table.  ThunderEP §2.2: tokens for
 * the same expert are grouped contiguously).
 *   With R = T*k and logical slot i = t*k + j, e_i = topk_idx[i]:
 *     counts[e]   = #{i : e_i == e}
 *     offsets[e]  = sum_{e' < e} counts[e'],  offsets[E] = R
 *     row_of[i]   = offsets[e_i] + #{i' < i : e_i' == e_i}   (stable by token)
 *     src_of[row_of[i]] = i
 *   topk_idx [T, k] int32 in [0, E), or -1 for a dropped slot (see
 *   moe_route_ex), which takes no row: row_of = -1, and offsets[E] counts the
 *   kept slots only; rows r >= offsets[E] get src_of[r] = -1.  Any other id
 *   sets MOE_DEV_BAD_EXPERT_ID and is treated as dropped.
 *   counts [E], offsets [E+1], row_of [R], src_of [R] int32.
 *   ws: at least moe_layout_workspace_size(T, E, k) bytes; its contents are
 *   scratch (look-back status words for the multi-block scan).
 * ------------------------------------------------------------------------- */
size_t moe_layout_workspace_size(int32_t T, int32_t E, int32_t k);
moe_status moe_layout(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k, int32_t* counts,
                      int32_t* offsets, int32_t* row_of, int32_t* src_of, void* ws,
                      size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_route_layout -- moe_route_ex followed by moe_layout, with the layout's
 * ranking folded into the routing kernel (the layer's own path): each CTA of
 * the routing kernel ranks its tile's kept slots within their experts, in
 * slot order, and adds the counts of all earlier tiles found by a decoupled
 * look-back over per-tile status words (tiles taken in ticket order; every
 * wait bounded); the last tile writes counts and offsets.  A second short
 * kernel turns ranks into rows (row_of) and fills src_of.  Two launches
 * instead of two or three (moe_route, then one layout kernel up to 8192 slots
 * with at most 32 experts or 4096 otherwise, two past that), and no
 * single-CTA pass.
 *   Arguments and results as moe_route_ex and moe_layout, bit for bit.
 *   ws: at least moe_route_layout_workspace_size(T, E) bytes (look-back
 *   status words, zeroed by the call).
 * ------------------------------------------------------------------------- */
size_t moe_route_layout_workspace_size(int32_t T, int32_t E);
moe_status moe_route_layout(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                            int32_t renormalize, float temperature, float min_prob,
                            int32_t* topk_idx, float* gates, int32_t* counts, int32_t* offsets,
                            int32_t* row_of, int32_t* src_of, void* ws, size_t ws_bytes,
                            void* stream);

/* ---------------------------------------------------------------------------
 * moe_layout_static -- moe_layout without a workspace argument, for callers
 * that cannot allocate device memory.  The pages have no counterpart: this
 * is a convenience of this library, not a step of the method.
 *   Some callers have no way to get scratch memory on the GPU: code running
 *   inside another framework's callback that is handed only the tensors it
 *   works on, with no allocator; or code that must not allocate after
 *   start-up.  This variant keeps the layout's scratch (the multi-block
 *   scan's look-back words and tile ticket) in a 1 MiB array inside the
 *   library, which every GPU that loads the library holds until the process
 *   exits.  It allocates nothing and calls no allocating routine.
 *   Same arguments and results as moe_layout, minus ws / ws_bytes.  Shapes
 *   whose scratch would exceed 1 MiB (moe_layout_workspace_size(T, E, k) >
 *   1048576, e.g. more than about 2 million slots with 1024 experts) are
 *   rejected with MOE_ERR_UNSUPPORTED before any launch.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  Every call on a device shares the one array
 *   and leaves its contents behind; the kernels re-arm what must start at
 *   zero on each call.  Calls whose kernels may overlap on the GPU (other
 *   streams, other host threads) race on the array: serialise them.
 * ------------------------------------------------------------------------- */
moe_status moe_layout_static(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k,
                             int32_t* counts, int32_t* offsets, int32_t* row_of, int32_t* src_of,
                             void* stream);

/* ---------------------------------------------------------------------------
 * moe_dispatch -- copy each token to its k experts' rows (DySHARP §1: the same
 * token data goes to each of its k experts; ThunderEP §1.1).
 *   Xe[r, :] = X[src_of[r] / k, :]   for r in [0, T*k) with src_of[r] >= 0;
 *   rows with src_of[r] = -1 (past the kept slots) are left untouched.
 *   X [T, d] bf16, src_of [T*k] int32, Xe [T*k, d] bf16.
 * ------------------------------------------------------------------------- */
moe_status moe_dispatch(const void* X, const int32_t* src_of, int32_t T, int32_t d, int32_t k,
                        void* Xe, void* stream);

/* ---------------------------------------------------------------------------
 * moe_dispatch_by_token -- the same copy as moe_dispatch, walked by token:
 *   Xe[row_of[t*k + j], :] = X[t, :]   for every slot with row_of >= 0.
 *   Each token row is read once and written to its k rows.  moe_dispatch walks
 *   the rows instead and reads a token once per slot, which goes back to HBM
 *   when X does not stay in L2 (many tokens, large k).  Rows no slot maps to
 *   are left untouched; a row_of entry outside [-1, T*k) sets MOE_DEV_BAD_ROW
 *   and is skipped.  moe_layer_forward uses this form.
 *   X [T, d] bf16, row_of [T*k] int32 (from moe_layout), Xe [T*k, d] bf16.
 * ------------------------------------------------------------------------- */
moe_status moe_dispatch_by_token(const void* X, const int32_t* row_of, int32_t T, int32_t d,
                                 int32_t k, void* Xe, void* stream);

/* ---------------------------------------------------------------------------
 * moe_expert_gemm -- one grouped expert linear layer over variable-size row
 * blocks (GPT-4 "2%" article §3.1 table: each expert is Linear -> GELU ->
 * Linear; DySHARP §3.2: GEMM-1 then GEMM-2 per expert).
 *   For each expert e and row r in [offsets[e], offsets[e+1]):
 *     out[r, n] = act( sum_c A[r, c] * W[e, n, c] ),  act = GELU (exact erf
 *     form, 0.5 x (1 + erf(x / sqrt 2))) when gelu != 0, identity otherwise;
 *   accumulated in fp32 on the tensor cores, rounded once to bf16.
 *   A [R, K] bf16, offsets [E+1] int32 (non-decreasing, offsets[E] <= R),
 *   W [E, N, K] bf16, out [R, N] bf16.  Rows at or past offsets[E] are not
 *   written.  K % 8 == 0, N % 8 == 0.
 * ------------------------------------------------------------------------- */
moe_status moe_expert_gemm(const void* A, const int32_t* offsets, const void* W, int32_t E,
                           int32_t R, int32_t N, int32_t K, int32_t gelu, void* out,
                           void* stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn -- both expert layers:  H = GELU(Xe W1[e]^T),  Ye = H W2[e]^T.
 *   Xe [R, d] bf16, offsets [E+1], W1 [E, f, d] bf16, W2 [E, d, f] bf16,
 *   H [R, f] bf16 (output, kept), Ye [R, d] bf16.
 * ------------------------------------------------------------------------- */
moe_status moe_expert_ffn(const void* Xe, const int32_t* offsets, const void* W1, const void* W2,
                          int32_t E, int32_t R, int32_t d, int32_t f, void* H, void* Ye,
                          void* stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn_fused -- moe_expert_ffn as ONE persistent kernel (the GEMM
 * part of the token-centric pipeline in the DySHARP review §3.2: GEMM-2
 * work on a block of tokens starts as soon as GEMM-1 has produced that
 * block's H, with no kernel boundary in between).
 *   Same arguments and results as moe_expert_ffn (bitwise), plus scratch:
 *   ws of at least moe_expert_ffn_fused_workspace_size(E, R) bytes holding
 *   one readiness counter per 256-row token block (zeroed by the call).
 *   Every device wait is bounded; a timeout sets MOE_DEV_TIMEOUT.
 * moe_expert_ffn_fused_fp8 -- the same with GEMM-1 on E4M3 operands
 *   (Xeq, x_scale from moe_dispatch_fp8; W1q, w1_scale from
 *   moe_quantize_experts_fp8); GEMM-2 stays bf16.  d % 16 == 0.
 * ------------------------------------------------------------------------- */
size_t moe_expert_ffn_fused_workspace_size(int32_t E, int32_t R);
moe_status moe_expert_ffn_fused(const void* Xe, const int32_t* offsets, const void* W1,
                                const void* W2, int32_t E, int32_t R, int32_t d, int32_t f,
                                void* H, void* Ye, void* ws, size_t ws_bytes, void* stream);
moe_status moe_expert_ffn_fused_fp8(const void* Xeq, const float* x_scale,
                                    const int32_t* offsets, const void* W1q,
                                    const float* w1_scale, const void* W2, int32_t E, int32_t R,
                                    int32_t d, int32_t f, void* H, void* Ye, void* ws,
                                    size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_ffn_pipeline -- dispatch, both expert layers and the combine as ONE
 * persistent kernel: the token-centric pipeline of the DySHARP review §3.2
 * (work on a group of tokens starts as soon as the data it needs is ready,
 * with no kernel boundary between the stages), after route and layout.
 *   Work items, taken by the SM pairs in this order from an atomic ticket:
 *   dispatch chunks of 64 expert rows (Xe[r] = X[src_of[r] / k]), GEMM-1 +
 *   GELU tiles (each waits for the chunks under its rows), GEMM-2 tiles (each
 *   waits for its token block's H).  An item only waits on items before it,
 *   so every wait ends, whatever share of the GPU the launch gets.  For
 *   k <= 2 the combine runs in GEMM-2's epilogue (see MOE_LAYER_FUSED_COMBINE:
 *   a token's output is written by the second of its two slot results to
 *   arrive, or at once when it has one kept slot); for k > 2 the kernel
 *   writes Ye and moe_combine's kernel follows.
 *   Results: Y within the float tolerance of moe_dispatch + moe_expert_ffn +
 *   moe_combine (bitwise for k > 2).  Rows of Y for tokens with no kept slot
 *   (every row_of entry -1) are not written.
 *   X [T, d] bf16; src_of [T*k], row_of [T*k], offsets [E+1] from moe_layout;
 *   gates [T, k] fp32; W1 [E, f, d], W2 [E, d, f] bf16; Y [T, d] bf16.
 *   ws: at least moe_ffn_pipeline_workspace_size(T, d, E, k, f) bytes
 *   (dispatched rows, H, partial rows, readiness counters; zeroed counters
 *   are set up by the call).  Every device wait is bounded; a timeout sets
 *   MOE_DEV_TIMEOUT.
 * ------------------------------------------------------------------------- */
size_t moe_ffn_pipeline_workspace_size(int32_t T, int32_t d, int32_t E, int32_t k, int32_t f);
moe_status moe_ffn_pipeline(const void* X, const int32_t* src_of, const int32_t* row_of,
                            const float* gates, const int32_t* offsets, const void* W1,
                            const void* W2, int32_t T, int32_t d, int32_t E, int32_t k,
                            int32_t f, void* Y, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- gate-weighted reduction of each token's k expert outputs
 * (DySHARP §1: the k results are summed into one; ThunderEP §2.1: the gate
 * values weight the combine sum).
 *   Y[t, :] = bf16( sum_{j<k} gates[t, j] * Ye[row_of[t*k + j], :] ),
 *   summed in fp32 in slot order j = 0..k-1; a dropped slot (row_of = -1)
 *   contributes nothing (its Ye row is not read).
 *   Ye [T*k, d] bf16, row_of [T*k] int32, gates [T, k] fp32, Y [T, d] bf16.
 * ------------------------------------------------------------------------- */
moe_status moe_combine(const void* Ye, const int32_t* row_of, const float* gates, int32_t T,
                       int32_t d, int32_t k, void* Y, void* stream);

/* ---------------------------------------------------------------------------
 * moe_layer_forward -- the whole layer in one call: [router_logits] -> route ->
 * layout -> dispatch -> GEMM-1 + GELU -> GEMM-2 -> combine, all on `stream`,
 * no host synchronisation.
 *   Exactly one of `logits` ([T, E] fp32) and `Wr` ([E, d] bf16) is non-NULL.
 *   X [T, d] bf16, W1 [E, f, d], W2 [E, d, f] bf16, Y [T, d] bf16.
 *   topk_idx_out [T, k], gates_out [T, k], counts_out [E]: optional copies
 *   of the routing (NULL to skip).
 *   ws: at least moe_workspace_size(desc) bytes.
 *   desc->flags & MOE_LAYER_FUSED_FFN runs both expert GEMMs as one persistent
 *   kernel (moe_expert_ffn_fused); the output is identical.
 *   desc->flags & MOE_LAYER_GATHER_ON_LOAD fuses the dispatch into GEMM-1
 *   (no dispatch kernel, no dispatched copy of X); the output is identical.
 *   On a B200 it is slower than the default for every shape measured (the
 *   gathered loads cost more tensor-memory-access time than the dispatch
 *   saves), so it is off by default.
 * ------------------------------------------------------------------------- */
size_t moe_workspace_size(const moe_layer_desc* desc);
moe_status moe_layer_forward(const moe_layer_desc* desc, const void* X, const float* logits,
                             const void* Wr, const void* W1, const void* W2, void* Y,
                             int32_t* topk_idx_out, float* gates_out, int32_t* counts_out,
                             void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * moe_layer_forward_host -- moe_layer_forward over `nbatch` batches whose
 * tokens and outputs live in HOST memory (the end-to-end form of the layer:
 * the pages' dispatch/combine path starts and ends with token rows that have
 * to move, ThunderEP blog §1.2 and §5.3 on overlapping transfer with compute).
 *   Batch i: X_host[i] [T, d] bf16 (and logits_host[i] [T, E] fp32 when the
 *   router is not given) is copied to the device, the layer runs, and its
 *   output is copied to Y_host[i] [T, d] bf16 -- one cudaMemcpyAsync per
 *   copy.  The library orders the work on three streams of its own per
 *   device (copies in, compute, copies out) with events, and two device
 *   buffer sets in `ws`, so the copies of neighbouring batches overlap the
 *   current forward and a batch costs about the slowest of the three.
 *   All batches share `desc` and the weights (device pointers: Wr or the
 *   logits_host array, W1, W2; w1_scale non-NULL selects the FP8 mode with
 *   W1 holding moe_quantize_experts_fp8 codes, as moe_layer_forward_fp8).
 *   Host buffers should be pinned (page-locked) for the copies to run
 *   asynchronously; pageable memory gives the same results, serialised.
 *   The call returns once the work is enqueued.  Work already on `stream`
 *   runs first, and `stream` waits for the last copy out: synchronising
 *   `stream` (or enqueueing after this call on it) sees every Y_host[i]
 *   complete.  The host buffers must stay valid until then.  Calls on one
 *   device are serialised on the library's streams; they are not for CUDA
 *   graph capture (the streams are the library's).
 *   ws: at least moe_host_workspace_size(desc, with_logits) bytes.
 * ------------------------------------------------------------------------- */
size_t moe_host_workspace_size(const moe_layer_desc* desc, int32_t with_logits);
moe_status moe_layer_forward_host(const moe_layer_desc* desc, int32_t nbatch,
                                  const void* const* X_host, const float* const* logits_host,
                                  const void* Wr, const void* W1, const float* w1_scale,
                                  const void* W2, void* const* Y_host, void* ws, size_t ws_bytes,
                                  void* stream);

/* ---------------------------------------------------------------------------
 * FP8 mode (ThunderEP PCIe blog §3.3 "transport-side bit reduction" and §5.2:
 * the activations a dispatch moves are cast to FP8 with one dynamic
 * per-tensor scale before they move and cast back after, halving the bytes;
 * FP8-capable tensor cores consume them directly).  Here: the dispatched
 * token rows are E4M3 codes (1 byte per value) with one scale for all of X,
 * and GEMM-1 runs on FP8 tensor cores against per-expert-quantised W1.
 * GEMM-2 and combine stay bf16.
 *
 * Quantisation of a tensor x (identical wherever the library does it):
 *   amax  = max |x|;  inv = 448 / amax  (fp32, round to nearest; 1 if amax = 0)
 *   code  = E4M3(x * inv)  (fp32 product; round to nearest even; magnitudes
 *           past 448 saturate to +-448; E4M3 = 1 sign, 4 exponent bits with
 *           bias 7, 3 mantissa bits, no infinities)
 *   scale = amax / 448     (fp32; 1 if amax = 0);  x ~= scale * code.
 * Inputs must be finite.  FP8 calls need d % 16 == 0 and K % 16 == 0 (rows of
 * codes are 16-byte aligned).
 *
 * moe_quantize_experts_fp8 -- per-expert quantisation of expert weights (done
 *   once, when the weights are loaded; the pages leave weight quantisation
 *   open, and one scale per expert matrix is the plainest choice).
 *   W [E, rows, cols] bf16 -> Wq [E, rows, cols] E4M3 codes (uint8),
 *   scales [E] fp32 (expert e's `scale`).  cols % 16 == 0.
 *
 * moe_dispatch_fp8 -- moe_dispatch writing E4M3 codes:
 *   Xeq[r, :] = E4M3(X[src_of[r] / k, :] * inv), one scale over all of X [T, d].
 *   x_scale: device float[2]; on return x_scale[0] = scale (what GEMM-1 reads),
 *   x_scale[1] = amax.  Rows with src_of = -1 are left untouched.
 *
 * moe_expert_gemm_fp8 -- moe_expert_gemm on E4M3 operands:
 *   out[r, n] = act( a_scale[0] * w_scale[e] * sum_c Aq[r, c] * Wq[e, n, c] ),
 *   products exact, sums in fp32 on the tensor cores, the scaled result
 *   rounded once to bf16.  Aq [R, K] uint8, a_scale device float[1],
 *   Wq [E, N, K] uint8, w_scale [E] fp32, out [R, N] bf16.
 *
 * moe_layer_forward_fp8 -- moe_layer_forward with FP8 dispatch and FP8 GEMM-1:
 *   W1q / w1_scale from moe_quantize_experts_fp8(W1); other arguments as in
 *   moe_layer_forward; ws: at least moe_workspace_size(desc) bytes (the same
 *   workspace serves both modes).
 * moe_kernel_launches_per_forward_fp8 -- its kernel count (memsets excluded).
 * ------------------------------------------------------------------------- */
moe_status moe_quantize_experts_fp8(const void* W, int32_t E, int32_t rows, int32_t cols,
                                    void* Wq, float* scales, void* stream);
moe_status moe_dispatch_fp8(const void* X, const int32_t* src_of, int32_t T, int32_t d,
                            int32_t k, void* Xeq, float* x_scale, void* stream);
/* moe_dispatch_fp8_by_token: moe_dispatch_fp8 walked by token through row_of
 * (see moe_dispatch_by_token); the same codes and x_scale. */
moe_status moe_dispatch_fp8_by_token(const void* X, const int32_t* row_of, int32_t T, int32_t d,
                                     int32_t k, void* Xeq, float* x_scale, void* stream);
moe_status moe_expert_gemm_fp8(const void* Aq, const float* a_scale, const int32_t* offsets,
                               const void* Wq, const float* w_scale, int32_t E, int32_t R,
                               int32_t N, int32_t K, int32_t gelu, void* out, void* stream);
moe_status moe_layer_forward_fp8(const moe_layer_desc* desc, const void* X, const float* logits,
                                 const void* Wr, const void* W1q, const float* w1_scale,
                                 const void* W2, void* Y, int32_t* topk_idx_out,
                                 float* gates_out, int32_t* counts_out, void* ws,
                                 size_t ws_bytes, void* stream);
int32_t moe_kernel_launches_per_forward_fp8(const moe_layer_desc* desc, int32_t with_router);

/* moe_quantize_fp8 -- per-tensor E4M3 quantisation of a bf16 matrix by the
 *   rule above: X [rows, cols] bf16 -> Xq [rows, cols] codes, x_scale device
 *   float[2] = {scale, amax}.  cols % 16 == 0.  Feeds the gather-on-load
 *   FP8 GEMM below (the tokens are quantised once, not once per expert slot). */
moe_status moe_quantize_fp8(const void* X, int32_t rows, int32_t cols, void* Xq, float* x_scale,
                            void* stream);

/* ---------------------------------------------------------------------------
 * Gather-on-load expert GEMM (DySHARP review §3.2: dispatch fused into the
 * expert GEMM, so the dispatched copy of the tokens is never written).
 *   moe_expert_gemm_gather: for each expert e and row r in
 *     [offsets[e], offsets[e+1]):
 *       out[r, n] = act( sum_c X[src_of[r] / k, c] * W[e, n, c] ),
 *     i.e. moe_expert_gemm applied to the rows moe_dispatch would produce.
 *     X [T, K] bf16, src_of [T*k] int32 (from moe_layout), offsets [E+1],
 *     W [E, N, K] bf16, out [T*k, N] bf16.  Rows at or past offsets[E] are not
 *     written.  A src_of entry inside an expert block outside [0, T*k) sets
 *     MOE_DEV_BAD_ROW and reads token 0.
 *   moe_expert_gemm_gather_fp8: the same on E4M3 codes (moe_quantize_fp8 of
 *     X, moe_quantize_experts_fp8 of W):
 *       out[r, n] = act( x_scale[0] * w_scale[e] *
 *                        sum_c Xq[src_of[r] / k, c] * Wq[e, n, c] ).
 *     K % 16 == 0.
 * ------------------------------------------------------------------------- */
moe_status moe_expert_gemm_gather(const void* X, const int32_t* src_of, int32_t T, int32_t k,
                                  const int32_t* offsets, const void* W, int32_t E, int32_t N,
                                  int32_t K, int32_t gelu, void* out, void* stream);
moe_status moe_expert_gemm_gather_fp8(const void* Xq, const float* x_scale, const int32_t* src_of,
                                      int32_t T, int32_t k, const int32_t* offsets,
                                      const void* Wq, const float* w_scale, int32_t E, int32_t N,
                                      int32_t K, int32_t gelu, void* out, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 *   moe_last_error_string: a description of the last failed call on this
 *   host thread ("" if none).  The pointer stays valid until the next call.
 *   moe_device_status: synchronises the current device, then stores the
 *   sticky MOE_DEV_* bits into *bits (clearing them when clear != 0).  Returns
 *   MOE_ERR_DEVICE when any bit was set, MOE_OK otherwise.
 *   moe_kernel_launches_per_forward: the number of kernels moe_layer_forward
 *   launches for this shape, with (with_router != 0) or without the router
 *   linear (for launch accounting; memsets excluded).
 * ------------------------------------------------------------------------- */
const char* moe_last_error_string(void);

/* moe_selftest_bounded_wait -- runs one of the library's bounded device waits
 * on a condition that nothing ever satisfies, so that a caller (or a test)
 * can check the failure path without faulting or hanging the GPU: the wait
 * gives up after limit_us microseconds, the kernel sets MOE_DEV_TIMEOUT in
 * the status word and returns; read it with moe_device_status().
 *   which = 0: the readiness-count wait of the fused forms (counter: a
 *              device uint32 holding 0, which nothing increments;
 *              caller-owned);
 *   which = 1: the shared-memory mbarrier wait of the grouped GEMM's ring
 *              (counter unused, may be NULL);
 *   which = 2: the flag wait of the combine in GEMM-2's epilogue (counter: a
 *              device uint32 holding 0, whose flag bit nothing sets);
 *   which = 3: the cluster-scope mbarrier wait of the work-item queue
 *              (counter unused, may be NULL).
 *   1 <= limit_us <= 10^7. */
moe_status moe_selftest_bounded_wait(int32_t which, uint32_t limit_us, uint32_t* counter,
                                     void* stream);
moe_status moe_device_status(uint32_t* bits, int32_t clear);
int32_t moe_kernel_launches_per_forward(const moe_layer_desc* desc, int32_t with_router);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
