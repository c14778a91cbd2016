// The C ABI of libmoe.so (declared in include/moe.h): argument validation,
// per-device state, workspace layout and the fused layer forward.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.h"

// Per-stage NVTX ranges around the layer's launches (build with -DMOE_NVTX=1;
// header-only NVTX v3, so nothing to link).  A profiler's timeline then shows
// router / route / layout / dispatch / GEMM-1 / GEMM-2 / combine by name: the
// kernel-level view of the GPT-4 "2%" article §5.2 (a GPU kernel flame graph
// of the router and expert GEMM kernels).  Off by default: they cost host time.
#if MOE_NVTX
#include <nvtx3/nvToolsExt.h>
struct NvtxStage {
  explicit NvtxStage(const char* name) { nvtxRangePushA(name); }
  ~NvtxStage() { nvtxRangePop(); }
};
#define MOE_STAGE(name) NvtxStage moe_nvtx_stage_(name)
#else
#define MOE_STAGE(name) \
  do {                  \
  } while (0)
#endif

// Sticky per-device status word set by kernels (MOE_DEV_* bits).
__device__ uint32_t g_moe_device_status;

namespace moe {
namespace {

thread_local std::string g_last_error;

moe_status fail(moe_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

moe_status cuda_fail(cudaError_t e, const char* where) {
  return fail(MOE_ERR_CUDA, std::string(where) + ": " + cudaGetErrorName(e) + " (" +
                                cudaGetErrorString(e) + ")");
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
cudaError_t g_dev_err[kMaxDevices];

}  // namespace

int set_last_error(int status, const std::string& msg) {
  g_last_error = msg;
  return status;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("MOE_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

const DeviceInfo* current_device_info(std::string* err) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = std::string("cudaGetDevice: ") + cudaGetErrorString(e);
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *err = "device ordinal out of range";
    return nullptr;
  }
  std::call_once(g_dev_once[dev], [dev] {
    DeviceInfo& d = g_dev[dev];
    d.device = dev;
    cudaError_t e1 = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    void* p = nullptr;
    cudaError_t e2 = cudaGetSymbolAddress(&p, g_moe_device_status);
    d.status = static_cast<uint32_t*>(p);
    g_dev_err[dev] = e1 != cudaSuccess ? e1 : e2;
  });
  if (g_dev_err[dev] != cudaSuccess) {
    *err = std::string("device set-up: ") + cudaGetErrorString(g_dev_err[dev]);
    return nullptr;
  }
  return &g_dev[dev];
}

}  // namespace moe

using moe::cuda_fail;
using moe::fail;

namespace {

moe_status get_dev(const moe::DeviceInfo** out) {
  std::string err;
  *out = moe::current_device_info(&err);
  if (!*out) return fail(MOE_ERR_CUDA, err);
  return MOE_OK;
}

moe_status check_ET(int32_t T, int32_t E, int32_t k) {
  if (T < 0) return fail(MOE_ERR_INVALID_ARG, "T must be >= 0");
  if (E < 1) return fail(MOE_ERR_INVALID_ARG, "E must be >= 1");
  if (k < 1 || k > E) return fail(MOE_ERR_INVALID_ARG, "k must be in [1, E]");
  if (E > moe::kMaxExperts) return fail(MOE_ERR_UNSUPPORTED, "E > 1024 is not supported");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  return MOE_OK;
}

moe_status check_dim(int32_t v, const char* name) {
  if (v < 1) return fail(MOE_ERR_INVALID_ARG, std::string(name) + " must be >= 1");
  if (v % 8) return fail(MOE_ERR_UNSUPPORTED, std::string(name) + " must be a multiple of 8");
  return MOE_OK;
}

moe_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (!moe::aligned16(p)) return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is not 16-byte aligned");
  return MOE_OK;
}

moe_status check_ptr4(const void* p, const char* name) {
  if (!p) return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is NULL");
  if (reinterpret_cast<uintptr_t>(p) & 3u)
    return fail(MOE_ERR_INVALID_ARG, std::string(name) + " is not 4-byte aligned");
  return MOE_OK;
}

#define MOE_TRY(x)                \
  do {                            \
    moe_status _s = (x);          \
    if (_s != MOE_OK) return _s;  \
  } while (0)

#define MOE_CUDA(x, where)                        \
  do {                                            \
    cudaError_t _e = (x);                         \
    if (_e != cudaSuccess) return cuda_fail(_e, where); \
  } while (0)

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Workspace of the fused forward: sub-buffers, each 256-byte aligned.
struct LayerWs {
  size_t logits, idx, gates, counts, offsets, row_of, src_of, layout, Xe, H, Ye, scale, ctr, part,
      lb, lpart, total;
};

// Counter words of the layer workspace (all zeroed by one memset per forward):
// the fused FFN's ticket and readiness counters (or GEMM-1's ticket), GEMM-2's
// ticket, the dispatch chunks' counters, the fused combine's arrival words.
struct LayerCtr {
  int ffn, g2, disp, comb, used;
};

LayerCtr layer_ctr(const moe_layer_desc& d) {
  const int R = d.T * d.k;
  LayerCtr c;
  c.ffn = 0;
  c.g2 = moe::ffn_counter_words(R, d.E);
  c.disp = c.g2 + 1;
  c.comb = c.disp + moe::dispatch_counter_words(R);
  const bool fused = (d.flags & MOE_LAYER_FUSED_FFN) != 0;
  const bool comb = (d.flags & MOE_LAYER_FUSED_COMBINE) && d.k <= 2;
  c.used = comb ? c.comb + moe::combine_counter_words(d.T, d.d)
                : (fused && (d.flags & MOE_LAYER_FUSED_DISPATCH)) ? c.comb : c.disp;
  return c;
}

size_t up256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

LayerWs layer_ws(const moe_layer_desc& d) {
  LayerWs w;
  const size_t T = (size_t)d.T, R = (size_t)d.T * d.k;
  size_t o = 0;
  w.logits = o;  o += up256(T * d.E * sizeof(float));
  w.idx = o;     o += up256(R * sizeof(int32_t));
  w.gates = o;   o += up256(R * sizeof(float));
  w.counts = o;  o += up256((size_t)d.E * sizeof(int32_t));
  w.offsets = o; o += up256((size_t)(d.E + 1) * sizeof(int32_t));
  w.row_of = o;  o += up256(R * sizeof(int32_t));
  w.src_of = o;  o += up256(R * sizeof(int32_t));
  w.layout = o;  o += up256(moe::layout_workspace_bytes((int64_t)R, d.E));
  w.Xe = o;      o += up256(R * d.d * 2);  // bf16 rows, or E4M3 rows in the first half
  w.H = o;       o += up256(R * d.f * 2);
  w.Ye = o;      o += up256(R * d.d * 2);
  w.scale = o;   o += up256(2 * sizeof(float));  // FP8 mode: activation scale and amax
  w.ctr = o;     o += up256((size_t)(moe::ffn_counter_words((int)R, d.E) + 1 +
                                     moe::dispatch_counter_words((int)R) +
                                     moe::combine_counter_words(d.T, d.d)) * sizeof(uint32_t));
  w.part = o;    o += up256(T * d.d * sizeof(float));  // fused combine: fp32 partial rows
  w.lb = o;      o += up256(moe::route_rank_lookback_words(d.T, d.E) * sizeof(uint32_t));
  // split router's partial logits (small batches on the ranked path)
  w.lpart = o;
  if (d.T <= moe::kSplitMaxT && d.E <= moe::kRankedMaxExperts)
    o += up256((size_t)moe::router_split_count(d.d) * T * d.E * sizeof(float));
  w.total = o;
  return w;
}

moe_status check_desc(const moe_layer_desc* desc) {
  if (!desc) return fail(MOE_ERR_INVALID_ARG, "desc is NULL");
  MOE_TRY(check_ET(desc->T, desc->E, desc->k));
  MOE_TRY(check_dim(desc->d, "d"));
  MOE_TRY(check_dim(desc->f, "f"));
  if (desc->score != MOE_SCORE_SOFTMAX && desc->score != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown score");
  if (desc->renormalize != 0 && desc->renormalize != 1)
    return fail(MOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (desc->flags & ~(MOE_LAYER_GATHER_ON_LOAD | MOE_LAYER_FUSED_FFN | MOE_LAYER_FUSED_COMBINE |
                      MOE_LAYER_FUSED_DISPATCH))
    return fail(MOE_ERR_INVALID_ARG, "unknown flags");
  if ((desc->flags & MOE_LAYER_GATHER_ON_LOAD) && (desc->flags & MOE_LAYER_FUSED_FFN))
    return fail(MOE_ERR_UNSUPPORTED, "MOE_LAYER_GATHER_ON_LOAD with MOE_LAYER_FUSED_FFN");
  if ((desc->flags & MOE_LAYER_FUSED_DISPATCH) && !(desc->flags & MOE_LAYER_FUSED_FFN))
    return fail(MOE_ERR_INVALID_ARG, "MOE_LAYER_FUSED_DISPATCH needs MOE_LAYER_FUSED_FFN");
  if (!std::isfinite(desc->temperature) || desc->temperature < 0.f)
    return fail(MOE_ERR_INVALID_ARG, "temperature must be >= 0 (0 reads as 1)");
  if (!std::isfinite(desc->min_prob)) return fail(MOE_ERR_INVALID_ARG, "min_prob must be finite");
  return MOE_OK;
}

float desc_temperature(const moe_layer_desc& d) { return d.temperature > 0.f ? d.temperature : 1.f; }

moe_status check_fp8_dim(int32_t v, const char* name) {
  if (v % 16) return fail(MOE_ERR_UNSUPPORTED, std::string(name) + " must be a multiple of 16 in FP8 mode");
  return MOE_OK;
}

moe_status gemm_fail(cudaError_t e, const std::string& err, const char* where) {
  return err.empty() ? cuda_fail(e, where) : fail(MOE_ERR_CUDA, std::string(where) + ": " + err);
}

// The layer forward of both modes: W1s == nullptr runs bf16, otherwise
// W1 holds E4M3 codes with per-expert scales W1s (FP8 dispatch + GEMM-1).
moe_status layer_forward(const moe_layer_desc* desc, const void* X, const float* logits,
                         const void* Wr, const void* W1, const float* W1s, const void* W2,
                         void* Y, int32_t* topk_idx_out, float* gates_out, int32_t* counts_out,
                         void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc d = *desc;
  const bool fp8 = W1s != nullptr;
  if ((logits == nullptr) == (Wr == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "give exactly one of logits and Wr");
  if (fp8) MOE_TRY(check_fp8_dim(d.d, "d"));
  if (d.T == 0) return MOE_OK;
  if ((int64_t)d.E * d.f >= (1ll << 31) || (int64_t)d.E * d.d >= (1ll << 31))
    return fail(MOE_ERR_UNSUPPORTED, "E*f and E*d must be < 2^31");
  MOE_TRY(check_ptr(X, "X"));
  if (logits) MOE_TRY(check_ptr4(logits, "logits"));
  if (Wr) MOE_TRY(check_ptr(Wr, "Wr"));
  MOE_TRY(check_ptr(W1, fp8 ? "W1q" : "W1"));
  if (fp8) MOE_TRY(check_ptr4(W1s, "w1_scale"));
  MOE_TRY(check_ptr(W2, "W2"));
  MOE_TRY(check_ptr(Y, "Y"));
  if (topk_idx_out) MOE_TRY(check_ptr4(topk_idx_out, "topk_idx_out"));
  if (gates_out) MOE_TRY(check_ptr4(gates_out, "gates_out"));
  if (counts_out) MOE_TRY(check_ptr4(counts_out, "counts_out"));
  const LayerWs w = layer_ws(d);
  if (ws_bytes < w.total) return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  cudaStream_t s = as_stream(stream);
  char* base = static_cast<char*>(ws);
  float* L = logits ? const_cast<float*>(logits) : reinterpret_cast<float*>(base + w.logits);
  int32_t* idx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t*>(base + w.idx);
  float* gates = gates_out ? gates_out : reinterpret_cast<float*>(base + w.gates);
  int32_t* counts = counts_out ? counts_out : reinterpret_cast<int32_t*>(base + w.counts);
  int32_t* offsets = reinterpret_cast<int32_t*>(base + w.offsets);
  int32_t* row_of = reinterpret_cast<int32_t*>(base + w.row_of);
  int32_t* src_of = reinterpret_cast<int32_t*>(base + w.src_of);
  void* lws = base + w.layout;
  void* Xe = base + w.Xe;
  void* H = base + w.H;
  void* Ye = base + w.Ye;
  float* x_scale = reinterpret_cast<float*>(base + w.scale);
  uint32_t* ctr = reinterpret_cast<uint32_t*>(base + w.ctr);
  const LayerCtr lc = layer_ctr(d);
  const int R = d.T * d.k;
  const bool fused = (d.flags & MOE_LAYER_FUSED_FFN) != 0;
  const bool gather = (d.flags & MOE_LAYER_GATHER_ON_LOAD) != 0;
  const bool comb = (d.flags & MOE_LAYER_FUSED_COMBINE) && d.k <= 2;
  const bool fdisp = fused && (d.flags & MOE_LAYER_FUSED_DISPATCH) && !fp8;
  // Routing fused with the layout's ranking, the rows finished by the
  // token-walking dispatch: the layer's bf16 path (the gathered, dispatch-item
  // and FP8 forms read src_of before any dispatch kernel, or dispatch
  // quantised rows, and keep the separate layout kernel).
  // Up to 32 experts (one look-back per warp of the routing kernel); with
  // more, the per-expert look-backs of a tile run one after another and the
  // separate layout kernels measured faster (256 experts: 103 us vs 27 us).
  const bool ranked = !gather && !fdisp && !fp8 && d.E <= moe::kRankedMaxExperts;
  uint32_t* lb = reinterpret_cast<uint32_t*>(base + w.lb);

  // The ranked routing's look-back words start at zero in every forward: the
  // router kernel clears them as a side job, or a memset when the logits are
  // given.  Small batches (up to 32 experts) take the split router, whose
  // partial logits the routing kernel sums; every form of the layer does, so
  // the forms route on the same logits.
  const int lb_words = ranked ? (int)moe::route_rank_lookback_words(d.T, d.E) : 0;
  const bool split = Wr && d.T <= moe::kSplitMaxT && d.E <= moe::kRankedMaxExperts;
  const int nsplit = split ? moe::router_split_count(d.d) : 1;
  const float* Lr = split ? reinterpret_cast<const float*>(base + w.lpart) : L;
  if (Wr) {
    MOE_STAGE("moe.router_logits");
    if (split)
      MOE_CUDA(moe::launch_router_split(X, Wr, d.T, d.d, d.E, const_cast<float*>(Lr), *dev, s,
                                        lb, lb_words),
               "router_split");
    else
      MOE_CUDA(moe::launch_router_logits(X, Wr, d.T, d.d, d.E, L, *dev, s, lb, lb_words),
               "router_logits");
  }
  // The routing kernel also clears the tickets, readiness and combine
  // counters (they start at zero in every forward) and, with the combine in
  // GEMM-2's epilogue, writes the zero outputs of tokens whose slots were all
  // dropped (no expert row reaches them).
  const bool drops = d.min_prob > 0.f;
  if (ranked) {
    MOE_STAGE("moe.route");
    if (!Wr)
      MOE_CUDA(cudaMemsetAsync(lb, 0, (size_t)lb_words * sizeof(uint32_t), s), "memset look-back");
    MOE_CUDA(moe::launch_route_rank(Lr, d.T, d.E, d.k, d.score, d.renormalize,
                                    desc_temperature(d), d.min_prob, idx, gates, row_of, counts,
                                    offsets, lb, *dev, s, (comb && drops) ? Y : nullptr, d.d, ctr,
                                    lc.used, nsplit),
             "route_rank");
  } else {
    {
      MOE_STAGE("moe.route");
      MOE_CUDA(moe::launch_route(Lr, d.T, d.E, d.k, d.score, d.renormalize, desc_temperature(d),
                                 d.min_prob, idx, gates, s, (comb && drops) ? Y : nullptr, d.d,
                                 ctr, lc.used, nsplit),
               "route");
    }
    MOE_STAGE("moe.layout");
    MOE_CUDA(moe::launch_layout(idx, R, d.E, counts, offsets, row_of, src_of, lws, *dev, s),
             "layout");
  }
  // The two-launch path keeps the static balanced schedule (measured faster
  // than tickets on uniform tiles); the fused launch always takes tickets.
  moe::GemmExtras ex1, ex2;
  // bf16 dispatch: with the ranks from the routing kernel it also turns them
  // into rows (row_of, src_of); otherwise the layout kernel already did
  auto dispatch_bf16 = [&]() {
    return ranked ? moe::launch_dispatch_scatter(X, idx, row_of, offsets, d.T, d.d, d.k, d.E,
                                                 Xe, src_of, *dev, s)
                  : moe::launch_dispatch_rows(X, row_of, d.T, d.d, d.k, Xe, *dev, s);
  };
  if (comb) {
    ex2.comb_Y = Y;
    ex2.comb_src = src_of;
    ex2.comb_row_of = row_of;
    ex2.comb_gates = gates;
    ex2.comb_part = reinterpret_cast<float*>(base + w.part);
    ex2.comb_cnt = ctr + lc.comb;
    ex2.comb_k = d.k;
    ex2.comb_T = d.T;
  }
  std::string err;
  cudaError_t e;
  if (fused) {  // both GEMMs in one persistent launch
    if (fdisp) {  // dispatch chunks run inside it
      ex2.disp_X = X;
      ex2.disp_src = src_of;
      ex2.disp_k = d.k;
      ex2.disp_T = d.T;
      ex2.dready = ctr + lc.disp;
    } else if (fp8) {
      MOE_STAGE("moe.dispatch");
      MOE_CUDA(moe::launch_dispatch_fp8_rows(X, row_of, d.T, d.d, d.k, Xe, x_scale, *dev, s),
               "dispatch_fp8");
    } else {
      MOE_STAGE("moe.dispatch");
      MOE_CUDA(dispatch_bf16(), "dispatch");
    }
    MOE_STAGE("moe.fused_ffn");
    e = moe::launch_fused_ffn(Xe, x_scale, offsets, W1, W1s, W2, d.E, R, d.d, d.f, fp8, H, Ye,
                              ctr + lc.ffn, true, *dev, s, &err, &ex2);
    if (e != cudaSuccess) return gemm_fail(e, err, "fused_ffn");
    if (!comb)
      MOE_CUDA(moe::launch_combine(Ye, row_of, gates, d.T, d.d, d.k, Y, *dev, s), "combine");
    return MOE_OK;
  }
  if (gather) {  // dispatch fused into GEMM-1: its rows are read through src_of
    const void* A = X;
    if (fp8) {   // the tokens are quantised once (T rows), into the Xe slot
      MOE_CUDA(moe::launch_quantize_tensor(X, (int64_t)d.T * d.d, Xe, x_scale, *dev, s),
               "quantize_fp8");
      A = Xe;
    }
    e = moe::launch_grouped_gemm_gather(A, x_scale, src_of, d.T, d.k, offsets, W1, W1s, d.E, d.f,
                                        d.d, true, fp8, H, *dev, s, &err);
  } else if (fp8) {
    {
      MOE_STAGE("moe.dispatch");
      MOE_CUDA(moe::launch_dispatch_fp8_rows(X, row_of, d.T, d.d, d.k, Xe, x_scale, *dev, s),
               "dispatch_fp8");
    }
    MOE_STAGE("moe.gemm1");
    e = moe::launch_grouped_gemm_fp8(Xe, x_scale, offsets, W1, W1s, d.E, R, d.f, d.d, true, H,
                                     *dev, s, &err, &ex1);
  } else {
    {
      MOE_STAGE("moe.dispatch");
      MOE_CUDA(dispatch_bf16(), "dispatch");
    }
    MOE_STAGE("moe.gemm1");
    e = moe::launch_grouped_gemm(Xe, offsets, W1, d.E, R, d.f, d.d, true, H, *dev, s, &err, &ex1);
  }
  if (e != cudaSuccess) return gemm_fail(e, err, "gemm1");
  {
    MOE_STAGE("moe.gemm2");
    e = moe::launch_grouped_gemm(H, offsets, W2, d.E, R, d.d, d.f, false, Ye, *dev, s, &err, &ex2);
  }
  if (e != cudaSuccess) return gemm_fail(e, err, "gemm2");
  if (!comb) {
    MOE_STAGE("moe.combine");
    MOE_CUDA(moe::launch_combine(Ye, row_of, gates, d.T, d.d, d.k, Y, *dev, s), "combine");
  }
  return MOE_OK;
}

moe_status check_gemm_shape(int32_t E, int32_t R, int32_t N, int32_t K, int32_t gelu) {
  if (E < 1) return fail(MOE_ERR_INVALID_ARG, "E must be >= 1");
  if (E > moe::kMaxExperts) return fail(MOE_ERR_UNSUPPORTED, "E > 1024 is not supported");
  if (R < 0) return fail(MOE_ERR_INVALID_ARG, "R must be >= 0");
  if (R >= (1 << 30)) return fail(MOE_ERR_UNSUPPORTED, "R must be < 2^30");
  MOE_TRY(check_dim(N, "N"));
  MOE_TRY(check_dim(K, "K"));
  if ((int64_t)E * N >= (1ll << 31)) return fail(MOE_ERR_UNSUPPORTED, "E*N must be < 2^31");
  if (gelu != 0 && gelu != 1) return fail(MOE_ERR_INVALID_ARG, "gelu must be 0 or 1");
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_last_error_string(void) { return moe::g_last_error.c_str(); }

moe_status moe_device_status(uint32_t* bits, int32_t clear) {
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
  uint32_t v = 0;
  MOE_CUDA(cudaMemcpy(&v, dev->status, sizeof(v), cudaMemcpyDeviceToHost), "read status");
  if (clear) MOE_CUDA(cudaMemset(dev->status, 0, sizeof(uint32_t)), "clear status");
  if (bits) *bits = v;
  if (v) return fail(MOE_ERR_DEVICE, "device status bits set: " + std::to_string(v));
  return MOE_OK;
}

moe_status moe_selftest_bounded_wait(int32_t which, uint32_t limit_us, uint32_t* counter,
                                     void* stream) {
  if (which < 0 || which > 3) return fail(MOE_ERR_INVALID_ARG, "which must be 0, 1, 2 or 3");
  if (limit_us < 1 || limit_us > 10u * 1000u * 1000u)
    return fail(MOE_ERR_INVALID_ARG, "limit_us must be in [1, 10^7]");
  if (which == 0 || which == 2) MOE_TRY(check_ptr4(counter, "counter"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_selftest_wait(which, (uint64_t)limit_us * 1000u, counter, *dev,
                                     as_stream(stream)),
           "selftest_wait");
  return MOE_OK;
}

moe_status moe_router_logits(const void* X, const void* Wr, int32_t T, int32_t d, int32_t E,
                             float* logits, void* stream) {
  MOE_TRY(check_ET(T, E, 1));
  MOE_TRY(check_dim(d, "d"));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(X, "X"));
  MOE_TRY(check_ptr(Wr, "Wr"));
  MOE_TRY(check_ptr4(logits, "logits"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_router_logits(X, Wr, T, d, E, logits, *dev, as_stream(stream)),
           "router_logits");
  return MOE_OK;
}

moe_status moe_route_ex(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                        int32_t renormalize, float temperature, float min_prob,
                        int32_t* topk_idx, float* gates, void* stream) {
  MOE_TRY(check_ET(T, E, k));
  if (score != MOE_SCORE_SOFTMAX && score != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown score");
  if (renormalize != 0 && renormalize != 1)
    return fail(MOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (!std::isfinite(temperature) || !(temperature > 0.f))
    return fail(MOE_ERR_INVALID_ARG, "temperature must be > 0");
  if (!std::isfinite(min_prob)) return fail(MOE_ERR_INVALID_ARG, "min_prob must be finite");
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr4(logits, "logits"));
  MOE_TRY(check_ptr4(topk_idx, "topk_idx"));
  MOE_TRY(check_ptr4(gates, "gates"));
  MOE_CUDA(moe::launch_route(logits, T, E, k, score, renormalize, temperature, min_prob, topk_idx,
                             gates, as_stream(stream)),
           "route");
  return MOE_OK;
}

moe_status moe_route(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                     int32_t renormalize, int32_t* topk_idx, float* gates, void* stream) {
  return moe_route_ex(logits, T, E, k, score, renormalize, 1.0f, 0.0f, topk_idx, gates, stream);
}

size_t moe_layout_workspace_size(int32_t T, int32_t E, int32_t k) {
  if (T < 0 || E < 1 || k < 1) return 0;
  return up256(moe::layout_workspace_bytes((int64_t)T * k, E));
}

moe_status moe_layout(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k, int32_t* counts,
                      int32_t* offsets, int32_t* row_of, int32_t* src_of, void* ws,
                      size_t ws_bytes, void* stream) {
  MOE_TRY(check_ET(T, E, k));
  MOE_TRY(check_ptr4(counts, "counts"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  const size_t need = moe_layout_workspace_size(T, E, k);
  if (T > 0) {
    MOE_TRY(check_ptr4(topk_idx, "topk_idx"));
    MOE_TRY(check_ptr4(row_of, "row_of"));
    MOE_TRY(check_ptr4(src_of, "src_of"));
  }
  if (ws_bytes < need) return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  if (need > 0) MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  cudaStream_t s = as_stream(stream);
  if (T == 0) {  // every expert empty
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), s), "memset counts");
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s), "memset offsets");
    return MOE_OK;
  }
  MOE_CUDA(moe::launch_layout(topk_idx, T * k, E, counts, offsets, row_of, src_of, ws, *dev, s),
           "layout");
  return MOE_OK;
}

size_t moe_route_layout_workspace_size(int32_t T, int32_t E) {
  if (T < 0 || E < 1) return 0;
  return up256(moe::route_rank_lookback_words(T, E) * sizeof(uint32_t));
}

moe_status moe_route_layout(const float* logits, int32_t T, int32_t E, int32_t k, int32_t score,
                            int32_t renormalize, float temperature, float min_prob,
                            int32_t* topk_idx, float* gates, int32_t* counts, int32_t* offsets,
                            int32_t* row_of, int32_t* src_of, void* ws, size_t ws_bytes,
                            void* stream) {
  MOE_TRY(check_ET(T, E, k));
  if (score != MOE_SCORE_SOFTMAX && score != MOE_SCORE_SIGMOID)
    return fail(MOE_ERR_INVALID_ARG, "unknown score");
  if (renormalize != 0 && renormalize != 1)
    return fail(MOE_ERR_INVALID_ARG, "renormalize must be 0 or 1");
  if (!std::isfinite(temperature) || !(temperature > 0.f))
    return fail(MOE_ERR_INVALID_ARG, "temperature must be > 0");
  if (!std::isfinite(min_prob)) return fail(MOE_ERR_INVALID_ARG, "min_prob must be finite");
  MOE_TRY(check_ptr4(counts, "counts"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  cudaStream_t s = as_stream(stream);
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, (size_t)E * sizeof(int32_t), s), "memset counts");
    MOE_CUDA(cudaMemsetAsync(offsets, 0, (size_t)(E + 1) * sizeof(int32_t), s), "memset offsets");
    return MOE_OK;
  }
  MOE_TRY(check_ptr4(logits, "logits"));
  MOE_TRY(check_ptr4(topk_idx, "topk_idx"));
  MOE_TRY(check_ptr4(gates, "gates"));
  MOE_TRY(check_ptr4(row_of, "row_of"));
  MOE_TRY(check_ptr4(src_of, "src_of"));
  if (ws_bytes < moe_route_layout_workspace_size(T, E))
    return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  uint32_t* lb = static_cast<uint32_t*>(ws);
  MOE_CUDA(cudaMemsetAsync(lb, 0, moe::route_rank_lookback_words(T, E) * sizeof(uint32_t), s),
           "memset look-back");
  MOE_CUDA(moe::launch_route_rank(logits, T, E, k, score, renormalize, temperature, min_prob,
                                  topk_idx, gates, row_of, counts, offsets, lb, *dev, s),
           "route_rank");
  MOE_CUDA(moe::launch_dispatch_scatter(nullptr, topk_idx, row_of, offsets, T, 8, k, E, nullptr,
                                        src_of, *dev, s),
           "rows");
  return MOE_OK;
}

moe_status moe_dispatch(const void* X, const int32_t* src_of, int32_t T, int32_t d, int32_t k,
                        void* Xe, void* stream) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_dim(d, "d"));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(X, "X"));
  MOE_TRY(check_ptr4(src_of, "src_of"));
  MOE_TRY(check_ptr(Xe, "Xe"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_dispatch(X, src_of, T, d, k, Xe, *dev, as_stream(stream)), "dispatch");
  return MOE_OK;
}

moe_status moe_dispatch_by_token(const void* X, const int32_t* row_of, int32_t T, int32_t d,
                                 int32_t k, void* Xe, void* stream) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_dim(d, "d"));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(X, "X"));
  MOE_TRY(check_ptr4(row_of, "row_of"));
  MOE_TRY(check_ptr(Xe, "Xe"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_dispatch_rows(X, row_of, T, d, k, Xe, *dev, as_stream(stream)),
           "dispatch_by_token");
  return MOE_OK;
}

moe_status moe_dispatch_fp8_by_token(const void* X, const int32_t* row_of, int32_t T, int32_t d,
                                     int32_t k, void* Xeq, float* x_scale, void* stream) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_dim(d, "d"));
  MOE_TRY(check_fp8_dim(d, "d"));
  MOE_TRY(check_ptr4(x_scale, "x_scale"));
  if (T > 0) {
    MOE_TRY(check_ptr(X, "X"));
    MOE_TRY(check_ptr4(row_of, "row_of"));
    MOE_TRY(check_ptr(Xeq, "Xeq"));
  }
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_dispatch_fp8_rows(X, row_of, T, d, k, Xeq, x_scale, *dev,
                                         as_stream(stream)),
           "dispatch_fp8_by_token");
  return MOE_OK;
}

moe_status moe_expert_gemm(const void* A, const int32_t* offsets, const void* W, int32_t E,
                           int32_t R, int32_t N, int32_t K, int32_t gelu, void* out,
                           void* stream) {
  MOE_TRY(check_gemm_shape(E, R, N, K, gelu));
  if (R == 0) return MOE_OK;
  MOE_TRY(check_ptr(A, "A"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  MOE_TRY(check_ptr(W, "W"));
  MOE_TRY(check_ptr(out, "out"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  std::string err;
  cudaError_t e = moe::launch_grouped_gemm(A, offsets, W, E, R, N, K, gelu != 0, out, *dev,
                                           as_stream(stream), &err);
  if (e != cudaSuccess) return gemm_fail(e, err, "expert_gemm");
  return MOE_OK;
}

moe_status moe_expert_gemm_fp8(const void* Aq, const float* a_scale, const int32_t* offsets,
                               const void* Wq, const float* w_scale, int32_t E, int32_t R,
                               int32_t N, int32_t K, int32_t gelu, void* out, void* stream) {
  MOE_TRY(check_gemm_shape(E, R, N, K, gelu));
  MOE_TRY(check_fp8_dim(K, "K"));
  if (R == 0) return MOE_OK;
  MOE_TRY(check_ptr(Aq, "Aq"));
  MOE_TRY(check_ptr4(a_scale, "a_scale"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  MOE_TRY(check_ptr(Wq, "Wq"));
  MOE_TRY(check_ptr4(w_scale, "w_scale"));
  MOE_TRY(check_ptr(out, "out"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  std::string err;
  cudaError_t e = moe::launch_grouped_gemm_fp8(Aq, a_scale, offsets, Wq, w_scale, E, R, N, K,
                                               gelu != 0, out, *dev, as_stream(stream), &err);
  if (e != cudaSuccess) return gemm_fail(e, err, "expert_gemm_fp8");
  return MOE_OK;
}

moe_status moe_quantize_fp8(const void* X, int32_t rows, int32_t cols, void* Xq, float* x_scale,
                            void* stream) {
  if (rows < 0 || cols < 1) return fail(MOE_ERR_INVALID_ARG, "need rows >= 0 and cols >= 1");
  MOE_TRY(check_fp8_dim(cols, "cols"));
  MOE_TRY(check_ptr4(x_scale, "x_scale"));
  const int64_t n = (int64_t)rows * cols;
  if (n > 0) {
    MOE_TRY(check_ptr(X, "X"));
    MOE_TRY(check_ptr(Xq, "Xq"));
  }
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_quantize_tensor(X, n, Xq, x_scale, *dev, as_stream(stream)), "quantize_fp8");
  return MOE_OK;
}

namespace {
moe_status gemm_gather(const void* X, const float* x_scale, const int32_t* src_of, int32_t T,
                       int32_t k, const int32_t* offsets, const void* W, const float* w_scale,
                       int32_t E, int32_t N, int32_t K, int32_t gelu, void* out, void* stream,
                       bool fp8) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_gemm_shape(E, T * k, N, K, gelu));
  if (fp8) MOE_TRY(check_fp8_dim(K, "K"));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(X, "X"));
  MOE_TRY(check_ptr4(src_of, "src_of"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  MOE_TRY(check_ptr(W, "W"));
  MOE_TRY(check_ptr(out, "out"));
  if (fp8) {
    MOE_TRY(check_ptr4(x_scale, "x_scale"));
    MOE_TRY(check_ptr4(w_scale, "w_scale"));
  }
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  std::string err;
  cudaError_t e = moe::launch_grouped_gemm_gather(X, x_scale, src_of, T, k, offsets, W, w_scale,
                                                  E, N, K, gelu != 0, fp8, out, *dev,
                                                  as_stream(stream), &err);
  if (e != cudaSuccess) return gemm_fail(e, err, fp8 ? "expert_gemm_gather_fp8" : "expert_gemm_gather");
  return MOE_OK;
}
}  // namespace

moe_status moe_expert_gemm_gather(const void* X, const int32_t* src_of, int32_t T, int32_t k,
                                  const int32_t* offsets, const void* W, int32_t E, int32_t N,
                                  int32_t K, int32_t gelu, void* out, void* stream) {
  return gemm_gather(X, nullptr, src_of, T, k, offsets, W, nullptr, E, N, K, gelu, out, stream,
                     false);
}

moe_status moe_expert_gemm_gather_fp8(const void* Xq, const float* x_scale, const int32_t* src_of,
                                      int32_t T, int32_t k, const int32_t* offsets,
                                      const void* Wq, const float* w_scale, int32_t E, int32_t N,
                                      int32_t K, int32_t gelu, void* out, void* stream) {
  return gemm_gather(Xq, x_scale, src_of, T, k, offsets, Wq, w_scale, E, N, K, gelu, out, stream,
                     true);
}

moe_status moe_quantize_experts_fp8(const void* W, int32_t E, int32_t rows, int32_t cols,
                                    void* Wq, float* scales, void* stream) {
  if (E < 1 || rows < 0 || cols < 1) return fail(MOE_ERR_INVALID_ARG, "need E >= 1, rows >= 0, cols >= 1");
  if (E > 65535) return fail(MOE_ERR_UNSUPPORTED, "E > 65535 is not supported");
  MOE_TRY(check_fp8_dim(cols, "cols"));
  MOE_TRY(check_ptr4(scales, "scales"));
  const int64_t per = (int64_t)rows * cols;
  if (per > 0) {
    MOE_TRY(check_ptr(W, "W"));
    MOE_TRY(check_ptr(Wq, "Wq"));
  }
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_quantize_experts(W, E, per, Wq, scales, *dev, as_stream(stream)),
           "quantize_experts_fp8");
  return MOE_OK;
}

moe_status moe_dispatch_fp8(const void* X, const int32_t* src_of, int32_t T, int32_t d,
                            int32_t k, void* Xeq, float* x_scale, void* stream) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_dim(d, "d"));
  MOE_TRY(check_fp8_dim(d, "d"));
  MOE_TRY(check_ptr4(x_scale, "x_scale"));
  if (T > 0) {
    MOE_TRY(check_ptr(X, "X"));
    MOE_TRY(check_ptr4(src_of, "src_of"));
    MOE_TRY(check_ptr(Xeq, "Xeq"));
  }
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_dispatch_fp8(X, src_of, T, d, k, Xeq, x_scale, *dev, as_stream(stream)),
           "dispatch_fp8");
  return MOE_OK;
}

moe_status moe_expert_ffn(const void* Xe, const int32_t* offsets, const void* W1, const void* W2,
                          int32_t E, int32_t R, int32_t d, int32_t f, void* H, void* Ye,
                          void* stream) {
  MOE_TRY(moe_expert_gemm(Xe, offsets, W1, E, R, f, d, 1, H, stream));
  return moe_expert_gemm(H, offsets, W2, E, R, d, f, 0, Ye, stream);
}

size_t moe_expert_ffn_fused_workspace_size(int32_t E, int32_t R) {
  if (E < 1 || R < 0) return 0;
  return up256((size_t)moe::ffn_counter_words(R, E) * sizeof(uint32_t));
}

namespace {
moe_status ffn_fused(const void* A, const float* a_scale, const int32_t* offsets, const void* W1,
                     const float* w1_scale, const void* W2, int32_t E, int32_t R, int32_t d,
                     int32_t f, void* H, void* Ye, void* ws, size_t ws_bytes, void* stream,
                     bool fp8) {
  MOE_TRY(check_gemm_shape(E, R, f, d, 1));
  MOE_TRY(check_gemm_shape(E, R, d, f, 0));
  if (fp8) MOE_TRY(check_fp8_dim(d, "d"));
  if (R == 0) return MOE_OK;
  MOE_TRY(check_ptr(A, fp8 ? "Xeq" : "Xe"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  MOE_TRY(check_ptr(W1, fp8 ? "W1q" : "W1"));
  MOE_TRY(check_ptr(W2, "W2"));
  MOE_TRY(check_ptr(H, "H"));
  MOE_TRY(check_ptr(Ye, "Ye"));
  if (fp8) {
    MOE_TRY(check_ptr4(a_scale, "x_scale"));
    MOE_TRY(check_ptr4(w1_scale, "w1_scale"));
  }
  if (ws_bytes < moe_expert_ffn_fused_workspace_size(E, R))
    return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  std::string err;
  cudaError_t e = moe::launch_fused_ffn(A, a_scale, offsets, W1, w1_scale, W2, E, R, d, f, fp8,
                                        H, Ye, static_cast<uint32_t*>(ws), false, *dev,
                                        as_stream(stream), &err);
  if (e != cudaSuccess) return gemm_fail(e, err, "expert_ffn_fused");
  return MOE_OK;
}
}  // namespace

moe_status moe_expert_ffn_fused(const void* Xe, const int32_t* offsets, const void* W1,
                                const void* W2, int32_t E, int32_t R, int32_t d, int32_t f,
                                void* H, void* Ye, void* ws, size_t ws_bytes, void* stream) {
  return ffn_fused(Xe, nullptr, offsets, W1, nullptr, W2, E, R, d, f, H, Ye, ws, ws_bytes,
                   stream, false);
}

moe_status moe_expert_ffn_fused_fp8(const void* Xeq, const float* x_scale,
                                    const int32_t* offsets, const void* W1q,
                                    const float* w1_scale, const void* W2, int32_t E, int32_t R,
                                    int32_t d, int32_t f, void* H, void* Ye, void* ws,
                                    size_t ws_bytes, void* stream) {
  return ffn_fused(Xeq, x_scale, offsets, W1q, w1_scale, W2, E, R, d, f, H, Ye, ws, ws_bytes,
                   stream, true);
}

namespace {
// Workspace of moe_ffn_pipeline: Xe, H, (k > 2) Ye, fp32 partial rows, counters.
struct PipeWs {
  size_t Xe, H, Ye, part, ctr, total;
  int ctr_words;
};
PipeWs pipe_ws(int32_t T, int32_t d, int32_t E, int32_t k, int32_t f) {
  PipeWs w;
  const size_t R = (size_t)T * k;
  size_t o = 0;
  w.Xe = o;   o += up256(R * d * 2);
  w.H = o;    o += up256(R * f * 2);
  w.Ye = o;   o += k > 2 ? up256(R * d * 2) : 0;
  w.part = o; o += k <= 2 ? up256((size_t)T * d * sizeof(float)) : 0;
  w.ctr_words = moe::ffn_counter_words((int)R, E) + moe::dispatch_counter_words((int)R) +
                (k <= 2 ? moe::combine_counter_words(T, d) : 0);
  w.ctr = o;  o += up256((size_t)w.ctr_words * sizeof(uint32_t));
  w.total = o;
  return w;
}
}  // namespace

size_t moe_ffn_pipeline_workspace_size(int32_t T, int32_t d, int32_t E, int32_t k, int32_t f) {
  if (T < 0 || d < 1 || E < 1 || k < 1 || f < 1) return 0;
  return pipe_ws(T, d, E, k, f).total;
}

moe_status moe_ffn_pipeline(const void* X, const int32_t* src_of, const int32_t* row_of,
                            const float* gates, const int32_t* offsets, const void* W1,
                            const void* W2, int32_t T, int32_t d, int32_t E, int32_t k,
                            int32_t f, void* Y, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_ET(T, E, k));
  MOE_TRY(check_dim(d, "d"));
  MOE_TRY(check_dim(f, "f"));
  const int R = T * k;
  MOE_TRY(check_gemm_shape(E, R, f, d, 1));
  MOE_TRY(check_gemm_shape(E, R, d, f, 0));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(X, "X"));
  MOE_TRY(check_ptr4(src_of, "src_of"));
  MOE_TRY(check_ptr4(row_of, "row_of"));
  MOE_TRY(check_ptr4(gates, "gates"));
  MOE_TRY(check_ptr4(offsets, "offsets"));
  MOE_TRY(check_ptr(W1, "W1"));
  MOE_TRY(check_ptr(W2, "W2"));
  MOE_TRY(check_ptr(Y, "Y"));
  const PipeWs w = pipe_ws(T, d, E, k, f);
  if (ws_bytes < w.total) return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  cudaStream_t s = as_stream(stream);
  char* base = static_cast<char*>(ws);
  uint32_t* ctr = reinterpret_cast<uint32_t*>(base + w.ctr);
  MOE_CUDA(cudaMemsetAsync(ctr, 0, (size_t)w.ctr_words * sizeof(uint32_t), s), "memset counters");
  const int nffn = moe::ffn_counter_words(R, E);
  moe::GemmExtras ex;
  ex.disp_X = X;
  ex.disp_src = src_of;
  ex.disp_k = k;
  ex.disp_T = T;
  ex.dready = ctr + nffn;
  const bool comb = k <= 2;
  if (comb) {
    ex.comb_Y = Y;
    ex.comb_src = src_of;
    ex.comb_row_of = row_of;
    ex.comb_gates = gates;
    ex.comb_part = reinterpret_cast<float*>(base + w.part);
    ex.comb_cnt = ctr + nffn + moe::dispatch_counter_words(R);
    ex.comb_k = k;
    ex.comb_T = T;
  }
  void* Ye = comb ? nullptr : base + w.Ye;
  std::string err;
  cudaError_t e = moe::launch_fused_ffn(base + w.Xe, nullptr, offsets, W1, nullptr, W2, E, R, d,
                                        f, false, base + w.H, Ye, ctr, true, *dev, s, &err, &ex);
  if (e != cudaSuccess) return gemm_fail(e, err, "ffn_pipeline");
  if (!comb)
    MOE_CUDA(moe::launch_combine(Ye, row_of, gates, T, d, k, Y, *dev, s), "combine");
  return MOE_OK;
}

moe_status moe_combine(const void* Ye, const int32_t* row_of, const float* gates, int32_t T,
                       int32_t d, int32_t k, void* Y, void* stream) {
  if (T < 0 || k < 1) return fail(MOE_ERR_INVALID_ARG, "need T >= 0 and k >= 1");
  if (k > moe::kMaxTopK) return fail(MOE_ERR_UNSUPPORTED, "k > 16 is not supported");
  if ((int64_t)T * k >= (1ll << 30)) return fail(MOE_ERR_UNSUPPORTED, "T*k must be < 2^30");
  MOE_TRY(check_dim(d, "d"));
  if (T == 0) return MOE_OK;
  MOE_TRY(check_ptr(Ye, "Ye"));
  MOE_TRY(check_ptr4(row_of, "row_of"));
  MOE_TRY(check_ptr4(gates, "gates"));
  MOE_TRY(check_ptr(Y, "Y"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  MOE_CUDA(moe::launch_combine(Ye, row_of, gates, T, d, k, Y, *dev, as_stream(stream)), "combine");
  return MOE_OK;
}

size_t moe_workspace_size(const moe_layer_desc* desc) {
  if (check_desc(desc) != MOE_OK) return 0;
  return layer_ws(*desc).total;
}

int32_t moe_kernel_launches_per_forward(const moe_layer_desc* desc, int32_t with_router) {
  if (check_desc(desc) != MOE_OK || desc->T == 0) return 0;
  // [router linear] + route + layout + [dispatch] + 2 GEMMs (1 fused) + [combine]
  const int f = desc->flags;
  const bool fused = (f & MOE_LAYER_FUSED_FFN) != 0;
  const int dispatch =
      ((f & MOE_LAYER_GATHER_ON_LOAD) || (fused && (f & MOE_LAYER_FUSED_DISPATCH))) ? 0 : 1;
  const int gemms = fused ? 1 : 2;
  const int combine = ((f & MOE_LAYER_FUSED_COMBINE) && desc->k <= 2) ? 0 : 1;
  // the bf16 layer ranks the slots inside the routing kernel (no layout
  // launch) unless it gathers or dispatches inside the fused FFN
  const bool ranked = !(f & MOE_LAYER_GATHER_ON_LOAD) &&
                      !(fused && (f & MOE_LAYER_FUSED_DISPATCH)) &&
                      desc->E <= moe::kRankedMaxExperts;
  const int layout = ranked ? 0 : moe::layout_kernel_count((int64_t)desc->T * desc->k, desc->E);
  return (with_router ? 1 : 0) + 1 + layout + dispatch + gemms + combine;
}

int32_t moe_kernel_launches_per_forward_fp8(const moe_layer_desc* desc, int32_t with_router) {
  if (check_desc(desc) != MOE_OK || desc->T == 0) return 0;
  // the quantising dispatch (or, gathering, the quantisation of X) is the
  // absmax kernel plus one; FP8 mode has no dispatch items
  moe_layer_desc d = *desc;
  d.flags &= ~MOE_LAYER_FUSED_DISPATCH;
  const int dispatch = (d.flags & MOE_LAYER_GATHER_ON_LOAD) ? 0 : 1;
  // FP8 mode keeps the separate layout kernel (the bf16 count has none when
  // it ranks in the routing kernel)
  const bool ranked = !(d.flags & MOE_LAYER_GATHER_ON_LOAD) && d.E <= moe::kRankedMaxExperts;
  const int layout = ranked ? moe::layout_kernel_count((int64_t)desc->T * desc->k, desc->E) : 0;
  return moe_kernel_launches_per_forward(&d, with_router) - dispatch + layout +
         moe::fp8_dispatch_kernel_count(desc->T);
}

moe_status moe_layer_forward(const moe_layer_desc* desc, const void* X, const float* logits,
                             const void* Wr, const void* W1, const void* W2, void* Y,
                             int32_t* topk_idx_out, float* gates_out, int32_t* counts_out,
                             void* ws, size_t ws_bytes, void* stream) {
  return layer_forward(desc, X, logits, Wr, W1, nullptr, W2, Y, topk_idx_out, gates_out,
                       counts_out, ws, ws_bytes, stream);
}

// ---------------------------------------------------------------------------
// Host-buffer batches (moe_layer_forward_host): per-device streams and events
// owned by the library, created on first use.
// ---------------------------------------------------------------------------
namespace {
struct HostLanes {
  std::mutex mu;  // one enqueue at a time per device (the events are shared)
  bool ready = false;
  cudaError_t err = cudaSuccess;
  cudaStream_t h2d = nullptr, comp = nullptr, d2h = nullptr;
  cudaEvent_t entry = nullptr, done = nullptr;
  cudaEvent_t x_ready[2] = {}, x_free[2] = {}, y_ready[2] = {}, y_free[2] = {};
};
HostLanes g_lanes[64];

cudaError_t lanes_init(HostLanes& h) {
  cudaError_t e = cudaSuccess;
  auto ev = [&](cudaEvent_t* p) {
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(p, cudaEventDisableTiming);
  };
  for (cudaStream_t* st : {&h.h2d, &h.comp, &h.d2h})
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(st, cudaStreamNonBlocking);
  ev(&h.entry);
  ev(&h.done);
  for (int i = 0; i < 2; ++i) {
    ev(&h.x_ready[i]);
    ev(&h.x_free[i]);
    ev(&h.y_ready[i]);
    ev(&h.y_free[i]);
  }
  return e;
}

struct HostWs {
  size_t X[2], Y[2], L[2], layer, total;
};
HostWs host_ws(const moe_layer_desc& d, bool with_logits) {
  HostWs w;
  size_t o = 0;
  for (int i = 0; i < 2; ++i) {
    w.X[i] = o; o += up256((size_t)d.T * d.d * 2);
    w.Y[i] = o; o += up256((size_t)d.T * d.d * 2);
    w.L[i] = o; o += with_logits ? up256((size_t)d.T * d.E * sizeof(float)) : 0;
  }
  w.layer = o;
  o += layer_ws(d).total;
  w.total = o;
  return w;
}
}  // namespace

size_t moe_host_workspace_size(const moe_layer_desc* desc, int32_t with_logits) {
  if (check_desc(desc) != MOE_OK) return 0;
  return host_ws(*desc, with_logits != 0).total;
}

moe_status moe_layer_forward_host(const moe_layer_desc* desc, int32_t nbatch,
                                  const void* const* X_host, const float* const* logits_host,
                                  const void* Wr, const void* W1, const float* w1_scale,
                                  const void* W2, void* const* Y_host, void* ws, size_t ws_bytes,
                                  void* stream) {
  MOE_TRY(check_desc(desc));
  const moe_layer_desc d = *desc;
  if (nbatch < 0) return fail(MOE_ERR_INVALID_ARG, "nbatch must be >= 0");
  if (nbatch == 0 || d.T == 0) return MOE_OK;
  if (!X_host || !Y_host) return fail(MOE_ERR_INVALID_ARG, "X_host and Y_host are required");
  if ((logits_host == nullptr) == (Wr == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "give exactly one of logits_host and Wr");
  for (int i = 0; i < nbatch; ++i) {
    if (!X_host[i] || !Y_host[i] || (logits_host && !logits_host[i]))
      return fail(MOE_ERR_INVALID_ARG, "batch " + std::to_string(i) + ": a host pointer is NULL");
  }
  const bool with_logits = logits_host != nullptr;
  const HostWs w = host_ws(d, with_logits);
  if (ws_bytes < w.total) return fail(MOE_ERR_INVALID_ARG, "workspace too small");
  MOE_TRY(check_ptr(ws, "ws"));
  const moe::DeviceInfo* dev;
  MOE_TRY(get_dev(&dev));
  HostLanes& h = g_lanes[dev->device & 63];
  std::lock_guard<std::mutex> lock(h.mu);
  if (!h.ready) {
    h.err = lanes_init(h);
    h.ready = h.err == cudaSuccess;
    if (!h.ready) return cuda_fail(h.err, "host-batch streams");
  }
  char* base = static_cast<char*>(ws);
  const size_t xb = (size_t)d.T * d.d * 2, lb = (size_t)d.T * d.E * sizeof(float);
  cudaStream_t caller = as_stream(stream);
  // everything enqueued on `stream` before this call comes first
  MOE_CUDA(cudaEventRecord(h.entry, caller), "record entry");
  for (cudaStream_t st : {h.h2d, h.comp, h.d2h})
    MOE_CUDA(cudaStreamWaitEvent(st, h.entry, 0), "wait entry");
  for (int i = 0; i < nbatch; ++i) {
    const int s = i & 1;
    void* Xd = base + w.X[s];
    void* Yd = base + w.Y[s];
    float* Ld = with_logits ? reinterpret_cast<float*>(base + w.L[s]) : nullptr;
    // inputs of batch i into buffer set s, once the forward two batches back
    // (this call's or a previous call's) has read it
    MOE_CUDA(cudaStreamWaitEvent(h.h2d, h.x_free[s], 0), "wait x_free");
    MOE_CUDA(cudaMemcpyAsync(Xd, X_host[i], xb, cudaMemcpyHostToDevice, h.h2d), "copy X");
    if (with_logits)
      MOE_CUDA(cudaMemcpyAsync(Ld, logits_host[i], lb, cudaMemcpyHostToDevice, h.h2d),
               "copy logits");
    MOE_CUDA(cudaEventRecord(h.x_ready[s], h.h2d), "record x_ready");
    // the forward, once its inputs are in and Y[s] has been copied out
    MOE_CUDA(cudaStreamWaitEvent(h.comp, h.x_ready[s], 0), "wait x_ready");
    MOE_CUDA(cudaStreamWaitEvent(h.comp, h.y_free[s], 0), "wait y_free");
    MOE_TRY(layer_forward(&d, Xd, Ld, Wr, W1, w1_scale, W2, Yd, nullptr, nullptr, nullptr,
                          base + w.layer, ws_bytes - w.layer, h.comp));
    MOE_CUDA(cudaEventRecord(h.x_free[s], h.comp), "record x_free");
    MOE_CUDA(cudaEventRecord(h.y_ready[s], h.comp), "record y_ready");
    // the output back to the host
    MOE_CUDA(cudaStreamWaitEvent(h.d2h, h.y_ready[s], 0), "wait y_ready");
    MOE_CUDA(cudaMemcpyAsync(Y_host[i], Yd, xb, cudaMemcpyDeviceToHost, h.d2h), "copy Y");
    MOE_CUDA(cudaEventRecord(h.y_free[s], h.d2h), "record y_free");
  }
  MOE_CUDA(cudaEventRecord(h.done, h.d2h), "record done");
  MOE_CUDA(cudaStreamWaitEvent(caller, h.done, 0), "wait done");
  return MOE_OK;
}

moe_status moe_layer_forward_fp8(const moe_layer_desc* desc, const void* X, const float* logits,
                                 const void* Wr, const void* W1q, const float* w1_scale,
                                 const void* W2, void* Y, int32_t* topk_idx_out,
                                 float* gates_out, int32_t* counts_out, void* ws,
                                 size_t ws_bytes, void* stream) {
  if (!w1_scale) return fail(MOE_ERR_INVALID_ARG, "w1_scale is NULL");
  return layer_forward(desc, X, logits, Wr, W1q, w1_scale, W2, Y, topk_idx_out, gates_out,
                       counts_out, ws, ws_bytes, stream);
}

}  // extern "C"
