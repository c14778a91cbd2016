// Host-side launch wrappers of libmoe.so (internal; the public ABI is include/moe.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>
#include <utility>

namespace moe {

// Programmatic dependent launch.  Every kernel of the library starts with
// griddepcontrol.wait (it reads nothing a stream predecessor writes, and
// writes nothing it reads, before that point) and then lets its own
// dependents launch.  Launched with the stream-serialisation attribute, a
// kernel's blocks are therefore scheduled while its predecessor's last
// blocks run, and its launch latency and set-up overlap them; the wait keeps
// the stream order of every memory access.  MOE_PDL=0 in the environment
// launches without the attribute (plain stream order).
bool pdl_enabled();

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  if (pdl_enabled()) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Limits checked by the ABI before any launch.
constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 16;

// Per-device facts the launchers need, filled once per device.
struct DeviceInfo {
  int device = -1;
  int sm_count = 0;
  uint32_t* status = nullptr;  // device address of the sticky status word
};

// Returns the info of the current device, initialising it on first use
// (cudaGetSymbolAddress, attribute queries).  nullptr on a CUDA error, with
// the message in *err.
const DeviceInfo* current_device_info(std::string* err);

// zero_words (optional): n_zero_words words cleared by the same launch.
cudaError_t launch_router_logits(const void* X, const void* Wr, int T, int d, int E, float* L,
                                 const DeviceInfo& dev, cudaStream_t stream,
                                 uint32_t* zero_words = nullptr, int n_zero_words = 0);

// zero_rows (optional): [T, zero_d] bf16 rows zeroed for tokens with no kept slot.
// zero_words (optional): n_zero_words counter words cleared by the same launch.
cudaError_t launch_route(const float* L, int T, int E, int k, int score, int renormalize,
                         float temperature, float min_prob, int32_t* idx, float* gates,
                         cudaStream_t stream, void* zero_rows = nullptr, int zero_d = 0,
                         uint32_t* zero_words = nullptr, int n_zero_words = 0, int nsplit = 1);

// Routing fused with the layout's ranking (see route.cu): idx, gates, the
// stable rank of each kept slot within its expert (into rank[], -1 for a
// dropped slot), counts and offsets.  lookback: route_rank_lookback_words(T,
// E) words, zeroed before the launch.
size_t route_rank_lookback_words(int T, int E);
constexpr int kRankedMaxExperts = 32;  // the layer ranks in its routing kernel up to this E
// Split router (small batches, ranked path): partial logits P[s][T][E] over
// router_split_count(d) column slices, summed by the routing kernel.
constexpr int kSplitMaxT = 64;
int router_split_count(int d);
cudaError_t launch_router_split(const void* X, const void* Wr, int T, int d, int E, float* P,
                                const DeviceInfo& dev, cudaStream_t stream,
                                uint32_t* zero_words = nullptr, int n_zero_words = 0);
cudaError_t launch_route_rank(const float* L, int T, int E, int k, int score, int renormalize,
                              float temperature, float min_prob, int32_t* idx, float* gates,
                              int32_t* rank, int32_t* counts, int32_t* offsets, uint32_t* lookback,
                              const DeviceInfo& dev, cudaStream_t stream, void* zero_rows = nullptr,
                              int zero_d = 0, uint32_t* zero_words = nullptr,
                              int n_zero_words = 0, int nsplit = 1);
// Token-ordered dispatch finishing the layout from route_rank's ranks
// (row_of holds the ranks on entry and the rows on return; src_of written).
cudaError_t launch_dispatch_scatter(const void* X, const int32_t* idx, int32_t* row_of,
                                    const int32_t* offsets, int T, int d, int k, int E, void* Xe,
                                    int32_t* src_of, const DeviceInfo& dev, cudaStream_t stream);

size_t layout_workspace_bytes(int64_t R, int E);
// Number of kernels launch_layout issues for R slots.
int layout_kernel_count(int64_t R, int E);
cudaError_t launch_layout(const int32_t* idx, int R, int E, int32_t* counts, int32_t* offsets,
                          int32_t* row_of, int32_t* src_of, void* ws, const DeviceInfo& dev,
                          cudaStream_t stream);

cudaError_t launch_dispatch(const void* X, const int32_t* src_of, int T, int d, int k, void* Xe,
                            const DeviceInfo& dev, cudaStream_t stream);

// Token-ordered dispatch through row_of (each token row read once).
cudaError_t launch_dispatch_rows(const void* X, const int32_t* row_of, int T, int d, int k,
                                 void* Xe, const DeviceInfo& dev, cudaStream_t stream);
cudaError_t launch_dispatch_fp8_rows(const void* X, const int32_t* row_of, int T, int d, int k,
                                     void* Xeq, float* x_scale, const DeviceInfo& dev,
                                     cudaStream_t stream);

cudaError_t launch_combine(const void* Ye, const int32_t* row_of, const float* gates, int T,
                           int d, int k, void* Y, const DeviceInfo& dev, cudaStream_t stream);

// Optional parts of a grouped GEMM launch.
struct GemmExtras {
  // Dynamic schedule: clusters take work items from this counter in order
  // (the caller zeroes it before the launch); null: static round-robin.
  uint32_t* ticket = nullptr;
  // Gate-weighted combine in the epilogue of the GEMM without GELU (k <= 2):
  // Y [T, N] bf16 written instead of `out`; part [T, N] fp32 scratch; cnt
  // [T * ceil(N / 32)] words zeroed by the caller (combine_counter_words).
  void* comb_Y = nullptr;
  const int32_t* comb_src = nullptr;     // src_of [R]
  const int32_t* comb_row_of = nullptr;  // row_of [T*k]
  const float* comb_gates = nullptr;     // [T, k]
  float* comb_part = nullptr;
  uint32_t* comb_cnt = nullptr;
  int comb_k = 0, comb_T = 0;
  // Dispatch items (fused FFN with a ticket): A[r] = disp_X[disp_src[r] / disp_k]
  // copied inside the launch; dready: dispatch_counter_words(R) words, zeroed.
  const void* disp_X = nullptr;
  const int32_t* disp_src = nullptr;
  int disp_k = 0, disp_T = 0;
  uint32_t* dready = nullptr;
};
int combine_counter_words(int T, int N);
int dispatch_counter_words(int R);

// Grouped GEMM over per-expert row blocks (tcgen05 + TMA).  On a failure to
// build the TMA descriptors, returns cudaErrorInvalidValue with *err set.
cudaError_t launch_grouped_gemm(const void* A, const int32_t* offsets, const void* W, int E,
                                int R, int N, int K, bool gelu, void* out,
                                const DeviceInfo& dev, cudaStream_t stream, std::string* err,
                                const GemmExtras* ex = nullptr);

// FP8 (E4M3) mode: grouped GEMM on codes with per-tensor scales, the
// quantising dispatch (x_scale: [scale, amax]) and per-expert weight quantisation.
cudaError_t launch_grouped_gemm_fp8(const void* Aq, const float* a_scale, const int32_t* offsets,
                                    const void* Wq, const float* w_scale, int E, int R, int N,
                                    int K, bool gelu, void* out, const DeviceInfo& dev,
                                    cudaStream_t stream, std::string* err,
                                    const GemmExtras* ex = nullptr);
// Gather-on-load grouped GEMM: row r of the GEMM reads X[src_of[r] / k]
// (X: [T, K] bf16, or E4M3 codes with scale x_scale[0] when fp8).
cudaError_t launch_grouped_gemm_gather(const void* X, const float* x_scale, const int32_t* src_of,
                                       int T, int k, const int32_t* offsets, const void* W,
                                       const float* w_scale, int E, int N, int K, bool gelu,
                                       bool fp8, void* out, const DeviceInfo& dev,
                                       cudaStream_t stream, std::string* err);
// Fused FFN (GEMM-1 + GELU, then GEMM-2) in one persistent launch; A is Xe
// (bf16) or E4M3 codes with scale a_scale[0] and per-expert w1_scale (fp8).
// `ctr`: ffn_counter_words(R, E) words of scratch (a ticket and one readiness
// counter per token block), zeroed by the launcher unless `zeroed`.  `ex`
// may add dispatch items and the combine epilogue (its ticket is ignored).
int ffn_ready_count(int R, int E);
int ffn_counter_words(int R, int E);
cudaError_t launch_fused_ffn(const void* A, const float* a_scale, const int32_t* offsets,
                             const void* W1, const float* w1_scale, const void* W2, int E, int R,
                             int d, int f, bool fp8, void* H, void* Ye, uint32_t* ctr,
                             bool zeroed, const DeviceInfo& dev, cudaStream_t stream,
                             std::string* err, const GemmExtras* ex = nullptr);
// Per-tensor E4M3 quantisation of n bf16 values (n % 8 == 0): x_scale = [scale, amax].
cudaError_t launch_quantize_tensor(const void* X, int64_t n, void* Xq, float* x_scale,
                                   const DeviceInfo& dev, cudaStream_t stream);
cudaError_t launch_dispatch_fp8(const void* X, const int32_t* src_of, int T, int d, int k,
                                void* Xeq, float* x_scale, const DeviceInfo& dev,
                                cudaStream_t stream);
int fp8_dispatch_kernel_count(int64_t T);
cudaError_t launch_quantize_experts(const void* W, int E, int64_t per_expert, void* Wq,
                                    float* scales, const DeviceInfo& dev, cudaStream_t stream);

// Diagnostics: one bounded wait on a condition nothing satisfies (see selftest.cu).
cudaError_t launch_selftest_wait(int which, uint64_t limit_ns, uint32_t* counter,
                                 const DeviceInfo& dev, cudaStream_t stream);

// Records `msg` as this thread's moe_last_error_string() and returns `status`.
int set_last_error(int status, const std::string& msg);

}  // namespace moe
