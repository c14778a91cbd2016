// moe_layout_static: moe_layout for callers that cannot allocate device memory.
//
// Some callers have no way to obtain scratch space on the GPU: code that runs
// inside another framework's callback and is handed only the tensors it works
// on, with no allocator behind them; or code that must not allocate once it
// has started (a fixed memory budget, or allocation forbidden after set-up).
// For them this entry point keeps the layout's scratch (the multi-block
// scan's look-back words and tile ticket) in a fixed array that lives in the
// library itself.  The caller still passes every input and output.
//
// The array is file-scope device memory: every GPU that loads the library
// holds kStaticScratchBytes of it until the process exits.  In host code its
// name is only a host-side stand-in, so the kernels get its device address,
// looked up once per device with cudaGetSymbolAddress.  The lookup happens on
// the first call on each device (and again after a failed one); make that
// first call before any stream capture.  All calls on a device share the one
// array, so calls whose kernels could overlap on the GPU (different streams,
// or several host threads) race on it; the kernels re-arm what must start at
// zero on every call (look-back words, ticket), and the last call's contents
// stay behind.
#include <mutex>
#include <string>

#include "common.cuh"
#include "launch.h"

namespace moe {
namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB per device

static __device__ __align__(256) uint8_t g_layout_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices];  // non-null once this device's lookup succeeded

// Device address of this device's scratch array, looked up with the device
// current.  Only a successful lookup is kept: a failed one (say, a first
// call made during a stream capture) is retried on the next call, and its
// error is cleared from the runtime's last-error state so that no later call
// reports it as its own.  nullptr on failure, with the message set.
void* static_scratch(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_ptr[dev]) return g_scratch_ptr[dev];
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_layout_scratch);
  if (e != cudaSuccess || !p) {
    (void)cudaGetLastError();
    set_last_error(MOE_ERR_CUDA, std::string("moe_layout_static: cudaGetSymbolAddress: ") +
                                     cudaGetErrorString(e));
    return nullptr;
  }
  g_scratch_ptr[dev] = p;
  return p;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_layout_static(const int32_t* topk_idx, int32_t T, int32_t E, int32_t k,
                                        int32_t* counts, int32_t* offsets, int32_t* row_of,
                                        int32_t* src_of, void* stream) {
  using namespace moe;
  const bool shape_ok = T >= 0 && E >= 1 && E <= kMaxExperts && k >= 1 && k <= E &&
                        k <= kMaxTopK && (int64_t)T * k < (1ll << 30);
  // Invalid shapes: moe_layout reports the precise status and message.
  if (!shape_ok) return moe_layout(topk_idx, T, E, k, counts, offsets, row_of, src_of, nullptr, 0, stream);
  const size_t need = moe_layout_workspace_size(T, E, k);
  if (need > kStaticScratchBytes) {
    return (moe_status)set_last_error(
        MOE_ERR_UNSUPPORTED,
        "moe_layout_static: T*k = " + std::to_string((int64_t)T * k) + " slots over E = " +
            std::to_string(E) + " experts need " + std::to_string(need) +
            " bytes of scratch, more than the " + std::to_string(kStaticScratchBytes) +
            "-byte static array; call moe_layout with a workspace instead");
  }
  if (need == 0)  // the one-block path uses no scratch
    return moe_layout(topk_idx, T, E, k, counts, offsets, row_of, src_of, nullptr, 0, stream);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess)
    return (moe_status)set_last_error(MOE_ERR_CUDA, std::string("moe_layout_static: cudaGetDevice: ") +
                                                        cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices)
    return (moe_status)set_last_error(MOE_ERR_CUDA, "moe_layout_static: device ordinal out of range");
  void* scratch = static_scratch(dev);
  if (!scratch) return MOE_ERR_CUDA;
  return moe_layout(topk_idx, T, E, k, counts, offsets, row_of, src_of, scratch,
                    kStaticScratchBytes, stream);
}
