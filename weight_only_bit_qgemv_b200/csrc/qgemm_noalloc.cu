// qgemm_bf16_noalloc: the tensor-core qgemm for callers that cannot allocate device memory.
//
// The ordinary qgemm asks its caller for a workspace (the bf16 copy of X that the tensor
// cores read). Some callers have no way to provide one: a plugin whose host hands it only
// its input and output buffers, a serving runtime that has already reserved all device
// memory for its own pool and forbids any other allocation, or a latency-critical loop in
// which cudaMalloc's implicit device-wide synchronisation cannot be afforded. For them this
// entry point uses a fixed scratch array that lives in the library's own device image.
//
// That array is a file-scope __device__ symbol of kScratchBytes (32 MiB). Every GPU that
// loads the library holds it until the process exits. In host code its name is only a
// host-side stand-in for the symbol, never a device address, so the real address is
// looked up with cudaGetSymbolAddress (with that device current) on a device's first call
// and cached once the lookup has succeeded. All calls on a device share the one array; its contents after a call are that
// call's bf16 copy of X, and every call overwrites the part it reads before reading it, so
// nothing has to be cleared. Two calls whose kernels overlap on the GPU (for example on two
// streams without ordering between them) race on the array.
#include <atomic>

#include "woq.h"
#include "woq_internal.h"

namespace woq {
namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void *> g_ptr[kMaxDevices];

// Device address of the scratch array on the current device. Only a successful lookup is
// cached: a failed one (for example a first call made while a stream is being captured)
// fails that call alone, and the next call looks the address up again.
int scratch_address(int device, void **out) {
  if (device < 0 || device >= kMaxDevices) return WOQ_EDEVICE;
  void *p = g_ptr[device].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // reset the runtime's last-error state, which the lookup set
      return WOQ_ECUDA;
    }
    g_ptr[device].store(p, std::memory_order_release);
  }
  *out = p;
  return WOQ_OK;
}

}  // namespace
}  // namespace woq

extern "C" int qgemm_bf16_noalloc(const float *X, int64_t m, const woq_weight *w, float *Y,
                                  void *stream) {
  if (!w || !w->packed || !w->scales) return WOQ_EINVAL;
  if (w->bits != 4 && w->bits != 8) return WOQ_EINVAL;
  if (w->block != 32) return WOQ_EINVAL;
  if (w->n <= 0 || w->k <= 0 || w->k % 32 != 0) return WOQ_ESHAPE;
  if (w->n > INT32_MAX || w->k > INT32_MAX / 8) return WOQ_ESHAPE;
  if (!X || !Y) return WOQ_EINVAL;
  if (m < 1 || m > INT32_MAX) return WOQ_EINVAL;
  if ((reinterpret_cast<uintptr_t>(w->packed) & 63) || (reinterpret_cast<uintptr_t>(w->scales) & 63))
    return WOQ_EALIGN;
  if ((reinterpret_cast<uintptr_t>(X) & 15) || (reinterpret_cast<uintptr_t>(Y) & 15)) return WOQ_EALIGN;
  // The bf16 copy of X must fit in the fixed scratch array (K-split partials are used only
  // as far as the rest of it allows).
  if (woq::plan_gemm_tc(m, w->n, w->k, 0, woq::kScratchBytes).xb > woq::kScratchBytes) return WOQ_ESHAPE;
  woq::DevInfo dev;
  int rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  void *scratch = nullptr;
  rc = woq::scratch_address(dev.device, &scratch);
  if (rc != WOQ_OK) return rc;
  const woq::GemmPlan plan = woq::plan_gemm_tc(m, w->n, w->k, dev.sm_count, woq::kScratchBytes);
  return woq::launch_gemm_tc(X, m, *w, Y, scratch, plan, static_cast<cudaStream_t>(stream), dev);
}
