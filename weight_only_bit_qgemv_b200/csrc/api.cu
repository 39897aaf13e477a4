// C-ABI entry points of libwoq (declared in include/woq.h): argument checks, the device
// check and dispatch to the kernel launchers. Nothing here allocates device memory or
// synchronises a stream (woq_device_status excepted, which exists to synchronise).
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "woq.h"
#include "woq_internal.h"

namespace woq {
namespace {

std::atomic<uint64_t> g_launches{0};

constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];
int g_dev_rc[kMaxDevices];

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_weight(const woq_weight *w) {
  if (!w || !w->packed || !w->scales) return WOQ_EINVAL;
  if (w->bits != 4 && w->bits != 5 && w->bits != 8) return WOQ_EINVAL;
  if (w->block != 32) return WOQ_EINVAL;
  if (w->n <= 0 || w->k <= 0 || w->k % 32 != 0) return WOQ_ESHAPE;
  if (w->bits == 5 && w->k % 128 != 0) return WOQ_ESHAPE;  // int5 rows on 16-byte boundaries
  if (w->n > INT32_MAX || w->k > INT32_MAX / 8) return WOQ_ESHAPE;
  if (!aligned(w->packed, 64) || !aligned(w->scales, 64)) return WOQ_EALIGN;
  return WOQ_OK;
}

}  // namespace

void count_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int current_device(DevInfo *out) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return WOQ_ECUDA;
  if (d < 0 || d >= kMaxDevices) return WOQ_EDEVICE;
  std::call_once(g_dev_once[d], [d] {
    DevInfo info;
    info.device = d;
    int v = 0;
    int rc = WOQ_OK;
    if (cudaDeviceGetAttribute(&info.cc_major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.cc_minor, cudaDevAttrComputeCapabilityMinor, d) != cudaSuccess ||
        cudaDeviceGetAttribute(&info.sm_count, cudaDevAttrMultiProcessorCount, d) != cudaSuccess ||
        cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, d) != cudaSuccess) {
      rc = WOQ_ECUDA;
    } else {
      info.smem_optin = static_cast<size_t>(v);
      if (info.cc_major != 10 || info.cc_minor != 0) rc = WOQ_EDEVICE;
    }
    g_dev[d] = info;
    g_dev_rc[d] = rc;
  });
  *out = g_dev[d];
  return g_dev_rc[d];
}

}  // namespace woq

using woq::DevInfo;

extern "C" {

// qgemv's automatic choice, measured on B200 (graphs of calls over L2-cold copies). Matrices
// wide enough that 128-row tiles cover every SM (the lm_head): the CUDA-core kernel for
// m <= 2; for 3 <= m <= 4 the integer tensor cores (int8: 63.5 / 71.0 us against 77.1 on the
// CUDA cores) or the small-batch mma.sync form (int4: 60.8 us against 94.9); the mma.sync form
// up to m = 32 (int8 80-115 us, int4 61-109 us, where the tcgen05 split GEMM takes 146-164);
// the split GEMM from m = 33 (at m = 47: 173 us against 272). Narrower matrices (the decoder's
// projections): the CUDA-core kernel below m = 16, the split GEMM from there (m = 16: qkv 10.1
// us against 11.8, down 11.2 against 12.05). int5 always takes the CUDA-core kernel.
constexpr int64_t kTcMinMWide = 3;
constexpr int64_t kI8TcMaxMWide = 4;
constexpr int64_t kGemmMinM = 16;
constexpr int64_t kGemmMinMWide = 33;

int qgemv_path(const float *x, int64_t m, const woq_weight *w, float *y, int32_t path,
               void *stream) {
  int rc = woq::check_weight(w);
  if (rc != WOQ_OK) return rc;
  if (!x || !y) return WOQ_EINVAL;
  if (m < 1 || m > 64) return WOQ_EINVAL;
  if (path != WOQ_GEMV_AUTO && path != WOQ_GEMV_CUDA_CORE && path != WOQ_GEMV_SPLIT_TC &&
      path != WOQ_GEMV_SPLIT_GEMM && path != WOQ_GEMV_INT8_TC)
    return WOQ_EINVAL;
  if (w->k > 32768) return WOQ_ESHAPE;
  if (!woq::aligned(x, 16) || !woq::aligned(y, 16)) return WOQ_EALIGN;
  DevInfo dev;
  rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (w->bits == 5) {  // int5: the CUDA-core kernel only
    if (path != WOQ_GEMV_AUTO && path != WOQ_GEMV_CUDA_CORE) return WOQ_EINVAL;
    return woq::launch_gemv_fp32(x, m, *w, y, s, dev, true);
  }
  if (path == WOQ_GEMV_INT8_TC) {
    rc = woq::launch_gemv_i8tc(x, m, *w, y, s, dev);
    return rc == 1 ? WOQ_ESHAPE : rc;
  }
  const bool wide = (w->n + 127) / 128 >= dev.sm_count;
  if (path == WOQ_GEMV_SPLIT_GEMM ||
      (path == WOQ_GEMV_AUTO && m >= (wide ? kGemmMinMWide : kGemmMinM))) {
    const woq::GemmPlan plan = woq::plan_gemm_tc(m, w->n, w->k, dev.sm_count, SIZE_MAX, true);
    return woq::launch_gemm_tc(x, m, *w, y, nullptr, plan, s, dev);
  }
  if (path == WOQ_GEMV_AUTO && wide && w->bits == 8 && m >= kTcMinMWide && m <= kI8TcMaxMWide) {
    rc = woq::launch_gemv_i8tc(x, m, *w, y, s, dev);
    if (rc != 1) return rc;  // shapes it does not take go on below
  }
  const bool tc = path == WOQ_GEMV_SPLIT_TC || (path == WOQ_GEMV_AUTO && m >= kTcMinMWide && wide);
  if (tc) {
    rc = woq::launch_gemv_tc(x, m, *w, y, s, dev);
    if (rc != 1) return rc;
    if (path == WOQ_GEMV_SPLIT_TC) return WOQ_ESHAPE;  // shape outside the kernel's limits
  }
  return woq::launch_gemv_fp32(x, m, *w, y, s, dev, true);
}

int qgemv(const float *x, int64_t m, const woq_weight *w, float *y, void *stream) {
  return qgemv_path(x, m, w, y, WOQ_GEMV_AUTO, stream);
}

int qgemv_swiglu(const float *x, int64_t m, const woq_weight *w, float *y, void *stream) {
  int rc = woq::check_weight(w);
  if (rc != WOQ_OK) return rc;
  if (!x || !y) return WOQ_EINVAL;
  if (m < 1 || m > 64) return WOQ_EINVAL;
  if (w->n % 2 != 0 || w->k > 8192) return WOQ_ESHAPE;
  if (!woq::aligned(x, 16) || !woq::aligned(y, 4)) return WOQ_EALIGN;
  DevInfo dev;
  rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  return woq::launch_gemv_swiglu(x, m, *w, y, static_cast<cudaStream_t>(stream), dev);
}

int qgemv_residual(const float *x, int64_t m, const woq_weight *w, const float *r, float *y,
                   void *stream) {
  int rc = woq::check_weight(w);
  if (rc != WOQ_OK) return rc;
  if (!x || !r || !y) return WOQ_EINVAL;
  if (m < 1 || m > 64) return WOQ_EINVAL;
  if (w->k > 8192) return WOQ_ESHAPE;
  // r may be y itself; any other overlap of the two [m, n] arrays is refused
  const uintptr_t rb = reinterpret_cast<uintptr_t>(r), yb = reinterpret_cast<uintptr_t>(y);
  const uintptr_t bytes = static_cast<uintptr_t>(m) * static_cast<uintptr_t>(w->n) * sizeof(float);
  if (rb != yb && rb < yb + bytes && yb < rb + bytes) return WOQ_EINVAL;
  if (!woq::aligned(x, 16) || !woq::aligned(r, 4) || !woq::aligned(y, 4)) return WOQ_EALIGN;
  DevInfo dev;
  rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  return woq::launch_gemv_residual(x, m, *w, r, y, static_cast<cudaStream_t>(stream), dev);
}

int qgemv_argmax(const float *x, int64_t m, const woq_weight *w, int64_t *idx, float *val,
                 void *stream) {
  int rc = woq::check_weight(w);
  if (rc != WOQ_OK) return rc;
  if (!x || !idx || !val) return WOQ_EINVAL;
  if (m < 1 || m > 8) return WOQ_EINVAL;
  if (w->k > 8192 || w->n >= (int64_t(1) << 31)) return WOQ_ESHAPE;
  if (!woq::aligned(x, 16) || !woq::aligned(idx, 8) || !woq::aligned(val, 4)) return WOQ_EALIGN;
  DevInfo dev;
  rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  return woq::launch_gemv_argmax(x, m, *w, idx, val, static_cast<cudaStream_t>(stream), dev);
}

size_t qgemv_chain_workspace_bytes(void) { return 256; }

int qgemv_chain(const woq_chain_item *items, int32_t count, int64_t m, void *workspace,
                size_t workspace_bytes, void *stream) {
  if (!items || count < 1 || count > WOQ_CHAIN_MAX_ITEMS) return WOQ_EINVAL;
  if (m < 1 || m > 8) return WOQ_EINVAL;
  if (!workspace || workspace_bytes < qgemv_chain_workspace_bytes()) return WOQ_EWORKSPACE;
  if (!woq::aligned(workspace, 256)) return WOQ_EALIGN;
  auto overlap = [](const void *a, size_t na, const void *b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
  };
  for (int32_t i = 0; i < count; ++i) {
    const woq_chain_item &it = items[i];
    int rc = woq::check_weight(it.w);
    if (rc != WOQ_OK) return rc;
    if (!it.x || !it.y) return WOQ_EINVAL;
    if (it.epilogue != WOQ_EPI_NONE && it.epilogue != WOQ_EPI_SWIGLU && it.epilogue != WOQ_EPI_RESIDUAL)
      return WOQ_EINVAL;
    if (it.w->k % 256 != 0 || it.w->k > 8192) return WOQ_ESHAPE;
    if (it.epilogue == WOQ_EPI_SWIGLU && it.w->n % 2 != 0) return WOQ_ESHAPE;
    if (!woq::aligned(it.x, 16) || !woq::aligned(it.y, 16)) return WOQ_EALIGN;
    const size_t xb = static_cast<size_t>(m) * it.w->k * 4;
    const size_t yb = static_cast<size_t>(m) * (it.epilogue == WOQ_EPI_SWIGLU ? it.w->n / 2 : it.w->n) * 4;
    if (overlap(it.x, xb, it.y, yb)) return WOQ_EINVAL;
    if (it.epilogue == WOQ_EPI_RESIDUAL) {
      if (!it.r) return WOQ_EINVAL;
      if (!woq::aligned(it.r, 16)) return WOQ_EALIGN;
      if (it.r != it.y && overlap(it.r, yb, it.y, yb)) return WOQ_EINVAL;
    }
  }
  DevInfo dev;
  int rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  return woq::launch_gemv_chain(items, count, m, static_cast<unsigned *>(workspace),
                                static_cast<cudaStream_t>(stream), dev);
}

// SM count the tensor-core plan is made for: the current device's, or 0 (no K-splits) when
// no device can be queried, so that sizing never fails.
static int plan_sm_count() {
  DevInfo dev;
  return woq::current_device(&dev) == WOQ_OK ? dev.sm_count : 0;
}

// qgemm's automatic choice: the bf16 tensor-core GEMM for prefill-sized m, the FP32-accurate
// split tensor-core GEMM for batched decode from kSplitMinM rows on (measured on B200 over
// the decoder projections and the lm_head: faster than the CUDA-core kernel from there on),
// and the CUDA-core kernel below that.
constexpr int64_t kSplitMinM = 16;

static int resolve_path(int32_t path, int64_t m, int32_t bits) {
  if (path == WOQ_PATH_AUTO) {
    if (bits == 5) return WOQ_PATH_FP32;  // int5: the CUDA-core kernel only
    return m >= 128 ? WOQ_PATH_BF16_TC : m >= kSplitMinM ? WOQ_PATH_SPLIT_TC : WOQ_PATH_FP32;
  }
  return path;
}

static bool known_path(int32_t path) {
  return path == WOQ_PATH_AUTO || path == WOQ_PATH_FP32 || path == WOQ_PATH_BF16_TC ||
         path == WOQ_PATH_SPLIT_TC;
}

size_t qgemm_workspace_bytes(int64_t m, const woq_weight *w, int32_t path) {
  if (woq::check_weight(w) != WOQ_OK || m < 1) return 0;
  if (!known_path(path)) return 0;
  const int p = resolve_path(path, m, w->bits);
  if (p == WOQ_PATH_FP32 || w->bits == 5) return 0;
  return woq::plan_gemm_tc(m, w->n, w->k, plan_sm_count(), SIZE_MAX, p == WOQ_PATH_SPLIT_TC).total;
}

int qgemm(const float *X, int64_t m, const woq_weight *w, float *Y, int32_t path,
          void *workspace, size_t workspace_bytes, void *stream) {
  int rc = woq::check_weight(w);
  if (rc != WOQ_OK) return rc;
  if (!X || !Y) return WOQ_EINVAL;
  if (m < 1 || m > INT32_MAX) return WOQ_EINVAL;
  if (!known_path(path)) return WOQ_EINVAL;
  if (!woq::aligned(X, 16) || !woq::aligned(Y, 16)) return WOQ_EALIGN;
  const int p = resolve_path(path, m, w->bits);
  if (w->bits == 5 && p != WOQ_PATH_FP32) return WOQ_EINVAL;  // no tensor-core int5 form
  if (p == WOQ_PATH_FP32 && w->k > 32768) return WOQ_ESHAPE;
  woq::GemmPlan plan;
  if (p != WOQ_PATH_FP32) {
    plan = woq::plan_gemm_tc(m, w->n, w->k, plan_sm_count(), SIZE_MAX, p == WOQ_PATH_SPLIT_TC);
    if (plan.total > 0) {
      if (!workspace || workspace_bytes < plan.total) return WOQ_EWORKSPACE;
      if (!woq::aligned(workspace, 256)) return WOQ_EALIGN;
    }
  }
  DevInfo dev;
  rc = woq::current_device(&dev);
  if (rc != WOQ_OK) return rc;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (p == WOQ_PATH_FP32) return woq::launch_gemv_fp32(X, m, *w, Y, s, dev, true);
  return woq::launch_gemm_tc(X, m, *w, Y, workspace, plan, s, dev);
}

int woq_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return WOQ_ECUDA;
  unsigned v = 0, g = 0, t = 0, i = 0, c = 0;
  int rc = woq::read_wait_timeout_flag(clear, &v);
  if (rc != WOQ_OK) return rc;
  rc = woq::read_gemv_timeout_flag(clear, &g);
  if (rc != WOQ_OK) return rc;
  rc = woq::read_gemv_tc_timeout_flag(clear, &t);
  if (rc != WOQ_OK) return rc;
  rc = woq::read_i8tc_timeout_flag(clear, &i);
  if (rc != WOQ_OK) return rc;
  rc = woq::read_chain_timeout_flag(clear, &c);
  if (rc != WOQ_OK) return rc;
  return (v || g || t || i || c) ? WOQ_ETIMEOUT : WOQ_OK;
}

void woq_debug_set_wait_limit(long long cycles) { woq::set_wait_limit_cycles(cycles); }

const char *woq_status_str(int status) {
  switch (status) {
    case WOQ_OK: return "ok";
    case WOQ_EINVAL: return "invalid argument";
    case WOQ_ESHAPE: return "unsupported shape";
    case WOQ_EALIGN: return "misaligned pointer";
    case WOQ_ERANGE: return "value out of range (non-finite weight or binary16 scale overflow)";
    case WOQ_EDEVICE: return "device is not compute capability 10.0 (B200)";
    case WOQ_ECUDA: return "CUDA runtime error";
    case WOQ_ETIMEOUT: return "a bounded device-side wait gave up";
    case WOQ_EWORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
  }
}

uint64_t woq_launch_count(void) { return woq::g_launches.load(std::memory_order_relaxed); }

int woq_abi_version(void) { return 1; }

}  // extern "C"
