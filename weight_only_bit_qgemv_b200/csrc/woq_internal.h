// Internal interfaces between the C-ABI layer (api.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda.h>
#include <cuda_runtime.h>

#include "woq.h"

namespace woq {

struct DevInfo {
  int device = -1;
  int sm_count = 0;
  int cc_major = 0, cc_minor = 0;
  size_t smem_optin = 0;  // max dynamic shared memory per block (opt-in)
};

// Properties of the current device (cached per device). WOQ_EDEVICE unless it is
// compute capability 10.0; WOQ_ECUDA if the runtime cannot be queried.
int current_device(DevInfo *out);

// Adds n to the process-wide launch counter reported by woq_launch_count().
void count_launches(uint64_t n);

// 2-D tensor map (TMA descriptor) over a row-major [rows, cols] array of `esize`-byte
// elements, box [box_rows, box_cols]; false if the driver refuses it. (qgemm_tc.cu)
bool make_tensor_map_2d(CUtensorMap *m, CUtensorMapDataType type, size_t esize, const void *base,
                        uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
                        CUtensorMapSwizzle swz);

// ---- qgemv.cu ----
// FP32 CUDA-core GEMV/GEMM: y[m, n] = x[m, k] . W_hat^T for any m >= 1. Arguments
// already validated. `pdl` launches with programmatic stream serialization.
int launch_gemv_fp32(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                     const DevInfo &dev, bool pdl);
// qgemv_swiglu: y[m, n/2] = silu(rows 2i) * rows 2i+1 of x . W_hat^T.
int launch_gemv_swiglu(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                       const DevInfo &dev);
// qgemv_residual: y[m, n] = x . W_hat^T + r (r may be y).
int launch_gemv_residual(const float *x, int64_t m, const woq_weight &w, const float *r, float *y,
                         cudaStream_t s, const DevInfo &dev);
// qgemv_argmax: zero the keys in idx, the argmax GEMV, then keys -> (idx, val).
int launch_gemv_argmax(const float *x, int64_t m, const woq_weight &w, int64_t *idx, float *val,
                       cudaStream_t s, const DevInfo &dev);

// Reads (and optionally clears) the GEMV kernels' record of bounded waits that gave up.
int read_gemv_timeout_flag(int clear, unsigned *value);

// ---- qgemv_tc.cu ----
// Small-batch GEMV on tensor cores (2 <= m <= 64, FP32-accurate via a hi/lo bf16 split of x).
// Returns 1 (nothing launched) for shapes it does not take.
int launch_gemv_tc(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                   const DevInfo &dev);
int read_gemv_tc_timeout_flag(int clear, unsigned *value);

// ---- qgemv_i8tc.cu ----
// Small-batch GEMV on the integer tensor cores (1 <= m <= 4; x as three signed digits per
// 32-block, exact int32 block sums). Returns 1 (nothing launched) for shapes it does not take.
int launch_gemv_i8tc(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                     const DevInfo &dev);
int read_i8tc_timeout_flag(int clear, unsigned *value);

// ---- qgemv_chain.cu ----
// A decode step's GEMV items as one persistent launch (arguments already validated).
int launch_gemv_chain(const woq_chain_item *items, int count, int64_t m, unsigned *counters,
                      cudaStream_t s, const DevInfo &dev);
int read_chain_timeout_flag(int clear, unsigned *value);

// ---- qgemm_tc.cu ----
// How the tensor-core path runs a problem: tile width, K-splits and workspace layout
// ([bf16 copy of X][FP32 partials of the splits], each 256-byte aligned).
struct GemmPlan {
  int bn = 128;   // output columns per tile
  int mh = 1;     // 128-row M halves per tile (2: both share each dequantised weight tile)
  int splits = 1;
  bool split = false;  // FP32-accurate form: X and W each as bf16 hi + bf16 lo
  size_t xb = 0, part = 0, total = 0;
};
// Plan for (m, n, k) on a device with sm_count SMs, using at most `budget` workspace bytes
// (the bf16 copy of X itself is always needed).
GemmPlan plan_gemm_tc(int64_t m, int64_t n, int64_t k, int sm_count, size_t budget,
                      bool split = false);
// tcgen05 GEMM with FP32 accumulation in tensor memory: Y = bf16(X) . bf16(W_hat)^T, or in
// the split form Y = (X_hi + X_lo) . (W_hi + W_lo)^T with all four products.
int launch_gemm_tc(const float *X, int64_t m, const woq_weight &w, float *Y, void *workspace,
                   const GemmPlan &plan, cudaStream_t s, const DevInfo &dev);
// Reads (and optionally clears) the device-side record of bounded waits that gave up on
// the current device. Synchronous.
int read_wait_timeout_flag(int clear, unsigned *value);
// Test hook: cycle budget of every bounded wait in the tensor-core kernel and the chained
// GEMV (0 = default); wait_limit_cycles() reads it back.
void set_wait_limit_cycles(long long cycles);
long long wait_limit_cycles();

}  // namespace woq
