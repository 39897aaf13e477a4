// tcgen05 qgemm (prefill): Y[m, n] = bf16(X) . bf16(W_hat)^T with FP32 accumulation in
// tensor memory. "TinyMOSS-Diarize", "How we built it": the prefill GEMM unpacks each
// weight group once into an on-chip tile and reuses it across all activation rows; here
// the tile is dequantised once into shared memory per (N-tile, K-stage) and is read by the
// tensor core for all 128 rows of the M-tile.
//
// Per CTA: one 128 x BN output tile, K in stages of 64.
//   warp 0        producer: bulk tensor copies (TMA) of the bf16 X tile (128B-swizzled) and
//                 of the raw packed weight tile, one mbarrier per stage (byte counted)
//   warp 1        TMEM allocation; one elected thread issues tcgen05.mma (M=128, N=BN,
//                 K=16, bf16 x bf16 -> f32) and commits completions to mbarriers
//   warps 2..9    dequantisers: raw codes + binary16 scales -> bf16(scale * code) written in
//                 the 128B-swizzled K-major layout the MMA descriptor names; afterwards the
//                 same warps drain the accumulator (tcgen05.ld) and store FP32 Y
// Every mbarrier wait is bounded; a wait that gives up records the event in a device flag,
// makes the CTA's other roles stop, drains the copies and MMAs already issued, frees TMEM
// and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstring>
#include <mutex>

#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_wait_timeout_flag = 0;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;           // bf16 elements per stage = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kWinStages = 32;   // K-stages whose scales each dequantiser holds in shared memory
constexpr int kTmaScaleCols = 128;  // scale tile copied whole by TMA when K/32 <= this
constexpr int kDequantWarps = 8;
constexpr int kThreads = 64 + kDequantWarps * 32;  // 320
constexpr long long kDrainLimit = 1LL << 31;       // cycles (~1 s) for draining on abort
constexpr long long kDefaultWaitLimit = 1LL << 32;  // cycles (~2 s) for ordinary waits

long long g_wait_limit_cycles = 0;  // test hook: > 0 wait limit, < 0 inject a stuck wait

template <int BITS, int BN>
struct Cfg {
  static constexpr int kABytes = BM * BK * 2;               // 16 KB
  static constexpr int kBBytes = BN * BK * 2;               // 16/32 KB
  static constexpr int kRawRow = BK * BITS / 8;             // 32 or 64 bytes
  static constexpr int kRawBytes = BN * kRawRow;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kStages * kABytes;
  static constexpr int kOffRaw = kOffB + kStages * kBBytes;
  static constexpr int kOffScale = kOffRaw + kStages * kRawBytes;
  // either per-thread slots (kWinStages per job) or the whole [BN, K/32] tile (K <= 4096)
  static constexpr int kScaleBytes = (kWinStages * (BN * 2) * 2 > BN * kTmaScaleCols * 2)
                                         ? kWinStages * (BN * 2) * 2
                                         : BN * kTmaScaleCols * 2;
  static constexpr int kOffBar = (kOffScale + kScaleBytes + 15) & ~15;
  static constexpr int kSmem = kOffBar + 256 + 1024;        // barriers + alignment slack
  static constexpr uint32_t kTmemCols = BN;                 // power of two >= 32
  // Instruction descriptor: D f32, A/B bf16, both K-major, N = BN, M = 128.
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     (static_cast<uint32_t>(BN >> 3) << 17) |
                                     (static_cast<uint32_t>(BM >> 4) << 24);
};

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) |
         (1ull << 46) | (2ull << 61);
}

struct Shared {
  uint64_t wfull[kStages];  // raw weight tile landed (TMA bytes)
  uint64_t afull[kStages];  // bf16 X tile landed (TMA bytes)
  uint64_t bfull[kStages];  // bf16 weight tile written by the dequantisers
  uint64_t empty[kStages];  // MMAs reading the stage completed
  uint64_t acc_full;        // all MMAs of the tile completed
  uint64_t sfull;           // scale tile landed (TMA bytes)
  uint64_t never;           // nothing arrives here: target of the injected stuck wait
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void record_timeout(volatile int *abort) {
  *abort = 1;
  atomicOr(&g_wait_timeout_flag, 1u);
}

// One 32-bit word of int4 codes -> 8 bf16 values s*q (exact in f32, rounded once to bf16),
// packed as 4 bf16x2 words in element order.
__device__ __forceinline__ uint4 dequant_int4_word(uint32_t w, const float (&sj)[4]) {
  const uint32_t hi = w >> 16;
  float2 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t mask = 0xFu << (4 * j);
    const uint32_t magic = 0x4B000000u | (0x8u << (4 * j));
    const float bias = 8388608.0f + 8.0f * static_cast<float>(1u << (4 * j));
    const float lo_f = __uint_as_float((w & mask) ^ magic);
    const float hi_f = __uint_as_float((hi & mask) ^ magic);
    v[j] = __fadd2_rn(make_float2(lo_f, hi_f), make_float2(-bias, -bias));  // q * 2^(4j)
    v[j] = __fmul2_rn(v[j], make_float2(sj[j], sj[j]));                        // s * q
  }
  // v[j] = (e_j, e_{4+j})
  uint4 out;
  __nv_bfloat162 t;
  t = __floats2bfloat162_rn(v[0].x, v[1].x); out.x = *reinterpret_cast<uint32_t *>(&t);
  t = __floats2bfloat162_rn(v[2].x, v[3].x); out.y = *reinterpret_cast<uint32_t *>(&t);
  t = __floats2bfloat162_rn(v[0].y, v[1].y); out.z = *reinterpret_cast<uint32_t *>(&t);
  t = __floats2bfloat162_rn(v[2].y, v[3].y); out.w = *reinterpret_cast<uint32_t *>(&t);
  return out;
}

// Two 32-bit words of int8 codes (8 elements) -> 8 bf16 values s*q.
__device__ __forceinline__ uint4 dequant_int8_words(uint32_t w0, uint32_t w1, float s) {
  const float bias = 8388608.0f + 128.0f;
  const uint32_t u0 = w0 ^ 0x80808080u, u1 = w1 ^ 0x80808080u;
  float2 p[4];
  p[0] = make_float2(__uint_as_float(__byte_perm(u0, 0x4B000000u, 0x7540)),
                     __uint_as_float(__byte_perm(u0, 0x4B000000u, 0x7541)));
  p[1] = make_float2(__uint_as_float(__byte_perm(u0, 0x4B000000u, 0x7542)),
                     __uint_as_float(__byte_perm(u0, 0x4B000000u, 0x7543)));
  p[2] = make_float2(__uint_as_float(__byte_perm(u1, 0x4B000000u, 0x7540)),
                     __uint_as_float(__byte_perm(u1, 0x4B000000u, 0x7541)));
  p[3] = make_float2(__uint_as_float(__byte_perm(u1, 0x4B000000u, 0x7542)),
                     __uint_as_float(__byte_perm(u1, 0x4B000000u, 0x7543)));
  uint4 out;
  uint32_t *o = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 v = __fadd2_rn(p[i], make_float2(-bias, -bias));
    v = __fmul2_rn(v, make_float2(s, s));
    __nv_bfloat162 t = __floats2bfloat162_rn(v.x, v.y);
    o[i] = *reinterpret_cast<uint32_t *>(&t);
  }
  return out;
}

template <int BITS, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    qgemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_s, const uint16_t *__restrict__ scales,
                    float *__restrict__ Y, int M, int N, int K, int scales_tma,
                    long long wait_limit, long long stuck_wait) {
  using C = Cfg<BITS, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + C::kOffBar);
  uint16_t *ssc = reinterpret_cast<uint16_t *>(smem + C::kOffScale);  // per-thread scale slots
  volatile int *abort = &sh.abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * BM;
  const int num_k = (K + BK - 1) / BK;
  const int pro = num_k < kStages ? num_k : kStages;  // stages issued before the PDL wait

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&sh.wfull[s], 1);
      ptx::mbar_init(&sh.afull[s], 1);
      ptx::mbar_init(&sh.bfull[s], kDequantWarps);  // one elected arrival per warp
      ptx::mbar_init(&sh.empty[s], 1);
    }
    ptx::mbar_init(&sh.acc_full, 1);
    ptx::mbar_init(&sh.sfull, 1);
    ptx::mbar_init(&sh.never, 1);
    sh.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_x);
    ptx::prefetch_tmap(&tm_w);
    if (scales_tma) ptx::prefetch_tmap(&tm_s);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh.tmem_base, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // Only X (produced by the conversion kernel) and Y depend on preceding kernels; the
  // weight copies, the scale window and the first dequantisations run before the wait.
  int issued_w = 0, issued_a = 0;  // producer: stages whose copies were issued
  bool mma_issued = false;

  if (warp == 0) {
    if (lane == 0) {
      if (scales_tma) {
        ptx::mbar_arrive_expect_tx(&sh.sfull, static_cast<uint32_t>(BN * (K >> 5) * 2));
        ptx::tma_load_2d(ssc, &tm_s, &sh.sfull, 0, n0);
      }
      for (int ks = 0; ks < pro; ++ks) {
        ptx::mbar_arrive_expect_tx(&sh.wfull[ks], C::kRawBytes);
        ptx::tma_load_2d(smem + C::kOffRaw + ks * C::kRawBytes, &tm_w, &sh.wfull[ks],
                         ks * C::kRawRow, n0);
      }
      issued_w = pro;
      ptx::pdl_wait();
      for (int ks = 0; ks < pro; ++ks) {
        ptx::mbar_arrive_expect_tx(&sh.afull[ks], C::kABytes);
        ptx::tma_load_2d(smem + C::kOffA + ks * C::kABytes, &tm_x, &sh.afull[ks], ks * BK, m0);
      }
      issued_a = pro;
      for (int ks = pro; ks < num_k; ++ks) {
        const int s = ks % kStages;
        const uint32_t ph = (ks / kStages) & 1;
        if (!ptx::mbar_wait_bounded(&sh.empty[s], ph ^ 1, wait_limit, abort)) {
          record_timeout(abort);
          break;
        }
        ptx::mbar_arrive_expect_tx(&sh.wfull[s], C::kRawBytes);
        ptx::tma_load_2d(smem + C::kOffRaw + s * C::kRawBytes, &tm_w, &sh.wfull[s],
                         ks * C::kRawRow, n0);
        issued_w = ks + 1;
        ptx::mbar_arrive_expect_tx(&sh.afull[s], C::kABytes);
        ptx::tma_load_2d(smem + C::kOffA + s * C::kABytes, &tm_x, &sh.afull[s], ks * BK, m0);
        issued_a = ks + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      // Test hook: a wait on a barrier nothing arrives on, which must run out.
      if (stuck_wait > 0 && !ptx::mbar_wait_bounded(&sh.never, 0, stuck_wait, abort)) {
        record_timeout(abort);
        ok = false;
      }
      for (int ks = 0; ks < num_k && ok; ++ks) {
        const int s = ks % kStages;
        const uint32_t ph = (ks / kStages) & 1;
        ok = ptx::mbar_wait_bounded(&sh.afull[s], ph, wait_limit, abort) &&
             ptx::mbar_wait_bounded(&sh.bfull[s], ph, wait_limit, abort);
        if (!ok) {
          record_timeout(abort);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t a0 = ptx::smem_u32(smem + C::kOffA + s * C::kABytes);
        const uint32_t b0 = ptx::smem_u32(smem + C::kOffB + s * C::kBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          ptx::tc_mma_f16(tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), C::kIdesc,
                          (ks | kk) != 0 ? 1u : 0u);
        }
        mma_issued = true;
        ptx::tc_commit(&sh.empty[s]);
      }
      ptx::tc_commit(&sh.acc_full);  // also covers a partial tile after an abort
    }
  } else {
    // ---- dequantisers ----
    const int t = threadIdx.x - 64;  // 0 .. 255
    const int spr = K >> 5;
    constexpr int kJobs = BN * 2 / (kDequantWarps * 32);  // (row, half) jobs per thread
    int wst0 = -kWinStages;                                // first stage of the loaded window
    bool ok = true;
    // Wait outcomes are made warp-uniform: the loop below contains warp-collective steps.
    if (scales_tma &&
        !__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.sfull, 0, wait_limit, abort))) {
      record_timeout(abort);
      ok = false;
    }
    for (int ks = 0; ks < num_k && ok; ++ks) {
      const int s = ks % kStages;
      const uint32_t ph = (ks / kStages) & 1;
      if (!scales_tma && ks >= wst0 + kWinStages) {
        // This thread's own scales for the next kWinStages stages, into its private slots
        // of shared memory (only it reads them, so no barrier is involved). Rows past N and
        // blocks past K/32 read as zero.
        wst0 = ks;
#pragma unroll 4
        for (int j = 0; j < kWinStages; ++j) {
#pragma unroll
          for (int jj = 0; jj < kJobs; ++jj) {
            const int job = t + jj * kDequantWarps * 32;
            const int gr = n0 + job % BN, kb = 2 * (ks + j) + job / BN;
            ssc[(j * kJobs + jj) * (kDequantWarps * 32) + t] =
                (gr < N && kb < spr) ? __ldg(scales + static_cast<size_t>(gr) * spr + kb) : 0;
          }
        }
      }
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.wfull[s], ph, wait_limit, abort))) {
        record_timeout(abort);
        ok = false;
        break;
      }
      const uint8_t *raw = smem + C::kOffRaw + s * C::kRawBytes;
      uint8_t *btile = smem + C::kOffB + s * C::kBBytes;
#pragma unroll
      for (int j = 0; j < kJobs; ++j) {
        const int job = t + j * kDequantWarps * 32;
        const int row = job % BN, h = job / BN;  // h: which 32-element half of the stage
        const float s0 = __half2float(__ushort_as_half(
            scales_tma ? ssc[row * spr + 2 * ks + h]
                       : ssc[((ks - wst0) * kJobs + j) * (kDequantWarps * 32) + t]));
        uint8_t *brow = btile + row * 128;
        const int sw = row & 7;
        if constexpr (BITS == 4) {
          const uint4 wq = *reinterpret_cast<const uint4 *>(raw + row * C::kRawRow + h * 16);
          const float sj[4] = {s0, s0 * 0.0625f, s0 * 0.00390625f, s0 * 0.000244140625f};
          const uint32_t ws[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int chunk = h * 4 + i;  // 16-byte chunk = 8 bf16 = 8 elements
            *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) = dequant_int4_word(ws[i], sj);
          }
        } else {
          const uint4 wa = *reinterpret_cast<const uint4 *>(raw + row * C::kRawRow + h * 32);
          const uint4 wb = *reinterpret_cast<const uint4 *>(raw + row * C::kRawRow + h * 32 + 16);
          const uint32_t ws[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int chunk = h * 4 + i;
            *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) =
                dequant_int8_words(ws[2 * i], ws[2 * i + 1], s0);
          }
        }
      }
      // Each lane makes its tile writes visible to the async proxy (the tensor core), the
      // warp converges, and one lane arrives for the warp.
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.bfull[s]);
    }

    // ---- epilogue: TMEM -> registers -> Y ----
    // Y may be read by a preceding kernel: write it only after that grid completed.
    ptx::pdl_wait();
    // tcgen05.ld is warp-collective, so the whole warp decides together.
    const bool mine = ok && ptx::mbar_wait_bounded(&sh.acc_full, 0, wait_limit, abort) && !*abort;
    const bool go = __all_sync(0xffffffffu, mine);
    if (go) {
      ptx::tc_fence_after();
      const int q = warp & 3;                        // TMEM lanes 32q .. 32q+31
      const int half = (warp - 2) >> 2;              // which half of the columns
      const int row = m0 + q * 32 + lane;
      const bool vec = (N & 3) == 0;
      for (int c0 = half * (BN / 2); c0 < (half + 1) * (BN / 2); c0 += 16) {
        uint32_t r[16];
        ptx::tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(q * 32) << 16) + c0, r);
        ptx::tmem_ld_wait();
        if (row < M) {
          float *yr = Y + static_cast<size_t>(row) * N + n0 + c0;
          if (vec && n0 + c0 + 16 <= N) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              reinterpret_cast<float4 *>(yr)[v] =
                  make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                              __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
          } else {
#pragma unroll
            for (int v = 0; v < 16; ++v)
              if (n0 + c0 + v < N) yr[v] = __uint_as_float(r[v]);
          }
        }
      }
    } else if (ok && !mine) {
      record_timeout(abort);
    }
  }

  ptx::pdl_launch_dependents();

  // ---- teardown: drain what this CTA issued, then free TMEM ----
  if (warp == 0 && lane == 0 && *abort) {
    // Only the last issue to each stage can still be in flight.
    int no_abort = 0;
    for (int ks = issued_w - 1; ks >= 0 && ks >= issued_w - kStages; --ks)
      ptx::mbar_wait_bounded(&sh.wfull[ks % kStages], (ks / kStages) & 1, kDrainLimit, &no_abort);
    for (int ks = issued_a - 1; ks >= 0 && ks >= issued_a - kStages; --ks)
      ptx::mbar_wait_bounded(&sh.afull[ks % kStages], (ks / kStages) & 1, kDrainLimit, &no_abort);
    if (scales_tma) ptx::mbar_wait_bounded(&sh.sfull, 0, kDrainLimit, &no_abort);
  }
  if (warp == 1 && lane == 0 && *abort && mma_issued) {
    // acc_full was committed after the last MMA this thread issued.
    int no_abort = 0;
    ptx::mbar_wait_bounded(&sh.acc_full, 0, kDrainLimit, &no_abort);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// X fp32 [m, k] -> bf16 [m, k], round to nearest even; 8 elements per thread.
__global__ void __launch_bounds__(256) x_to_bf16_kernel(const float4 *__restrict__ x,
                                                        uint4 *__restrict__ xb, size_t n8) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const float4 a = x[2 * i], b = x[2 * i + 1];
    uint4 o;
    __nv_bfloat162 t;
    t = __floats2bfloat162_rn(a.x, a.y); o.x = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2bfloat162_rn(a.z, a.w); o.y = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2bfloat162_rn(b.x, b.y); o.z = *reinterpret_cast<uint32_t *>(&t);
    t = __floats2bfloat162_rn(b.z, b.w); o.w = *reinterpret_cast<uint32_t *>(&t);
    xb[i] = o;
  }
}

// ---- host side -------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] array.
bool make_map(CUtensorMap *m, CUtensorMapDataType type, size_t esize, const void *base,
              uint64_t cols, uint64_t rows, uint32_t box_cols, uint32_t box_rows,
              CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * esize};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, type, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BITS, int BN>
int launch_tc(const float *X, int64_t m, const woq_weight &w, float *Y, void *workspace,
              cudaStream_t s, const DevInfo &dev) {
  using C = Cfg<BITS, BN>;
  (void)dev;
  auto kern = qgemm_tc_kernel<BITS, BN>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (attr_err != cudaSuccess) return WOQ_ECUDA;

  CUtensorMap tm_x, tm_w, tm_s;
  const int64_t spr = w.k / 32;
  // The whole scale tile [BN, K/32] comes by TMA when its rows are 16-byte multiples and
  // it fits the shared-memory slot; otherwise each dequantiser loads its own scales.
  const int scales_tma = (spr % 8 == 0 && spr <= kTmaScaleCols) ? 1 : 0;
  if (scales_tma) {
    if (!make_map(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w.scales, spr, w.n,
                  static_cast<uint32_t>(spr), BN, CU_TENSOR_MAP_SWIZZLE_NONE))
      return WOQ_ECUDA;
  } else {
    std::memset(&tm_s, 0, sizeof(tm_s));
  }
  if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, workspace, w.k, m, BK, BM,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return WOQ_ECUDA;
  if (!make_map(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, w.k * BITS / 8, w.n,
                C::kRawRow, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WOQ_ECUDA;

  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;

  // 1) X -> bf16 into the workspace.
  const size_t n8 = static_cast<size_t>(m) * w.k / 8;
  {
    cudaLaunchConfig_t cfg = {};
    size_t blocks = (n8 + 255) / 256;
    if (blocks > static_cast<size_t>(dev.sm_count) * 8) blocks = static_cast<size_t>(dev.sm_count) * 8;
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, x_to_bf16_kernel, reinterpret_cast<const float4 *>(X),
                           reinterpret_cast<uint4 *>(workspace), n8) != cudaSuccess)
      return WOQ_ECUDA;
    count_launches(1);
  }
  // 2) the GEMM.
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((w.n + BN - 1) / BN),
                       static_cast<unsigned>((m + BM - 1) / BM), 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const long long lim = g_wait_limit_cycles > 0 ? g_wait_limit_cycles : kDefaultWaitLimit;
    const long long stuck = g_wait_limit_cycles < 0 ? -g_wait_limit_cycles : 0;
    if (cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w, tm_s, w.scales, Y, static_cast<int>(m),
                           static_cast<int>(w.n), static_cast<int>(w.k), scales_tma, lim,
                           stuck) != cudaSuccess)
      return WOQ_ECUDA;
    count_launches(1);
  }
  return WOQ_OK;
}

}  // namespace

size_t gemm_tc_workspace_bytes(int64_t m, int64_t k) {
  const size_t b = static_cast<size_t>(m) * static_cast<size_t>(k) * 2;
  return (b + 255) & ~static_cast<size_t>(255);
}

int launch_gemm_tc(const float *X, int64_t m, const woq_weight &w, float *Y, void *workspace,
                   cudaStream_t s, const DevInfo &dev) {
  return w.bits == 4 ? launch_tc<4, 128>(X, m, w, Y, workspace, s, dev)
                     : launch_tc<8, 128>(X, m, w, Y, workspace, s, dev);
}

int read_wait_timeout_flag(int clear, unsigned *value) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_wait_timeout_flag, sizeof(v)) != cudaSuccess) return WOQ_ECUDA;
  if (clear && v) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_wait_timeout_flag, &z, sizeof(z)) != cudaSuccess) return WOQ_ECUDA;
  }
  *value = v;
  return WOQ_OK;
}

void set_wait_limit_cycles(long long cycles) { g_wait_limit_cycles = cycles; }

}  // namespace woq
