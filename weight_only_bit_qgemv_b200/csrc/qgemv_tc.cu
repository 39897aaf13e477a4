// Small-batch qgemv on tensor cores (decode with 2 <= m <= 64), FP32-accurate.
//
// y[m, n] = x[m, k] . W_hat^T with the same exact-block arithmetic as the CUDA-core GEMV,
// moved onto mma.sync (m16n8k16, bf16 inputs, f32 accumulate):
//   * the codes q are exact in bf16, so A = the codes of 16 weight rows;
//   * x is split into two bf16 terms, x = x_hi + x_lo (about 16 significant bits), so the
//     products keep FP32-level accuracy; B = x_hi or x_lo of 8 activation rows;
//   * each 32-code block is reduced by four MMAs (two K=16 steps, hi and lo) into a zeroed
//     block accumulator, which is then scaled by the block's binary16 scale and added to
//     the FP32 output accumulator ("TinyMOSS-Diarize", "How we built it": weight-only,
//     FP32 activations, dequantisation fused into the multiply).
// Within each 8-code group the K order is permuted (0,4,1,5 | 2,6,3,7) on both operands;
// a permutation applied to both sides of a dot product leaves it unchanged, and it lets one
// LOP3 turn two 4-bit codes into a bf16 pair.
//
// Per CTA: one producer warp streams 128-row x 128-byte code tiles (TMA, 128B-swizzled) into
// a ring and each row tile's [128, K/32] scale tile into a double buffer; eight compute
// warps own 16 rows each. For every K-chunk the compute warps convert that chunk of x into
// hi/lo bf16 in shared memory, synchronised through mbarriers. Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_gemv_tc_timeout_flag = 0;

namespace {

constexpr int kRows = 128;                 // weight rows per tile (16 per compute warp)
constexpr int kWarps = 8;                  // compute warps
constexpr int kThreads = (kWarps + 1) * 32;
constexpr int kTileBytes = kRows * 128;    // one code stage: 128 rows x 128 bytes
constexpr int kMaxStages = 8;
constexpr int kSmemMax = 227 * 1024;
constexpr long long kWaitLimit = 1LL << 32;  // cycles (~2 s)
constexpr long long kDrainLimit = 1LL << 31;

struct Shared {
  uint64_t cfull[kMaxStages];   // code tile landed (TMA bytes)
  uint64_t cempty[kMaxStages];  // code tile consumed (one arrival per compute warp)
  uint64_t sfull[2];            // scale tile landed
  uint64_t sempty[2];           // scale tile consumed (one arrival per compute warp)
  uint64_t xready;              // x chunk converted (one arrival per compute warp)
  uint64_t xfree;               // x chunk consumed (one arrival per compute warp)
  int abort;
};

// Bytes of one activation row of x in shared memory, holding `chunks` K-chunks: per chunk,
// for each K=16 step (2 per block) and each of hi/lo, 8 bytes per 8-code group; plus 32
// bytes of padding so that rows 0..3 of a half-warp fall on different banks.
__host__ __device__ constexpr int x_row_bytes(int kc, int chunks) { return 4 * kc * chunks + 32; }

struct Layout {
  int x, codes, sc, hdr, total;
};
__host__ __device__ inline Layout make_layout(int nt, int kc, int stages, int sc_bytes, int xchunks) {
  Layout L;
  L.codes = 0;  // 1024-aligned for the 128B swizzle
  L.sc = stages * kTileBytes;
  L.x = L.sc + 2 * sc_bytes;
  L.hdr = (L.x + 8 * nt * x_row_bytes(kc, xchunks) + 127) & ~127;
  L.total = L.hdr + static_cast<int>(sizeof(Shared)) + 1024;
  return L;
}

__device__ __forceinline__ void record_timeout(volatile int *abort) {
  *abort = 1;
  atomicOr(&g_gemv_tc_timeout_flag, 1u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t *>(&t);
}

// Two 4-bit codes (at bits 0-3 and 16-19 after the shift) -> exact bf16 pair (q_lo, q_hi).
__device__ __forceinline__ uint32_t int4_pair_bf16(uint32_t w) {
  const uint32_t v = (w & 0x000F000Fu) ^ 0x43084308u;  // bf16 128 + (q + 8)
  __nv_bfloat162 t = *reinterpret_cast<const __nv_bfloat162 *>(&v);
  t = __hsub2(t, __floats2bfloat162_rn(136.f, 136.f));  // exact: q
  return *reinterpret_cast<uint32_t *>(&t);
}

// Byte j of wa and byte j of wb (8-bit codes) -> exact bf16 pair.
__device__ __forceinline__ uint32_t int8_pair_bf16(uint32_t wa, uint32_t wb, int j) {
  const float bias = 8388608.0f + 128.0f;
  const float fa = __uint_as_float(__byte_perm(wa ^ 0x80808080u, 0x4B000000u, 0x7540 | j));
  const float fb = __uint_as_float(__byte_perm(wb ^ 0x80808080u, 0x4B000000u, 0x7540 | j));
  const float2 q = __fadd2_rn(make_float2(fa, fb), make_float2(-bias, -bias));
  return pack_bf16x2(q.x, q.y);
}

// D = A . B + C, m16n8k16, bf16 x bf16 -> f32.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1, const float (&c)[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]),
        "f"(c[2]), "f"(c[3]));
}

// grid.x: CTAs striding over 128-row tiles; one pass over all m (<= 8 * NT) activation rows.
template <int BITS, int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_s,
                   const float *__restrict__ x, float *__restrict__ y, int m, int n, int k,
                   int stages, int sc_bytes, int xres) {
  constexpr int KC = 1024 / BITS;         // codes per K-chunk: 128 bytes of a row
  constexpr int BPC = KC / 32;            // 32-code blocks per chunk
  constexpr int G = KC / 8;               // 8-code groups per chunk
  const int num_c = (k + KC - 1) / KC;
  // xres: all of x is converted once per CTA (it fits); else one chunk at a time.
  const int xchunks = xres ? num_c : 1;
  const int RS = x_row_bytes(KC, xchunks);
  const Layout L = make_layout(NT, KC, stages, sc_bytes, xchunks);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + L.hdr);
  volatile int *abort = &sh.abort;
  uint8_t *xs = smem + L.x;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int spr = k >> 5;
  const int num_tiles = (n + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&sh.cfull[s], 1);
      ptx::mbar_init(&sh.cempty[s], kWarps);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&sh.sfull[s], 1);
      ptx::mbar_init(&sh.sempty[s], kWarps);
    }
    ptx::mbar_init(&sh.xready, kWarps);
    ptx::mbar_init(&sh.xfree, kWarps);
    sh.abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ---- producer (one lane): weights only, so no wait on the preceding grid ----
    if (lane == 0) {
      ptx::prefetch_tmap(&tm_c);
      ptx::prefetch_tmap(&tm_s);
      int it = 0, tc = 0, issued_c = 0, issued_s = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tc) {
        const int sb = tc & 1;
        if (tc >= 2 && !ptx::mbar_wait_bounded(&sh.sempty[sb], ((tc >> 1) - 1) & 1, kWaitLimit, abort)) {
          record_timeout(abort);
          break;
        }
        ptx::mbar_arrive_expect_tx(&sh.sfull[sb], static_cast<uint32_t>(kRows * spr * 2));
        ptx::tma_load_2d(smem + L.sc + sb * sc_bytes, &tm_s, &sh.sfull[sb], 0, tile * kRows);
        issued_s = tc + 1;
        for (int c = 0; c < num_c; ++c, ++it) {
          const int s = it % stages, r = it / stages;
          if (r > 0 && !ptx::mbar_wait_bounded(&sh.cempty[s], (r - 1) & 1, kWaitLimit, abort)) {
            record_timeout(abort);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&sh.cfull[s], kTileBytes);
          ptx::tma_load_2d(smem + L.codes + s * kTileBytes, &tm_c, &sh.cfull[s], c * 128, tile * kRows);
          issued_c = it + 1;
        }
      }
      if (*abort) {  // drain: only the last issue to each buffer can still be in flight
        int no_abort = 0;
        for (int i = issued_c - 1; i >= 0 && i >= issued_c - stages; --i)
          ptx::mbar_wait_bounded(&sh.cfull[i % stages], (i / stages) & 1, kDrainLimit, &no_abort);
        for (int i = issued_s - 1; i >= 0 && i >= issued_s - 2; --i)
          ptx::mbar_wait_bounded(&sh.sfull[i & 1], (i >> 1) & 1, kDrainLimit, &no_abort);
      }
    }
    return;
  }

  // ---- compute warps: rows r0 = 16 * warp + g and r0 + 8 of each tile ----
  const int g = lane >> 2, tq = lane & 3;
  const int r0 = warp * 16 + g;
  ptx::pdl_wait();  // x and y belong to the preceding kernels from here on
  int it = 0, tc = 0;
  bool ok = true;
  for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++tc) {
    const int sb = tc & 1;
    if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.sfull[sb], (tc >> 1) & 1, kWaitLimit, abort))) {
      record_timeout(abort);
      ok = false;
      break;
    }
    const uint16_t *sct = reinterpret_cast<const uint16_t *>(smem + L.sc + sb * sc_bytes);
    float acc[NT][4];
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[t][i] = 0.f;

    for (int c = 0; c < num_c; ++c, ++it) {
      // 1) convert this chunk of x (rows 0 .. 8*NT-1) into hi/lo bf16 once the previous chunk
      //    is no longer read by any warp.
      const bool convert = xres ? it == 0 : true;  // resident x: only before the first chunk
      if (convert && it > 0 &&
          !__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.xfree, (it - 1) & 1, kWaitLimit, abort))) {
        record_timeout(abort);
        ok = false;
        break;
      }
      // Four items per thread per round: their global loads are all in flight before any
      // is converted.
      const int items = convert ? 8 * NT * G * xchunks : 0;
      for (int base = threadIdx.x; base < items; base += 4 * kWarps * 32) {
        float v[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = base + u * kWarps * 32;
          const int xr = idx / (G * xchunks), gi = idx - xr * (G * xchunks);
          const int cc = xres ? gi / G : c, grp = gi % G;
          const int kg = cc * KC + grp * 8;
          if (idx < items && xr < m && kg < k) {
            const float4 a4 = *reinterpret_cast<const float4 *>(x + static_cast<size_t>(xr) * k + kg);
            const float4 b4 = *reinterpret_cast<const float4 *>(x + static_cast<size_t>(xr) * k + kg + 4);
            v[u][0] = a4.x; v[u][1] = a4.y; v[u][2] = a4.z; v[u][3] = a4.w;
            v[u][4] = b4.x; v[u][5] = b4.y; v[u][6] = b4.z; v[u][7] = b4.w;
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[u][i] = 0.f;
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int idx = base + u * kWarps * 32;
          if (idx >= items) break;
          const int xr = idx / (G * xchunks), gi = idx - xr * (G * xchunks);
          const int cc = xres ? gi / G : c, grp = gi % G;
          uint8_t *row = xs + xr * RS + (xres ? cc : 0) * 4 * KC;
#pragma unroll
          for (int st = 0; st < 2; ++st) {
            // order within the step: e_{2st}, e_{2st+4}, e_{2st+1}, e_{2st+5}
            const float e[4] = {v[u][2 * st], v[u][2 * st + 4], v[u][2 * st + 1], v[u][2 * st + 5]};
            float h[4], l[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              h[i] = __bfloat162float(__float2bfloat16_rn(e[i]));
              l[i] = e[i] - h[i];  // exact in FP32
            }
            *reinterpret_cast<uint2 *>(row + ((st * 2 + 0) * G + grp) * 8) =
                make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
            *reinterpret_cast<uint2 *>(row + ((st * 2 + 1) * G + grp) * 8) =
                make_uint2(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]));
          }
        }
      }
      const int xph = xres ? 0 : (it & 1);
      if (convert) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.xready);
      }
      const int s = it % stages;
      if (!__all_sync(0xffffffffu,
                      ptx::mbar_wait_bounded(&sh.xready, xph, kWaitLimit, abort) &&
                          ptx::mbar_wait_bounded(&sh.cfull[s], (it / stages) & 1, kWaitLimit, abort))) {
        record_timeout(abort);
        ok = false;
        break;
      }
      // 2) the chunk's blocks: A from the 128B-swizzled code tile, B from the x chunk.
      const uint8_t *ct = smem + L.codes + s * kTileBytes;
#pragma unroll 2
      for (int b = 0; b < BPC; ++b) {
        uint32_t wr[2][2];  // [row r0 / r0+8][word]: this thread's 8 codes of block b
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int r = r0 + 8 * h;
          if constexpr (BITS == 4) {
            wr[h][0] = *reinterpret_cast<const uint32_t *>(ct + r * 128 + ((b ^ (r & 7)) << 4) + 4 * tq);
            wr[h][1] = 0u;
          } else {
            const int ch = 2 * b + (tq >> 1);
            const uint2 v = *reinterpret_cast<const uint2 *>(ct + r * 128 + ((ch ^ (r & 7)) << 4) + 8 * (tq & 1));
            wr[h][0] = v.x;
            wr[h][1] = v.y;
          }
        }
        uint32_t a[2][4];  // [step][fragment register]
#pragma unroll
        for (int st = 0; st < 2; ++st) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if constexpr (BITS == 4) {
              a[st][h] = int4_pair_bf16(wr[h][0] >> (8 * st));          // (e_{2st}, e_{2st+4})
              a[st][2 + h] = int4_pair_bf16(wr[h][0] >> (8 * st + 4));  // (e_{2st+1}, e_{2st+5})
            } else {
              a[st][h] = int8_pair_bf16(wr[h][0], wr[h][1], 2 * st);
              a[st][2 + h] = int8_pair_bf16(wr[h][0], wr[h][1], 2 * st + 1);
            }
          }
        }
        const int kb = c * BPC + b;
        const float s0 = __half2float(__ushort_as_half(sct[r0 * spr + kb]));
        const float s1 = __half2float(__ushort_as_half(sct[(r0 + 8) * spr + kb]));
        const int grp = b * 4 + tq;
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const uint8_t *xrow = xs + (t * 8 + g) * RS + (xres ? c : 0) * 4 * KC + grp * 8;
          float cb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int st = 0; st < 2; ++st) {
            const uint2 bh = *reinterpret_cast<const uint2 *>(xrow + (st * 2 + 0) * G * 8);
            const uint2 bl = *reinterpret_cast<const uint2 *>(xrow + (st * 2 + 1) * G * 8);
            mma_bf16(cb, a[st], bh.x, bh.y, cb);
            mma_bf16(cb, a[st], bl.x, bl.y, cb);
          }
          acc[t][0] = fmaf(s0, cb[0], acc[t][0]);
          acc[t][1] = fmaf(s0, cb[1], acc[t][1]);
          acc[t][2] = fmaf(s1, cb[2], acc[t][2]);
          acc[t][3] = fmaf(s1, cb[3], acc[t][3]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&sh.cempty[s]);
        if (!xres) ptx::mbar_arrive(&sh.xfree);
      }
    }
    if (!ok) break;
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&sh.sempty[sb]);
    // 3) y[m][row]: acc[t][0/1] rows r0, columns m = 8t + 2tq (+1); acc[t][2/3] row r0 + 8.
    ptx::pdl_launch_dependents();
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int mm = t * 8 + 2 * tq + (i & 1);
        const int row = tile * kRows + r0 + 8 * (i >> 1);
        if (mm < m && row < n) y[static_cast<size_t>(mm) * n + row] = acc[t][i];
      }
  }
}

template <int BITS, int NT>
int launch_t(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
             const DevInfo &dev) {
  constexpr int KC = 1024 / BITS;
  auto kern = gemv_tc_kernel<BITS, NT>;
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
  });
  if (attr_err != cudaSuccess) return WOQ_ECUDA;
  const int64_t spr = w.k / 32;
  const int sc_bytes = static_cast<int>((kRows * spr * 2 + 127) & ~int64_t(127));
  // Keep all of x resident when that still leaves three code stages.
  const int num_c = static_cast<int>((w.k + KC - 1) / KC);
  int xres = 1;
  if ((kSmemMax - make_layout(NT, KC, 0, sc_bytes, num_c).total) / kTileBytes < 3) xres = 0;
  const int xchunks = xres ? num_c : 1;
  const int stages = std::min(kMaxStages, (kSmemMax - make_layout(NT, KC, 0, sc_bytes, xchunks).total) / kTileBytes);
  if (stages < 2) return 1;
  const int smem = make_layout(NT, KC, stages, sc_bytes, xchunks).total;

  CUtensorMap tm_c, tm_s;
  if (!make_tensor_map_2d(&tm_c, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, w.k * BITS / 8, w.n,
                          128, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return WOQ_ECUDA;
  if (!make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w.scales, spr, w.n,
                          static_cast<uint32_t>(spr), kRows, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WOQ_ECUDA;
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, smem) != cudaSuccess || occ < 1)
    return WOQ_ECUDA;
  const int64_t tiles = (w.n + kRows - 1) / kRows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(tiles, static_cast<int64_t>(dev.sm_count) * occ)), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, tm_c, tm_s, x, y, static_cast<int>(m), static_cast<int>(w.n),
                         static_cast<int>(w.k), stages, sc_bytes, xres) != cudaSuccess)
    return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

template <int BITS>
int pick_nt(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
            const DevInfo &dev) {
  if (m <= 8) return launch_t<BITS, 1>(x, m, w, y, s, dev);
  if (m <= 16) return launch_t<BITS, 2>(x, m, w, y, s, dev);
  if (m <= 32) return launch_t<BITS, 4>(x, m, w, y, s, dev);
  return launch_t<BITS, 8>(x, m, w, y, s, dev);
}

}  // namespace

int launch_gemv_tc(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                   const DevInfo &dev) {
  // Shapes this path takes: 2 <= m <= 64; whole 128-byte code chunks and a scale tile that
  // one bulk tensor copy can bring (K/32 a multiple of 8, at most 256).
  if (m < 2 || m > 64 || w.k % 256 != 0 || w.k / 32 > 256) return 1;
  return w.bits == 4 ? pick_nt<4>(x, m, w, y, s, dev) : pick_nt<8>(x, m, w, y, s, dev);
}

int read_gemv_tc_timeout_flag(int clear, unsigned *value) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_tc_timeout_flag, sizeof(v)) != cudaSuccess) return WOQ_ECUDA;
  if (clear && v) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_gemv_tc_timeout_flag, &z, sizeof(z)) != cudaSuccess) return WOQ_ECUDA;
  }
  *value = v;
  return WOQ_OK;
}

}  // namespace woq
