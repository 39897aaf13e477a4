// FP32 CUDA-core qgemv: y[m, n] = x[m, k] . W_hat^T with W packed int4/int8 in blocks of 32
// along k and one binary16 scale per block ("TinyMOSS-Diarize", "How we built it": the
// decode GEMV multiplies straight out of the packed weights, FP32 activations, no
// dequantised weight tensor).
//
// Design (HBM-bound at small m):
//   * Each warp owns R consecutive weight rows at a time; lane l reads 16-byte chunks
//     l, l+32, ... of every row (one int4 block or half an int8 block per chunk) with
//     128-bit streaming loads, so a warp reads 512 contiguous bytes per row per step.
//   * x rows are staged once per CTA in shared memory, 16-byte units XOR-swizzled so a
//     quarter-warp reading 8 different chunks hits 8 different bank groups.
//   * Codes become exact FP32 values with a single LOP3 per element: the 4-bit field
//     (offset by 8) is placed in the low mantissa bits of 2^23 and the bias is removed
//     with one exact packed subtraction (f32x2). int4 fields at nibble position j of a
//     16-bit half carry a factor 2^(4j) that is removed, exactly, once per block.
//   * Products accumulate per block in FP32 (f32x2 FMA), the block sum is scaled once by
//     the binary16 scale, and rows are reduced across the warp with shuffles in a fixed
//     order (deterministic).
#include <cuda_fp16.h>

#include <algorithm>
#include <mutex>
#include <type_traits>
#include <unordered_map>

#include "gemv_math.cuh"
#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_gemv_timeout_flag = 0;

namespace {

using namespace gemv;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

// Dot products of RW consecutive weight rows with MT staged x rows over blocks [b0, b1) of
// each row, lane l taking blocks b0+l, b0+l+32, ... . SMEM: rows come from a shared-memory stage (all RW rows present);
// otherwise from global memory, rows at or past `valid` reading as zero.
template <int BITS, int MT, int RW, bool SMEM>
__device__ __forceinline__ void rows_dot(const float4 *__restrict__ xs4, int units_row, int spr,
                                         int lane, const uint8_t *codes, size_t row_stride,
                                         const uint16_t *scs, int valid, float (&acc)[RW][MT],
                                         int b0, int b1) {
  if constexpr (BITS == 5) {
    // int5: a block's 16 bytes of low nibbles at 16 b, its high-bit word at k/2 + 4 b
    const int half = spr * 16;
    for (int b = b0 + lane; b < b1; b += 32) {
      uint4 lo[RW];
      uint32_t hw[RW];
      float sc[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        const uint8_t *pr = codes + r * row_stride;
        if (SMEM || r < valid) {
          if constexpr (SMEM) {
            lo[r] = *reinterpret_cast<const uint4 *>(pr + b * 16);
            hw[r] = *reinterpret_cast<const uint32_t *>(pr + half + b * 4);
            sc[r] = half_bits_to_float(scs[r * spr + b]);
          } else {
            lo[r] = ptx::ldg_stream_v4(pr + b * 16);
            hw[r] = __ldg(reinterpret_cast<const uint32_t *>(pr + half + b * 4));
            sc[r] = half_bits_to_float(__ldg(scs + r * spr + b));
          }
        } else {
          lo[r] = make_uint4(0u, 0u, 0u, 0u);
          hw[r] = 0xFFFFFFFFu;  // with zero nibbles: code -16 times a zero scale
          sc[r] = 0.f;
        }
      }
      chunk_int5<MT, RW>(xs4, units_row, b, lo, hw, sc, acc);
    }
  } else {
  constexpr int kBlockBytes = BITS * 4;  // 16 (int4) or 32 (int8)
  for (int b = b0 + lane; b < b1; b += 32) {
    uint4 lo[RW], hi[RW];
    float sc[RW];
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const uint8_t *pr = codes + r * row_stride + b * kBlockBytes;
      if (SMEM || r < valid) {
        if constexpr (SMEM) {
          lo[r] = *reinterpret_cast<const uint4 *>(pr);
          if constexpr (BITS == 8) hi[r] = *reinterpret_cast<const uint4 *>(pr + 16);
          sc[r] = half_bits_to_float(scs[r * spr + b]);
        } else {
          lo[r] = ptx::ldg_stream_v4(pr);
          if constexpr (BITS == 8) hi[r] = ptx::ldg_stream_v4(pr + 16);
          sc[r] = half_bits_to_float(__ldg(scs + r * spr + b));
        }
      } else {
        lo[r] = make_uint4(0u, 0u, 0u, 0u);
        hi[r] = lo[r];
        sc[r] = 0.f;
      }
    }
    if constexpr (BITS == 4)
      chunk_int4<MT, RW>(xs4, units_row, b, lo, sc, acc);
    else
      block_int8<MT, RW>(xs4, units_row, b, lo, hi, sc, acc);
  }
  }
}

// Loads one batch of weight chunks: chunks cb + 32u + lane (u < U) of rows row0 .. row0+R-1.
// Rows at or past n, and chunks at or past cpr, read as zero codes with zero scale.
template <int BITS, int R, int U>
__device__ __forceinline__ void load_batch(const uint8_t *__restrict__ packed,
                                           const uint16_t *__restrict__ scales, int n, int cpr,
                                           int spr, size_t row_bytes, int row0, int cb, int lane,
                                           uint4 (&wv)[U][R], float (&sc)[U][R]) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = cb + 32 * u + lane;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int row = row0 + r;
      if (c < cpr && row < n) {
        wv[u][r] = ptx::ldg_stream_v4(packed + static_cast<size_t>(row) * row_bytes +
                                      static_cast<size_t>(c) * 16);
        sc[u][r] = half_bits_to_float(
            __ldg(scales + static_cast<size_t>(row) * spr + (BITS == 4 ? c : (c >> 1))));
      } else {
        wv[u][r] = make_uint4(0u, 0u, 0u, 0u);
        sc[u][r] = 0.f;
      }
    }
  }
}

// grid.x: CTAs striding over units of R rows; grid.y: passes of MT x rows.
//
// The weights never depend on the preceding kernel, so each warp issues the loads of its
// first batch before waiting on the preceding grid (programmatic dependent launch): their
// DRAM latency overlaps that grid's tail and the staging of x. Afterwards every batch's
// loads are issued one batch ahead of its arithmetic.
template <int BITS, int MT, int R, int U>
__global__ void __launch_bounds__(kThreads)
    gemv_kernel(const float *__restrict__ x, const uint8_t *__restrict__ packed,
                const uint16_t *__restrict__ scales, float *__restrict__ y, int m, int n, int k) {
  extern __shared__ float4 xs4[];
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int m0 = blockIdx.y * MT;
  const int units_row = k >> 2;
  const int cpr = (k * BITS) >> 7;  // 16-byte chunks per weight row
  const int spr = k >> 5;           // scales per row
  const size_t row_bytes = static_cast<size_t>(k) * BITS / 8;
  const int units = (n + R - 1) / R;
  const int stride = gridDim.x * kWarps;
  int unit = blockIdx.x * kWarps + warp;

  uint4 wv[U][R];
  float sc[U][R];
  load_batch<BITS, R, U>(packed, scales, n, cpr, spr, row_bytes, unit * R, 0, lane, wv, sc);

  // Everything below reads x or writes y, which a preceding kernel may produce or read.
  ptx::pdl_wait();

  // Stage x rows [m0, m0 + MT): 8-element groups; int4 interleaves (0,4,1,5 | 2,6,3,7)
  // so that each f32x2 pair lines up with the code pair (q_j, q_{4+j}).
  const int groups = k >> 3;
  for (int idx = tid; idx < MT * groups; idx += kThreads) {
    const int mm = idx / groups;
    const int g = idx - mm * groups;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (m0 + mm < m) {
      const float4 *src = reinterpret_cast<const float4 *>(x + static_cast<size_t>(m0 + mm) * k) + 2 * g;
      a = src[0];
      b = src[1];
    }
    float4 pa = a, pb = b;
    if constexpr (BITS != 8) {  // int4 and int5: nibble pairs
      pa = make_float4(a.x, b.x, a.y, b.y);
      pb = make_float4(a.z, b.z, a.w, b.w);
    }
    float4 *row = xs4 + mm * units_row;
    row[swz(2 * g)] = pa;
    row[swz(2 * g + 1)] = pb;
  }
  __syncthreads();
  ptx::pdl_launch_dependents();

  for (; unit < units; unit += stride) {
    const int row0 = unit * R;
    float acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) acc[r][mm] = 0.f;

    for (int cb = 0; cb < cpr; cb += 32 * U) {
      // Issue the next batch (rest of this row group, else the next unit) before computing.
      const bool same = cb + 32 * U < cpr;
      uint4 nwv[U][R];
      float nsc[U][R];
      load_batch<BITS, R, U>(packed, scales, n, cpr, spr, row_bytes,
                             same ? row0 : (unit + stride) * R, same ? cb + 32 * U : 0, lane,
                             nwv, nsc);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = cb + 32 * u + lane;
        if (c < cpr) {
          if constexpr (BITS == 4)
            chunk_int4<MT, R>(xs4, units_row, c, wv[u], sc[u], acc);
          else
            chunk_int8<MT, R>(xs4, units_row, c, wv[u], sc[u], acc);
        }
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int r = 0; r < R; ++r) {
          wv[u][r] = nwv[u][r];
          sc[u][r] = nsc[u][r];
        }
    }

#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        float v = acc[r][mm];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        acc[r][mm] = v;
      }
    // Lane (r * MT + mm) stores one result.
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
        if (lane == r * MT + mm && row0 + r < n && m0 + mm < m)
          y[static_cast<size_t>(m0 + mm) * n + row0 + r] = acc[r][mm];
  }
}

// ---------------------------------------------------------------------------------------
// Bulk-copy pipeline variant (the default when a tile of rows fits a shared-memory stage).
//
// A tile is TR = 8 * RW consecutive weight rows; its codes and its scales are each one
// contiguous range of memory, so one producer lane streams a tile with two 1-D bulk copies
// (cp.async.bulk) into a ring of shared-memory stages, completion counted in bytes on an
// mbarrier. Eight compute warps each take RW rows of a tile: lane l reads chunks l, l+32, ...
// of its rows from shared memory and runs the same exact FP32 arithmetic as above. Memory
// parallelism is the ring depth, not registers; the producer never touches x or y, so it
// issues its copies before the wait on the preceding grid and they overlap that grid. A
// partial last tile is read straight from global memory by the compute warps.
// ---------------------------------------------------------------------------------------

// Compute warps per CTA (NW): 8, or 16 for a single activation row over a matrix small
// enough that every CTA sees at most a couple of tiles. There the launch is latency-bound:
// the arithmetic after x arrives is on the critical path and twice the warps halve it,
// while two such CTAs (registers capped for it) still fit on an SM, so the next launch's
// CTAs can stream their weights beside this one's.
__host__ __device__ constexpr int bulk_threads(int nw) { return (nw + 1) * 32; }
constexpr int kMaxStages = 8;
constexpr int kBulkHeader = 256;  // mbarriers + abort flag (BulkShared, padded)
constexpr long long kGemvWaitLimit = 1LL << 32;   // cycles (~2 s)
constexpr long long kGemvDrainLimit = 1LL << 31;  // cycles (~1 s)

struct BulkShared {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];
  unsigned long long amax[8];  // argmax mode: this CTA's best key per activation row
  int abort;
  int stop[2];  // split-K: a compute warp's stage wait gave up on a tile of this parity
};
static_assert(sizeof(BulkShared) <= kBulkHeader, "header too small");

__device__ __forceinline__ void gemv_record_timeout(volatile int *abort) {
  *abort = 1;
  atomicOr(&g_gemv_timeout_flag, 1u);
}

// Argmax keys: the output's bits mapped to an unsigned order that agrees with the float
// order, every NaN (of either sign) above +inf, then the complement of the row so that ties
// go to the smaller row.
__device__ __forceinline__ unsigned long long argmax_key(float v, int row) {
  const uint32_t b = __float_as_uint(v);
  const uint32_t o = (v != v) ? 0xFFFFFFFFu : (b & 0x80000000u) ? ~b : (b | 0x80000000u);
  return (static_cast<unsigned long long>(o) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(row));
}

// Epilogues. kEpiWrite: y[m, n] is written. kEpiArgmax: nothing is written to y; for each
// activation row the CTA's largest key over its outputs goes into keys[row] by a 64-bit
// atomicMax. kEpiSwiglu: rows 2i and 2i+1 are a gate and an up projection (RW even, so a
// warp holds both); y[m, n/2] gets silu(gate) * up. kEpiResidual: y[m, n] = the output +
// resid[m, n], one FP32 add (resid may be y itself: each element is read, then written, by
// the one lane that owns it).
constexpr int kEpiWrite = 0, kEpiArgmax = 1, kEpiSwiglu = 2, kEpiResidual = 3;

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Registers for two CTAs per SM: the 17 warps of a 16-warp CTA need <= 56 (the launch bound);
// the 9 warps of an 8-warp CTA need <= 96, as a sub-partition holding five of the 18 warps has
// 16384 registers. The single-x-row 8-warp forms are held to 96 (the int4 lm_head form used
// 100, which left one CTA per SM); forms with more x rows keep what they use, one CTA per SM.
__host__ __device__ constexpr int bulk_max_regs(int nw, int mt) { return nw == 8 && mt == 1 ? 96 : 255; }

// y carries no __restrict__: in residual mode `resid` may be y itself.
//
// KS > 1 (split-K inside the CTA, one x row, any epilogue but SwiGLU): the KS consecutive
// warps of a group share the group's RW rows, warp part p taking blocks
// [p * spr / KS, (p + 1) * spr / KS) of each row. After each tile every warp leaves its
// reduced partial sums in shared memory (two buffers, by tile parity), the compute warps meet
// at a barrier, and the group's first warp adds the KS partials in part order, so the result
// does not depend on timing. The barrier is reached by every compute warp on every tile: a
// warp whose stage wait gave up skips the arithmetic and raises the tile's stop flag, and
// all compute warps leave the loop together after that tile's barrier.
template <int BITS, int MT, int RW, int NW, int EPI = kEpiWrite, int KS = 1>
__global__ void __launch_bounds__(bulk_threads(NW), NW == 16 ? 2 : 1) __maxnreg__(bulk_max_regs(NW, MT))
    gemv_bulk_kernel(const float *__restrict__ x, const uint8_t *__restrict__ packed,
                     const uint16_t *__restrict__ scales, float *y, int m, int n,
                     int k, int stages, int stage_bytes, int x_bytes,
                     unsigned long long *__restrict__ keys = nullptr, const float *resid = nullptr) {
  constexpr int kBulkWarps = NW;
  constexpr int TR = kBulkWarps / KS * RW;
  constexpr bool AMAX = EPI == kEpiArgmax;
  static_assert(EPI != kEpiSwiglu || RW % 2 == 0, "gate/up pairs need an even row count");
  static_assert(KS == 1 || (MT == 1 && NW % KS == 0 && EPI != kEpiSwiglu),
                "split-K takes one x row and the plain, residual or argmax epilogue");
  extern __shared__ __align__(128) uint8_t smem[];
  BulkShared &sh = *reinterpret_cast<BulkShared *>(smem);
  float4 *xs4 = reinterpret_cast<float4 *>(smem + kBulkHeader);
  uint8_t *ring = smem + kBulkHeader + x_bytes;
  volatile int *abort = &sh.abort;

  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int warp = tid >> 5;
  const int m0 = blockIdx.y * MT;
  const int units_row = k >> 2;
  const int spr = k >> 5;
  const size_t row_bytes = static_cast<size_t>(k) * BITS / 8;
  const uint32_t code_bytes = static_cast<uint32_t>(TR * row_bytes);
  const uint32_t scale_bytes = static_cast<uint32_t>(TR * spr * 2);
  const int full_tiles = n / TR;
  const int num_tiles = (n + TR - 1) / TR;

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(&sh.full[s], 1);
      ptx::mbar_init(&sh.empty[s], kBulkWarps);
    }
    sh.abort = 0;
    sh.stop[0] = sh.stop[1] = 0;
    for (int mm = 0; mm < MT; ++mm) sh.amax[mm] = 0ull;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kBulkWarps) {
    // ---- producer: weights only, so no wait on the preceding grid ----
    if (lane == 0) {
      int issued = 0;
      for (int tile = blockIdx.x, i = 0; tile < full_tiles; tile += gridDim.x, ++i) {
        const int s = i % stages;
        const int round = i / stages;
        if (round > 0 && !ptx::mbar_wait_bounded(&sh.empty[s], (round - 1) & 1, kGemvWaitLimit, abort,
                                                 NW == 8 ? 1000u : 0u)) {
          gemv_record_timeout(abort);
          break;
        }
        if (*abort) break;
        uint8_t *dst = ring + static_cast<size_t>(s) * stage_bytes;
        ptx::mbar_arrive_expect_tx(&sh.full[s], code_bytes + scale_bytes);
        ptx::bulk_load(dst, packed + static_cast<size_t>(tile) * code_bytes, code_bytes, &sh.full[s]);
        ptx::bulk_load(dst + code_bytes, scales + static_cast<size_t>(tile) * TR * spr, scale_bytes,
                       &sh.full[s]);
        issued = i + 1;
      }
      if (*abort) {
        int no_abort = 0;  // only the last issue to each stage can still be in flight
        for (int i = issued - 1; i >= 0 && i >= issued - stages; --i)
          ptx::mbar_wait_bounded(&sh.full[i % stages], (i / stages) & 1, kGemvDrainLimit, &no_abort);
      }
    }
    return;
  }

  // ---- compute warps ----
  ptx::pdl_wait();
  const int groups = k >> 3;
  for (int idx = tid; idx < MT * groups; idx += kBulkWarps * 32) {
    const int mm = idx / groups;
    const int g = idx - mm * groups;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (m0 + mm < m) {
      const float4 *src = reinterpret_cast<const float4 *>(x + static_cast<size_t>(m0 + mm) * k) + 2 * g;
      a = src[0];
      b = src[1];
    }
    float4 pa = a, pb = b;
    if constexpr (BITS != 8) {  // int4 and int5: nibble pairs
      pa = make_float4(a.x, b.x, a.y, b.y);
      pb = make_float4(a.z, b.z, a.w, b.w);
    }
    float4 *row = xs4 + mm * units_row;
    row[swz(2 * g)] = pa;
    row[swz(2 * g + 1)] = pb;
  }
  asm volatile("bar.sync 1, %0;" ::"n"(kBulkWarps * 32) : "memory");
  ptx::pdl_launch_dependents();
  unsigned long long best = 0ull;  // argmax mode: this lane's best key (activation row lane % MT)

  const int part = warp % KS;  // split-K: this warp's share of each row's blocks
  const int b0 = part * (spr / KS), b1 = KS == 1 ? spr : b0 + spr / KS;
  float *pbuf = reinterpret_cast<float *>(ring + static_cast<size_t>(stages) * stage_bytes);

  for (int tile = blockIdx.x, i = 0; tile < num_tiles; tile += gridDim.x, ++i) {
    const bool staged = tile < full_tiles;
    const int s = i % stages;
    // The outcome is made warp-uniform: shuffles and the elected arrival follow.
    // Bandwidth-bound launches (NW = 8) let waiting warps sleep so that the computing ones
    // get the issue slots; latency-bound ones (NW = 16) poll.
    const bool ok = !staged || __all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.full[s], (i / stages) & 1,
                                                                              kGemvWaitLimit, abort,
                                                                              NW == 8 ? 1000u : 0u));
    if (!ok) {
      gemv_record_timeout(abort);
      if constexpr (KS == 1) break;
      sh.stop[i & 1] = 1;  // written only by compute warps, read by all after this tile's barrier
    }
    const uint8_t *stage = ring + static_cast<size_t>(s) * stage_bytes;
    const int lrow0 = warp / KS * RW;  // this warp's first row within the tile
    const int row0 = tile * TR + lrow0;
    // Residual mode: the lane that will store output (row0 + lane / MT, x row lane % MT)
    // fetches its residual now, so that the load's latency hides behind the dot products.
    float res = 0.f;
    if constexpr (EPI == kEpiResidual) {
      const int rr = lane / MT, mm = lane % MT;
      if (part == 0 && rr < RW && row0 + rr < n && m0 + mm < m)
        res = resid[static_cast<size_t>(m0 + mm) * n + row0 + rr];
    }
    float acc[RW][MT];
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) acc[r][mm] = 0.f;

    if (staged && ok) {
      rows_dot<BITS, MT, RW, true>(xs4, units_row, spr, lane, stage + lrow0 * row_bytes, row_bytes,
                                   reinterpret_cast<const uint16_t *>(stage + code_bytes) + lrow0 * spr,
                                   RW, acc, b0, b1);
    } else if (!staged) {
      rows_dot<BITS, MT, RW, false>(xs4, units_row, spr, lane,
                                    packed + static_cast<size_t>(row0) * row_bytes, row_bytes,
                                    scales + static_cast<size_t>(row0) * spr, n - row0, acc, b0, b1);
    }
    if (staged && ok) {
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.empty[s]);
    }
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        float v = acc[r][mm];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        acc[r][mm] = v;
      }
    if constexpr (KS > 1) {
      float *pb = pbuf + (i & 1) * (kBulkWarps * RW);
      if (lane < RW) {
#pragma unroll
        for (int r = 0; r < RW; ++r)
          if (lane == r) pb[warp * RW + r] = acc[r][0];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kBulkWarps * 32) : "memory");
      // Every compute warp reads the same flag after the same barrier, so all leave together;
      // the next tile's flag is the other one, so a warp already on that tile cannot change
      // this outcome for a warp still reading it.
      if (*static_cast<volatile int *>(&sh.stop[i & 1])) break;
      if (part != 0) continue;
#pragma unroll
      for (int r = 0; r < RW; ++r) {
        float v = pb[warp * RW + r];
#pragma unroll
        for (int p = 1; p < KS; ++p) v += pb[(warp + p) * RW + r];
        acc[r][0] = v;
      }
    }
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
        if (lane == r * MT + mm && row0 + r < n && m0 + mm < m) {
          if constexpr (AMAX) {
            const unsigned long long key = argmax_key(acc[r][mm], row0 + r);
            best = key > best ? key : best;
          } else if constexpr (EPI == kEpiResidual) {
            y[static_cast<size_t>(m0 + mm) * n + row0 + r] = acc[r][mm] + res;
          } else if constexpr (EPI == kEpiSwiglu) {
            // every lane holds every row's sum after the butterfly: the up row r + 1 is here
            if (r % 2 == 0)
              y[static_cast<size_t>(m0 + mm) * (n / 2) + (row0 + r) / 2] =
                  silu(acc[r][mm]) * acc[r + 1 < RW ? r + 1 : r][mm];
          } else {
            y[static_cast<size_t>(m0 + mm) * n + row0 + r] = acc[r][mm];
          }
        }
  }
  if constexpr (AMAX) {
    // Lanes l and l ^ d with d >= MT hold keys of the same activation row (lane % MT): reduce
    // over them, then one shared atomic per warp and row.
#pragma unroll
    for (int d = 16; d >= MT; d >>= 1) {
      const unsigned long long o = __shfl_xor_sync(0xffffffffu, best, d);
      best = o > best ? o : best;
    }
    if (lane < MT) atomicMax(&sh.amax[lane], best);
    // Every compute warp reaches this barrier (a warp that gave up on a wait leaves its loop
    // and arrives here too); then one thread publishes the CTA's keys.
    asm volatile("bar.sync 1, %0;" ::"n"(kBulkWarps * 32) : "memory");
    if (tid == 0)
      for (int mm = 0; mm < MT; ++mm)
        if (m0 + mm < m) atomicMax(&keys[m0 + mm], sh.amax[mm]);
  }
}

struct OccKey {
  const void *fn;
  size_t smem;
  int device;
  bool operator==(const OccKey &o) const {
    return fn == o.fn && smem == o.smem && device == o.device;
  }
};
struct OccHash {
  size_t operator()(const OccKey &k) const {
    return std::hash<const void *>()(k.fn) ^ (k.smem * 1315423911u) ^ (size_t(k.device) << 48);
  }
};

// Resident CTAs per SM for (kernel, dynamic smem) on the device. Cached. Every kernel's
// dynamic shared-memory limit is raised once per device, on first use, to the most any of
// its launches asks for (`smem_max`), so that no launch depends on which sizes came first.
int blocks_per_sm(const void *fn, size_t smem, const DevInfo &dev, int threads, size_t smem_max) {
  static std::mutex mu;
  static std::unordered_map<OccKey, int, OccHash> cache;
  const OccKey key{fn, smem, dev.device};
  const OccKey raised{fn, 0, dev.device};
  bool need_raise = false;
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    need_raise = cache.find(raised) == cache.end();
  }
  if (need_raise) {
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_max)) != cudaSuccess)
      return -1;
    std::lock_guard<std::mutex> g(mu);
    cache[raised] = 1;
  }
  if (smem > smem_max) return -1;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, threads, smem) != cudaSuccess)
    return -1;
  std::lock_guard<std::mutex> g(mu);
  cache[key] = nb;
  return nb;
}

constexpr size_t kRegSmemMax = 200 * 1024;  // x rows staged by the register-path kernel

template <int BITS, int MT, int R, int U>
int launch_t(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
             const DevInfo &dev, bool pdl) {
  auto kern = gemv_kernel<BITS, MT, R, U>;
  const size_t smem = static_cast<size_t>(MT) * w.k * sizeof(float);
  const int nb = blocks_per_sm(reinterpret_cast<const void *>(kern), smem, dev, kThreads,
                               kRegSmemMax);
  if (nb <= 0) return WOQ_ECUDA;
  const int64_t units = (w.n + R - 1) / R;
  int64_t gx = (units + kWarps - 1) / kWarps;
  const int64_t cap = static_cast<int64_t>(dev.sm_count) * nb;
  if (gx > cap) gx = cap;
  const int64_t gy = (m + MT - 1) / MT;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, x, w.packed, w.scales, y, static_cast<int>(m),
                                           static_cast<int>(w.n), static_cast<int>(w.k));
  if (e != cudaSuccess) return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

template <int BITS, int MT>
int pick_ru(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
            const DevInfo &dev, bool pdl) {
  const int64_t cpr = w.k * BITS / 128;
  const bool two = cpr > 32;
  // Enough warps to cover the machine a few times over with R rows each.
  const int64_t want = static_cast<int64_t>(dev.sm_count) * 16;
  int R = 1;
  if (MT <= 2) {
    if ((w.n + 3) / 4 >= want) R = 4;
    else if ((w.n + 1) / 2 >= want) R = 2;
  } else if ((w.n + 1) / 2 >= want) {
    R = 2;
  }
  if constexpr (MT <= 2) {
    if (R == 4) return two ? launch_t<BITS, MT, 4, 2>(x, m, w, y, s, dev, pdl)
                           : launch_t<BITS, MT, 4, 1>(x, m, w, y, s, dev, pdl);
  }
  if (R == 2) return two ? launch_t<BITS, MT, 2, 2>(x, m, w, y, s, dev, pdl)
                         : launch_t<BITS, MT, 2, 1>(x, m, w, y, s, dev, pdl);
  return two ? launch_t<BITS, MT, 1, 2>(x, m, w, y, s, dev, pdl)
             : launch_t<BITS, MT, 1, 1>(x, m, w, y, s, dev, pdl);
}

// Bulk-pipeline launch. Returns 1 (not launched) when the shape does not suit it.
constexpr size_t kStageTarget = 20 * 1024;   // bytes per ring stage to aim for
// 8-warp (bandwidth-bound, wide-matrix) launches: a larger stage lets a warp take more rows
// (more independent work per lane between waits); two such stages still fit the budget.
constexpr size_t kStageTargetWide = 36 * 1024;
constexpr size_t kCtaSmemBudget = 100 * 1024;  // so that two CTAs fit on an SM

template <int BITS, int MT, int RW, int NW, int EPI = kEpiWrite, int KS = 1>
int launch_bulk_t(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                  const DevInfo &dev, bool pdl, size_t stage_bytes, size_t x_bytes,
                  unsigned long long *keys = nullptr, const float *resid = nullptr) {
  auto kern = gemv_bulk_kernel<BITS, MT, RW, NW, EPI, KS>;
  constexpr int kBulkThreads = bulk_threads(NW);
  constexpr int TR = NW / KS * RW;
  constexpr size_t kPartialBytes = KS > 1 ? 2 * NW * RW * sizeof(float) : 0;
  const int64_t num_tiles = (w.n + TR - 1) / TR;
  const int64_t full_tiles = w.n / TR;
  // stages: enough for the tiles one CTA will see, within the smem budget
  const int64_t want_grid = std::min<int64_t>(num_tiles, static_cast<int64_t>(dev.sm_count) * 2);
  int64_t stages = want_grid > 0 ? (full_tiles + want_grid - 1) / want_grid : 1;
  const int64_t fit = (static_cast<int64_t>(kCtaSmemBudget) - kBulkHeader - static_cast<int64_t>(x_bytes) -
                       static_cast<int64_t>(kPartialBytes)) /
                      static_cast<int64_t>(stage_bytes);
  stages = std::max<int64_t>(1, std::min<int64_t>({stages, fit, kMaxStages}));
  const size_t smem = kBulkHeader + x_bytes + stages * stage_bytes + kPartialBytes;
  const int nb = blocks_per_sm(reinterpret_cast<const void *>(kern), smem, dev, kBulkThreads,
                               kCtaSmemBudget);
  if (nb <= 0) return WOQ_ECUDA;
  const int64_t gx = std::max<int64_t>(1, std::min<int64_t>(num_tiles, static_cast<int64_t>(dev.sm_count) * nb));
  const int64_t gy = (m + MT - 1) / MT;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy), 1);
  cfg.blockDim = dim3(kBulkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, x, w.packed, w.scales, y, static_cast<int>(m),
                                           static_cast<int>(w.n), static_cast<int>(w.k),
                                           static_cast<int>(stages), static_cast<int>(stage_bytes),
                                           static_cast<int>(x_bytes), keys, resid);
  if (e != cudaSuccess) return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

// Rows per warp for NW compute warps: as many as fit a stage of about kStageTarget bytes; for
// 8 warps over a wide matrix, more (up to kStageTargetWide) while the tiles still number at
// least two per SM.
inline int bulk_rows_per_warp(int nw, int rw_max, size_t row_total, int64_t n = 0, int sms = 0) {
  int rw = rw_max;
  while (rw > 1 && static_cast<size_t>(nw) * rw * row_total > kStageTarget) rw /= 2;
  while (nw == 8 && rw < rw_max && static_cast<size_t>(nw) * rw * 2 * row_total <= kStageTargetWide &&
         n / (nw * rw * 2) >= 2 * static_cast<int64_t>(sms))
    rw *= 2;
  return rw;
}

template <int BITS, int MT, int NW, int EPI = kEpiWrite>
int launch_bulk_nw(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                   const DevInfo &dev, bool pdl, size_t row_total, size_t x_bytes,
                   unsigned long long *keys = nullptr, const float *resid = nullptr) {
  // More rows per warp only where registers allow.
  int rw = bulk_rows_per_warp(NW, NW == 16 ? 2 : MT <= 2 ? 4 : 2, row_total, w.n, dev.sm_count);
  const size_t stage_bytes = (static_cast<size_t>(NW) * rw * row_total + 127) & ~size_t(127);
  if (kBulkHeader + x_bytes + stage_bytes > kCtaSmemBudget) return 1;
  if (w.n < NW * rw) rw = 1;  // tiny n: one row per warp, all from global memory
  if constexpr (MT <= 2 && NW == 8) {
    if (rw == 4)
      return launch_bulk_t<BITS, MT, 4, NW, EPI>(x, m, w, y, s, dev, pdl, stage_bytes, x_bytes, keys,
                                                 resid);
  }
  if constexpr (NW == 8 || MT == 1) {
    if (rw >= 2)
      return launch_bulk_t<BITS, MT, 2, NW, EPI>(x, m, w, y, s, dev, pdl, stage_bytes, x_bytes, keys,
                                                 resid);
  }
  return launch_bulk_t<BITS, MT, 1, NW, EPI>(x, m, w, y, s, dev, pdl,
                                              (static_cast<size_t>(NW) * row_total + 127) & ~size_t(127),
                                              x_bytes, keys, resid);
}

// Split-K for the 16-warp launch of an int5 call with one x row (m == 1): while a warp's share
// of a row is more than one block per lane, halve it (up to 4 parts), as long as the CTAs
// still number at most two per SM and the scale ranges of a tile stay 16-byte multiples.
// Returns 1 when it does not split.
//
// Measured on B200 over the decoder block (four dependent launches, programmatic dependent
// launch): int5 11 % faster per step (15.7 -> 14.0 us), its unpack being the heaviest; int4
// 19 % slower (11.0 -> 13.2 us) even though o and down alone each got 0.1 us faster, because
// the split launches' extra CTAs leave no room on the SMs for the next launch's CTAs to start
// streaming their weights early. So int4 and int8 do not split.
//
// Calls with m > 1 never split, also where their x rows go one at a time, so that qgemv,
// qgemv_argmax and qgemv_residual at the same m add a row's products in the same order
// (bitwise the same outputs); an int5 row at m = 1 may differ in the last bits from the same
// row in a batch.
inline int bulk_splits(const woq_weight &w, int64_t m, int sms) {
  if (m != 1 || w.bits != 5) return 1;
  const int64_t spr = w.k / 32;
  int ks = 1;
  while (ks < 4 && spr / ks > 32 && spr % (2 * ks) == 0 && w.n / (16 / (2 * ks)) <= 2 * static_cast<int64_t>(sms) &&
         w.n >= 16 / (2 * ks))
    ks *= 2;
  return ks;
}

template <int BITS, int EPI>
int launch_bulk_split(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                      const DevInfo &dev, bool pdl, size_t row_total, size_t x_bytes, int ks,
                      const float *resid = nullptr, unsigned long long *keys = nullptr) {
  const size_t stage_bytes = (static_cast<size_t>(16 / ks) * row_total + 127) & ~size_t(127);
  if (kBulkHeader + x_bytes + stage_bytes + 2 * 16 * sizeof(float) > kCtaSmemBudget) return 1;
  if (ks == 2)
    return launch_bulk_t<BITS, 1, 1, 16, EPI, 2>(x, m, w, y, s, dev, pdl, stage_bytes, x_bytes, keys, resid);
  if (ks == 4)
    return launch_bulk_t<BITS, 1, 1, 16, EPI, 4>(x, m, w, y, s, dev, pdl, stage_bytes, x_bytes, keys, resid);
  return 1;
}

template <int BITS, int MT>
int try_bulk(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
             const DevInfo &dev, bool pdl) {
  const size_t row_total = static_cast<size_t>(w.k) * BITS / 8 + static_cast<size_t>(w.k) / 16;
  const size_t x_bytes = (static_cast<size_t>(MT) * w.k * sizeof(float) + 127) & ~size_t(127);
  if constexpr (MT == 1) {
    const int ks = bulk_splits(w, m, dev.sm_count);
    if (ks > 1) {
      const int rc = launch_bulk_split<BITS, kEpiWrite>(x, m, w, y, s, dev, pdl, row_total, x_bytes, ks);
      if (rc != 1) return rc;
    }
    // 16 warps where each CTA of the grid gets at most two tiles (latency-bound launches).
    const int rw16 = bulk_rows_per_warp(16, 2, row_total);
    const int64_t tiles16 = w.n / (16 * rw16);
    if (tiles16 >= 1 && tiles16 <= 2 * static_cast<int64_t>(dev.sm_count)) {
      const int rc = launch_bulk_nw<BITS, MT, 16>(x, m, w, y, s, dev, pdl, row_total, x_bytes);
      if (rc != 1) return rc;
    }
  }
  return launch_bulk_nw<BITS, MT, 8>(x, m, w, y, s, dev, pdl, row_total, x_bytes);
}

template <int BITS>
int pick_mt(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
            const DevInfo &dev, bool pdl) {
  int mt = m == 1 ? 1 : m == 2 ? 2 : m <= 4 ? 4 : 8;
  const size_t limit = dev.smem_optin < kRegSmemMax ? dev.smem_optin : kRegSmemMax;
  while (mt > 1 && static_cast<size_t>(mt) * w.k * sizeof(float) > limit) mt /= 2;
  if (static_cast<size_t>(mt) * w.k * sizeof(float) > limit) return WOQ_ESHAPE;
  int rc = 1;
  auto bulk = [&](int t) {
    switch (t) {
      case 1: return try_bulk<BITS, 1>(x, m, w, y, s, dev, pdl);
      case 2: return try_bulk<BITS, 2>(x, m, w, y, s, dev, pdl);
      case 4: return try_bulk<BITS, 4>(x, m, w, y, s, dev, pdl);
      default: return try_bulk<BITS, 8>(x, m, w, y, s, dev, pdl);
    }
  };
  rc = bulk(mt);
  if (rc != 1) return rc;
  if constexpr (BITS == 5) {
    // int5 has the staged kernel only: fewer x rows per CTA until they fit beside a stage
    for (int t = mt / 2; t >= 1; t /= 2) {
      rc = bulk(t);
      if (rc != 1) return rc;
    }
    return WOQ_ESHAPE;
  } else {
    switch (mt) {
      case 1: return pick_ru<BITS, 1>(x, m, w, y, s, dev, pdl);
      case 2: return pick_ru<BITS, 2>(x, m, w, y, s, dev, pdl);
      case 4: return pick_ru<BITS, 4>(x, m, w, y, s, dev, pdl);
      default: return pick_ru<BITS, 8>(x, m, w, y, s, dev, pdl);
    }
  }
}

// qgemv_argmax's first and last steps: zero the keys; turn each key back into
// (row, output). Both wait on the preceding grid before touching memory.
__global__ void __launch_bounds__(32) argmax_init_kernel(unsigned long long *keys, int m) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  if (static_cast<int>(threadIdx.x) < m) keys[threadIdx.x] = 0ull;
}

__global__ void __launch_bounds__(32) argmax_final_kernel(unsigned long long *keys, float *val,
                                                          int m) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  const int i = threadIdx.x;
  if (i >= m) return;
  const unsigned long long key = keys[i];
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  const uint32_t b = (o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o;
  val[i] = __uint_as_float(b);
  reinterpret_cast<long long *>(keys)[i] =
      static_cast<long long>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
}

// Calls go(MT) for x-row tiles of MT = the smallest of 1, 2, 4, 8 that covers m, then for
// smaller MT while the launch does not fit in a CTA's shared memory (go returns 1): fewer x
// rows per CTA leave room for longer rows. Returns 1 if not even MT = 1 fits.
template <typename Go>
int with_fitting_mt(int64_t m, Go &&go) {
  const int want = m == 1 ? 1 : m == 2 ? 2 : m <= 4 ? 4 : 8;
  int rc = 1;
  if (want >= 8 && (rc = go(std::integral_constant<int, 8>())) != 1) return rc;
  if (want >= 4 && (rc = go(std::integral_constant<int, 4>())) != 1) return rc;
  if (want >= 2 && (rc = go(std::integral_constant<int, 2>())) != 1) return rc;
  return go(std::integral_constant<int, 1>());
}

// qgemv_swiglu: the bulk GEMV with two rows (gate, up) per warp.
template <int BITS>
int swiglu_bulk(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                const DevInfo &dev) {
  const size_t row_total = static_cast<size_t>(w.k) * BITS / 8 + static_cast<size_t>(w.k) / 16;
  auto go = [&](auto mt_tag, auto nw_tag) -> int {
    constexpr int MT = decltype(mt_tag)::value;
    constexpr int NW = decltype(nw_tag)::value;
    const size_t x_bytes = (static_cast<size_t>(MT) * w.k * sizeof(float) + 127) & ~size_t(127);
    const size_t stage_bytes = (static_cast<size_t>(NW) * 2 * row_total + 127) & ~size_t(127);
    if (kBulkHeader + x_bytes + stage_bytes > kCtaSmemBudget) return 1;
    return launch_bulk_t<BITS, MT, 2, NW, kEpiSwiglu>(x, m, w, y, s, dev, true, stage_bytes, x_bytes);
  };
  using I8 = std::integral_constant<int, 8>;
  using I16 = std::integral_constant<int, 16>;
  return with_fitting_mt(m, [&](auto mt_tag) -> int {
    if constexpr (decltype(mt_tag)::value == 1) {
      // as qgemv: 16 warps while each CTA gets at most two tiles
      if (w.n / 32 <= 2 * static_cast<int64_t>(dev.sm_count)) {
        const int rc = go(mt_tag, I16());
        if (rc != 1) return rc;
      }
    }
    return go(mt_tag, I8());
  });
}

template <int BITS>
int argmax_bulk(const float *x, int64_t m, const woq_weight &w, unsigned long long *keys,
                cudaStream_t s, const DevInfo &dev) {
  const size_t row_total = static_cast<size_t>(w.k) * BITS / 8 + static_cast<size_t>(w.k) / 16;
  return with_fitting_mt(m, [&](auto mt_tag) -> int {
    constexpr int MT = decltype(mt_tag)::value;
    const size_t x_bytes = (static_cast<size_t>(MT) * w.k * sizeof(float) + 127) & ~size_t(127);
    if constexpr (MT == 1) {
      // where qgemv splits K, the pick does too, so that it sees the same output bits
      const int ks = bulk_splits(w, m, dev.sm_count);
      if (ks > 1) {
        const int rc = launch_bulk_split<BITS, kEpiArgmax>(x, m, w, nullptr, s, dev, true, row_total, x_bytes,
                                                           ks, nullptr, keys);
        if (rc != 1) return rc;
      }
    }
    return launch_bulk_nw<BITS, MT, 8, kEpiArgmax>(x, m, w, nullptr, s, dev, true, row_total, x_bytes, keys);
  });
}

// qgemv_residual: the bulk GEMV (row and warp choices as qgemv's) with the residual add.
template <int BITS>
int residual_bulk(const float *x, int64_t m, const woq_weight &w, const float *r, float *y,
                  cudaStream_t s, const DevInfo &dev) {
  const size_t row_total = static_cast<size_t>(w.k) * BITS / 8 + static_cast<size_t>(w.k) / 16;
  return with_fitting_mt(m, [&](auto mt_tag) -> int {
    constexpr int MT = decltype(mt_tag)::value;
    const size_t x_bytes = (static_cast<size_t>(MT) * w.k * sizeof(float) + 127) & ~size_t(127);
    if constexpr (MT == 1) {
      const int ks = bulk_splits(w, m, dev.sm_count);
      if (ks > 1) {
        const int rc = launch_bulk_split<BITS, kEpiResidual>(x, m, w, y, s, dev, true, row_total, x_bytes,
                                                             ks, r);
        if (rc != 1) return rc;
      }
      const int rw16 = bulk_rows_per_warp(16, 2, row_total);
      const int64_t tiles16 = w.n / (16 * rw16);
      if (tiles16 >= 1 && tiles16 <= 2 * static_cast<int64_t>(dev.sm_count)) {
        const int rc = launch_bulk_nw<BITS, MT, 16, kEpiResidual>(x, m, w, y, s, dev, true, row_total,
                                                                  x_bytes, nullptr, r);
        if (rc != 1) return rc;
      }
    }
    return launch_bulk_nw<BITS, MT, 8, kEpiResidual>(x, m, w, y, s, dev, true, row_total, x_bytes,
                                                     nullptr, r);
  });
}

}  // namespace

int read_gemv_timeout_flag(int clear, unsigned *value) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_gemv_timeout_flag, sizeof(v)) != cudaSuccess) return WOQ_ECUDA;
  if (clear && v) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_gemv_timeout_flag, &z, sizeof(z)) != cudaSuccess) return WOQ_ECUDA;
  }
  *value = v;
  return WOQ_OK;
}

int launch_gemv_fp32(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                     const DevInfo &dev, bool pdl) {
  return w.bits == 4 ? pick_mt<4>(x, m, w, y, s, dev, pdl)
       : w.bits == 5 ? pick_mt<5>(x, m, w, y, s, dev, pdl)
                     : pick_mt<8>(x, m, w, y, s, dev, pdl);
}

int launch_gemv_swiglu(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                       const DevInfo &dev) {
  const int rc = w.bits == 4 ? swiglu_bulk<4>(x, m, w, y, s, dev)
               : w.bits == 5 ? swiglu_bulk<5>(x, m, w, y, s, dev)
                             : swiglu_bulk<8>(x, m, w, y, s, dev);
  return rc == 1 ? WOQ_ESHAPE : rc;
}

int launch_gemv_residual(const float *x, int64_t m, const woq_weight &w, const float *r, float *y,
                         cudaStream_t s, const DevInfo &dev) {
  const int rc = w.bits == 4 ? residual_bulk<4>(x, m, w, r, y, s, dev)
               : w.bits == 5 ? residual_bulk<5>(x, m, w, r, y, s, dev)
                             : residual_bulk<8>(x, m, w, r, y, s, dev);
  return rc == 1 ? WOQ_ESHAPE : rc;
}

int launch_gemv_argmax(const float *x, int64_t m, const woq_weight &w, int64_t *idx, float *val,
                       cudaStream_t s, const DevInfo &dev) {
  unsigned long long *keys = reinterpret_cast<unsigned long long *>(idx);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(32, 1, 1);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, argmax_init_kernel, keys, static_cast<int>(m)) != cudaSuccess)
    return WOQ_ECUDA;
  count_launches(1);
  const int rc = w.bits == 4 ? argmax_bulk<4>(x, m, w, keys, s, dev)
               : w.bits == 5 ? argmax_bulk<5>(x, m, w, keys, s, dev)
                             : argmax_bulk<8>(x, m, w, keys, s, dev);
  if (rc == 1) return WOQ_ESHAPE;
  if (rc != WOQ_OK) return rc;
  if (cudaLaunchKernelEx(&cfg, argmax_final_kernel, keys, val, static_cast<int>(m)) != cudaSuccess)
    return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

}  // namespace woq
