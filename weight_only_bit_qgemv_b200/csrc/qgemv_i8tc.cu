// qgemv on the integer tensor cores: y[m, n] = x[m, k] . W_hat^T for small m (decode), with
// the weight codes multiplied exactly by tcgen05.mma kind::i8 and FP32 accuracy kept by
// splitting x into signed 8-bit digits. "TinyMOSS-Diarize", "What's next": an i8mm GEMM path
// that does not quantise the activations; "How we built it": weight-only, FP32 activations,
// dequantisation fused into the multiply, no dequantised weight tensor.
//
// Arithmetic. Per activation row a and 32-block b of K, x is written as
//   x = 2^E (d0 + d1 * 2^-7 + d2 * 2^-14),  d_i integers in [-64, 64],
// with E = p - 6 where max |x| over the block lies in [2^(p-1), 2^p); the remainder is below
// 2^(E-15), i.e. under 2^-20 of the block's largest |x|. The weight operand is the codes as
// s8: int8 codes as they are, int4 codes as 16 * q (the nibble in the top half of a byte,
// which is its two's-complement value times 16). One K = 32 MMA per block multiplies a
// 128-row tile of codes against the block's digits into accumulator columns of its own, so
// every block's three exact int32 sums S_i = sum over the block of code * d_i stay apart
// (the weight scale differs from block to block). The epilogue forms
// T = S0 + S1 2^-7 + S2 2^-14 in FP32 and accumulates s_b 2^E T over the blocks in FP32
// (with 1/16 for int4). Deterministic: fixed block and split order.
//
// Layout. A stage is 128 weight rows x 128 K (4 blocks): the s8 code tile is one 128-byte
// row per weight row in the 128B-swizzled K-major layout the MMA's shared-memory descriptor
// names (int8: copied in that form by TMA; int4: TMA of the packed rows, then converter warps
// write it). The B tile of a stage has N = 16 * ceil(3 m / 16) rows: row 3 a + i holds digit
// i of activation row a, block j of the stage in bytes 32 j .. 32 j + 31. Block j's MMA reads
// only those bytes and writes its own N-column group of the stage's slot of tensor memory (a
// ring of slots of 4 N columns), so a stage's four MMAs do not depend on one another; the
// epilogue reads the slot, combines and frees it.
//
// Work. A unit is a 128-row tile and a range of K-stages. Few tiles (the decoder's
// projections): K is split across the CTAs of a thread-block cluster (one unit per CTA) and
// the partial outputs are summed through distributed shared memory in rank order. Many tiles
// (the lm_head): one persistent CTA per SM walks tiles over the whole of K.
//
// Roles (320 threads): warp 0 producer (TMA of the code tiles, no multicast), warp 1 tensor
// memory owner and MMA issuer, warps 2-5 epilogue (x digits into the B tiles, then
// accumulator read-out), warps 6-9 int4 converters. Every mbarrier wait is bounded; a wait
// that gives up records the event, stops the CTA's roles, drains what was issued, frees
// tensor memory and returns.
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_i8tc_timeout_flag = 0;

namespace {

constexpr int kRows = 128;           // weight rows per tile (MMA M)
constexpr int kStageK = 128;         // K per stage: 4 blocks, one 128-byte swizzle row of s8
constexpr int kBlocksPerStage = kStageK / 32;
constexpr int kATile = kRows * kStageK;  // 16 KB of s8 codes
constexpr int kRawTile = kRows * 64;     // 8 KB of packed int4 codes
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2, kEpiWarps = 4;
constexpr int kCvtWarp0 = 6, kCvtWarps = 4;
constexpr int kThreads = (kCvtWarp0 + kCvtWarps) * 32;  // 320
constexpr int kMaxA = 10;     // s8 code tiles
constexpr int kMaxRaw = 12;   // packed int4 tiles
constexpr int kMaxSlots = 16; // tensor-memory stage slots
constexpr int kMaxM = 4;
constexpr int kScaleChunk = 4;  // stages of scales fetched ahead by each read-out lane
constexpr long long kWaitLimit = 1LL << 32;   // cycles (~2 s)
constexpr long long kDrainLimit = 1LL << 31;  // cycles (~1 s)

struct Shared {
  uint64_t rawfull[kMaxRaw], rawempty[kMaxRaw];
  uint64_t afull[kMaxA], aempty[kMaxA];
  uint64_t accfull[kMaxSlots], accempty[kMaxSlots];
  uint64_t bready;   // B tiles and digit scales written (one arrival per epilogue warp)
  uint64_t drain;    // every MMA issued has completed
  uint32_t tmem_base;
  int abort;
  int gexp[kMaxM];   // per activation row: the largest block exponent of this CTA's K range
};

// Byte offsets of the dynamic shared-memory regions (the base is aligned to 1024 bytes).
struct Layout {
  int a, raw, b, cexp, eexp, part, bar, total;
};
__host__ __device__ inline Layout make_layout(int sa, int sraw, int bstages, int nb, int blocks, int m) {
  Layout L;
  L.a = 0;                                   // s8 code tiles (1024-aligned)
  L.raw = L.a + sa * kATile;                 // packed int4 tiles
  L.b = L.raw + sraw * kRawTile;             // B tiles (1024-aligned: both above are)
  L.cexp = L.b + bstages * nb * 128;         // float [m][blocks]: 2^(E - G) (1/16 for int4)
  L.eexp = L.cexp + ((m * blocks * 4 + 15) & ~15);  // int [m][blocks]: E
  L.part = L.eexp + ((m * blocks * 4 + 15) & ~15);  // float [m][128]: partial outputs
  L.bar = L.part + m * kRows * 4;
  L.total = L.bar + static_cast<int>(sizeof(Shared)) + 1024;  // + base alignment slack
  return L;
}

// Instruction descriptor, kind::i8: D s32, A and B s8, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_i8(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(kRows >> 4) << 24);
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void tc_mma_i8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{.reg .pred p; setp.ne.b32 p, %4, 0;"
      " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void record_timeout(volatile int *abort) {
  *abort = 1;
  atomicOr(&g_i8tc_timeout_flag, 1u);
}

// 2^e, exact; built from the bit pattern where e is a normal exponent.
__device__ __forceinline__ float pow2f(int e) {
  return (e >= -126 && e <= 127) ? __int_as_float((e + 127) << 23) : ldexpf(1.0f, e);
}

// p with v = f 2^p, 0.5 <= |f| < 1 (0 for v == 0), for finite v.
__device__ __forceinline__ int frexp_exp(float v) {
  const int ef = (__float_as_int(v) >> 23) & 0xFF;
  if (ef != 0) return ef - 126;
  int p = 0;
  frexpf(v, &p);  // zero or subnormal
  return p;
}

// Byte offset of (row, K byte) in a tile of 128-byte rows, 128B-swizzled.
__device__ __forceinline__ int sw128_off(int row, int kb) {
  return row * 128 + ((((kb >> 4) ^ row) & 7) << 4) + (kb & 15);
}

// Position, within its 8-element group, that element e of x takes in the K order of the s8
// code tile: int4 tiles hold each packed word's even codes, then its odd codes.
template <int BITS>
__device__ __forceinline__ int k_pos(int e) {
  if constexpr (BITS == 4) {
    const int g = e & ~7, r = e & 7;
    return g + ((r & 1) ? 4 + (r >> 1) : (r >> 1));
  } else {
    return e;
  }
}

template <int BITS, int M>
__global__ void __launch_bounds__(kThreads, 2)
    qgemv_i8tc_kernel(const __grid_constant__ CUtensorMap tm_w, const float *__restrict__ x,
                      const uint16_t *__restrict__ scales, float *__restrict__ y, int N, int K,
                      int splits, int sa, int sraw, int slots, int nb, long long wait_limit) {
  const int spr = K >> 5;                              // blocks per row
  const int num_stages = (K + kStageK - 1) / kStageK;
  const int num_tiles = (N + kRows - 1) / kRows;
  const int kps = (num_stages + splits - 1) / splits;  // stages per split
  const int num_units = num_tiles * splits;
  // This CTA's K-stage range: a split's range when K is split (one unit per CTA), else all.
  const int cs0 = splits > 1 ? (blockIdx.x % splits) * kps : 0;
  const int cs1 = splits > 1 ? min(num_stages, cs0 + kps) : num_stages;
  const int blk0 = cs0 * kBlocksPerStage;
  const int nblk = min(spr, cs1 * kBlocksPerStage) - blk0;  // blocks in the range
  const Layout L = make_layout(sa, sraw, cs1 - cs0, nb, nblk, M);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + L.bar);
  volatile int *abort = &sh.abort;
  float *cexp = reinterpret_cast<float *>(smem + L.cexp);
  int *eexp = reinterpret_cast<int *>(smem + L.eexp);
  float *part = reinterpret_cast<float *>(smem + L.part);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool kCvt = BITS == 4;

  if (threadIdx.x == 0) {
    for (int s = 0; s < sraw; ++s) {
      ptx::mbar_init(&sh.rawfull[s], 1);
      ptx::mbar_init(&sh.rawempty[s], kCvtWarps);
    }
    for (int s = 0; s < sa; ++s) {
      ptx::mbar_init(&sh.afull[s], kCvt ? kCvtWarps : 1);
      ptx::mbar_init(&sh.aempty[s], 1);
    }
    for (int s = 0; s < slots; ++s) {
      ptx::mbar_init(&sh.accfull[s], 1);
      ptx::mbar_init(&sh.accempty[s], kEpiWarps);
    }
    ptx::mbar_init(&sh.bready, kEpiWarps);
    ptx::mbar_init(&sh.drain, 1);
    sh.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) ptx::prefetch_tmap(&tm_w);
  uint32_t tmem_cols = 32;
  while (tmem_cols < static_cast<uint32_t>(slots * 4 * nb)) tmem_cols <<= 1;
  if (warp == kMmaWarp) {
    ptx::tmem_alloc(&sh.tmem_base, tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // drain bookkeeping: slots issued at least once and the parity of their last issue
  uint32_t imask = 0, ipar = 0;
  bool mma_issued = false;

  if (warp == 0) {
    // ---- producer (one lane): weights only, so no wait on the preceding grid ----
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      const int nslot = kCvt ? sraw : sa;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int tile = u / splits;
        const int s0 = splits > 1 ? cs0 : 0, s1 = splits > 1 ? cs1 : num_stages;
        for (int st = s0; st < s1; ++st) {
          uint64_t *empty = kCvt ? &sh.rawempty[s] : &sh.aempty[s];
          uint64_t *full = kCvt ? &sh.rawfull[s] : &sh.afull[s];
          if (!ptx::mbar_wait_bounded(empty, ph ^ 1, wait_limit, abort)) {
            record_timeout(abort);
            ok = false;
            break;
          }
          uint8_t *dst = smem + (kCvt ? L.raw + s * kRawTile : L.a + s * kATile);
          ptx::mbar_arrive_expect_tx(full, kCvt ? kRawTile : kATile);
          ptx::tma_load_2d(dst, &tm_w, full, st * (kStageK * BITS / 8), tile * kRows);
          imask |= 1u << s;
          ipar = (ipar & ~(1u << s)) | (ph << s);
          if (++s == nslot) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---- MMA issuer (one lane) ----
    if (lane == 0) {
      bool ok = ptx::mbar_wait_bounded(&sh.bready, 0, wait_limit, abort);
      if (!ok) record_timeout(abort);
      const uint32_t idesc = idesc_i8(nb);
      const uint64_t adesc0 = sw128_desc(ptx::smem_u32(smem + L.a));
      const uint64_t bdesc0 = sw128_desc(ptx::smem_u32(smem + L.b));
      int a = 0, slot = 0;
      uint32_t aph = 0, sph = 0;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int s0 = splits > 1 ? cs0 : 0, s1 = splits > 1 ? cs1 : num_stages;
        for (int st = s0; st < s1; ++st) {
          ok = ptx::mbar_wait_bounded(&sh.accempty[slot], sph ^ 1, wait_limit, abort) &&
               ptx::mbar_wait_bounded(&sh.afull[a], aph, wait_limit, abort);
          if (!ok) {
            record_timeout(abort);
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem + static_cast<uint32_t>(slot * 4 * nb);
          // start-address field counts 16-byte units: one block (32 bytes of K) = 2 units
          const uint64_t ad = adesc0 + static_cast<uint64_t>(a * (kATile >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((st - cs0) * ((nb * 128) >> 4));
          const int nvalid = min(kBlocksPerStage, spr - st * kBlocksPerStage);
          for (int j = 0; j < nvalid; ++j) tc_mma_i8(d + j * nb, ad + 2 * j, bd + 2 * j, idesc, 0u);
          mma_issued = true;
          ptx::tc_commit(&sh.aempty[a]);
          ptx::tc_commit(&sh.accfull[slot]);
          if (++a == sa) {
            a = 0;
            aph ^= 1;
          }
          if (++slot == slots) {
            slot = 0;
            sph ^= 1;
          }
        }
      }
      ptx::tc_commit(&sh.drain);  // arrives once every MMA issued above has completed
    }
  } else if (warp < kCvtWarp0) {
    // ---- epilogue: x digits into the B tiles, then accumulator read-out ----
    const int et = threadIdx.x - kEpiWarp0 * 32;  // 0..127
    const int ew = et >> 5;
    const int q = warp & 3;        // TMEM lanes 32q .. 32q+31
    const int rl = q * 32 + lane;  // weight row within the tile
    bool ok = true;
    // Scales of this lane's row for the f-th .. (f+7)-th stage of the CTA's stage sequence.
    const int su0 = splits > 1 ? cs0 : 0, su1 = splits > 1 ? cs1 : num_stages;
    auto load_scale_chunk = [&](int f, uint2 (&buf)[kScaleChunk]) {
      const int units_here = blockIdx.x < num_units ? (num_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
#pragma unroll
      for (int i = 0; i < kScaleChunk; ++i) {
        buf[i] = make_uint2(0u, 0u);
        const int fi = f + i, ui = fi / (su1 - su0);
        if (ui < units_here) {
          const int st = su0 + fi - ui * (su1 - su0);
          const int rw = min((blockIdx.x + ui * gridDim.x) / splits * kRows + rl, N - 1);
          buf[i] = __ldg(reinterpret_cast<const uint2 *>(scales + static_cast<size_t>(rw) * spr + st * 4));
        }
      }
    };
    uint2 scur[kScaleChunk], snext[kScaleChunk];
    load_scale_chunk(0, scur);
    // (1) zero the B tiles (only digit bytes are written below)
    {
      uint4 *bt = reinterpret_cast<uint4 *>(smem + L.b);
      const int n16 = (cs1 - cs0) * nb * 128 / 16;
      for (int i = et; i < n16; i += kEpiWarps * 32) bt[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    ptx::pdl_wait();  // x is written by preceding kernels, and y may be read by them
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    // (2) per (activation row, block): exponent and digits, one block per warp at a time; each
    // warp issues the x loads of eight of its blocks before using any (one L2 round trip)
    constexpr int kBatch = 8;
    for (int job0 = ew; job0 < M * nblk; job0 += kEpiWarps * kBatch) {
      float vb[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int job = job0 + i * kEpiWarps;
        vb[i] = 0.f;
        if (job < M * nblk) {
          const int a = job / nblk, b = blk0 + job - (job / nblk) * nblk;
          vb[i] = x[static_cast<size_t>(a) * K + 32 * b + lane];
        }
      }
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const int job = job0 + i * kEpiWarps;
        if (job >= M * nblk) break;  // warp-uniform
        const int a = job / nblk, bl = job - a * nblk;
        const int b = blk0 + bl;
        const float v = vb[i];
        float mx = fabsf(v);
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const int e = frexp_exp(mx) - 6;
        const float t = e >= -127 ? v * pow2f(-e) : ldexpf(v, -e);  // |t| < 64
        const float d0 = rintf(t);
        const float r1 = (t - d0) * 128.0f;
        const float d1 = rintf(r1);
        const float d2 = rintf((r1 - d1) * 128.0f);
        const int st = b / kBlocksPerStage - cs0, j = b % kBlocksPerStage;
        uint8_t *bt = smem + L.b + st * nb * 128;
        const int kb = 32 * j + k_pos<BITS>(lane);
        const int r0 = a * 3;
        bt[sw128_off(r0, kb)] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<int>(d0)));
        bt[sw128_off(r0 + 1, kb)] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<int>(d1)));
        bt[sw128_off(r0 + 2, kb)] = static_cast<uint8_t>(static_cast<int8_t>(static_cast<int>(d2)));
        // a block holding a non-finite x (fmaxf above skips NaN) makes its outputs NaN
        const bool finite = __all_sync(0xffffffffu, isfinite(v));
        if (lane == 0) eexp[a * nblk + bl] = finite ? e : INT32_MIN;
      }
    }
    ptx::fence_proxy_async_smem();
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    // (3) per activation row the largest exponent G; per block 2^(E - G) (1/16 for int4)
    if (et < M) {
      int g = INT32_MIN + 1;
      for (int bl = 0; bl < nblk; ++bl) g = max(g, eexp[et * nblk + bl]);
      sh.gexp[et] = g;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    for (int i = et; i < M * nblk; i += kEpiWarps * 32) {
      const int a = i / nblk;
      const int e = eexp[i];
      cexp[i] = e == INT32_MIN ? __int_as_float(0x7fc00000)
                               : (BITS == 4 ? 0.0625f : 1.0f) * pow2f(max(e - sh.gexp[a], -200));
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kEpiWarps * 32) : "memory");
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&sh.bready);
    ptx::pdl_launch_dependents();

    // (4) read-out: TMEM lane = weight row; per stage slot nb columns. The CTA's stages are
    // walked as one sequence over its units; each row's binary16 scales (8 bytes a stage) are
    // loaded a chunk of four stages ahead, the first chunk before the wait on the preceding
    // grid, so no stage waits on a scale load.
    int slot = 0;
    uint32_t sph = 0;
    const int s0 = splits > 1 ? cs0 : 0, s1 = splits > 1 ? cs1 : num_stages;
    const int spu = s1 - s0;  // stages per unit
    const int my_units = blockIdx.x < num_units ? (num_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int nst = my_units * spu;
    float acc[M];
#pragma unroll
    for (int a = 0; a < M; ++a) acc[a] = 0.f;
    int row = 0;
    for (int f0 = 0; f0 < nst && ok; f0 += kScaleChunk) {
      if (f0 + kScaleChunk < nst) load_scale_chunk(f0 + kScaleChunk, snext);
#pragma unroll
      for (int i = 0; i < kScaleChunk; ++i) {
        const int f = f0 + i;
        if (f >= nst) break;  // warp-uniform
        const int ui = f / spu, st = s0 + f - ui * spu;
        const int tile = (blockIdx.x + ui * gridDim.x) / splits;
        row = tile * kRows + rl;
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.accfull[slot], sph, wait_limit, abort))) {
          record_timeout(abort);
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(slot * 4 * nb);
        // block j's columns start at j * nb: 3 m of them hold its sums (column 3 a + i); the
        // blocks are read in groups of G (all four at once for m <= 2, pairs above, so that
        // the loaded columns fit in registers)
        constexpr int C = M == 1 ? 4 : M == 2 ? 8 : 16;
        constexpr int G = M <= 2 ? kBlocksPerStage : 2;
        const __half2 h01 = *reinterpret_cast<const __half2 *>(&scur[i].x);
        const __half2 h23 = *reinterpret_cast<const __half2 *>(&scur[i].y);
        const float sc[kBlocksPerStage] = {__low2float(h01), __high2float(h01), __low2float(h23),
                                           __high2float(h23)};
#pragma unroll
        for (int j0 = 0; j0 < kBlocksPerStage; j0 += G) {
          uint32_t r[G][C];
#pragma unroll
          for (int g = 0; g < G; ++g) {
            if constexpr (C == 4) ptx::tmem_ld_32x32b_x4(tb + (j0 + g) * nb, r[g]);
            else if constexpr (C == 8) ptx::tmem_ld_32x32b_x8(tb + (j0 + g) * nb, r[g]);
            else ptx::tmem_ld_32x32b_x16(tb + (j0 + g) * nb, r[g]);
          }
#pragma unroll
          for (int g = 0; g < G; ++g) ptx::tmem_ld_wait(r[g]);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const int b = st * kBlocksPerStage + j0 + g;
            if (b < spr) {
#pragma unroll
              for (int a = 0; a < M; ++a) {
                const int c = a * 3;
                const float t = fmaf(static_cast<float>(static_cast<int>(r[g][c + 2])), 6.103515625e-05f,
                                     fmaf(static_cast<float>(static_cast<int>(r[g][c + 1])), 0.0078125f,
                                          static_cast<float>(static_cast<int>(r[g][c]))));
                acc[a] = fmaf(sc[j0 + g] * cexp[a * nblk + (b - blk0)], t, acc[a]);
              }
            }
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.accempty[slot]);
        if (++slot == slots) {
          slot = 0;
          sph ^= 1;
        }
        if (st == s1 - 1) {  // the unit's last stage: its outputs are complete
          if (splits == 1) {
            if (row < N)
#pragma unroll
              for (int a = 0; a < M; ++a) y[static_cast<size_t>(a) * N + row] = ldexpf(acc[a], sh.gexp[a]);
          } else {
#pragma unroll
            for (int a = 0; a < M; ++a) part[a * kRows + rl] = ldexpf(acc[a], sh.gexp[a]);
          }
#pragma unroll
          for (int a = 0; a < M; ++a) acc[a] = 0.f;
        }
      }
#pragma unroll
      for (int i = 0; i < kScaleChunk; ++i) scur[i] = snext[i];
    }
  } else if constexpr (kCvt) {
    // ---- int4 converters: packed rows -> s8 tile (16 q per byte), 128B-swizzled ----
    const int ct = threadIdx.x - kCvtWarp0 * 32;  // 0..127
    int r = 0, a = 0;
    uint32_t rph = 0, aph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
      const int s0 = splits > 1 ? cs0 : 0, s1 = splits > 1 ? cs1 : num_stages;
      for (int st = s0; st < s1; ++st) {
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.rawfull[r], rph, wait_limit, abort) &&
                                         ptx::mbar_wait_bounded(&sh.aempty[a], aph ^ 1, wait_limit, abort))) {
          record_timeout(abort);
          ok = false;
          break;
        }
        const uint8_t *raw = smem + L.raw + r * kRawTile;
        uint8_t *at = smem + L.a + a * kATile;
#pragma unroll
        for (int i = 0; i < kRows * 4 / (kCvtWarps * 32); ++i) {
          const int job = ct + i * kCvtWarps * 32;
          const int row = job >> 2, c = job & 3;  // 16-byte chunk c (one block) of the row
          const uint4 w = *reinterpret_cast<const uint4 *>(raw + row * 64 + c * 16);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          uint32_t o[8];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            o[2 * t] = (ws[t] << 4) & 0xF0F0F0F0u;  // even codes, times 16
            o[2 * t + 1] = ws[t] & 0xF0F0F0F0u;      // odd codes, times 16
          }
          *reinterpret_cast<uint4 *>(at + row * 128 + ((((2 * c) ^ row) & 7) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4 *>(at + row * 128 + ((((2 * c + 1) ^ row) & 7) << 4)) =
              make_uint4(o[4], o[5], o[6], o[7]);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&sh.afull[a]);
          ptx::mbar_arrive(&sh.rawempty[r]);
        }
        if (++r == sraw) {
          r = 0;
          rph ^= 1;
        }
        if (++a == sa) {
          a = 0;
          aph ^= 1;
        }
      }
    }
  }

  // K split across the cluster: sum the staged partials in rank order through distributed
  // shared memory. Every thread of every CTA reaches both cluster barriers (all waits above
  // are bounded), which make the partials visible and keep each CTA's shared memory alive
  // until all reads are done.
  __syncwarp();  // the cluster barrier is warp-aligned: single-lane roles rejoin their warps
  if (splits > 1) {
    ptx::cluster_sync();
    ptx::pdl_wait();  // y may be read by preceding kernels (passed already by the epilogue)
    const int tile = blockIdx.x / splits, rank = blockIdx.x % splits;
    const int per = (kRows + splits - 1) / splits;
    const int r0 = rank * per, r1 = min(kRows, r0 + per);
    const uint32_t pbase = ptx::smem_u32(part);
    for (int i = threadIdx.x; i < (r1 - r0) * M; i += kThreads) {
      const int a = i / (r1 - r0), rl = r0 + i % (r1 - r0);
      const int row = tile * kRows + rl;
      const uint32_t off = static_cast<uint32_t>((a * kRows + rl) * 4);
      float v[8];  // every rank's partial in flight at once, then summed in rank order
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        v[k] = 0.f;
        if (k < splits)
          asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v[k]) : "r"(ptx::mapa_shared(pbase + off, k)));
      }
      float s = v[0];
#pragma unroll
      for (int k = 1; k < 8; ++k)
        if (k < splits) s += v[k];
      if (row < N && !*abort) y[static_cast<size_t>(a) * N + row] = s;
    }
    ptx::cluster_sync();
  }

  // ---- teardown: drain what this CTA issued, then free tensor memory ----
  if (warp == 0 && lane == 0 && *abort) {
    int no_abort = 0;  // only the last issue to each slot can still be in flight
    const int nslot = kCvt ? sraw : sa;
    for (int i = 0; i < nslot; ++i)
      if ((imask >> i) & 1)
        ptx::mbar_wait_bounded(kCvt ? &sh.rawfull[i] : &sh.afull[i], (ipar >> i) & 1, kDrainLimit, &no_abort);
  }
  if (warp == kMmaWarp && lane == 0 && mma_issued) {
    int no_abort = 0;
    ptx::mbar_wait_bounded(&sh.drain, 0, kDrainLimit, &no_abort);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tmem_cols);
  }
}

// B-tile rows (MMA N) for m activation rows: m rows x 3 digits, rounded up to 16.
int b_rows(int m) { return ((3 * m + 15) / 16) * 16; }

constexpr int kSmemMax = 227 * 1024;
// Every CTA asks for at least this much shared memory, so that at most two share an SM and
// their tensor memory (at most 256 columns each) never has to wait for a third CTA's: K-split
// CTAs wait for each other at cluster barriers, so no CTA may block in tcgen05.alloc behind a
// CTA of another cluster.
constexpr int kSmemFloor = 80 * 1024;

template <int BITS, int M>
int launch_i8tc_t(const float *x, const woq_weight &w, float *y, cudaStream_t s, const DevInfo &dev) {
  auto kern = qgemv_i8tc_kernel<BITS, M>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
  });
  if (attr_err != cudaSuccess) return WOQ_ECUDA;

  const int K = static_cast<int>(w.k), N = static_cast<int>(w.n);
  if (K % kStageK != 0) return 1;  // whole stages only (every decoder shape)
  const int nb = b_rows(M);
  const int spr = K / 32;
  const int stages = (K + kStageK - 1) / kStageK;
  const int tiles = (N + kRows - 1) / kRows;
  // Few tiles: split K across a cluster of at most 8 CTAs (the portable size), as many splits
  // as keep the CTAs within the SM count, every split with at least one stage.
  int splits = 1;
  if (tiles < dev.sm_count) {
    splits = std::max(1, std::min({8, stages, dev.sm_count / tiles}));
    while (splits > 1 && (splits - 1) * ((stages + splits - 1) / splits) >= stages) --splits;
  }
  const int kps = (stages + splits - 1) / splits;
  const int cta_stages = splits > 1 ? kps : stages;
  const int blocks = std::min(spr, cta_stages * kBlocksPerStage);
  // Rings: every stage of a unit in flight at once when they fit (decoder projections);
  // tensor-memory slots so that at most 256 columns are held (two CTAs may share an SM).
  // K split: every stage of the CTA's unit in flight at once. Persistent: rings as deep as
  // about 200 KB of shared memory allows (HBM latency times bandwidth is ~10 MB across the
  // SMs): int8 code tiles straight from TMA; int4 four s8 tiles and a deep packed-tile ring.
  const int slots = std::max(1, std::min({kMaxSlots, 256 / (4 * nb), cta_stages}));
  int sa = std::min(kMaxA, cta_stages);
  int sraw = BITS == 4 ? std::min(kMaxRaw, cta_stages) : 0;
  if (splits == 1) {
    const int rest = make_layout(0, 0, cta_stages, nb, blocks, M).total;
    const int budget = 200 * 1024 - rest;
    if (BITS == 8) {
      sa = std::max(2, std::min(kMaxA, budget / kATile));
    } else {
      sa = 4;
      sraw = std::max(2, std::min(kMaxRaw, (budget - sa * kATile) / kRawTile));
    }
  }
  const Layout L = make_layout(sa, sraw, cta_stages, nb, blocks, M);
  if (L.total > kSmemMax) return 1;  // B tiles too large for this K: not taken
  const int smem = std::max(L.total, kSmemFloor);

  CUtensorMap tm;
  const bool ok = BITS == 4
      ? make_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, w.k / 2, w.n, 64, kRows,
                           CU_TENSOR_MAP_SWIZZLE_NONE)
      : make_tensor_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, w.k, w.n, 128, kRows,
                           CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return WOQ_ECUDA;

  const int units = tiles * splits;
  int grid = units;
  if (splits == 1) {
    int nbk = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nbk, kern, kThreads, smem) != cudaSuccess || nbk < 1)
      return WOQ_ECUDA;
    grid = std::min(units, dev.sm_count * std::min(nbk, 2));
  }
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (splits > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(splits);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, kern, tm, x, w.scales, y, N, K, splits, sa, sraw, slots, nb,
                         kWaitLimit) != cudaSuccess)
    return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

template <int BITS>
int launch_i8tc_bits(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                     const DevInfo &dev) {
  switch (m) {
    case 1: return launch_i8tc_t<BITS, 1>(x, w, y, s, dev);
    case 2: return launch_i8tc_t<BITS, 2>(x, w, y, s, dev);
    case 3: return launch_i8tc_t<BITS, 3>(x, w, y, s, dev);
    case 4: return launch_i8tc_t<BITS, 4>(x, w, y, s, dev);
    default: return 1;
  }
}

}  // namespace

int launch_gemv_i8tc(const float *x, int64_t m, const woq_weight &w, float *y, cudaStream_t s,
                     const DevInfo &dev) {
  if (m < 1 || m > kMaxM) return 1;
  return w.bits == 4 ? launch_i8tc_bits<4>(x, m, w, y, s, dev) : launch_i8tc_bits<8>(x, m, w, y, s, dev);
}

int read_i8tc_timeout_flag(int clear, unsigned *value) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_i8tc_timeout_flag, sizeof(v)) != cudaSuccess) return WOQ_ECUDA;
  if (clear && v) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_i8tc_timeout_flag, &z, sizeof(z)) != cudaSuccess) return WOQ_ECUDA;
  }
  *value = v;
  return WOQ_OK;
}

}  // namespace woq
