// tcgen05 qgemm (prefill): Y[m, n] = bf16(X) . bf16(W_hat)^T with FP32 accumulation in
// tensor memory. "TinyMOSS-Diarize", "How we built it": the prefill GEMM unpacks each
// weight group once into an on-chip tile and reuses it across all activation rows; here
// each weight tile is dequantised once into shared memory per (output tile, K-stage) and
// read by the tensor core for all 128 rows of the M-tile.
//
// Persistent, warp-specialised kernel; one CTA per SM walks (128 * MH) x BN output tiles.
//   warp 0        weight producer: bulk tensor copies (TMA, no multicast) of the raw code
//                 tiles into a deep ring (up to 8 stages, freed by the dequantisers), and of
//                 each output tile's [BN, K/32] scale tile into a double buffer
//   warp 1        TMEM owner; one thread issues tcgen05.mma (K=16, bf16 x bf16 -> f32) into
//                 one of two accumulator sets and commits completions: M=128 activation rows x
//                 N=BN for MH = 1; for MH = 2 the operands swap, M=128 weight rows x N=256
//                 activation rows
//   warp 2        X producer: TMA copies of the bf16 X tile (128B-swizzled, 128 * MH rows)
//                 into a ring of up to 4 stages, freed by the MMA commits
//   warps 3..18   dequantisers: raw codes + binary16 scales -> bf16(scale * code) written
//                 into a short ring of B tiles in the 128B-swizzled K-major layout that the
//                 MMA's shared-memory descriptor names; with MH = 2 each weight tile meets 256
//                 activation rows, so the dequantisation per FLOP is halved
//   warps 19..22  epilogue: tcgen05.ld of the finished accumulators -> FP32 Y, while the MMA
//                 thread already fills the other set with the next tile
// Raw codes and X tiles travel in separate rings so that each is freed by its own reader:
// a shared load slot could only be reused once the MMAs had read its X tile, which held
// the raw codes (and with them the dequantisers) to the MMAs' pace.
// Every mbarrier wait is bounded. A wait that gives up records the event in a device flag
// and stops the CTA's other roles; the CTA drains the copies and MMAs it issued, frees
// tensor memory and returns.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_wait_timeout_flag = 0;

namespace {

constexpr int BM = 128;
constexpr int BK = 64;              // bf16 elements per stage = one 128-byte swizzle row
// Three rings, each freed by its own consumer: raw code tiles (read by the dequantisers),
// X tiles (read by the MMAs) and dequantised weight tiles (written by the dequantisers, read
// by the MMAs). Raw codes are small, so their ring is deep and the dequantisers never wait
// for the MMAs to free a load slot.
constexpr int kMaxSW = 8;  // raw code stages
constexpr int kMaxSX = 4;  // X stages
constexpr int kMaxSB = 3;  // dequantised weight tiles
// Weight-tile ring depth: the dequantisers run up to this many K-steps ahead of the MMAs.
__host__ __device__ constexpr int sb_for(int bn, bool split = false) {
  return split || bn == 128 ? 3 : 2;
}
constexpr int kTmaScaleCols = 128;  // scale tile copied by TMA when K/32 <= this (and % 8 == 0)
constexpr int kDequantWarps = 16;  // four per scheduler: each warp's chain is latency-bound
constexpr int kDequantThreads = kDequantWarps * 32;
constexpr int kEpiWarps = 4;
// warp 0: raw-code and scale producer; 1: MMA issuer; 2: X producer; then the dequantisers,
// then the epilogue warps
constexpr int kDequantWarp0 = 3;
constexpr int kEpiWarp0 = kDequantWarp0 + kDequantWarps;
constexpr int kThreads = (kEpiWarp0 + kEpiWarps) * 32;  // 736
constexpr long long kDrainLimit = 1LL << 31;                    // cycles (~1 s)
constexpr long long kDefaultWaitLimit = 1LL << 32;              // cycles (~2 s)
constexpr int kSmemMax = 227 * 1024;
// The single-lane roles (producer, MMA issuer) and the epilogue wait with a suspend hint:
// back-to-back polling by them takes issue slots from the dequantising warps that share
// their schedulers.
constexpr uint32_t kRoleSleepNs = 200;

// Instruction descriptor: D f32, A/B bf16, both K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t idesc_for(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(BM >> 4) << 24);
}

long long g_wait_limit_cycles = 0;  // test hook: > 0 wait limit, < 0 inject a stuck wait

struct Shared {
  uint64_t wfull[kMaxSW];   // raw code tile landed (TMA bytes)
  uint64_t wempty[kMaxSW];  // raw code tile read (one arrival per dequant warp)
  uint64_t xfull[kMaxSX];   // X tile landed (TMA bytes; split form: one arrival per epilogue warp)
  uint64_t xempty[kMaxSX];  // X tile read by the MMAs (commit)
  uint64_t bfull[kMaxSB];   // B tile written (one arrival per dequant warp)
  uint64_t bempty[kMaxSB];  // B tile read by the MMAs (commit)
  uint64_t sfull[2];        // scale tile landed (TMA bytes)
  uint64_t sempty[2];       // scale tile done with (one arrival per dequant warp)
  uint64_t accfull[2];      // accumulator complete (commit)
  uint64_t accempty[2];     // accumulator drained (one arrival per epilogue warp)
  uint64_t never;           // nothing arrives here: target of the injected stuck wait
  uint64_t drain;           // MMA completion on abort
  uint32_t tmem_base;
  int abort;
};

// Shared-memory layout for given ring depths and scale-tile size.
struct Layout {
  int a, b, raw, sc, bar, total;
};
__host__ __device__ inline Layout make_layout(int bits, int bn, int x_stage, int b_slot, int sb,
                                              int sx, int sw, int sc_bytes, int sc_bufs) {
  Layout L;
  const int raw_bytes = bn * BK * bits / 8;
  L.a = 0;
  L.b = L.a + sx * x_stage;
  L.raw = L.b + sb * b_slot;
  L.sc = L.raw + sw * raw_bytes;
  L.bar = (L.sc + sc_bufs * sc_bytes + 127) & ~127;
  L.total = L.bar + static_cast<int>(sizeof(Shared)) + 1024;  // + base alignment slack
  return L;
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFF) | (1ull << 16) | (64ull << 32) |
         (1ull << 46) | (2ull << 61);
}

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

// Split forms for the FP32-accurate tensor-core path: the exact FP32 value v = s*q as
// bf16 hi = RNE(v) plus bf16 lo = RNE(v - hi). For int4, v has at most 15 significant bits,
// so hi + lo == v exactly; for int8 the remainder below lo is under 2^-16 of |v|.
__device__ __forceinline__ void split_pack(float a, float b, uint32_t &hi, uint32_t &lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t *>(&h);
  lo = *reinterpret_cast<const uint32_t *>(&l);
}

__device__ __forceinline__ void dequant_int4_word_split(uint32_t w, const float (&sj)[4], uint4 &hi,
                                                        uint4 &lo) {
  const uint32_t hw = w >> 16;
  float2 v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t mask = 0xFu << (4 * j);
    const uint32_t magic = 0x4B000000u | (0x8u << (4 * j));
    const float bias = 8388608.0f + 8.0f * static_cast<float>(1u << (4 * j));
    v[j] = __fadd2_rn(make_float2(__uint_as_float((w & mask) ^ magic), __uint_as_float((hw & mask) ^ magic)),
                      make_float2(-bias, -bias));
    v[j] = __fmul2_rn(v[j], make_float2(sj[j], sj[j]));
  }
  split_pack(v[0].x, v[1].x, hi.x, lo.x);
  split_pack(v[2].x, v[3].x, hi.y, lo.y);
  split_pack(v[0].y, v[1].y, hi.z, lo.z);
  split_pack(v[2].y, v[3].y, hi.w, lo.w);
}

__device__ __forceinline__ void dequant_int8_words_split(uint32_t w0, uint32_t w1, float s, uint4 &hi,
                                                         uint4 &lo) {
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
  uint32_t *h = reinterpret_cast<uint32_t *>(&hi), *l = reinterpret_cast<uint32_t *>(&lo);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 v = __fadd2_rn(p[i], make_float2(-bias, -bias));
    v = __fmul2_rn(v, make_float2(s, s));
    split_pack(v.x, v.y, h[i], l[i]);
  }
}

template <int BITS, int BN, int MH, bool SPLIT = false>
__global__ void __launch_bounds__(kThreads, 1)
    qgemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                    const __grid_constant__ CUtensorMap tm_s, const uint16_t *__restrict__ scales,
                    float *__restrict__ Y, int M, int N, int K, int sx_stages, int sw_stages,
                    int sc_bytes, int sc_bufs, int splits, float *__restrict__ partials,
                    const float *__restrict__ Xf, long long wait_limit, long long stuck_wait) {
  constexpr int kRawRow = BK * BITS / 8;  // bytes of one row's codes per stage
  constexpr int kRawBytes = BN * kRawRow;
  // SPLIT (FP32-accurate form): each X tile holds 64 activation rows as bf16 hi then bf16 lo
  // (128 rows), each weight slot holds the bf16 hi and lo tiles of the dequantised weights,
  // and per K-step two M=128, N=128 MMAs (A = weight hi, then weight lo; B = the X tile)
  // accumulate all four products; the epilogue adds the hi and lo column halves. The
  // epilogue warps, idle during the main loop, also write the X tiles from FP32 X (no
  // pre-pass), and the K-splits of one output tile run as one thread-block cluster that sums
  // its partials through distributed shared memory (no workspace, no reduction launch).
  // One work unit per CTA: the host launches one CTA per unit.
  static_assert(!SPLIT || (MH == 1 && BN == BM), "the split form uses 128-row weight tiles");
  constexpr bool kSwap = MH == 2 || SPLIT;       // A = weight tile, B = X tile
  constexpr int kBBytes1 = BN * BK * 2;          // one dequantised weight tile
  constexpr int kBBytes = (SPLIT ? 2 : 1) * kBBytes1;  // one weight ring slot
  constexpr int kSB = sb_for(BN, SPLIT);         // weight-tile ring depth
  constexpr int TM = SPLIT ? 64 : BM * MH;       // output rows (activation rows) per tile
  constexpr int kXRows = SPLIT ? 128 : TM;       // X tile rows per stage
  constexpr int kAStage = kXRows * BK * 2;       // X bytes per load stage
  // MH = 1: the MMA's A is the X tile and B the weight tile; the accumulator holds
  // [128 activation rows x BN]. MH = 2: the roles swap, A = the 128-row weight tile and
  // B = the 256-row X tile, so one M=128, N=256 MMA per K-step covers the whole tile (long
  // MMAs keep the tensor pipe fed between stages); the accumulator holds [BN = 128 weight
  // rows x 256 activation rows].
  static_assert(MH == 1 || BN == BM, "swapped tiles need 128 weight rows");
  constexpr int kAccCols = kSwap ? kXRows : BN;  // accumulator columns per set (= MMA N)
  constexpr uint32_t kTmemCols = 2 * kAccCols;   // two accumulator sets
  static_assert(kTmemCols <= 512, "accumulators exceed tensor memory");
  constexpr uint32_t kIdesc = idesc_for(kAccCols);
  constexpr uint32_t kIdescLo = idesc_for(SPLIT ? TM : kAccCols);  // split form: x hi rows only
  const Layout L = make_layout(BITS, BN, kAStage, kBBytes, kSB, sx_stages, sw_stages, sc_bytes, sc_bufs);
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  Shared &sh = *reinterpret_cast<Shared *>(smem + L.bar);
  volatile int *abort = &sh.abort;
  const bool sc_tma = sc_bytes > 0;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int num_k = (K + BK - 1) / BK;
  const int num_m = (M + TM - 1) / TM;
  // Work unit u covers output tile u / splits and K-stages [ks0, ks1) of split u % splits.
  const int num_units = num_m * ((N + BN - 1) / BN) * splits;
  const int kps = (num_k + splits - 1) / splits;
  const int SX = sx_stages, SW = sw_stages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SW; ++s) {
      ptx::mbar_init(&sh.wfull[s], 1);
      ptx::mbar_init(&sh.wempty[s], kDequantWarps);
    }
    for (int s = 0; s < SX; ++s) {
      ptx::mbar_init(&sh.xfull[s], SPLIT ? kEpiWarps : 1);
      ptx::mbar_init(&sh.xempty[s], 1);
    }
    for (int s = 0; s < kSB; ++s) {
      ptx::mbar_init(&sh.bfull[s], kDequantWarps);
      ptx::mbar_init(&sh.bempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(&sh.sfull[s], 1);
      ptx::mbar_init(&sh.sempty[s], kDequantWarps);
      ptx::mbar_init(&sh.accfull[s], 1);
      ptx::mbar_init(&sh.accempty[s], kEpiWarps);
    }
    ptx::mbar_init(&sh.never, 1);
    ptx::mbar_init(&sh.drain, 1);
    sh.abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    if (!SPLIT) ptx::prefetch_tmap(&tm_x);
    ptx::prefetch_tmap(&tm_w);
    if (sc_tma) ptx::prefetch_tmap(&tm_s);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&sh.tmem_base, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // producer bookkeeping for the drain: slots issued at least once, and the parity of
  // their last issue
  uint32_t wmask = 0, wpar = 0, smask = 0, spar = 0, xmask = 0, xpar = 0;
  bool mma_issued = false;

  if (warp == 0) {
    // ---- raw-code and scale producer (one lane): weights only, no wait on preceding grids.
    // Ring positions advance incrementally (no division on the issue path); a wait with the
    // opposite parity passes at once on a fresh barrier, so the first round needs no case.
    if (lane == 0) {
      int s = 0, sb = 0;
      uint32_t ph = 0, sph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int tile = u / splits, sp = u - (u / splits) * splits;
        const int nb = tile / num_m;
        const int ks0 = sp * kps, ks1 = min(num_k, ks0 + kps);
        if (sc_tma) {
          if (!ptx::mbar_wait_bounded(&sh.sempty[sb], sph ^ 1, wait_limit, abort, kRoleSleepNs)) {
            record_timeout(abort);
            break;
          }
          ptx::mbar_arrive_expect_tx(&sh.sfull[sb], static_cast<uint32_t>(BN * (K >> 5) * 2));
          ptx::tma_load_2d(smem + L.sc + sb * sc_bytes, &tm_s, &sh.sfull[sb], 0, nb * BN);
          smask |= 1u << sb;
          spar = (spar & ~(1u << sb)) | (sph << sb);
          if (++sb == sc_bufs) {
            sb = 0;
            sph ^= 1;
          }
        }
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!ptx::mbar_wait_bounded(&sh.wempty[s], ph ^ 1, wait_limit, abort, kRoleSleepNs)) {
            record_timeout(abort);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&sh.wfull[s], kRawBytes);
          ptx::tma_load_2d(smem + L.raw + s * kRawBytes, &tm_w, &sh.wfull[s], ks * kRawRow, nb * BN);
          wmask |= 1u << s;
          wpar = (wpar & ~(1u << s)) | (ph << s);
          if (++s == SW) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 2) {
    // ---- X producer (one lane; the split form's X tiles are written by the epilogue warps).
    // X is written by preceding kernels: wait for them before the first copy.
    if (!SPLIT && lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      ptx::pdl_wait();
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int tile = u / splits, sp = u - (u / splits) * splits;
        const int mb = tile % num_m;
        const int ks0 = sp * kps, ks1 = min(num_k, ks0 + kps);
        for (int ks = ks0; ks < ks1; ++ks) {
          if (!ptx::mbar_wait_bounded(&sh.xempty[s], ph ^ 1, wait_limit, abort)) {
            record_timeout(abort);
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&sh.xfull[s], kAStage);
          ptx::tma_load_2d(smem + L.a + s * kAStage, &tm_x, &sh.xfull[s], ks * BK, mb * kXRows);
          xmask |= 1u << s;
          xpar = (xpar & ~(1u << s)) | (ph << s);
          if (++s == SX) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (one lane): descriptors advance by constants, no division ----
    if (lane == 0) {
      bool ok = true;
      // Test hook: a wait on a barrier nothing arrives on, which must run out.
      if (stuck_wait > 0 && !ptx::mbar_wait_bounded(&sh.never, 0, stuck_wait, abort)) {
        record_timeout(abort);
        ok = false;
      }
      const uint64_t adesc0 = sw128_desc(ptx::smem_u32(smem + L.a));
      const uint64_t bdesc0 = sw128_desc(ptx::smem_u32(smem + L.b));
      int s = 0, bs = 0, ab = 0;
      uint32_t ph = 0, bph = 0, aph = 0;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        const int ks0 = (u - (u / splits) * splits) * kps, ks1 = min(num_k, ks0 + kps);
        if (!ptx::mbar_wait_bounded(&sh.accempty[ab], aph ^ 1, wait_limit, abort, kRoleSleepNs)) {
          record_timeout(abort);
          break;
        }
        ptx::tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(ab * kAccCols);
        for (int ks = ks0; ks < ks1; ++ks) {
          ok = ptx::mbar_wait_bounded(&sh.bfull[bs], bph, wait_limit, abort) &&
               ptx::mbar_wait_bounded(&sh.xfull[s], ph, wait_limit, abort);
          if (!ok) {
            record_timeout(abort);
            break;
          }
          ptx::tc_fence_after();
          // start-address field counts 16-byte units; K=16 bf16 = 32 bytes = 2 units; in the
          // split form the lo half of the weight tile starts kBBytes1 further on
          const uint64_t ad = adesc0 + static_cast<uint64_t>(s * (kAStage >> 4));
          const uint64_t bd = bdesc0 + static_cast<uint64_t>(bs * (kBBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc = (ks != ks0 || kk != 0) ? 1u : 0u;
            if constexpr (SPLIT) {
              // weight hi against x hi and x lo (N = 128); weight lo against x hi only
              // (N = 64, the first 64 X tile rows): the dropped lo x lo product is below
              // 2^-16 of each term.
              ptx::tc_mma_f16(d, bd + 2 * kk, ad + 2 * kk, kIdesc, acc);
              ptx::tc_mma_f16(d, bd + (kBBytes1 >> 4) + 2 * kk, ad + 2 * kk, kIdescLo, 1u);
            } else if constexpr (MH == 2) {
              ptx::tc_mma_f16(d, bd + 2 * kk, ad + 2 * kk, kIdesc, acc);
            } else {
              ptx::tc_mma_f16(d, ad + 2 * kk, bd + 2 * kk, kIdesc, acc);
            }
          }
          mma_issued = true;
          ptx::tc_commit(&sh.xempty[s]);
          ptx::tc_commit(&sh.bempty[bs]);
          if (++s == SX) {
            s = 0;
            ph ^= 1;
          }
          if (++bs == kSB) {
            bs = 0;
            bph ^= 1;
          }
        }
        if (!ok) break;
        ptx::tc_commit(&sh.accfull[ab]);
        if (++ab == 2) {
          ab = 0;
          aph ^= 1;
        }
      }
      ptx::tc_commit(&sh.drain);  // arrives once every MMA issued above has completed
    }
  } else if (warp < kEpiWarp0) {
    // ---- dequantisers: 512 threads, one job of E codes per stage each: part t % P of row
    //      t / P, P = 64 / E parts per row (E = 32 at BN = 256, 16 at BN = 128). A warp's lanes
    //      cover 32 / P whole rows, so their raw-code loads are one contiguous range and their
    //      swizzled B stores hit distinct bank groups ----
    constexpr int E = BN * BK / kDequantThreads;  // codes per job
    constexpr int CH = E / 8;                     // 16-byte B chunks per job
    constexpr int P = BK / E;                     // jobs per row
    const int t = threadIdx.x - kDequantWarp0 * 32;
    const int row = t / P, part = t % P;
    const int spr = K >> 5;
    const int sw = row & 7;
    const int kbo = (part * E) >> 5;  // which 32-code block of the stage
    int s = 0, bs = 0, sb = 0;
    uint32_t ph = 0, bph = 0, sph = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
      const int tile = u / splits;
      const int ks0 = (u - tile * splits) * kps, ks1 = min(num_k, ks0 + kps);
      const int nb = tile / num_m;
      const int gr = nb * BN + row;
      // Wait outcomes are made warp-uniform: warp-collective steps follow.
      if (sc_tma && !__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.sfull[sb], sph, wait_limit, abort))) {
        record_timeout(abort);
        ok = false;
        break;
      }
      const uint16_t *sct = reinterpret_cast<const uint16_t *>(smem + L.sc + sb * sc_bytes);
      for (int ks = ks0; ks < ks1; ++ks) {
        const int kb = 2 * ks + kbo;
        float s0 = 0.f;
        if (!sc_tma && gr < N && kb < spr)  // fallback: this thread's own scale from global
          s0 = __half2float(__ushort_as_half(__ldg(scales + static_cast<size_t>(gr) * spr + kb)));
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.wfull[s], ph, wait_limit, abort) &&
                                         ptx::mbar_wait_bounded(&sh.bempty[bs], bph ^ 1, wait_limit, abort))) {
          record_timeout(abort);
          ok = false;
          break;
        }
        if (sc_tma) s0 = __half2float(__ushort_as_half(sct[row * spr + kb]));
        const uint8_t *raw = smem + L.raw + s * kRawBytes + row * kRawRow + part * (E * BITS / 8);
        uint8_t *brow = smem + L.b + bs * kBBytes + row * 128;
        if constexpr (BITS == 4) {
          uint32_t ws[CH];  // one word = 8 codes = one 16-byte chunk of bf16
          if constexpr (CH == 4) {
            const uint4 v = *reinterpret_cast<const uint4 *>(raw);
            ws[0] = v.x; ws[1] = v.y; ws[2] = v.z; ws[3] = v.w;
          } else {
            const uint2 v = *reinterpret_cast<const uint2 *>(raw);
            ws[0] = v.x; ws[1] = v.y;
          }
          const float sj[4] = {s0, s0 * 0.0625f, s0 * 0.00390625f, s0 * 0.000244140625f};
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int chunk = part * CH + i;
            if constexpr (SPLIT) {
              uint4 hi, lo;
              dequant_int4_word_split(ws[i], sj, hi, lo);
              *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) = hi;
              *reinterpret_cast<uint4 *>(brow + kBBytes1 + ((chunk ^ sw) << 4)) = lo;
            } else {
              *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) = dequant_int4_word(ws[i], sj);
            }
          }
        } else {
          uint32_t ws[2 * CH];  // two words = 8 codes = one chunk
#pragma unroll
          for (int i = 0; i < CH / 2; ++i) {
            const uint4 v = reinterpret_cast<const uint4 *>(raw)[i];
            ws[4 * i] = v.x; ws[4 * i + 1] = v.y; ws[4 * i + 2] = v.z; ws[4 * i + 3] = v.w;
          }
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const int chunk = part * CH + i;
            if constexpr (SPLIT) {
              uint4 hi, lo;
              dequant_int8_words_split(ws[2 * i], ws[2 * i + 1], s0, hi, lo);
              *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) = hi;
              *reinterpret_cast<uint4 *>(brow + kBBytes1 + ((chunk ^ sw) << 4)) = lo;
            } else {
              *reinterpret_cast<uint4 *>(brow + ((chunk ^ sw) << 4)) =
                  dequant_int8_words(ws[2 * i], ws[2 * i + 1], s0);
            }
          }
        }
        // Each lane makes its writes visible to the async proxy (the tensor core), the warp
        // converges, and one lane arrives for the warp: its B rows are written and its raw
        // codes read.
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&sh.bfull[bs]);
          ptx::mbar_arrive(&sh.wempty[s]);
        }
        if (++s == SW) {
          s = 0;
          ph ^= 1;
        }
        if (++bs == kSB) {
          bs = 0;
          bph ^= 1;
        }
      }
      if (ok && sc_tma) {
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.sempty[sb]);
        if (++sb == sc_bufs) {
          sb = 0;
          sph ^= 1;
        }
      }
    }
  } else if constexpr (SPLIT) {
    // ---- split form, epilogue warps: write the X tiles, then accumulator -> Y ----
    const int q = warp & 3;                                  // TMEM lanes 32q .. 32q+31
    const int et = threadIdx.x - kEpiWarp0 * 32;             // 0 .. 127
    const int u = blockIdx.x;                                // one work unit per CTA
    const int tile = u / splits, sp = u - tile * splits;
    const int mb = tile % num_m, nb = tile / num_m;
    const int ks0 = sp * kps, ks1 = min(num_k, ks0 + kps);
    const int rows = min(TM, M - mb * TM);                   // activation rows of the tile
    const int n0 = nb * BN;
    bool ok = u < num_units;
    ptx::pdl_wait();  // X is written, and Y may be read, by preceding kernels
    // (1) X tiles: 64 FP32 rows -> bf16 hi in tile rows 0..63 and bf16 lo in rows 64..127,
    // in the 128-byte-swizzled order a TMA copy would produce. Columns past K are zero
    // (K % 32 == 0, so an 8-column chunk is wholly inside or outside). Tile rows past the
    // last activation row are left as they are: they only feed accumulator columns that are
    // never read.
    {
      const float *xt = Xf + static_cast<size_t>(mb * TM) * K;
      int s = 0;
      uint32_t ph = 0;
      for (int ks = ks0; ks < ks1 && ok; ++ks) {
        if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.xempty[s], ph ^ 1, wait_limit, abort))) {
          record_timeout(abort);
          ok = false;
          break;
        }
        uint8_t *xs = smem + L.a + s * kAStage;
        // A stage is at most TM * 8 = 512 jobs of 8 values, four per epilogue thread: all of a
        // thread's loads are issued before any is used, so a stage costs one L2 round trip.
        constexpr int kJobsPerThread = TM * 8 / (kEpiWarps * 32);
        float4 va[kJobsPerThread], vb[kJobsPerThread];
#pragma unroll
        for (int i = 0; i < kJobsPerThread; ++i) {
          const int job = et + i * kEpiWarps * 32;
          const int r = job >> 3, c = job & 7;
          const int col = ks * BK + c * 8;
          va[i] = make_float4(0.f, 0.f, 0.f, 0.f);
          vb[i] = va[i];
          if (r < rows && col < K) {
            const float4 *src = reinterpret_cast<const float4 *>(xt + static_cast<size_t>(r) * K + col);
            va[i] = __ldg(src);
            vb[i] = __ldg(src + 1);
          }
        }
#pragma unroll
        for (int i = 0; i < kJobsPerThread; ++i) {
          const int job = et + i * kEpiWarps * 32;
          const int r = job >> 3, c = job & 7;
          if (r < rows) {
            uint4 h, l;
            split_pack(va[i].x, va[i].y, h.x, l.x);
            split_pack(va[i].z, va[i].w, h.y, l.y);
            split_pack(vb[i].x, vb[i].y, h.z, l.z);
            split_pack(vb[i].z, vb[i].w, h.w, l.w);
            const int off = (c ^ (r & 7)) << 4;
            *reinterpret_cast<uint4 *>(xs + r * 128 + off) = h;
            *reinterpret_cast<uint4 *>(xs + (TM + r) * 128 + off) = l;
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&sh.xfull[s]);
        if (++s == SX) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    // (2) Accumulator: TMEM lane = weight row, column t = activation row t's hi part, column
    // 64 + t its lo part; their sum goes to Y (one split) or to this CTA's staged partial
    // [64][BN] in the X ring, now idle (every MMA, the only reader, has completed), which
    // the cluster sums after the roles end.
    if (ok && !__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.accfull[0], 0, wait_limit, abort,
                                                              kRoleSleepNs))) {
      record_timeout(abort);
      ok = false;
    }
    float *stage = reinterpret_cast<float *>(smem + L.a);
    if (ok) {
      ptx::tc_fence_after();
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const int nl = q * 32 + lane;
      for (int c0 = 0; c0 < rows; c0 += 16) {  // warp-uniform trip count
        uint32_t ra[16], rb[16];
        ptx::tmem_ld_32x32b_x16(tb + c0, ra);
        ptx::tmem_ld_32x32b_x16(tb + TM + c0, rb);
        ptx::tmem_ld_wait(ra);
        ptx::tmem_ld_wait(rb);
        if (splits == 1) {
          // for each activation row the warp's lanes store 32 consecutive floats of Y
          float *p = Y + static_cast<size_t>(mb * TM + c0) * N + n0 + nl;
          if (n0 + nl < N) {
#pragma unroll
            for (int j = 0; j < 16; ++j, p += N)
              if (c0 + j < rows) *p = __uint_as_float(ra[j]) + __uint_as_float(rb[j]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < rows) stage[(c0 + j) * BN + nl] = __uint_as_float(ra[j]) + __uint_as_float(rb[j]);
        }
      }
      ptx::tc_fence_before();
    }
  } else {
    // ---- epilogue: TMEM accumulator -> registers -> Y ----
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    const bool vec = (N & 3) == 0;
    bool waited = false;
    int ab = 0;
    uint32_t aph = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
      const int tile = u / splits, sp = u - tile * splits;
      const int mb = tile % num_m, nb = tile / num_m;
      // One split writes Y; several write FP32 partials [split][M][N] for the reduction.
      float *out = splits == 1 ? Y : partials + static_cast<size_t>(sp) * M * N;
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.accfull[ab], aph, wait_limit, abort, kRoleSleepNs))) {
        record_timeout(abort);
        break;
      }
      ptx::tc_fence_after();
      if (!waited) {  // Y may be read by a preceding kernel: write it only after that grid
        ptx::pdl_wait();
        waited = true;
      }
      const int n0 = nb * BN;
      const uint32_t tb = tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * kAccCols;
      // 16-column chunks, software-pipelined: the next chunk's TMEM load is in flight while
      // this one is stored (two register buffers, each waited for before use).
      const int ncols = MH == 2 ? min(TM, M - mb * TM) : BN;
      const int nchunks = (ncols + 15) / 16;
      auto store_chunk = [&](const uint32_t (&r)[16], int c) {
        const int c0 = 16 * c;
        if constexpr (MH == 2) {
          // TMEM lane = weight row n, column = activation row m: for each column the warp's
          // 32 lanes store 32 consecutive floats of one Y row. The row pointer advances by
          // N per column; full chunks skip the row check.
          const int n = n0 + q * 32 + lane;
          const int mrem = M - (mb * TM + c0);
          float *p = out + static_cast<size_t>(mb * TM + c0) * N + n;
          if (n < N) {
            if (mrem >= 16) {
#pragma unroll
              for (int j = 0; j < 16; ++j, p += N) *p = __uint_as_float(r[j]);
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j, p += N)
                if (j < mrem) *p = __uint_as_float(r[j]);
            }
          }
        } else {
          const int grow = mb * TM + q * 32 + lane;
          if (grow < M) {
            float *yr = out + static_cast<size_t>(grow) * N + n0 + c0;
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
      };
      uint32_t ra[16], rb[16];
      ptx::tmem_ld_32x32b_x16(tb, ra);
      ptx::tmem_ld_wait(ra);
      for (int c = 0; c < nchunks; c += 2) {  // trip counts are warp-uniform
        if (c + 1 < nchunks) ptx::tmem_ld_32x32b_x16(tb + 16 * (c + 1), rb);
        store_chunk(ra, c);
        if (c + 1 < nchunks) {
          ptx::tmem_ld_wait(rb);
          if (c + 2 < nchunks) ptx::tmem_ld_32x32b_x16(tb + 16 * (c + 2), ra);
          store_chunk(rb, c + 1);
          if (c + 2 < nchunks) ptx::tmem_ld_wait(ra);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&sh.accempty[ab]);
      if (++ab == 2) {
        ab = 0;
        aph ^= 1;
      }
    }
  }

  if constexpr (SPLIT) {
    // Several K-splits: the cluster's CTAs (rank = split) sum their staged partials through
    // distributed shared memory, every thread of the cluster taking part. The cluster
    // barriers make the staged partials visible before the reads and keep every CTA (and
    // its shared memory) alive until all reads are done. Every thread arrives whatever its
    // role did before, and every role's waits are bounded, so the barriers are reached.
    if (splits > 1) {
      ptx::cluster_sync();
      ptx::pdl_wait();  // Y may be read by preceding kernels (passed already by the epilogue)
      const int u = blockIdx.x;
      const int tile = u / splits, sp = u - tile * splits;
      const int mb = tile % num_m, nb = tile / num_m;
      const int rows = min(TM, M - mb * TM);
      const int per = (rows + splits - 1) / splits;  // activation rows summed by this CTA
      const int j0 = sp * per, j1 = min(rows, j0 + per);
      const uint32_t st = ptx::smem_u32(smem + L.a);
      const bool vec = (N & 3) == 0;
      for (int i = threadIdx.x; i < (j1 - j0) * (BN / 4); i += kThreads) {
        const int j = j0 + i / (BN / 4), c4 = i % (BN / 4);
        const uint32_t off = static_cast<uint32_t>((j * BN + 4 * c4) * 4);
        float4 acc = ptx::ld_shared_cluster_v4(ptx::mapa_shared(st + off, 0));
        for (int r = 1; r < splits; ++r) {
          const float4 v = ptx::ld_shared_cluster_v4(ptx::mapa_shared(st + off, r));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const int n = nb * BN + 4 * c4;
        float *yr = Y + static_cast<size_t>(mb * TM + j) * N + n;
        if (vec && n + 4 <= N) {
          *reinterpret_cast<float4 *>(yr) = acc;
        } else {
          if (n < N) yr[0] = acc.x;
          if (n + 1 < N) yr[1] = acc.y;
          if (n + 2 < N) yr[2] = acc.z;
          if (n + 3 < N) yr[3] = acc.w;
        }
      }
      ptx::cluster_sync();
    }
  }

  ptx::pdl_launch_dependents();

  // ---- teardown: drain what this CTA issued, then free TMEM ----
  if (warp == 0 && lane == 0 && *abort) {
    int no_abort = 0;  // only the last issue to each slot can still be in flight
    for (int i = 0; i < SW; ++i) {
      if ((wmask >> i) & 1)
        ptx::mbar_wait_bounded(&sh.wfull[i], (wpar >> i) & 1, kDrainLimit, &no_abort);
    }
    for (int i = 0; i < sc_bufs; ++i)
      if ((smask >> i) & 1)
        ptx::mbar_wait_bounded(&sh.sfull[i], (spar >> i) & 1, kDrainLimit, &no_abort);
  }
  if (warp == 2 && lane == 0 && *abort) {
    int no_abort = 0;
    for (int i = 0; i < SX; ++i) {
      if ((xmask >> i) & 1)
        ptx::mbar_wait_bounded(&sh.xfull[i], (xpar >> i) & 1, kDrainLimit, &no_abort);
    }
  }
  if (warp == 1 && lane == 0 && mma_issued) {
    int no_abort = 0;
    ptx::mbar_wait_bounded(&sh.drain, 0, kDrainLimit, &no_abort);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
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

// Y = sum over splits of the FP32 partials, in split order (deterministic); 4 per thread.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4 *__restrict__ part,
                                                            float4 *__restrict__ y, size_t n4,
                                                            int splits) {
  ptx::pdl_wait();
  ptx::pdl_launch_dependents();
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float4 a = part[i];
    for (int s = 1; s < splits; ++s) {
      const float4 b = part[static_cast<size_t>(s) * n4 + i];
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    y[i] = a;
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

template <int BITS, int BN, int MH, bool SPLIT = false>
int launch_tc(const float *X, int64_t m, const woq_weight &w, float *Y, void *workspace,
              const GemmPlan &plan, cudaStream_t s, const DevInfo &dev) {
  auto kern = qgemm_tc_kernel<BITS, BN, MH, SPLIT>;
  constexpr int TM = SPLIT ? 64 : BM * MH;      // activation rows per output tile
  constexpr int kXRows = SPLIT ? 128 : TM;      // X workspace rows per output tile
  constexpr int kAStage = kXRows * BK * 2;
  constexpr int kBSlot = (SPLIT ? 2 : 1) * BN * BK * 2;
  constexpr int kSB = sb_for(BN, SPLIT);
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
  });
  if (attr_err != cudaSuccess) return WOQ_ECUDA;

  // The whole scale tile [BN, K/32] of an output tile comes by TMA when its rows are 16-byte
  // multiples and it is small; otherwise each dequantiser loads its own scales. Ring depths:
  // the first (X stages, raw stages) pair below that fits, with two scale buffers (the next
  // tile's scales load during this one) if they fit too. Four X stages cover the X copy
  // latency behind the MMAs; four or more raw stages (4 or 8 KB each) keep the dequantisers
  // ahead of the copy latency.
  const int64_t spr = w.k / 32;
  const bool sc_tma = spr % 8 == 0 && spr <= kTmaScaleCols;
  const int sc_bytes = sc_tma ? static_cast<int>((BN * spr * 2 + 127) & ~int64_t(127)) : 0;
  constexpr int kDepths[][2] = {{4, 8}, {4, 6}, {3, 8}, {3, 6}, {4, 4}, {3, 4}, {2, 8},
                                {2, 6}, {2, 4}, {4, 2}, {3, 2}, {2, 2}};
  int sx = 0, sw = 0, sc_bufs = 1;
  for (const auto &d : kDepths) {
    for (int bufs = sc_tma ? 2 : 1; bufs >= 1 && sx == 0; --bufs) {
      if (make_layout(BITS, BN, kAStage, kBSlot, kSB, d[0], d[1], sc_bytes, bufs).total <= kSmemMax) {
        sx = d[0];
        sw = d[1];
        sc_bufs = bufs;
      }
    }
    if (sx) break;
  }
  if (sx < 2) return WOQ_ESHAPE;
  const int smem = make_layout(BITS, BN, kAStage, kBSlot, kSB, sx, sw, sc_bytes, sc_bufs).total;

  const int64_t num_m = (m + TM - 1) / TM;
  CUtensorMap tm_x, tm_w, tm_s;
  if constexpr (SPLIT) {  // the kernel writes its X tiles itself
    std::memset(&tm_x, 0, sizeof(tm_x));
  } else if (!make_tensor_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, workspace, w.k, m, BK,
                                 kXRows, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return WOQ_ECUDA;
  }
  if (!make_tensor_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, w.packed, w.k * BITS / 8, w.n,
                BK * BITS / 8, BN, CU_TENSOR_MAP_SWIZZLE_NONE))
    return WOQ_ECUDA;
  if (sc_tma) {
    if (!make_tensor_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_UINT16, 2, w.scales, spr, w.n,
                  static_cast<uint32_t>(spr), BN, CU_TENSOR_MAP_SWIZZLE_NONE))
      return WOQ_ECUDA;
  } else {
    std::memset(&tm_s, 0, sizeof(tm_s));
  }

  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const long long lim = g_wait_limit_cycles > 0 ? g_wait_limit_cycles : kDefaultWaitLimit;
  const long long stuck = g_wait_limit_cycles < 0 ? -g_wait_limit_cycles : 0;
  const int64_t units = num_m * ((w.n + BN - 1) / BN) * plan.splits;

  if constexpr (SPLIT) {
    // One CTA per work unit; the K-splits of an output tile form one cluster.
    if (units > INT32_MAX) return WOQ_ESHAPE;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(units), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (plan.splits > 1) {
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = static_cast<unsigned>(plan.splits);
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      cfg.numAttrs = 2;
    }
    if (cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w, tm_s, w.scales, Y, static_cast<int>(m),
                           static_cast<int>(w.n), static_cast<int>(w.k), sx, sw, sc_bytes, sc_bufs,
                           plan.splits, static_cast<float *>(nullptr), X, lim, stuck) != cudaSuccess)
      return WOQ_ECUDA;
    count_launches(1);
    return WOQ_OK;
  }

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
  // 2) the persistent GEMM: one CTA per SM (or per work unit, if fewer).
  float *partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + plan.xb);
  {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(units, dev.sm_count)), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tm_x, tm_w, tm_s, w.scales, Y, static_cast<int>(m),
                           static_cast<int>(w.n), static_cast<int>(w.k), sx, sw, sc_bytes, sc_bufs,
                           plan.splits, partials, static_cast<const float *>(nullptr), lim,
                           stuck) != cudaSuccess)
      return WOQ_ECUDA;
    count_launches(1);
  }
  // 3) several K-splits: sum their partials into Y.
  if (plan.splits > 1) {
    const size_t n4 = static_cast<size_t>(m) * w.n / 4;
    cudaLaunchConfig_t cfg = {};
    size_t blocks = (n4 + 255) / 256;
    if (blocks > static_cast<size_t>(dev.sm_count) * 8) blocks = static_cast<size_t>(dev.sm_count) * 8;
    cfg.gridDim = dim3(static_cast<unsigned>(blocks), 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, reinterpret_cast<const float4 *>(partials),
                           reinterpret_cast<float4 *>(Y), n4, plan.splits) != cudaSuccess)
      return WOQ_ECUDA;
    count_launches(1);
  }
  return WOQ_OK;
}

}  // namespace

// 2-D tensor map over a row-major [rows, cols] array.
bool make_tensor_map_2d(CUtensorMap *m, CUtensorMapDataType type, size_t esize, const void *base,
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


GemmPlan plan_gemm_tc(int64_t m, int64_t n, int64_t k, int sm_count, size_t budget,
                      bool split) {
  auto align = [](size_t b) { return (b + 255) & ~static_cast<size_t>(255); };
  GemmPlan p;
  p.split = split;
  const int64_t num_k = (k + BK - 1) / BK;
  // Work units cover the SMs: split K (at most 8 ways) while the units stay within 1.25x the
  // SM count and every split keeps >= 4 K-stages.
  auto grow_splits = [&](int64_t tiles, auto &&fits) {
    while (p.splits < 8 && sm_count > 0 && tiles * p.splits * 2 <= sm_count + sm_count / 4 &&
           num_k / (p.splits * 2) >= 4 && fits(p.splits * 2))
      p.splits *= 2;
  };
  if (split) {
    // 64-row tiles; the kernel writes its own X tiles and a tile's K-splits (a cluster of at
    // most 8, the portable size) sum their partials on chip: no workspace.
    const int64_t tiles = ((m + 63) / 64) * ((n + 127) / 128);
    grow_splits(tiles, [](int) { return true; });
    return p;
  }
  p.xb = align(static_cast<size_t>(m) * static_cast<size_t>(k) * 2);
  // Past one 128-row M tile, 256 x 128 tiles (two M halves sharing each dequantised weight
  // tile) halve the dequantisation per FLOP. Otherwise 128 x 256 tiles, which do twice the
  // work per MMA instruction, when N allows.
  p.mh = m > 128 ? 2 : 1;
  p.bn = p.mh == 1 && n >= 256 ? 256 : 128;
  const int64_t mt = (m + 128 * p.mh - 1) / (128 * p.mh);
  const int64_t tiles = mt * ((n + p.bn - 1) / p.bn);
  // The splits need FP32 partials in the workspace and a vectorisable Y (n % 4 == 0).
  if (n % 4 == 0)
    grow_splits(tiles, [&](int sp) {
      return p.xb + align(static_cast<size_t>(sp) * m * n * 4) <= budget;
    });
  if (p.splits == 1 && p.bn == 256 && tiles * 2 <= sm_count) p.bn = 128;  // more tiles instead
  p.part = p.splits > 1 ? align(static_cast<size_t>(p.splits) * m * n * 4) : 0;
  p.total = p.xb + p.part;
  return p;
}

int launch_gemm_tc(const float *X, int64_t m, const woq_weight &w, float *Y, void *workspace,
                   const GemmPlan &plan, cudaStream_t s, const DevInfo &dev) {
  if (plan.split)
    return w.bits == 4 ? launch_tc<4, 128, 1, true>(X, m, w, Y, workspace, plan, s, dev)
                       : launch_tc<8, 128, 1, true>(X, m, w, Y, workspace, plan, s, dev);
  if (w.bits == 4) {
    if (plan.mh == 2) return launch_tc<4, 128, 2>(X, m, w, Y, workspace, plan, s, dev);
    return plan.bn == 256 ? launch_tc<4, 256, 1>(X, m, w, Y, workspace, plan, s, dev)
                          : launch_tc<4, 128, 1>(X, m, w, Y, workspace, plan, s, dev);
  }
  if (plan.mh == 2) return launch_tc<8, 128, 2>(X, m, w, Y, workspace, plan, s, dev);
  return plan.bn == 256 ? launch_tc<8, 256, 1>(X, m, w, Y, workspace, plan, s, dev)
                        : launch_tc<8, 128, 1>(X, m, w, Y, workspace, plan, s, dev);
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

long long wait_limit_cycles() { return g_wait_limit_cycles; }

}  // namespace woq
