// qgemv_chain: a decode step's GEMVs as one persistent launch ("TinyMOSS-Diarize", "What we
// learned": the thread granularity has to match the size of the operation; a decoder block's
// projections at one token are each far too small to fill the GPU on their own).
//
// The items run in order, each one computed exactly as qgemv's CUDA-core form computes it
// (exact codes, per-block FP32 sums scaled once by the binary16 scale, FP32 accumulation),
// with an optional fused epilogue (SwiGLU over row-interleaved gate|up rows, or a residual
// add). Item i reads its x only after every CTA has finished item i-1, so an input may be the
// output of an earlier item and the launch keeps the order that separate launches on one
// stream would have.
//
// Design (B200):
//   * One CTA per SM. Every item's rows are divided evenly among the CTAs (in gate/up pairs
//     for the SwiGLU), so each SM does 1/148 of every projection.
//   * The weights never depend on the inputs: one producer lane streams the CTA's rows of
//     every item, in item order, by 1-D bulk copies (codes and scales of consecutive rows are
//     each one contiguous range) into a ring of shared-memory stages. A decoder block is about
//     60 KB per SM, so the whole step's weights are in flight from the first cycle, also
//     before the wait on the preceding grid.
//   * 16 compute warps. When a CTA holds few rows (the K-tall o and down projections), each
//     row's K is split into parts taken by different warps (split-K inside the CTA), and the
//     parts are summed through shared memory in a fixed order: deterministic.
//   * Between items: the CTA's outputs are stored, one thread makes them visible device-wide
//     and adds 1 to the item's counter in the workspace; before the next item one thread
//     waits (bounded) until that counter equals the grid size. The last CTA to finish the
//     last item resets every counter, so each call leaves the workspace zeroed.
#include <cuda_fp16.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "gemv_math.cuh"
#include "ptx.cuh"
#include "woq_internal.h"

namespace woq {

__device__ unsigned int g_chain_timeout_flag = 0;

namespace {

using namespace gemv;

constexpr int kNW = 16;                    // compute warps
constexpr int kThreads = (kNW + 1) * 32;   // + one producer warp
constexpr int kMaxItems = 8;
constexpr int kMaxSlots = 8;
constexpr int kMaxJobs = 256;              // (row, K-part) jobs of one stage
constexpr int kHeader = 512;               // mbarriers, abort flag
constexpr long long kWaitLimit = 1LL << 32;   // cycles (~2 s)
constexpr long long kDrainLimit = 1LL << 31;  // cycles (~1 s)

constexpr int kEpiWrite = 0, kEpiSwiglu = 1, kEpiResidual = 2;

struct Item {
  const uint8_t *packed;
  const uint16_t *scales;
  const float *x;
  float *y;
  const float *r;
  int n, k, bits, epi;
  int parts;       // K-parts per row (split-K inside the CTA)
  int stage_rows;  // rows per ring stage (even for the SwiGLU)
};

struct Params {
  Item it[kMaxItems];
  int count, m, slot_bytes, slots, x_units;  // x_units: float4 per staged x row (max k / 4)
  unsigned *counters;
  long long wait_limit;
  int stuck;  // test hook: wait for one arrival more than the grid has (never comes)
};

struct Shared {
  uint64_t full[kMaxSlots];
  uint64_t empty[kMaxSlots];
  int abort;
};
static_assert(sizeof(Shared) <= kHeader, "header too small");

__device__ __forceinline__ void chain_timeout(volatile int *abort) {
  *abort = 1;
  atomicOr(&g_chain_timeout_flag, 1u);
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// The CTA's rows of item `it` on a grid of G CTAs: [r0, r1).
__device__ __forceinline__ void cta_rows(const Item &it, int c, int G, int &r0, int &r1) {
  const int w = it.epi == kEpiSwiglu ? 2 : 1;
  const long long units = it.n / w;
  r0 = static_cast<int>(units * c / G) * w;
  r1 = static_cast<int>(units * (c + 1) / G) * w;
}

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Dot products of one stage: `nr` rows whose codes start at `codes` and scales at `scs` in
// shared memory, each row split into `parts` ranges of blocks; job j = (row j / parts,
// part j % parts) is one warp's; its lanes take the part's blocks lane, lane + 32, ... and the
// warp's sum over them goes to psum[j][mm].
template <int BITS, int MT>
__device__ __forceinline__ void stage_dots(const float4 *xs4, int units_row, const uint8_t *codes,
                                           const uint16_t *scs, int nr, int k, int parts, int warp,
                                           int lane, float *psum) {
  constexpr int kBlockBytes = BITS == 8 ? 32 : 16;  // int4/int5: a block's (low) nibbles
  const int spr = k >> 5;
  const size_t row_bytes = static_cast<size_t>(k) * BITS / 8;
  for (int job = warp; job < nr * parts; job += kNW) {
    const int rl = job / parts, part = job - (job / parts) * parts;
    const int b0 = part * spr / parts, b1 = (part + 1) * spr / parts;
    float acc[1][MT];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) acc[0][mm] = 0.f;
    const uint8_t *crow = codes + rl * row_bytes;
    const uint16_t *srow = scs + rl * spr;
    for (int b = b0 + lane; b < b1; b += 32) {
      uint4 lo[1], hi[1];
      float sc[1];
      lo[0] = *reinterpret_cast<const uint4 *>(crow + b * kBlockBytes);
      if constexpr (BITS == 8) hi[0] = *reinterpret_cast<const uint4 *>(crow + b * kBlockBytes + 16);
      sc[0] = half_bits_to_float(srow[b]);
      if constexpr (BITS == 4) {
        chunk_int4<MT, 1>(xs4, units_row, b, lo, sc, acc);
      } else if constexpr (BITS == 5) {  // the block's high-bit word follows the row's nibbles
        const uint32_t hw[1] = {*reinterpret_cast<const uint32_t *>(crow + spr * 16 + b * 4)};
        chunk_int5<MT, 1>(xs4, units_row, b, lo, hw, sc, acc);
      } else {
        block_int8<MT, 1>(xs4, units_row, b, lo, hi, sc, acc);
      }
    }
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) {
      float v = acc[0][mm];
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (lane == 0) psum[job * MT + mm] = v;
    }
  }
}

// At m <= 2 two CTAs fit on an SM (registers capped for it), so the next launch's CTAs can
// start streaming their weights while this launch computes.
template <int MT>
__global__ void __launch_bounds__(kThreads, MT <= 2 ? 2 : 1)
    qgemv_chain_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(128) uint8_t smem[];
  Shared &sh = *reinterpret_cast<Shared *>(smem);
  volatile int *abort = &sh.abort;
  float4 *xs4 = reinterpret_cast<float4 *>(smem + kHeader);
  const int x_bytes = MT * P.x_units * 16;
  float *psum = reinterpret_cast<float *>(smem + kHeader + x_bytes);
  uint8_t *ring = smem + kHeader + x_bytes + kMaxJobs * MT * 4;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x, c = blockIdx.x;

  if (tid == 0) {
    for (int s = 0; s < P.slots; ++s) {
      ptx::mbar_init(&sh.full[s], 1);
      ptx::mbar_init(&sh.empty[s], 1);
    }
    sh.abort = 0;
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == kNW) {
    // ---- producer: weights only, so no wait on the preceding grid ----
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int p = 0; p < P.count && ok; ++p) {
        const Item &it = P.it[p];
        int r0, r1;
        cta_rows(it, c, G, r0, r1);
        const uint32_t rbytes = static_cast<uint32_t>(it.k) * it.bits / 8, sbytes = it.k / 16;
        for (int cr = r0; cr < r1; cr += it.stage_rows) {
          const int nr = min(it.stage_rows, r1 - cr);
          if (!ptx::mbar_wait_bounded(&sh.empty[s], ph ^ 1, P.wait_limit, abort)) {
            chain_timeout(abort);
            ok = false;
            break;
          }
          uint8_t *dst = ring + static_cast<size_t>(s) * P.slot_bytes;
          ptx::mbar_arrive_expect_tx(&sh.full[s], nr * (rbytes + sbytes));
          ptx::bulk_load(dst, it.packed + static_cast<size_t>(cr) * rbytes, nr * rbytes, &sh.full[s]);
          ptx::bulk_load(dst + nr * rbytes, reinterpret_cast<const uint8_t *>(it.scales) +
                                                static_cast<size_t>(cr) * sbytes,
                         nr * sbytes, &sh.full[s]);
          ++issued;
          if (++s == P.slots) {
            s = 0;
            ph ^= 1;
          }
        }
      }
      // Before this lane leaves, every copy it issued has landed, whatever the compute warps
      // did (after an abort they may skip stages): only the last issue to each slot can still
      // be in flight, since a slot is reissued only after its previous copy was consumed.
      int no_abort = 0;
      for (int i = issued - 1; i >= 0 && i >= issued - P.slots; --i)
        ptx::mbar_wait_bounded(&sh.full[i % P.slots], (i / P.slots) & 1, kDrainLimit, &no_abort);
    }
    return;
  }

  // ---- compute warps ----
  int s = 0;
  uint32_t ph = 0;
  for (int p = 0; p < P.count; ++p) {
    const Item &it = P.it[p];
    // (1) the inputs of item p: the preceding grid (item 0), else every CTA's item p - 1
    if (p == 0) {
      ptx::pdl_wait();
    } else if (tid == 0) {
      const long long t0 = clock64();
      const unsigned target = static_cast<unsigned>(G) + (P.stuck ? 1u : 0u);
      while (ld_acquire_gpu(P.counters + p - 1) < target) {
        if (*abort || clock64() - t0 > P.wait_limit) {
          chain_timeout(abort);
          break;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");
    if (*abort) break;
    // (2) stage x rows [0, m) of the item (read at L2: an earlier item may have written them)
    const int k = it.k, units_row = k >> 2, groups = k >> 3;
    for (int idx = tid; idx < MT * groups; idx += kNW * 32) {
      const int mm = idx / groups, g = idx - (idx / groups) * groups;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
      if (mm < P.m) {
        const float4 *src = reinterpret_cast<const float4 *>(it.x + static_cast<size_t>(mm) * k) + 2 * g;
        a = __ldcg(src);
        b = __ldcg(src + 1);
      }
      float4 pa = a, pb = b;
      if (it.bits != 8) {  // int4/int5 pairs (q_j, q_{4+j}) meet (x_j, x_{4+j})
        pa = make_float4(a.x, b.x, a.y, b.y);
        pb = make_float4(a.z, b.z, a.w, b.w);
      }
      float4 *row = xs4 + mm * units_row;
      row[swz(2 * g)] = pa;
      row[swz(2 * g + 1)] = pb;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");
    if (p == 0) ptx::pdl_launch_dependents();
    // (3) the CTA's rows, stage by stage
    int r0, r1;
    cta_rows(it, c, G, r0, r1);
    const uint32_t rbytes = static_cast<uint32_t>(k) * it.bits / 8;
    bool ok = true;
    for (int cr = r0; cr < r1; cr += it.stage_rows) {
      const int nr = min(it.stage_rows, r1 - cr);
      if (!__all_sync(0xffffffffu, ptx::mbar_wait_bounded(&sh.full[s], ph, P.wait_limit, abort))) {
        chain_timeout(abort);
        ok = false;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");  // every warp's outcome
      if (!ok || *abort) {
        ok = false;
        break;
      }
      const uint8_t *stage = ring + static_cast<size_t>(s) * P.slot_bytes;
      const uint16_t *scs = reinterpret_cast<const uint16_t *>(stage + nr * rbytes);
      if (it.bits == 4)
        stage_dots<4, MT>(xs4, units_row, stage, scs, nr, k, it.parts, warp, lane, psum);
      else if (it.bits == 5)
        stage_dots<5, MT>(xs4, units_row, stage, scs, nr, k, it.parts, warp, lane, psum);
      else
        stage_dots<8, MT>(xs4, units_row, stage, scs, nr, k, it.parts, warp, lane, psum);
      asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");
      if (tid == 0) ptx::mbar_arrive(&sh.empty[s]);  // the stage's codes are read
      if (++s == P.slots) {
        s = 0;
        ph ^= 1;
      }
      // epilogue: one thread per (output, activation row), K-parts summed in order
      const int outs = it.epi == kEpiSwiglu ? nr / 2 : nr;
      for (int i = tid; i < outs * P.m; i += kNW * 32) {
        const int o = i / P.m, mm = i - (i / P.m) * P.m;
        if (it.epi == kEpiSwiglu) {
          float g = 0.f, u = 0.f;
          for (int q = 0; q < it.parts; ++q) {
            g += psum[((2 * o) * it.parts + q) * MT + mm];
            u += psum[((2 * o + 1) * it.parts + q) * MT + mm];
          }
          it.y[static_cast<size_t>(mm) * (it.n / 2) + (cr / 2 + o)] = silu(g) * u;
        } else {
          float v = 0.f;
          for (int q = 0; q < it.parts; ++q) v += psum[(o * it.parts + q) * MT + mm];
          const size_t at = static_cast<size_t>(mm) * it.n + cr + o;
          if (it.epi == kEpiResidual) v += __ldcg(it.r + at);
          it.y[at] = v;
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kNW * 32) : "memory");  // psum is reused
    }
    if (!ok) break;
    // (4) item done on this CTA: outputs visible device-wide, then count the arrival; the last
    // CTA to finish the last item resets every counter for the next call
    if (tid == 0) {
      __threadfence();
      const unsigned old = atomicAdd(P.counters + p, 1u);
      if (p == P.count - 1 && old == static_cast<unsigned>(G) - 1u) {
        for (int q = 0; q < P.count; ++q) P.counters[q] = 0u;
        __threadfence();
      }
    }
  }
}

// Shared memory per CTA: at m <= 2 two CTAs (this launch's and the next's) share an SM; above
// that one CTA per SM may use most of it (the staged x rows grow with m).
constexpr int smem_budget(int mt) { return mt <= 2 ? 110 * 1024 : 200 * 1024; }

template <int MT>
int launch_chain_t(Params &P, const int (&rows)[kMaxItems], cudaStream_t s, const DevInfo &dev) {
  auto kern = qgemv_chain_kernel<MT>;
  constexpr int kBudget = smem_budget(MT);
  const int x_bytes = MT * P.x_units * 16;
  const int fixed = kHeader + x_bytes + kMaxJobs * MT * 4;
  // Stages: as many rows as fit a quarter of the space left (at most 32 KB), so that the ring
  // holds at least four of the largest stage; an item's rows on a CTA are usually one stage.
  const int room = kBudget - fixed;
  const int cap = std::min(32 * 1024, room / 4);
  int slot = 0;
  for (int p = 0; p < P.count; ++p) {
    Item &it = P.it[p];
    const int w = it.epi == kEpiSwiglu ? 2 : 1;
    const int rb = it.k * it.bits / 8 + it.k / 16;
    int sr = std::max(1, std::min({rows[p], cap / rb, kMaxJobs / it.parts}));
    if (w == 2) sr = std::max(2, sr & ~1);
    it.stage_rows = sr;
    slot = std::max(slot, sr * rb);
  }
  slot = (slot + 127) & ~127;
  const int slots = std::min(kMaxSlots, room / slot);
  if (slots < 2) return WOQ_ESHAPE;
  P.slot_bytes = slot;
  P.slots = slots;
  const int smem = fixed + slots * slot;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kBudget);
  });
  if (attr_err != cudaSuccess) return WOQ_ECUDA;
  int nb = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, smem) != cudaSuccess || nb < 1)
    return WOQ_ECUDA;
  // Every CTA waits for every other between items, so the grid must be resident at once:
  // one CTA per SM (at least one fits on each, by the occupancy query above).
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(dev.sm_count), 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, P) != cudaSuccess) return WOQ_ECUDA;
  count_launches(1);
  return WOQ_OK;
}

}  // namespace

int launch_gemv_chain(const woq_chain_item *items, int count, int64_t m, unsigned *counters,
                      cudaStream_t s, const DevInfo &dev) {
  Params P;
  std::memset(&P, 0, sizeof(P));
  P.count = count;
  P.m = static_cast<int>(m);
  P.counters = counters;
  const long long hook = wait_limit_cycles();
  P.wait_limit = hook > 0 ? hook : hook < 0 ? -hook : kWaitLimit;
  P.stuck = hook < 0;
  const int G = dev.sm_count;
  const int mt = m == 1 ? 1 : m == 2 ? 2 : m <= 4 ? 4 : 8;
  int kmax = 0;
  int rows[kMaxItems] = {};
  for (int p = 0; p < count; ++p) {
    const woq_chain_item &ci = items[p];
    Item &it = P.it[p];
    it.packed = ci.w->packed;
    it.scales = ci.w->scales;
    it.x = ci.x;
    it.y = ci.y;
    it.r = ci.r;
    it.n = static_cast<int>(ci.w->n);
    it.k = static_cast<int>(ci.w->k);
    it.bits = ci.w->bits;
    it.epi = ci.epilogue == WOQ_EPI_SWIGLU ? kEpiSwiglu : ci.epilogue == WOQ_EPI_RESIDUAL ? kEpiResidual : kEpiWrite;
    kmax = std::max(kmax, it.k);
    const int w = it.epi == kEpiSwiglu ? 2 : 1;
    rows[p] = static_cast<int>(((it.n / w) + G - 1) / G) * w;  // most rows a CTA gets
    // split-K inside the CTA while rows leave warps idle, each part at least 32 blocks
    it.parts = std::max(1, std::min(kNW / std::max(rows[p], 1), it.k / 32 / 32));
  }
  P.x_units = kmax / 4;
  switch (mt) {
    case 1: return launch_chain_t<1>(P, rows, s, dev);
    case 2: return launch_chain_t<2>(P, rows, s, dev);
    case 4: return launch_chain_t<4>(P, rows, s, dev);
    default: return launch_chain_t<8>(P, rows, s, dev);
  }
}

int read_chain_timeout_flag(int clear, unsigned *value) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_chain_timeout_flag, sizeof(v)) != cudaSuccess) return WOQ_ECUDA;
  if (clear && v) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_chain_timeout_flag, &z, sizeof(z)) != cudaSuccess) return WOQ_ECUDA;
  }
  *value = v;
  return WOQ_OK;
}

}  // namespace woq
