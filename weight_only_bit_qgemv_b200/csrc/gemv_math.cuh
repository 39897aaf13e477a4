// Exact FP32 arithmetic of the CUDA-core GEMV kernels (qgemv.cu, qgemv_chain.cu): packed
// int4/int5/int8 codes to exact FP32 values, products with staged x rows, one binary16 scale
// per 32-block applied to the block's sum.
//
// int8 and int5 codes become exact FP32 values with one PRMT / LOP3 per element: the field
// (offset to unsigned) is placed in the low mantissa bits of 2^23 and the bias is removed with
// one exact packed subtraction (f32x2); int5 fields at nibble position j of a 16-bit half
// carry a factor 2^(4j) that is removed, exactly, once per block. int4 takes one LOP3 per two
// codes into binary16 pairs (unpack_int4_word_h).
#pragma once

#include <cuda_fp16.h>
#include <cstdint>

namespace woq {
namespace gemv {

// 16-byte unit u of an x row lives at unit swz(u) in shared memory.
__device__ __forceinline__ int swz(int u) { return u ^ ((u >> 3) & 7); }

__device__ __forceinline__ float half_bits_to_float(uint16_t h) {
  return __half2float(__ushort_as_half(h));
}

// One 32-bit word of int8 codes (elements e0..e3 in bytes 0..3) -> (q0, q1), (q2, q3).
__device__ __forceinline__ void unpack_int8_word(uint32_t w, float2 (&p)[2]) {
  const uint32_t u = w ^ 0x80808080u;  // offset binary, q + 128
  const float bias = 8388608.0f + 128.0f;
  const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540));
  const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7541));
  const float f2 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7542));
  const float f3 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7543));
  p[0] = __fadd2_rn(make_float2(f0, f1), make_float2(-bias, -bias));
  p[1] = __fadd2_rn(make_float2(f2, f3), make_float2(-bias, -bias));
}

__device__ __forceinline__ float fold_int4(const float2 (&a)[4]) {
  float2 t = __ffma2_rn(a[1], make_float2(0.0625f, 0.0625f), a[0]);
  t = __ffma2_rn(a[2], make_float2(0.00390625f, 0.00390625f), t);
  t = __ffma2_rn(a[3], make_float2(0.000244140625f, 0.000244140625f), t);
  return t.x + t.y;
}

// Two int4 codes per LOP3: the 4-bit fields at nibble
// positions j and j + 4 of a word, sign bit flipped, land in the low mantissa bits of two
// binary16 values 1024 + (q + 8) * 16^(j % 2) (exact: below 2048, where binary16 steps by 1);
// a mixed-precision add widens each to FP32 and removes the bias exactly. Fewer LOP3s on the
// half-rate ALU pipe, more adds on the FMA pipe, which the unpack otherwise leaves half idle.
__device__ __forceinline__ float half_lo_plus(uint32_t h2, float c) {
  float d;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.f16 %0, l, %2; }" : "=f"(d) : "r"(h2), "f"(c));
  return d;
}
__device__ __forceinline__ float half_hi_plus(uint32_t h2, float c) {
  float d;
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.f16 %0, h, %2; }" : "=f"(d) : "r"(h2), "f"(c));
  return d;
}

// One 32-bit word of int4 codes -> four exact pairs p[j] = (q_j, q_{4+j}) * 16^(j % 2).
__device__ __forceinline__ void unpack_int4_word_h(uint32_t w, float2 (&p)[4]) {
  const uint32_t w8 = w >> 8;
  const uint32_t a0 = (w & 0x000F000Fu) ^ 0x64086408u;   // e0, e4
  const uint32_t a1 = (w & 0x00F000F0u) ^ 0x64806480u;   // e1, e5 (x 16)
  const uint32_t a2 = (w8 & 0x000F000Fu) ^ 0x64086408u;  // e2, e6
  const uint32_t a3 = (w8 & 0x00F000F0u) ^ 0x64806480u;  // e3, e7 (x 16)
  p[0] = make_float2(half_lo_plus(a0, -1032.f), half_hi_plus(a0, -1032.f));
  p[1] = make_float2(half_lo_plus(a1, -1152.f), half_hi_plus(a1, -1152.f));
  p[2] = make_float2(half_lo_plus(a2, -1032.f), half_hi_plus(a2, -1032.f));
  p[3] = make_float2(half_lo_plus(a3, -1152.f), half_hi_plus(a3, -1152.f));
}

// Block sum from the four pair accumulators of unpack_int4_word_h's products.
__device__ __forceinline__ float fold_int4_h(const float2 (&a)[4]) {
  float2 t = __fadd2_rn(a[0], a[2]);
  t = __ffma2_rn(__fadd2_rn(a[1], a[3]), make_float2(0.0625f, 0.0625f), t);
  return t.x + t.y;
}

// int4: one 16-byte chunk (one block of 32) of R rows against MT x rows.
template <int MT, int R>
__device__ __forceinline__ void chunk_int4(const float4 *__restrict__ xs4, int units_row, int c,
                                           const uint4 (&wv)[R], const float (&sc)[R],
                                           float (&acc)[R][MT]) {
  if constexpr (MT <= 2) {
    // words outer, rows inner: one pair of x units live at a time, reused by every row
    float2 a2[R][MT][4];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
#pragma unroll
        for (int j = 0; j < 4; ++j) a2[r][mm][j] = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float4 xa[MT], xb[MT];
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        xa[mm] = xs4[mm * units_row + swz(8 * c + 2 * i)];
        xb[mm] = xs4[mm * units_row + swz(8 * c + 2 * i + 1)];
      }
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t wi = i == 0 ? wv[r].x : i == 1 ? wv[r].y : i == 2 ? wv[r].z : wv[r].w;
        float2 p[4];
        unpack_int4_word_h(wi, p);
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          a2[r][mm][0] = __ffma2_rn(p[0], make_float2(xa[mm].x, xa[mm].y), a2[r][mm][0]);
          a2[r][mm][1] = __ffma2_rn(p[1], make_float2(xa[mm].z, xa[mm].w), a2[r][mm][1]);
          a2[r][mm][2] = __ffma2_rn(p[2], make_float2(xb[mm].x, xb[mm].y), a2[r][mm][2]);
          a2[r][mm][3] = __ffma2_rn(p[3], make_float2(xb[mm].z, xb[mm].w), a2[r][mm][3]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) acc[r][mm] = fmaf(sc[r], fold_int4_h(a2[r][mm]), acc[r][mm]);
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 p[4][4];
      const uint32_t ws[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) unpack_int4_word_h(ws[i], p[i]);
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        float2 a2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 xa = xs4[mm * units_row + swz(8 * c + 2 * i)];
          const float4 xb = xs4[mm * units_row + swz(8 * c + 2 * i + 1)];
          a2[0] = __ffma2_rn(p[i][0], make_float2(xa.x, xa.y), a2[0]);
          a2[1] = __ffma2_rn(p[i][1], make_float2(xa.z, xa.w), a2[1]);
          a2[2] = __ffma2_rn(p[i][2], make_float2(xb.x, xb.y), a2[2]);
          a2[3] = __ffma2_rn(p[i][3], make_float2(xb.z, xb.w), a2[3]);
        }
        acc[r][mm] = fmaf(sc[r], fold_int4_h(a2), acc[r][mm]);
      }
    }
  }
}

// int8: one 16-byte chunk (half a block) of R rows against MT x rows.
template <int MT, int R>
__device__ __forceinline__ void chunk_int8(const float4 *__restrict__ xs4, int units_row, int c,
                                           const uint4 (&wv)[R], const float (&sc)[R],
                                           float (&acc)[R][MT]) {
  if constexpr (MT <= 2) {
    float4 xv[MT][4];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
#pragma unroll
      for (int t = 0; t < 4; ++t) xv[mm][t] = xs4[mm * units_row + swz(4 * c + t)];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 a2[MT];
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) a2[mm] = make_float2(0.f, 0.f);
      const uint32_t ws[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float2 p[2];
        unpack_int8_word(ws[i], p);
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          a2[mm] = __ffma2_rn(p[0], make_float2(xv[mm][i].x, xv[mm][i].y), a2[mm]);
          a2[mm] = __ffma2_rn(p[1], make_float2(xv[mm][i].z, xv[mm][i].w), a2[mm]);
        }
      }
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) acc[r][mm] = fmaf(sc[r], a2[mm].x + a2[mm].y, acc[r][mm]);
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 p[4][2];
      const uint32_t ws[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) unpack_int8_word(ws[i], p[i]);
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 xa = xs4[mm * units_row + swz(4 * c + i)];
          a2 = __ffma2_rn(p[i][0], make_float2(xa.x, xa.y), a2);
          a2 = __ffma2_rn(p[i][1], make_float2(xa.z, xa.w), a2);
        }
        acc[r][mm] = fmaf(sc[r], a2.x + a2.y, acc[r][mm]);
      }
    }
  }
}

// int8: one whole block (32 codes = chunks 2b and 2b+1, x units 8b .. 8b+7) of R rows
// against MT x rows; one scale per row, applied once to the block sum.
template <int MT, int R>
__device__ __forceinline__ void block_int8(const float4 *__restrict__ xs4, int units_row, int b,
                                           const uint4 (&lo)[R], const uint4 (&hi)[R],
                                           const float (&sc)[R], float (&acc)[R][MT]) {
  if constexpr (MT <= 2) {
    float4 xv[MT][8];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
#pragma unroll
      for (int t = 0; t < 8; ++t) xv[mm][t] = xs4[mm * units_row + swz(8 * b + t)];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 a2[MT];
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) a2[mm] = make_float2(0.f, 0.f);
      const uint32_t ws[8] = {lo[r].x, lo[r].y, lo[r].z, lo[r].w, hi[r].x, hi[r].y, hi[r].z, hi[r].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float2 p[2];
        unpack_int8_word(ws[i], p);
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          a2[mm] = __ffma2_rn(p[0], make_float2(xv[mm][i].x, xv[mm][i].y), a2[mm]);
          a2[mm] = __ffma2_rn(p[1], make_float2(xv[mm][i].z, xv[mm][i].w), a2[mm]);
        }
      }
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) acc[r][mm] = fmaf(sc[r], a2[mm].x + a2[mm].y, acc[r][mm]);
    }
  } else {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float2 p[8][2];
      const uint32_t ws[8] = {lo[r].x, lo[r].y, lo[r].z, lo[r].w, hi[r].x, hi[r].y, hi[r].z, hi[r].w};
#pragma unroll
      for (int i = 0; i < 8; ++i) unpack_int8_word(ws[i], p[i]);
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        float2 a2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float4 xa = xs4[mm * units_row + swz(8 * b + i)];
          a2 = __ffma2_rn(p[i][0], make_float2(xa.x, xa.y), a2);
          a2 = __ffma2_rn(p[i][1], make_float2(xa.z, xa.w), a2);
        }
        acc[r][mm] = fmaf(sc[r], a2.x + a2.y, acc[r][mm]);
      }
    }
  }
}

}  // namespace gemv
}  // namespace woq

namespace woq {
namespace gemv {

// int5: one 32-bit word of low nibbles (elements e0..e7, e_p in bits 4p..4p+3, the int4 layout)
// and `nb`, the complemented fifth bits of the same elements (bit 4j for e_j, bit 16+4j for
// e_{4+j}; built by int5_fifth_bits). Each field becomes the offset-binary value
// u = code + 16 in the low mantissa bits of 2^23 (one LOP3 for the nibble, one for the fifth
// bit, moved just above its nibble: left by 4 for e_j, right by 12 for e_{4+j}); one exact
// packed subtraction removes 2^23 + 16, leaving the exact pairs p[j] = (q_j, q_{4+j}) * 2^(4j).
__device__ __forceinline__ void unpack_int5_word(uint32_t w, uint32_t nb, float2 (&p)[4]) {
  const uint32_t hi = w >> 16, nb4 = nb << 4, nbh = nb >> 12;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t mask = 0xFu << (4 * j);
    const uint32_t m5 = 0x10u << (4 * j);
    const float bias = 8388608.0f + 16.0f * static_cast<float>(1u << (4 * j));
    const float lo_f = __uint_as_float(((w & mask) | 0x4B000000u) | (nb4 & m5));
    const float hi_f = __uint_as_float(((hi & mask) | 0x4B000000u) | (nbh & m5));
    p[j] = __fadd2_rn(make_float2(lo_f, hi_f), make_float2(-bias, -bias));
  }
}

// The block's high-bit word H holds bit 4 of element e at bit e/8 + 4(e%4) + 16((e%8)/4); for
// the block's word i (elements 8i..8i+7) this returns their complemented fifth bits, e_{8i+j}
// at bit 4j and e_{8i+4+j} at bit 16+4j, as unpack_int5_word expects.
__device__ __forceinline__ uint32_t int5_fifth_bits(uint32_t H, int i) {
  return (~(H >> i)) & 0x11111111u;
}

// int5: one block of R rows (low nibbles `wv`, high-bit words `hw`) against MT x rows; the x
// units are those of chunk_int4, the 2^(4j) factors are removed by fold_int4.
template <int MT, int R>
__device__ __forceinline__ void chunk_int5(const float4 *__restrict__ xs4, int units_row, int c,
                                           const uint4 (&wv)[R], const uint32_t (&hw)[R],
                                           const float (&sc)[R], float (&acc)[R][MT]) {
  float4 xv[MT][8];
#pragma unroll
  for (int mm = 0; mm < MT; ++mm)
#pragma unroll
    for (int t = 0; t < 8; ++t) xv[mm][t] = xs4[mm * units_row + swz(8 * c + t)];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float2 a2[MT][4];
#pragma unroll
    for (int mm = 0; mm < MT; ++mm)
#pragma unroll
      for (int j = 0; j < 4; ++j) a2[mm][j] = make_float2(0.f, 0.f);
    const uint32_t ws[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 p[4];
      unpack_int5_word(ws[i], int5_fifth_bits(hw[r], i), p);
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        const float4 xa = xv[mm][2 * i], xb = xv[mm][2 * i + 1];
        a2[mm][0] = __ffma2_rn(p[0], make_float2(xa.x, xa.y), a2[mm][0]);
        a2[mm][1] = __ffma2_rn(p[1], make_float2(xa.z, xa.w), a2[mm][1]);
        a2[mm][2] = __ffma2_rn(p[2], make_float2(xb.x, xb.y), a2[mm][2]);
        a2[mm][3] = __ffma2_rn(p[3], make_float2(xb.z, xb.w), a2[mm][3]);
      }
    }
#pragma unroll
    for (int mm = 0; mm < MT; ++mm) acc[r][mm] = fmaf(sc[r], fold_int4(a2[mm]), acc[r][mm]);
  }
}

}  // namespace gemv
}  // namespace woq
