// Host-side quantiser: float32 W [n, k] -> packed int4/int8 codes + binary16 block scales.
//
// Formats: int4 in blocks of 32 ("MOSS-Transcribe-Diarize -- LiteRT (TFLite)", section
// "Files": the q4b32 production decoder), symmetric linear INT8 in blocks of 32 (soniqo
// Russian guide, section "Implementation notes") and 5-bit codes in blocks of 32 (soniqo
// English guide, section "INT5 vs INT8", which gives no layout: the one written here is this
// library's, documented in include/woq.h). Rule per row r and block j:
//   a = max |w| over the block (exact)
//   s = binary16(round-half-even((double)a / qmax))
//   q = clamp(round-half-even((double)w / (double)s), qmin, qmax), or 0 when s == 0.
// The layout written is the one documented in include/woq.h.
#include <cfenv>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

#include "woq.h"

namespace {

// Round a non-negative finite double once, half-to-even, to IEEE binary16; returns the bit
// pattern, or -1 if the result is infinite. Written from the binary16 definition: normal
// numbers are 1.f x 2^E with a 10-bit fraction and E in [-14, 15]; below 2^-14 the grid is
// the multiples of 2^-24.
int32_t half_bits_rne(double v) {
  if (v == 0.0) return 0;
  int e = 0;
  const double m = std::frexp(v, &e);  // v = m * 2^e, m in [0.5, 1)
  int E = e - 1;                       // v = (2m) * 2^E, 2m in [1, 2)
  if (E >= -14) {
    double sig = std::nearbyint(std::ldexp(m, 11));  // 11-bit significand, RNE
    if (sig == 2048.0) {
      sig = 1024.0;
      E += 1;
    }
    if (E > 15) return -1;
    return ((E + 15) << 10) | (static_cast<int32_t>(sig) - 1024);
  }
  const double f = std::nearbyint(std::ldexp(v, 24));  // multiples of 2^-24
  return static_cast<int32_t>(f);                        // 1024 is the smallest normal, 0x0400
}

double half_value(uint16_t h) {
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  const double mag = e == 0 ? std::ldexp(static_cast<double>(f), -24)
                            : std::ldexp(static_cast<double>(1024 + f), e - 25);
  return (h & 0x8000) ? -mag : mag;
}

int pack_rows(const float *W, int64_t r0, int64_t r1, int64_t k, int bits, uint8_t *packed,
              uint16_t *scales) {
  const int qmax = (1 << (bits - 1)) - 1;
  const int qmin = -(1 << (bits - 1));
  const int64_t nb = k / 32;
  const int64_t row_bytes = k * bits / 8;
  int q[32];
  for (int64_t r = r0; r < r1; ++r) {
    const float *wr = W + r * k;
    uint8_t *pr = packed + r * row_bytes;
    for (int64_t j = 0; j < nb; ++j) {
      const float *wb = wr + j * 32;
      float a = 0.0f;
      for (int i = 0; i < 32; ++i) {
        if (!std::isfinite(wb[i])) return WOQ_ERANGE;
        const float m = std::fabs(wb[i]);
        if (m > a) a = m;
      }
      const int32_t sb = half_bits_rne(static_cast<double>(a) / qmax);
      if (sb < 0) return WOQ_ERANGE;
      scales[r * nb + j] = static_cast<uint16_t>(sb);
      const double s = half_value(static_cast<uint16_t>(sb));
      for (int i = 0; i < 32; ++i) {
        if (s == 0.0) {
          q[i] = 0;
          continue;
        }
        double t = std::nearbyint(static_cast<double>(wb[i]) / s);
        if (t > qmax) t = qmax;
        if (t < qmin) t = qmin;
        q[i] = static_cast<int>(t);
      }
      if (bits == 8) {
        for (int i = 0; i < 32; ++i) pr[j * 32 + i] = static_cast<uint8_t>(static_cast<int8_t>(q[i]));
      } else if (bits == 5) {
        // low four bits as int4 in the row's first k/2 bytes; bit 4 of element i of the block in
        // bit (i / 8 + 4 * (i % 4) + 16 * ((i % 8) / 4)) of the block's word after them
        uint32_t high = 0;
        for (int i = 0; i < 16; ++i)
          pr[j * 16 + i] = static_cast<uint8_t>((q[2 * i] & 0xF) | ((q[2 * i + 1] & 0xF) << 4));
        for (int i = 0; i < 32; ++i)
          high |= static_cast<uint32_t>((q[i] >> 4) & 1) << (i / 8 + 4 * (i % 4) + 16 * ((i % 8) / 4));
        uint8_t *ph = pr + k / 2 + j * 4;
        for (int b = 0; b < 4; ++b) ph[b] = static_cast<uint8_t>(high >> (8 * b));
      } else {
        for (int i = 0; i < 16; ++i)
          pr[j * 16 + i] = static_cast<uint8_t>((q[2 * i] & 0xF) | ((q[2 * i + 1] & 0xF) << 4));
      }
    }
  }
  return WOQ_OK;
}

}  // namespace

extern "C" int qpack(const float *W, int64_t n, int64_t k, int32_t bits, uint8_t *packed,
                     uint16_t *scales) {
  if (!W || !packed || !scales) return WOQ_EINVAL;
  if (bits != 4 && bits != 5 && bits != 8) return WOQ_EINVAL;
  if (n <= 0 || k <= 0 || k % 32 != 0) return WOQ_ESHAPE;
  if (std::fegetround() != FE_TONEAREST) return WOQ_EINVAL;  // nearbyint must round to even

  const int64_t work = n * k;
  unsigned nt = std::thread::hardware_concurrency();
  if (nt == 0) nt = 1;
  if (nt > 16) nt = 16;
  if (work < (int64_t(1) << 22)) nt = 1;
  if (static_cast<int64_t>(nt) > n) nt = static_cast<unsigned>(n);
  if (nt == 1) return pack_rows(W, 0, n, k, bits, packed, scales);

  std::vector<int> rc(nt, WOQ_OK);
  std::vector<std::thread> th;
  const int64_t per = (n + nt - 1) / nt;
  for (unsigned t = 0; t < nt; ++t) {
    const int64_t r0 = t * per;
    const int64_t r1 = r0 + per < n ? r0 + per : n;
    if (r0 >= r1) break;
    th.emplace_back([&, t, r0, r1] { rc[t] = pack_rows(W, r0, r1, k, bits, packed, scales); });
  }
  for (auto &x : th) x.join();
  for (int c : rc)
    if (c != WOQ_OK) return c;
  return WOQ_OK;
}
