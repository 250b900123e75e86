// MXFP4 (E2M1 codes, E8M0 scale per 32 columns) -> bf16 decoding shared by
// the GEMM's in-kernel decode and the expansion kernel.  Every product
// e2m1 x 2^(e - 127) has at most two significant bits, so its bf16 value is
// exact; mx_decode32 decodes one scale group of 32 codes (16 bytes, low
// nibble first) into 32 bf16 values.
#pragma once
#include "qi_common.cuh"

namespace qi {

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Byte tables of the bf16 values of the 8 E2M1 magnitudes at scale 2^(e-127),
// for 2 <= e <= 252 (every value then a normal bf16): magnitude c has the
// exponent field e + E[c] (E = -1, 0, 0, 1, 1, 2, 2 for c = 1..7) and the
// mantissa bit 0x40 for c = 3, 5, 7; c = 0 is +0.  lo0/lo1 hold the low bytes
// of c = 0..3 / 4..7, hi0/hi1 the high bytes.
struct MxTable {
  uint32_t lo0, lo1, hi0, hi1;
};
__device__ __forceinline__ MxTable mx_table(uint32_t e) {
  const uint32_t p0 = (e & 1u) << 7, p1 = ((e + 1u) & 1u) << 7;   // exponent LSB in bit 7
  MxTable t;
  t.lo0 = (p1 << 8) | (p0 << 16) | ((p0 | 0x40u) << 24);             // c = 0 .. 3 (c1: e - 1 ~ e + 1)
  t.lo1 = p1 | ((p1 | 0x40u) << 8) | (p0 << 16) | ((p0 | 0x40u) << 24);
  t.hi0 = (((e - 1u) >> 1) << 8) | ((e >> 1) << 16) | ((e >> 1) << 24);
  t.hi1 = ((e + 1u) >> 1) | (((e + 1u) >> 1) << 8) | (((e + 2u) >> 1) << 16) | (((e + 2u) >> 1) << 24);
  return t;
}

// 8 E2M1 codes (one 32-bit word, low nibble first) -> 8 bf16 values (4 words).
__device__ __forceinline__ void mx_decode8(const MxTable& t, uint32_t w, uint32_t (&o)[4]) {
  const uint32_t sel = w & 0x77777777u;                 // magnitudes as byte selectors
  const uint32_t sg = (w << 4);                         // sign bit of every even nibble -> bit 7 of its byte
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t s = h ? (sel >> 16) : sel;
    const uint32_t lo = prmt(t.lo0, t.lo1, s);
    uint32_t hi = prmt(t.hi0, t.hi1, s);
    // bit 7 of each value's byte: nibble 4h+0 from (w << 4), 4h+1 from w, ...
    const uint32_t sbits = prmt(w, sg, h ? 0x3726u : 0x1504u);
    hi |= sbits & 0x80808080u;
    o[2 * h] = prmt(lo, hi, 0x5140u);
    o[2 * h + 1] = prmt(lo, hi, 0x7362u);
  }
}

// The general decode of 8 codes (any E8M0 byte, including the extremes and
// the NaN marker 255): the fp32 value e2m1 x 2^(e-127), rounded to bf16.
static __device__ __noinline__ void mx_decode8_general(uint32_t e, uint32_t w, uint32_t (&o)[4]) {
  const float scale = e == 255u ? __int_as_float(0x7FC00000) :
                      (e == 0u ? __int_as_float(0x00400000) : __int_as_float(static_cast<int>(e << 23)));
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t c = (w >> (4 * i)) & 15u;
    const uint32_t ex = (c >> 1) & 3u, m = c & 1u;
    const float mag = ex == 0u ? 0.5f * static_cast<float>(m)
                               : (1.0f + 0.5f * static_cast<float>(m)) * static_cast<float>(1u << (ex - 1u));
    v[i] = ((c & 8u) ? -mag : mag) * scale;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) o[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
}

// 32 codes (16 bytes) of one scale group -> 32 bf16 values (four 16-byte chunks).
__device__ __forceinline__ void mx_decode32(uint32_t e, const uint4& w, uint32_t (&o)[16]) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
  if (e >= 2u && e <= 252u) {
    const MxTable t = mx_table(e);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t q[4];
      mx_decode8(t, ws[i], q);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[4 * i + j] = q[j];
    }
  } else {
#pragma unroll 1
    for (int i = 0; i < 4; ++i) {
      uint32_t q[4];
      mx_decode8_general(e, ws[i], q);
#pragma unroll
      for (int j = 0; j < 4; ++j) o[4 * i + j] = q[j];
    }
  }
}

}  // namespace qi
