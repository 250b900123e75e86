// Per-token activation quantization, optionally fused with the non-affine
// LayerNorm and the adaLN modulate that precede every W8A8 Linear input of a
// block; and the one-time symmetric per-channel weight quantization.
//
// Activation scheme (FlagRelease "Qwen-Image-2.1-W8A8-arm-FlagOS",
// "Quantization and validation": dynamic asymmetric INT8 per token/row, FP32
// scales), all in fp32 with IEEE-rounded operations so that the codes are
// reproducible bit for bit:
//   lo = min(min_k u, 0), hi = max(max_k u, 0), s = (hi - lo) / 255
//   zp = clamp(rint(-128 - lo / s), -128, 127),  q = clamp(rint(u / s) + zp, -128, 127)
//   an all-zero row gets s = 1, zp = 0.
// Weight scheme (same section: symmetric INT8 per output channel, zero point
// 0, FP32 scales): s = max|w| / 127 (1 for a zero row), q = clamp(rint(w/s), +-127).
//
// One CTA per row, so the input is read once from HBM and the int8 codes are
// written once: the LayerNorm form holds its row in registers, the plain form
// stages it in shared memory.
#include "qi_common.cuh"
#include "qi_internal.h"

namespace qi {

constexpr int QT = 256;        // threads per row of the weight-preparation kernel

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reduction of one value over QT threads (weight preparation).
template <int OP>   // 0 sum, 1 min, 2 max
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  v = OP == 0 ? warp_sum(v) : (OP == 1 ? warp_min(v) : warp_max(v));
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < QT / 32; ++i)
    r = OP == 0 ? r + red[i] : (OP == 1 ? fminf(r, red[i]) : fmaxf(r, red[i]));
  return r;
}

// Block-wide reduction of a pair over blockDim.x threads: (sum, sum) or
// (min, max).  `red` holds 2 x 32 floats.
template <bool MINMAX>
__device__ __forceinline__ float2 block_reduce2(float a, float b, float* red) {
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (MINMAX) {
    a = warp_min(a);
    b = warp_max(b);
  } else {
    a = warp_sum(a);
    b = warp_sum(b);
  }
  __syncthreads();
  if (l == 0) {
    red[w] = a;
    red[32 + w] = b;
  }
  __syncthreads();
  float ra = red[0], rb = red[32];
  for (int i = 1; i < nw; ++i) {
    if (MINMAX) {
      ra = fminf(ra, red[i]);
      rb = fmaxf(rb, red[32 + i]);
    } else {
      ra += red[i];
      rb += red[32 + i];
    }
  }
  return make_float2(ra, rb);
}

// rint(v / s) for |v / s| <= 255 + rounding, by the exact IEEE quotient
// (the rare elements near a rounding tie; kept out of line).
__device__ __noinline__ int exact_code(float v, float s) { return __float2int_rn(__fdiv_rn(v, s)); }

// Codes q = rint(v / s) + zp of 2 NP values (NP fp32 pairs), not yet saturated.
// v * (1/s) is within ~3e-5 of the IEEE quotient (|v / s| <= 255), so it
// rounds the same way unless its fraction lies within 1e-4 of one half; a
// group holding such an element recomputes its codes from the exact quotient.
// Rounding uses the 1.5 * 2^23 shifter: t + 1.5 * 2^23 rounds t to an integer
// (ties to even, as rint) and leaves it in the low mantissa bits, so
// q = bits(t + shifter) - bits(shifter) + zp.
template <int NP>
__device__ __forceinline__ void quant_codes(const uint64_t (&v)[NP], float inv_s, float s, int zp,
                                            int (&q)[2 * NP]) {
  constexpr float kShift = 12582912.0f;
  const uint64_t inv2 = f2_pack(inv_s, inv_s), sh2 = f2_pack(kShift, kShift);
  const int bias = 0x4B400000 - zp;
  float worst = 0.f;
#pragma unroll
  for (int i = 0; i < NP; ++i) {
    const uint64_t t = f2_mul(v[i], inv2);
    const uint64_t y = f2_add(t, sh2);
    float f0, f1, y0, y1;
    f2_unpack(f2_sub(t, f2_sub(y, sh2)), f0, f1);   // t - rint(t), exact
    f2_unpack(y, y0, y1);
    worst = fmax3(worst, fabsf(f0), fabsf(f1));
    q[2 * i] = __float_as_int(y0) - bias;
    q[2 * i + 1] = __float_as_int(y1) - bias;
  }
  if (worst > 0.4999f) {
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      float e0, e1;
      f2_unpack(v[i], e0, e1);
      q[2 * i] = exact_code(e0, s) + zp;
      q[2 * i + 1] = exact_code(e1, s) + zp;
    }
  }
}

// Four codes, each saturated to [-128, 127], packed little-endian (a0 first).
// cvt.pack.sat.s8.s32.b32 d, a, b, c puts sat(b) in byte 0 and sat(a) in
// byte 1 of d, above the low bytes of c shifted up by 16.
__device__ __forceinline__ uint32_t pack4_sat_s8(int a0, int a1, int a2, int a3) {
  uint32_t hi, r;
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, 0;" : "=r"(hi) : "r"(a3), "r"(a2));
  asm("cvt.pack.sat.s8.s32.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a1), "r"(a0), "r"(hi));
  return r;
}

// bf16 words (2 values each, low half first) as fp32 pairs.
__device__ __forceinline__ uint64_t bf16x2_pair(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// 2 NP bf16 values from global memory (8 or 16 bytes) as NP fp32 pairs.
template <int NP>
__device__ __forceinline__ void load_bf16_pairs(const uint16_t* p, uint64_t (&d)[NP]) {
  if constexpr (NP == 4) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p);
    d[0] = bf16x2_pair(raw.x);
    d[1] = bf16x2_pair(raw.y);
    d[2] = bf16x2_pair(raw.z);
    d[3] = bf16x2_pair(raw.w);
  } else {
    const uint2 raw = *reinterpret_cast<const uint2*>(p);
    d[0] = bf16x2_pair(raw.x);
    d[1] = bf16x2_pair(raw.y);
  }
}

// One 16-byte unit of the staged row as fp32 pairs: 8 bf16 values (NP = 4)
// or 4 fp32 values (NP = 2).
template <bool XBF16>
__device__ __forceinline__ void unit_pairs(const uint4 u, uint64_t (&d)[XBF16 ? 4 : 2]) {
  if constexpr (XBF16) {
    d[0] = bf16x2_pair(u.x);
    d[1] = bf16x2_pair(u.y);
    d[2] = bf16x2_pair(u.z);
    d[3] = bf16x2_pair(u.w);
  } else {
    d[0] = f2_pack(__uint_as_float(u.x), __uint_as_float(u.y));
    d[1] = f2_pack(__uint_as_float(u.z), __uint_as_float(u.w));
  }
}

// ---------------------------------------------------------------- LayerNorm form
//
// One CTA per row with blockDim.x = max(32, K / 32) threads, each holding up
// to LN_CH chunks of 8 consecutive elements (as fp32 pairs) in registers:
// chunk c of thread t covers [8 (t + c blockDim), +8), so each load
// instruction of a warp reads one contiguous segment of the row.  The values
// are used by three passes (sums, modulate + range, codes), so they stay in
// registers.  Optionally the gated residual of the preceding Linear is added
// first (x + gate * y, one rounding; written out only if asked: the Linear
// after the LayerNorm can recompute it where it updates the stream).
constexpr int LN_CH = 4;

template <bool XBF16>
__global__ void __launch_bounds__(512) quant_ln_kernel(const QuantParams p) {
  __shared__ float red[64];
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int nchunk = p.K >> 3;
  uint64_t v[LN_CH][4];   // chunk c: elements (2i, 2i+1) in v[c][i]

#pragma unroll
  for (int c = 0; c < LN_CH; ++c) {
    const int ch = tid + c * nt;
    if (ch >= nchunk) continue;
    if (XBF16) {
      load_bf16_pairs<4>(static_cast<const uint16_t*>(p.x) + static_cast<int64_t>(row) * p.ldx + ch * 8, v[c]);
    } else {
      const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.x) +
                                                          static_cast<int64_t>(row) * p.ldx + ch * 8);
      const float4 a = src[0], b = src[1];
      v[c][0] = f2_pack(a.x, a.y);
      v[c][1] = f2_pack(a.z, a.w);
      v[c][2] = f2_pack(b.x, b.y);
      v[c][3] = f2_pack(b.z, b.w);
    }
  }
  if (p.zero_range && tid == 0) {
    p.zero_range[2 * static_cast<int64_t>(row)] = 0u;
    p.zero_range[2 * static_cast<int64_t>(row) + 1] = 0u;
  }
  if (p.zero_words && row == 0)
    for (int i = tid; i < p.n_zero_words; i += nt) p.zero_words[i] = 0u;
  const int rs = p.groups.row_set[group_of(p.groups, p.row0 + row)];
  if (!XBF16 && p.res_y) {
    const uint16_t* gt = p.res_gate + static_cast<int64_t>(rs) * p.mod_ld;
    float* xw = p.res_out ? p.res_out + static_cast<int64_t>(row) * p.ldx : nullptr;
#pragma unroll
    for (int c = 0; c < LN_CH; ++c) {
      const int ch = tid + c * nt;
      if (ch >= nchunk) continue;
      uint64_t fy[4], fg[4];
      load_bf16_pairs<4>(p.res_y + static_cast<int64_t>(row) * p.K + ch * 8, fy);
      load_bf16_pairs<4>(gt + ch * 8, fg);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[c][i] = f2_fma(fg[i], fy[i], v[c][i]);
      if (!xw) continue;
      float e[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(v[c][i], e[2 * i], e[2 * i + 1]);
      float4* o4 = reinterpret_cast<float4*>(xw + ch * 8);
      o4[0] = make_float4(e[0], e[1], e[2], e[3]);
      o4[1] = make_float4(e[4], e[5], e[6], e[7]);
    }
  }
  uint64_t s2 = 0ull, ss2 = 0ull;
#pragma unroll
  for (int c = 0; c < LN_CH; ++c)
    if (tid + c * nt < nchunk)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        s2 = f2_add(s2, v[c][i]);
        ss2 = f2_fma(v[c][i], v[c][i], ss2);
      }
  float s0, s1, q0, q1;
  f2_unpack(s2, s0, s1);
  f2_unpack(ss2, q0, q1);
  const float2 t = block_reduce2<false>(s0 + s1, q0 + q1, red);
  const float inv_k = 1.0f / static_cast<float>(p.K);
  const float mean = t.x * inv_k;
  const float var = fmaxf(t.y * inv_k - mean * mean, 0.0f);
  const float rstd = 1.0f / sqrtf(var + p.eps);
  const uint16_t* sh = p.shift + static_cast<int64_t>(rs) * p.mod_ld;
  const uint16_t* sc = p.scale + static_cast<int64_t>(rs) * p.mod_ld;
  const uint64_t mean2 = f2_pack(mean, mean), rstd2 = f2_pack(rstd, rstd), one2 = f2_pack(1.0f, 1.0f);
#pragma unroll
  for (int c = 0; c < LN_CH; ++c) {
    const int ch = tid + c * nt;
    if (ch >= nchunk) continue;
    uint64_t fsh[4], fsc[4];
    load_bf16_pairs<4>(sh + ch * 8, fsh);
    load_bf16_pairs<4>(sc + ch * 8, fsc);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      v[c][i] = f2_fma(f2_mul(f2_sub(v[c][i], mean2), rstd2), f2_add(one2, fsc[i]), fsh[i]);
  }
  if (p.u_bf16) {   // modulated activation for a BF16 Linear
#pragma unroll
    for (int c = 0; c < LN_CH; ++c) {
      const int ch = tid + c * nt;
      if (ch >= nchunk) continue;
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float e0, e1;
        f2_unpack(v[c][i], e0, e1);
        w[i] = pack_bf16x2(e0, e1);
      }
      *reinterpret_cast<uint4*>(p.u_bf16 + static_cast<int64_t>(row) * p.ldq + ch * 8) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (!p.quant_too) return;
  }
  if (p.u_f32) {   // tap: the exact fp32 values quantized below
#pragma unroll
    for (int c = 0; c < LN_CH; ++c) {
      const int ch = tid + c * nt;
      if (ch >= nchunk) continue;
      float e[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(v[c][i], e[2 * i], e[2 * i + 1]);
      float4* o4 = reinterpret_cast<float4*>(p.u_f32 + static_cast<int64_t>(row) * p.ldq + ch * 8);
      o4[0] = make_float4(e[0], e[1], e[2], e[3]);
      o4[1] = make_float4(e[4], e[5], e[6], e[7]);
    }
  }
  float lo = 0.f, hi = 0.f;
#pragma unroll
  for (int c = 0; c < LN_CH; ++c)
    if (tid + c * nt < nchunk)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float e0, e1;
        f2_unpack(v[c][i], e0, e1);
        lo = fmin3(lo, e0, e1);
        hi = fmax3(hi, e0, e1);
      }
  const float2 mm = block_reduce2<true>(lo, hi, red);
  float s = __fdiv_rn(__fsub_rn(mm.y, mm.x), 255.0f);
  int zp;
  if (s == 0.0f) {
    s = 1.0f;
    zp = 0;
  } else {
    const float z = rintf(__fsub_rn(-128.0f, __fdiv_rn(mm.x, s)));
    zp = static_cast<int>(fminf(fmaxf(z, -128.0f), 127.0f));
  }
  const float inv_s = __fdiv_rn(1.0f, s);
#pragma unroll
  for (int c = 0; c < LN_CH; ++c) {
    const int ch = tid + c * nt;
    if (ch >= nchunk) continue;
    int qv[8];
    quant_codes<4>(v[c], inv_s, s, zp, qv);
    *reinterpret_cast<uint2*>(p.q + static_cast<int64_t>(row) * p.ldq + ch * 8) =
        make_uint2(pack4_sat_s8(qv[0], qv[1], qv[2], qv[3]), pack4_sat_s8(qv[4], qv[5], qv[6], qv[7]));
  }
  if (tid == 0) {
    p.s[row] = s;
    p.zp[row] = zp;
  }
}

// ---------------------------------------------------------------- plain form
//
// One CTA per row.  Thread 0 brings the row into shared memory with one bulk
// copy; the CTA then works out of shared memory over 16-byte units (unit j of
// the row goes to thread j mod blockDim.x, so every warp access is one
// contiguous 512-byte segment), holding no row data in registers.  With about
// 40 registers per thread and one row of shared memory per CTA, 6 (K = 16384
// bf16) to 25 (K = 4096 bf16) rows are in flight per SM, against 2 to 8 for a
// row held in registers.  The range comes from a min/max pass, or (RANGE) was
// published by the producer as [bits of -min, bits of max] and is read while
// the copy is in flight, leaving one pass.
constexpr int QS_MAX_THREADS = 256;
constexpr int QS_UNITS_PER_THREAD = 8;
constexpr int QS_MAX_SMEM = 16384 * 4;   // an fp32 row at K = 16384

template <bool XBF16, bool RANGE>
__global__ void __launch_bounds__(QS_MAX_THREADS, 6) quant_kernel(const QuantParams p) {
  constexpr int NP = XBF16 ? 4 : 2;   // fp32 pairs per unit
  constexpr int VPU = 2 * NP;         // values per unit
  extern __shared__ __align__(128) uint8_t qs_row[];
  __shared__ float red[64];
  __shared__ uint64_t bar;
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int nunit = p.K / VPU;
  const uint32_t xbytes = static_cast<uint32_t>(p.K) * (XBF16 ? 2u : 4u);
  const uint4* xs = reinterpret_cast<const uint4*>(qs_row);
  pdl_wait();
  pdl_trigger();

  if (tid == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(&bar, xbytes);
    bulk_load_1d(qs_row,
                 static_cast<const uint8_t*>(p.x) + static_cast<int64_t>(row) * p.ldx * (XBF16 ? 2 : 4),
                 xbytes, &bar);
  }
  float lo = 0.f, hi = 0.f;
  if (RANGE) {
    lo = -__uint_as_float(p.range[2 * static_cast<int64_t>(row)]);
    hi = __uint_as_float(p.range[2 * static_cast<int64_t>(row) + 1]);
  }
  __syncthreads();   // the barrier's initialisation is visible to every thread
  if (!__syncthreads_and(mbar_wait(&bar, 0, p.status))) {
    if (tid == 0) {   // the copy may still be landing: bounded wait before leaving
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&bar, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
      }
    }
    return;
  }
  if (!RANGE) {
#pragma unroll 2
    for (int j = tid; j < nunit; j += nt) {
      uint64_t v[NP];
      unit_pairs<XBF16>(xs[j], v);
#pragma unroll
      for (int i = 0; i < NP; ++i) {
        float e0, e1;
        f2_unpack(v[i], e0, e1);
        lo = fmin3(lo, e0, e1);
        hi = fmax3(hi, e0, e1);
      }
    }
    const float2 mm = block_reduce2<true>(lo, hi, red);
    lo = mm.x;
    hi = mm.y;
  }
  float s = __fdiv_rn(__fsub_rn(hi, lo), 255.0f);
  int zp;
  if (s == 0.0f) {
    s = 1.0f;
    zp = 0;
  } else {
    const float z = rintf(__fsub_rn(-128.0f, __fdiv_rn(lo, s)));
    zp = static_cast<int>(fminf(fmaxf(z, -128.0f), 127.0f));
  }
  const float inv_s = __fdiv_rn(1.0f, s);
  int8_t* qrow = p.q + static_cast<int64_t>(row) * p.ldq;
#pragma unroll 2
  for (int j = tid; j < nunit; j += nt) {
    uint64_t v[NP];
    unit_pairs<XBF16>(xs[j], v);
    int qv[2 * NP];
    quant_codes<NP>(v, inv_s, s, zp, qv);
    if constexpr (NP == 4)
      *reinterpret_cast<uint2*>(qrow + j * 8) =
          make_uint2(pack4_sat_s8(qv[0], qv[1], qv[2], qv[3]), pack4_sat_s8(qv[4], qv[5], qv[6], qv[7]));
    else
      *reinterpret_cast<uint32_t*>(qrow + j * 4) = pack4_sat_s8(qv[0], qv[1], qv[2], qv[3]);
  }
  if (tid == 0) {
    p.s[row] = s;
    p.zp[row] = zp;
  }
}

template <bool XBF16>
static int launch_quant_ln_t(const QuantParams& p, cudaStream_t st) {
  int nt = (p.K / 8 + LN_CH - 1) / LN_CH;   // threads so that each holds <= LN_CH chunks
  nt = ((nt + 31) / 32) * 32;
  if (nt < 32) nt = 32;
  launch_pdl(quant_ln_kernel<XBF16>, dim3(p.M), dim3(nt), 0, st, 1, p);
  return launch_result();
}

template <bool XBF16, bool RANGE>
static int launch_quant_t(const QuantParams& p, cudaStream_t st) {
  static bool attr = false;   // per instantiation
  if (!attr) {
    if (cudaFuncSetAttribute(quant_kernel<XBF16, RANGE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QS_MAX_SMEM) != cudaSuccess) {
      launch_result();
      return -1;
    }
    attr = true;
  }
  const int nunit = p.K / (XBF16 ? 8 : 4);
  int nt = (nunit + QS_UNITS_PER_THREAD - 1) / QS_UNITS_PER_THREAD;
  nt = ((nt + 31) / 32) * 32;
  nt = nt < 32 ? 32 : (nt > QS_MAX_THREADS ? QS_MAX_THREADS : nt);
  const size_t smem = static_cast<size_t>(p.K) * (XBF16 ? 2 : 4);
  launch_pdl(quant_kernel<XBF16, RANGE>, dim3(p.M), dim3(nt), smem, st, 1, p);
  return launch_result();
}

int launch_quant(const QuantParams& p, cudaStream_t st) {
  if (p.M == 0) return 0;
  if (p.K <= 0 || p.K % 8 != 0 || p.K > 16384) return -1;
  if (p.ln && p.range) return -1;                 // LN computes its own range
  if (p.res_y && (!p.ln || p.x_bf16)) return -1;  // the residual add is on the fp32 stream
  if (p.ln) return p.x_bf16 ? launch_quant_ln_t<true>(p, st) : launch_quant_ln_t<false>(p, st);
  // the row copy needs 16-byte aligned rows
  const int esz = p.x_bf16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(p.x) % 16 != 0 || (static_cast<int64_t>(p.ldx) * esz) % 16 != 0) return -1;
  if (p.x_bf16) return p.range ? launch_quant_t<true, true>(p, st) : launch_quant_t<true, false>(p, st);
  return p.range ? launch_quant_t<false, true>(p, st) : launch_quant_t<false, false>(p, st);
}

// ---------------------------------------------------------------- weights

__global__ void __launch_bounds__(QT) prepare_w8_kernel(const float* __restrict__ w, int k,
                                                         int8_t* __restrict__ q,
                                                         float* __restrict__ s,
                                                         int32_t* __restrict__ rowsum) {
  __shared__ float red[QT / 32];
  __shared__ int ired[QT / 32];
  const int n = blockIdx.x;
  const float* row = w + static_cast<int64_t>(n) * k;
  float amax = 0.f;
  for (int i = threadIdx.x; i < k; i += QT) amax = fmaxf(amax, fabsf(row[i]));
  amax = block_reduce<2>(amax, red);
  const float sc = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 127.0f);
  int sum = 0;
  for (int i = threadIdx.x; i < k; i += QT) {
    const float r = fminf(fmaxf(rintf(__fdiv_rn(row[i], sc)), -127.0f), 127.0f);
    const int qi = static_cast<int>(r);
    q[static_cast<int64_t>(n) * k + i] = static_cast<int8_t>(qi);
    sum += qi;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) ired[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int i = 0; i < QT / 32; ++i) t += ired[i];
    rowsum[n] = t;
    s[n] = sc;
  }
}

int launch_prepare_w8(const float* w, int n, int k, int8_t* q, float* s, int32_t* rowsum,
                      cudaStream_t st) {
  if (n == 0) return 0;
  prepare_w8_kernel<<<n, QT, 0, st>>>(w, k, q, s, rowsum);
  return launch_result();
}

}  // namespace qi
