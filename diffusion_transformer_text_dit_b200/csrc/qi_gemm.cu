// Persistent tcgen05 GEMM for sm_100a: D[M,N] = A[M,K] . B[N,K]^T with both
// operands K-major, fed by TMA (128-byte swizzle) into a multi-stage shared
// memory ring, accumulated in TMEM and drained by a fused epilogue.
//
//  * kind::i8  : int8 x int8 -> int32 (the W8A8 Linear, FlagRelease
//    "Qwen-Image-2.1-W8A8-arm-FlagOS", "Quantization and validation": INT32
//    accumulation, FP32 scaling, BF16 output).  Epilogue:
//      y = (float)(acc - zp_a[m] * rowsum[n]) * s_a[m] * s_w[n] + bias[n]
//  * kind::f16 : bf16 x bf16 -> fp32 (the BF16 Linears: in/out projections).
//      y = acc + bias[n]
//
// Warp roles in a 320-thread CTA (one CTA per SM, persistent over tiles):
//   warp 0      TMA producer (one thread)
//   warp 1      TMEM allocator + MMA issuer (one thread)
//   warps 2..9  epilogue: warp w reads TMEM lanes 32*(w%4) .. +31; warps 2-5
//               take the first half of the tile's columns, warps 6-9 the second
//               (two warps per SM sub-partition hide the epilogue's latencies)
// Tiles are 128 x BN; the accumulator is double-buffered in TMEM (2*BN
// columns) so the epilogue of tile i overlaps the MMAs of tile i+1.
#include "qi_common.cuh"
#include "qi_mx.cuh"
#include "qi_internal.h"

namespace qi {

constexpr int GEMM_BM = 128;
constexpr int GEMM_BK_BYTES = 128;      // one 128-byte swizzle row per stage
constexpr int GEMM_THREADS = 320;
constexpr int GEMM_EPI_WARPS = 8;

template <int BN>
struct GemmCfg {
  static constexpr int A_BYTES = GEMM_BM * GEMM_BK_BYTES;
  static constexpr int B_BYTES = BN * GEMM_BK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;
  static constexpr int COL_BYTES = 2 * BN * 12;   // two tiles of (s_w, rowsum, bias)
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256 + COL_BYTES;
  static_assert(2 * STAGES + 8 <= 32, "barrier area");
};

// GELU, tanh form: 0.5 x (1 + tanh(z)), z = sqrt(2/pi) (x + 0.044715 x^3).
// Evaluated as x / (1 + e^(-2z)) (the same function: 0.5 (1 + tanh z) is the
// logistic of 2z), with the hardware base-2 exponential and a fast divide;
// relative error ~1e-6, far below the bf16 rounding of the result.
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k0 = 0.7978845608028654f;   // sqrt(2/pi)
  const float k1 = 0.044715f;
  const float z = k0 * fmaf(k1 * x, x * x, x);
  float e;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-2.8853900817779268f * z));   // e^(-2z)
  return __fdividef(x, 1.0f + e);
}

// Per-column constants of one tile (s_w, rowsum, bias as fp32), staged in
// shared memory by the epilogue warps so that each output element reads them
// with broadcast 16-byte loads instead of three global loads.  Indexed by the
// column's offset in the tile; columns past N hold zeros.
struct ColTable {
  const float* sw;
  const int32_t* rs;
  const float* b;
};

// Dequantise 32 accumulator columns (tile offset c0, a multiple of 32):
//   v = (acc - zp rowsum) s_a s_w + bias      (kind::i8)
//   v = acc + bias                            (kind::f16)
template <bool I8>
__device__ __forceinline__ void dequant32(const ColTable& t, const uint32_t (&r)[32], int c0,
                                          float sa, int32_t zp, float (&v)[32]) {
  const float4* sw4 = reinterpret_cast<const float4*>(t.sw + c0);
  const int4* rs4 = reinterpret_cast<const int4*>(t.rs + c0);
  const float4* b4 = reinterpret_cast<const float4*>(t.b + c0);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 bb = b4[q];
    const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
    if (I8) {
      const float4 ww = sw4[q];
      const int4 rr = rs4[q];
      const float wv[4] = {ww.x, ww.y, ww.z, ww.w};
      const int32_t rv[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int32_t corr = static_cast<int32_t>(r[4 * q + e]) - zp * rv[e];
        v[4 * q + e] = fmaf(static_cast<float>(corr) * sa, wv[e], bv[e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[4 * q + e] = __uint_as_float(r[4 * q + e]) + bv[e];
    }
  }
}

// 32 accumulator columns dequantized (W8A8) or biased (BF16) and rounded to
// bf16 (the Linear's output dtype).
template <bool I8>
__device__ __forceinline__ void dequant32_bf16(const ColTable& t, const uint32_t (&r)[32], int c0,
                                               float sa, int32_t zp, float (&y)[32]) {
  dequant32<I8>(t, r, c0, sa, zp, y);
#pragma unroll
  for (int j = 0; j < 32; ++j) y[j] = bf16_round_f(y[j]);
}

// Stage the constants of the tile's columns n0 .. n0 + BN - 1 (the 256
// epilogue threads, numbered et = 0 .. 255) and arrive on `ready` (one arrival
// per epilogue warp); the caller then waits on `ready` with a bounded wait.
// Buffers alternate with the accumulator buffer: a warp writes the buffer of
// tile i + 2 only after the wait of tile i + 1, which needs every warp's
// arrival for tile i + 1, made after that warp finished tile i.
template <bool I8, int BN>
__device__ __forceinline__ void stage_columns(const GemmParams& p, float* sw, int32_t* rs, float* b,
                                              int n0, int et, uint64_t* ready) {
#pragma unroll 1
  for (int c = et; c < BN; c += 32 * GEMM_EPI_WARPS) {
    const int n = n0 + c;
    const bool in = n < p.N;
    if (I8) {
      sw[c] = in ? __ldg(p.s_w + n) : 0.f;
      rs[c] = in ? __ldg(p.rowsum + n) : 0;
    }
    b[c] = (in && p.bias) ? bf16_bits_to_float(__ldg(p.bias + n)) : 0.f;
  }
  __threadfence_block();
  __syncwarp();
  if ((et & 31) == 0) mbar_arrive(ready);
}

// "Accumulator buffer drained" signal of one epilogue warp.  In a CTA pair
// the barrier lives in the even CTA, whose thread issues the MMAs for both.
template <bool PAIR>
__device__ __forceinline__ void tempty_signal(uint32_t addr) {
  if (PAIR)
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
  else
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(addr) : "memory");
}

// e4m3 codes (round to nearest even, saturating at +-448) of the two bf16
// values of a packed word, first value in the low byte.
__device__ __forceinline__ uint32_t e4m3x2_of_bf16x2(uint32_t w) {
  uint16_t h;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
      : "=h"(h)
      : "f"(__uint_as_float(w & 0xFFFF0000u)), "f"(__uint_as_float(w << 16)));
  return h;
}

// 32 stored bf16 values (16 packed words) as 32 e4m3 bytes at dst.
__device__ __forceinline__ void store_e4m3_32(uint8_t* dst, const uint32_t (&pk)[16]) {
  uint32_t e[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = e4m3x2_of_bf16x2(pk[2 * i]) | (e4m3x2_of_bf16x2(pk[2 * i + 1]) << 16);
  uint4* d = reinterpret_cast<uint4*>(dst);
  d[0] = make_uint4(e[0], e[1], e[2], e[3]);
  d[1] = make_uint4(e[4], e[5], e[6], e[7]);
}

// Fused epilogue of the QKV projection: the W columns handled by one epilogue
// warp are W/128 whole heads of q, k or v.  A q or k head row is read from
// TMEM once and held (dequantized, bf16-rounded) in registers for
//   r = 1/sqrt(mean(y^2) + eps), n = bf16(y r), y' = bf16(n w)   (cast before scale)
//   (a, b) -> (bf16(a c - b s), bf16(a s + b c))                 (RoPE, pair = column/2)
// with explicitly rounded fp32 operations; v is stored as bf16(y).  For fp8
// attention each stored bf16 row is also written as e4m3 (the value a
// separate cast of the bf16 tensor gives).
template <bool I8, int W, bool PAIR>
__device__ __forceinline__ void qkv_epilogue(const GemmParams& p, const ColTable& ct, int cb,
                                             uint32_t t_row, int m, bool row_ok, float sa,
                                             int32_t zp, int n0, int lane, uint32_t tempty_addr) {
  // column n of this GEMM is column n_base + n of the q | k | v projection
  // (a GEMM may cover only part of it: the W8A8 q, k rows and a BF16 v)
  const int gn = n0 + p.n_base;
  const int which = gn / p.H;
  const int col0 = gn - which * p.H;
  // q rows are contiguous; K/V rows of a second sequence go to its own buffer
  const bool second = which > 0 && p.k_out2 != nullptr && m >= p.kv_split;
  const int mo = second ? m - p.kv_split : m;
  uint16_t* out = which == 0 ? p.q_out
                             : (which == 1 ? (second ? p.k_out2 : p.k_out)
                                           : (second ? p.v_out2 : p.v_out_bf16));
  // e4m3 row of this head (read from the kernel parameters where it is used)
  auto row8 = [&](int hh) -> uint8_t* {
    uint8_t* o8 = which == 0 ? p.q8_out
                             : (which == 1 ? (second ? p.k8_out2 : p.k8_out) : (second ? p.v8_out2 : p.v8_out));
    return o8 + static_cast<size_t>(mo) * p.ldo + col0 + hh * 128;
  };
  const bool has8 = p.q8_out != nullptr;   // fp8 attention: all five are set
  const uint16_t* w = which == 0 ? p.wq : p.wk;
#pragma unroll 1
  for (int hh = 0; hh < W / 128; ++hh) {
    const bool last = hh == W / 128 - 1;   // this warp's last TMEM reads of the accumulator
    uint4* dst_row = reinterpret_cast<uint4*>(out + static_cast<size_t>(mo) * p.ldo + col0 + hh * 128);
    if (which == 2) {
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + hh * 128 + c * 32, r);
        if (last && c == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) tempty_signal<PAIR>(tempty_addr);
        }
        if (!row_ok) continue;
        float y[32];
        dequant32_bf16<I8>(ct, r, cb + hh * 128 + c * 32, sa, zp, y);
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
#pragma unroll
        for (int v = 0; v < 4; ++v)
          dst_row[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        if (has8) store_e4m3_32(row8(hh) + c * 32, pk);
      }
      continue;
    }
    // the head row as bf16 pairs (the dequantized values are bf16 already)
    uint32_t yp[4][16];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(t_row + hh * 128 + c * 32, r);
      if (last && c == 3) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) tempty_signal<PAIR>(tempty_addr);
      }
      if (row_ok) {
        float y[32];
        dequant32_bf16<I8>(ct, r, cb + hh * 128 + c * 32, sa, zp, y);
#pragma unroll
        for (int j = 0; j < 32; ++j) ss = __fadd_rn(ss, __fmul_rn(y[j], y[j]));
#pragma unroll
        for (int i = 0; i < 16; ++i) yp[c][i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      }
    }
    if (!row_ok) continue;
    const float rs = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, 128.0f), p.eps)));
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
      const float4* c4 = reinterpret_cast<const float4*>(p.rcos + static_cast<size_t>(m) * 64 + c * 16);
      const float4* s4 = reinterpret_cast<const float4*>(p.rsin + static_cast<size_t>(m) * 64 + c * 16);
      const uint4* w4 = reinterpret_cast<const uint4*>(w + c * 32);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const float4 cc = __ldg(c4 + g), sn = __ldg(s4 + g);
        const uint4 wv = __ldg(w4 + g);
        const float cs[4] = {cc.x, cc.y, cc.z, cc.w}, si[4] = {sn.x, sn.y, sn.z, sn.w};
        const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int i = 4 * g + t;   // pair index in the chunk
          const float y0 = __uint_as_float(yp[c][i] << 16), y1 = __uint_as_float(yp[c][i] & 0xFFFF0000u);
          const float a = bf16_round_f(__fmul_rn(bf16_round_f(__fmul_rn(y0, rs)),
                                                 __uint_as_float(ww[t] << 16)));
          const float b = bf16_round_f(__fmul_rn(bf16_round_f(__fmul_rn(y1, rs)),
                                                 __uint_as_float(ww[t] & 0xFFFF0000u)));
          pk[i] = pack_bf16x2(__fsub_rn(__fmul_rn(a, cs[t]), __fmul_rn(b, si[t])),
                              __fadd_rn(__fmul_rn(a, si[t]), __fmul_rn(b, cs[t])));
        }
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
        dst_row[c * 4 + v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
      if (has8) store_e4m3_32(row8(hh) + c * 32, pk);
    }
  }
}

// Epilogue of one accumulator tile, run by the 8 epilogue warps: warp
// (quarter, half) reads TMEM lanes 32*quarter .. +31 (rows m0 + 32*quarter + lane)
// and half `half` of the BN columns, signals the accumulator buffer free after
// its last TMEM read, and writes the fused result.
template <bool I8, int BN, int EPI, bool PAIR>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const ColTable& ct,
                                              uint32_t tmem_acc, int m0, int n0, int quarter,
                                              int half, int lane, uint32_t tempty_addr) {
  const int row_in_tile = quarter * 32 + lane;
  const int m = m0 + row_in_tile;
  const bool row_ok = m < p.M;
  float sa = 0.f;
  int32_t zp = 0;
  int rs = 0;
  if (row_ok) {
    if (I8) {
      sa = p.s_a[m];
      zp = p.zp_a[m];
    }
    if (EPI == EPI_GATED) rs = p.groups.row_set[group_of(p.groups, p.row0 + m)];
  }
  const uint32_t t_row = tmem_acc + (static_cast<uint32_t>(quarter * 32) << 16);
  if constexpr (EPI == EPI_QKV) {
    qkv_epilogue<I8, BN / 2, PAIR>(p, ct, half * (BN / 2), t_row + half * (BN / 2), m, row_ok, sa,
                               zp, n0 + half * (BN / 2), lane, tempty_addr);
    return;
  }
  float rlo = 0.f, rhi = 0.f;   // GELU: row range of this warp's half tile
#pragma unroll 1
  for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
    uint32_t r[32];
    tmem_ld32(t_row + c * 32, r);
    if (c == (half + 1) * (BN / 64) - 1) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) tempty_signal<PAIR>(tempty_addr);
    }
    const int nb = n0 + c * 32;
    if (!row_ok || nb >= p.N) continue;
    const int ncols = min(32, p.N - nb);
    if (p.acc_debug) {
      int4* dst = reinterpret_cast<int4*>(p.acc_debug + static_cast<size_t>(m) * p.N + nb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (4 * j < ncols)
          dst[j] = make_int4(static_cast<int>(r[4 * j]), static_cast<int>(r[4 * j + 1]),
                             static_cast<int>(r[4 * j + 2]), static_cast<int>(r[4 * j + 3]));
    }
    float v[32];
    dequant32<I8>(ct, r, c * 32, sa, zp, v);
    if (EPI == EPI_BF16 || EPI == EPI_GELU) {
      uint16_t* dst = p.y + static_cast<size_t>(m) * p.ldy + nb;
      uint32_t w[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float a0 = v[2 * j], a1 = v[2 * j + 1];
        if (EPI == EPI_GELU) {
          a0 = bf16_round_f(gelu_tanh_f(bf16_round_f(a0)));
          a1 = bf16_round_f(gelu_tanh_f(bf16_round_f(a1)));
          if (8 * (j >> 2) < ncols) {   // the stored values' range for the quantizer
            rlo = fminf(rlo, fminf(a0, a1));
            rhi = fmaxf(rhi, fmaxf(a0, a1));
          }
        }
        w[j] = pack_bf16x2(a0, a1);
      }
      if (ncols == 32) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      } else {
        // ragged N tail: ncols is a multiple of 16 (n % 16 == 0)
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (8 * j < ncols)
            d4[j] = make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
      }
    } else if (EPI == EPI_GATED) {
      // x += gate * bf16(y)  (fp32 residual stream); with res_y, x first
      // becomes x + gate1 * res_y, one rounding, as the LayerNorm before this
      // Linear computed it
      float4* dst = reinterpret_cast<float4*>(p.yf + static_cast<size_t>(m) * p.ldyf + nb);
      const uint4* g4 =
          reinterpret_cast<const uint4*>(p.gate + static_cast<size_t>(rs) * p.gate_ld + nb);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (8 * j >= ncols) break;
        const uint4 gr = __ldg(g4 + j);
        const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
        float4 a = dst[2 * j], b = dst[2 * j + 1];
        if (p.res_y) {
          const uint4 g1 = __ldg(reinterpret_cast<const uint4*>(
                                     p.gate1 + static_cast<size_t>(rs) * p.gate_ld + nb) + j);
          const uint4 y1 = __ldg(reinterpret_cast<const uint4*>(
                                     p.res_y + static_cast<size_t>(m) * p.ld_res_y + nb) + j);
          a.x = fmaf(__uint_as_float(g1.x << 16), __uint_as_float(y1.x << 16), a.x);
          a.y = fmaf(__uint_as_float(g1.x & 0xFFFF0000u), __uint_as_float(y1.x & 0xFFFF0000u), a.y);
          a.z = fmaf(__uint_as_float(g1.y << 16), __uint_as_float(y1.y << 16), a.z);
          a.w = fmaf(__uint_as_float(g1.y & 0xFFFF0000u), __uint_as_float(y1.y & 0xFFFF0000u), a.w);
          b.x = fmaf(__uint_as_float(g1.z << 16), __uint_as_float(y1.z << 16), b.x);
          b.y = fmaf(__uint_as_float(g1.z & 0xFFFF0000u), __uint_as_float(y1.z & 0xFFFF0000u), b.y);
          b.z = fmaf(__uint_as_float(g1.w << 16), __uint_as_float(y1.w << 16), b.z);
          b.w = fmaf(__uint_as_float(g1.w & 0xFFFF0000u), __uint_as_float(y1.w & 0xFFFF0000u), b.w);
        }
        a.x += __uint_as_float(gw[0] << 16) * bf16_round_f(v[8 * j + 0]);
        a.y += __uint_as_float(gw[0] & 0xFFFF0000u) * bf16_round_f(v[8 * j + 1]);
        a.z += __uint_as_float(gw[1] << 16) * bf16_round_f(v[8 * j + 2]);
        a.w += __uint_as_float(gw[1] & 0xFFFF0000u) * bf16_round_f(v[8 * j + 3]);
        b.x += __uint_as_float(gw[2] << 16) * bf16_round_f(v[8 * j + 4]);
        b.y += __uint_as_float(gw[2] & 0xFFFF0000u) * bf16_round_f(v[8 * j + 5]);
        b.z += __uint_as_float(gw[3] << 16) * bf16_round_f(v[8 * j + 6]);
        b.w += __uint_as_float(gw[3] & 0xFFFF0000u) * bf16_round_f(v[8 * j + 7]);
        dst[2 * j] = a;
        dst[2 * j + 1] = b;
      }
    } else if (EPI == EPI_F32) {
      float4* dst = reinterpret_cast<float4*>(p.yf + static_cast<size_t>(m) * p.ldyf + nb);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (4 * j < ncols) dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else if (EPI == EPI_EULER) {
      // FlowMatch Euler: x += (sigma_next - sigma) * v, fp32, no FMA
      float4* lat = reinterpret_cast<float4*>(p.yf + static_cast<size_t>(m) * p.ldyf + nb);
      float4* vo = p.v_out ? reinterpret_cast<float4*>(p.v_out + static_cast<size_t>(m) * p.ldyf + nb)
                           : nullptr;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (4 * j >= ncols) break;
        const float4 vv = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        if (vo) vo[j] = vv;
        float4 x = lat[j];
        x.x = __fadd_rn(x.x, __fmul_rn(p.dt, vv.x));
        x.y = __fadd_rn(x.y, __fmul_rn(p.dt, vv.y));
        x.z = __fadd_rn(x.z, __fmul_rn(p.dt, vv.z));
        x.w = __fadd_rn(x.w, __fmul_rn(p.dt, vv.w));
        lat[j] = x;
      }
    }
  }
  if (EPI == EPI_GELU && p.row_range && row_ok) {
    // non-negative floats order like their bit patterns; 0 - lo and hi + 0
    // turn a negative zero into +0 so it cannot win the unsigned max
    atomicMax(p.row_range + 2 * static_cast<size_t>(m), __float_as_uint(__fsub_rn(0.0f, rlo)));
    atomicMax(p.row_range + 2 * static_cast<size_t>(m) + 1, __float_as_uint(__fadd_rn(rhi, 0.0f)));
  }
}

// Tile order of the persistent loops.  Tiles are walked in groups of
// group_m consecutive M tiles: inside a group M varies fastest, then N; the
// groups follow each other along M.  The tiles in flight at one time then
// share a band of A rows and a band of B columns.  group_m = m_tiles is the
// plain M-fastest order, in which every wave of tiles re-reads all of A: right
// when A is small enough to stay in L2, wasteful when it is not (the MLP down
// projection's A is 75 MB at 4608 x 16384).
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int group_m, int n_tiles,
                                            int& mt, int& nt) {
  const int per_group = group_m * n_tiles;
  const int g = tile / per_group;
  const int first = g * group_m;
  const int gm = min(group_m, m_tiles - first);
  const int local = tile - g * per_group;
  mt = first + local % gm;
  nt = local / gm;
}

template <bool I8, int BN, int EPI>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmParams p) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;                       // [STAGES]
  uint64_t* empty = bars + C::STAGES;          // [STAGES]
  uint64_t* tfull = bars + 2 * C::STAGES;      // [2]
  uint64_t* tempty = bars + 2 * C::STAGES + 2; // [2]
  uint64_t* drain = bars + 2 * C::STAGES + 4;  // MMA drain on the error path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 5);
  uint64_t* cols_ready = bars + 2 * C::STAGES + 6;   // [2] column tables staged
  float* col_sw = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES + 256);   // [2][BN]
  int32_t* col_rs = reinterpret_cast<int32_t*>(col_sw + 2 * BN);                        // [2][BN]
  float* col_b = reinterpret_cast<float*>(col_rs + 2 * BN);                             // [2][BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int m_tiles = (p.M + GEMM_BM - 1) / GEMM_BM;
  const int n_tiles = (p.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = p.num_kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], GEMM_EPI_WARPS);
    }
    mbar_init(drain, 1);
    for (int a = 0; a < 2; ++a) mbar_init(&cols_ready[a], GEMM_EPI_WARPS);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();      // the previous kernel's outputs are complete from here on
  pdl_trigger();

  constexpr int ELEMS_PER_KB = I8 ? 128 : 64;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt;
        tile_coords(tile, m_tiles, p.group_m, n_tiles, mt, nt);
        const int m0 = mt * GEMM_BM;
        const int n0 = nt * BN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(&tmA, &full[stage], sA + stage * C::A_BYTES, kb * ELEMS_PER_KB, m0);
          tma_load_2d(&tmB, &full[stage], sB + stage * C::B_BYTES, kb * ELEMS_PER_KB, n0);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Drain: wait (bounded) for the last load armed on every stage to land
        // before the CTA may exit, so no bulk copy writes into released shared
        // memory.  Stages below `stage` were last armed in the current lap
        // (parity `phase`), the others in the previous lap (parity phase ^ 1;
        // a stage never armed passes that test at once).
        for (int s = 0; s < C::STAGES; ++s) {
          const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < QI_WAIT_NS) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc(I8, GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, p.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = umma_desc_kmajor_sw128(smem_u32(sA + stage * C::A_BYTES));
          const uint64_t bdesc = umma_desc_kmajor_sw128(smem_u32(sB + stage * C::B_BYTES));
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // 4 x 32 bytes of K per stage
            const uint64_t off = static_cast<uint64_t>(k * 32) >> 4;
            if (I8)
              umma_i8(d_tmem, adesc + off, bdesc + off, idesc, (kb | k) != 0);
            else
              umma_f16(d_tmem, adesc + off, bdesc + off, idesc, (kb | k) != 0);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        // make sure no MMA is still writing TMEM before it is released
        umma_commit(drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;          // 0: warps 2-5, 1: warps 6-9
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mt, nt;
      tile_coords(tile, m_tiles, p.group_m, n_tiles, mt, nt);
      const int m0 = mt * GEMM_BM;
      const int n0 = nt * BN;
      const ColTable ct{col_sw + acc * BN, col_rs + acc * BN, col_b + acc * BN};
      stage_columns<I8, BN>(p, col_sw + acc * BN, col_rs + acc * BN, col_b + acc * BN, n0,
                            threadIdx.x - 64, &cols_ready[acc]);
      if (!mbar_wait_warp(&cols_ready[acc], acc_phase, p.status)) break;
      if (!mbar_wait_warp(&tfull[acc], acc_phase, p.status)) break;
      tc_fence_after();
      epilogue_tile<I8, BN, EPI, false>(p, ct, tmem_base + static_cast<uint32_t>(acc * BN), m0, n0,
                                        quarter, half, lane, smem_u32(&tempty[acc]));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA-pair int8 GEMM
//
// Two CTAs of a cluster (one per SM) share one 256 x 256 tile: CTA r loads rows
// m0 + 128 r .. +127 of A and rows n0 + 128 r .. +127 of B into its own shared
// memory, and the even CTA issues tcgen05.mma.cta_group::2 (M = 256, N = 256),
// which reads both CTAs' operands and accumulates rows 128 r .. +127 of the
// tile into CTA r's TMEM.  Each SM then streams 256 bytes of operands per 128
// bytes of K instead of 384, the operand traffic that bounds the single-CTA
// 128 x 256 tile.  Barriers:
//   full[s]   even CTA: both CTAs' TMA loads of stage s complete on it (the even
//             CTA's producer arms it with the bytes of both)
//   empty[s]  in each CTA: stage s of that CTA may be refilled (multicast commit)
//   tfull[a]  in each CTA: accumulator buffer a is complete (multicast commit)
//   tempty[a] even CTA: all 16 epilogue warps of the pair have drained buffer a

constexpr int PAIR_STAGES = 6;
constexpr int PAIR_A_BYTES = 128 * GEMM_BK_BYTES;
constexpr int PAIR_B_BYTES = 128 * GEMM_BK_BYTES;
constexpr int PAIR_STAGE_BYTES = PAIR_A_BYTES + PAIR_B_BYTES;
constexpr int PAIR_COL_BYTES = 2 * 256 * 12;
constexpr int PAIR_SMEM_BYTES = 1024 + PAIR_STAGES * PAIR_STAGE_BYTES + 256 + PAIR_COL_BYTES;
static_assert(3 * PAIR_STAGES + 8 <= 32, "barrier area");
// MXFP4 B operand: each stage's E2M1 codes of this CTA's 128 B rows (32 bytes a
// row) are brought in by TMA before the converter warps decode them
constexpr int MX_CODE_BYTES = 128 * 32;
constexpr int PAIR_SMEM_BYTES_MX = PAIR_SMEM_BYTES + PAIR_STAGES * MX_CODE_BYTES;
static_assert(PAIR_SMEM_BYTES_MX <= 232448, "shared memory per CTA");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Every thread of both CTAs; orders shared-memory and barrier set-up (release /
// acquire at cluster scope).  The non-.aligned form: lanes may arrive apart.
__device__ __forceinline__ void cluster_sync_all() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
  __syncwarp();
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for a phase completed by arrivals from both CTAs of the pair.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int* status) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (has_error(status)) return false;
    if (globaltimer_ns() - t0 > QI_WAIT_NS) {
      set_error(status, QI_DEV_ERR_TIMEOUT);
      return false;
    }
  }
}

// TMA tile load into this CTA's shared memory whose completion is counted on
// an mbarrier of either CTA of the pair (`bar_cluster` is a shared::cluster
// address).  Plain load: no multicast.
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap* map, uint32_t bar_cluster,
                                                 void* smem, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t a, uint64_t b,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}

// Arrive on the barrier at this offset in every CTA of `mask` once all MMAs
// issued so far by this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// TMEM allocation / release for a CTA pair: one warp of each CTA executes it;
// the same columns are allocated in both SMs.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// ---------------------------------------------------------------- MXFP4 B operand
//
// MXFP4 weights (EliovpAI "Qwen_Image-2.1-MXFP4-Paiton-RDNA4", "What was
// quantized": E2M1 values packed two per byte, low nibble first, one E8M0
// scale per 32 input columns) are decoded to bf16 inside the GEMM's load
// path, so HBM holds 4.25 bits per weight.  E2M1 magnitudes are 0, 0.5, 1,
// 1.5, 2, 3, 4, 6 (exponent bias 1, one mantissa bit), E8M0 is 2^(e - 127)
// (255 = NaN); every product e2m1 x 2^(e - 127) has at most two significant
// bits, so its bf16 value is exact.
constexpr int MX_WARPS = 4;   // converter warps per CTA (one B row per thread)

// With MXB the B operand is MXFP4 (bf16 A, kind::f16): MX_WARPS extra warps
// per CTA decode this CTA's 128 B rows of each stage into the 128-byte
// swizzled bf16 layout that TMA would have written, fence the writes for the
// tensor core and arrive on the even CTA's full barrier.
template <bool I8, int EPI, bool MXB = false>
__global__ void __launch_bounds__(MXB ? GEMM_THREADS + 32 * MX_WARPS : GEMM_THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmParams p) {
  constexpr int BN = 256;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sA = smem;
  uint8_t* sB = smem + PAIR_STAGES * PAIR_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PAIR_STAGES * PAIR_STAGE_BYTES);
  uint64_t* full = bars;                          // [STAGES] (even CTA)
  uint64_t* empty = bars + PAIR_STAGES;           // [STAGES]
  uint64_t* tfull = bars + 2 * PAIR_STAGES;       // [2]
  uint64_t* tempty = bars + 2 * PAIR_STAGES + 2;  // [2] (even CTA)
  uint64_t* drain = bars + 2 * PAIR_STAGES + 4;   // MMA drain on the error path
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * PAIR_STAGES + 5);
  uint64_t* cols_ready = bars + 2 * PAIR_STAGES + 6;   // [2] column tables staged
  float* col_sw = reinterpret_cast<float*>(smem + PAIR_STAGES * PAIR_STAGE_BYTES + 256);   // [2][BN]
  int32_t* col_rs = reinterpret_cast<int32_t*>(col_sw + 2 * BN);                            // [2][BN]
  float* col_b = reinterpret_cast<float*>(col_rs + 2 * BN);                                 // [2][BN]
  uint8_t* sC = reinterpret_cast<uint8_t*>(col_b + 2 * BN);    // MXB: [STAGES][128 rows][32 B] codes
  uint64_t* c_full = bars + 2 * PAIR_STAGES + 8;               // MXB: [STAGES] codes landed (own CTA)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const int m_tiles = (p.M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  const int n_tiles = (p.N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int num_kb = p.num_kb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PAIR_STAGES; ++s) {
      mbar_init(&full[s], MXB ? 1 + 2 * MX_WARPS : 1);   // + the converter warps of both CTAs
      mbar_init(&empty[s], 1);
      if (MXB) mbar_init(&c_full[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * GEMM_EPI_WARPS);
      mbar_init(&cols_ready[a], GEMM_EPI_WARPS);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * BN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();   // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();      // the previous kernel's outputs are complete from here on
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        int mt, nt;
        tile_coords(tile, m_tiles, p.group_m, n_tiles, mt, nt);
        const int m0 = mt * (2 * GEMM_BM) + static_cast<int>(rank) * GEMM_BM;
        const int n0 = nt * BN + static_cast<int>(rank) * (BN / 2);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.status)) { ok = false; break; }
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&full[stage], MXB ? 2 * PAIR_A_BYTES : 2 * PAIR_STAGE_BYTES);
          // one 128-byte K row per stage: 128 int8 or 64 bf16 elements
          tma_load_2d_pair(&tmA, fb, sA + stage * PAIR_A_BYTES, kb * (I8 ? 128 : 64), m0);
          if (!MXB) {
            tma_load_2d_pair(&tmB, fb, sB + stage * PAIR_B_BYTES, kb * (I8 ? 128 : 64), n0);
          } else {
            // this CTA's rows of the stage's MXFP4 codes, for its converter warps
            mbar_arrive_expect_tx(&c_full[stage], MX_CODE_BYTES);
            tma_load_2d(&tmB, &c_full[stage], sC + stage * MX_CODE_BYTES, kb * 32, n0);
          }
          if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // Error path: the loads in flight must land before the CTAs exit.  The
        // even CTA waits (bounded) on the full barriers it armed, which also
        // count the odd CTA's bytes; the odd CTA, which cannot wait on the even
        // CTA's barriers, gives its last loads a fixed 200 us.
        if (MXB) {   // this CTA's own code loads
          for (int s = 0; s < PAIR_STAGES; ++s) {
            const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&c_full[s], par) && globaltimer_ns() - t0 < QI_WAIT_NS) {
            }
          }
        }
        if (rank == 0) {
          for (int s = 0; s < PAIR_STAGES; ++s) {
            const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < QI_WAIT_NS) {
            }
          }
        } else {
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 200000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = umma_idesc(I8, 2 * GEMM_BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
        if (!mbar_wait_cluster(&tempty[acc], acc_phase ^ 1u, p.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          // (with MXB the stage also holds the converters' shared-memory
          // writes of both CTAs, released at cluster scope)
          if (!(MXB ? mbar_wait_cluster(&full[stage], phase, p.status)
                    : mbar_wait(&full[stage], phase, p.status))) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = umma_desc_kmajor_sw128(smem_u32(sA + stage * PAIR_A_BYTES));
          const uint64_t bdesc = umma_desc_kmajor_sw128(smem_u32(sB + stage * PAIR_B_BYTES));
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // 4 x 32 bytes of K per stage
            const uint64_t off = static_cast<uint64_t>(k * 32) >> 4;
            if (I8)
              umma_i8_pair(d_tmem, adesc + off, bdesc + off, idesc, (kb | k) != 0);
            else
              umma_f16_pair(d_tmem, adesc + off, bdesc + off, idesc, (kb | k) != 0);
          }
          umma_commit_pair(&empty[stage], 0x3);
          if (++stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&tfull[acc], 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        // make sure no MMA is still writing TMEM before it is released
        umma_commit_pair(drain, 0x1);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
        }
      }
    }
  } else if (MXB && warp >= 2 + GEMM_EPI_WARPS) {
    // ------------------------------------------------------------ MXFP4 converters (both CTAs)
    // thread t decodes row n0 + t of this CTA's B half: per stage the row's 64
    // codes (32 bytes, brought to shared memory by the producer's TMA) and its
    // two E8M0 scales (read 8 bytes = 4 stages at a time, one batch ahead).
    // Stages are filled two at a time: one proxy fence and one arrival per
    // stage pair, so the hand-over to the tensor core is paid half as often.
    constexpr int MX_BATCH = 2;
    static_assert(PAIR_STAGES % MX_BATCH == 0, "stage pairs must not straddle the ring");
    const int t = threadIdx.x - 32 * (2 + GEMM_EPI_WARPS);
    const size_t kscl = static_cast<size_t>(p.K) / 32;
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = pair; tile < num_tiles && ok; tile += num_pairs) {
      int mt, nt;
      tile_coords(tile, m_tiles, p.group_m, n_tiles, mt, nt);
      const int n = nt * BN + static_cast<int>(rank) * (BN / 2) + t;
      const bool n_ok = n < p.N;
      const uint2* srow = reinterpret_cast<const uint2*>(p.b_scales + (n_ok ? n : 0) * kscl);
      uint2 sc_next = n_ok ? __ldg(srow) : make_uint2(0, 0);
      uint2 sc_cur = sc_next;
#pragma unroll 1
      for (int kb0 = 0; kb0 < num_kb; kb0 += MX_BATCH) {   // num_kb % 4 == 0 (k % 256 == 0)
        if ((kb0 & 3) == 0) {   // scales of stages kb0 .. kb0+3; prefetch the next four
          sc_cur = sc_next;
          if (n_ok && kb0 + 4 < num_kb) sc_next = __ldg(srow + (kb0 >> 2) + 1);
        }
        uint32_t o[MX_BATCH][32];
#pragma unroll
        for (int u = 0; u < MX_BATCH; ++u) {
          const int kb = kb0 + u;
          const uint32_t sw = (kb & 2) ? sc_cur.y : sc_cur.x;
          const uint32_t dsc = (kb & 1) ? (sw >> 16) : (sw & 0xFFFFu);
          if (!mbar_wait_warp(&c_full[stage + u], phase, p.status)) { ok = false; break; }
          const uint4* code = reinterpret_cast<const uint4*>(sC + (stage + u) * MX_CODE_BYTES + t * 32);
          const uint4 d0 = code[0], d1 = code[1];
          uint32_t a[16], b[16];
          mx_decode32(dsc & 0xFFu, d0, a);
          mx_decode32(dsc >> 8, d1, b);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            o[u][i] = n_ok ? a[i] : 0u;
            o[u][16 + i] = n_ok ? b[i] : 0u;
          }
        }
        if (!ok) break;
#pragma unroll
        for (int u = 0; u < MX_BATCH; ++u) {
          if (!mbar_wait_warp(&empty[stage + u], phase ^ 1u, p.status)) { ok = false; break; }
          // 128-byte swizzle: 16-byte chunk c of row t goes to chunk c ^ (t & 7)
          uint8_t* row = sB + (stage + u) * PAIR_B_BYTES + t * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(row + ((c ^ (t & 7)) << 4)) =
                make_uint4(o[u][4 * c], o[u][4 * c + 1], o[u][4 * c + 2], o[u][4 * c + 3]);
        }
        if (!ok) break;
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int u = 0; u < MX_BATCH; ++u) {
            const uint32_t fr = mapa_shared(smem_u32(&full[stage + u]), 0);
            asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(fr)
                         : "memory");
          }
        }
        stage += MX_BATCH;
        if (stage == PAIR_STAGES) { stage = 0; phase ^= 1u; }
      }
    }
  } else if (warp >= 2 && warp < 2 + GEMM_EPI_WARPS) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += num_pairs) {
      int mt, nt;
      tile_coords(tile, m_tiles, p.group_m, n_tiles, mt, nt);
      const int m0 = mt * (2 * GEMM_BM) + static_cast<int>(rank) * GEMM_BM;
      const int n0 = nt * BN;
      const ColTable ct{col_sw + acc * BN, col_rs + acc * BN, col_b + acc * BN};
      stage_columns<I8, BN>(p, col_sw + acc * BN, col_rs + acc * BN, col_b + acc * BN, n0,
                            threadIdx.x - 64, &cols_ready[acc]);
      if (!mbar_wait_warp(&cols_ready[acc], acc_phase, p.status)) break;
      if (!mbar_wait_warp(&tfull[acc], acc_phase, p.status)) break;
      tc_fence_after();
      epilogue_tile<I8, BN, EPI, true>(p, ct, tmem_base + static_cast<uint32_t>(acc * BN), m0, n0,
                                         quarter, half, lane, mapa_shared(smem_u32(&tempty[acc]), 0));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  // Neither CTA leaves (or frees TMEM) while the other may still read its
  // shared memory, arrive on its barriers, or have MMAs writing its TMEM.
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * BN);
  }
}

// ---------------------------------------------------------------- host side

template <bool I8, int BN, int EPI>
static int launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                         int num_sms, cudaStream_t st) {
  using C = GemmCfg<BN>;
  auto kern = gemm_kernel<I8, BN, EPI>;
  static bool attr_set = false;   // per instantiation
  if (!attr_set) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) {
      launch_result();
      return -1;
    }
    attr_set = true;
  }
  const int tiles = ((p.M + GEMM_BM - 1) / GEMM_BM) * ((p.N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  launch_pdl(kern, dim3(grid), dim3(GEMM_THREADS), C::SMEM_BYTES, st, 1, ta, tb, p);
  return launch_result();
}


// Clusters of two that can be resident at once (0 if the pair kernel cannot run).
template <bool I8, int EPI, bool MXB = false>
static int pair_capacity() {
  static int cap = -1;   // per instantiation
  if (cap < 0) {
    auto kern = gemm_pair_kernel<I8, EPI, MXB>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             MXB ? PAIR_SMEM_BYTES_MX : PAIR_SMEM_BYTES) != cudaSuccess) {
      launch_result();
      return cap = 0;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(MXB ? GEMM_THREADS + 32 * MX_WARPS : GEMM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = MXB ? PAIR_SMEM_BYTES_MX : PAIR_SMEM_BYTES;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
      launch_result();
      n = 0;
    }
    cap = n;
  }
  return cap;
}

template <bool I8, int EPI, bool MXB = false>
static int launch_gemm_pair(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                            int max_pairs, cudaStream_t st) {
  const int tiles = ((p.M + 2 * GEMM_BM - 1) / (2 * GEMM_BM)) * ((p.N + 255) / 256);
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  launch_pdl(gemm_pair_kernel<I8, EPI, MXB>, dim3(2 * pairs),
             dim3(MXB ? GEMM_THREADS + 32 * MX_WARPS : GEMM_THREADS),
             MXB ? PAIR_SMEM_BYTES_MX : PAIR_SMEM_BYTES, st, 2, ta, tb, p);
  return launch_result();
}

// BF16 GEMM whose B operand is MXFP4 (p.b_packed [N, K/2] codes, p.b_scales
// [N, K/32] E8M0), decoded in the load path; CTA pairs, N % 256 == 0.
static int launch_gemm_mx(int epi, const void* A, int lda, const GemmParams& p, int num_sms,
                          cudaStream_t st) {
  int max_pairs = 0;
  switch (epi) {
    case EPI_BF16: max_pairs = pair_capacity<false, EPI_BF16, true>(); break;
    case EPI_GELU: max_pairs = pair_capacity<false, EPI_GELU, true>(); break;
    case EPI_GATED: max_pairs = pair_capacity<false, EPI_GATED, true>(); break;
    case EPI_QKV: max_pairs = pair_capacity<false, EPI_QKV, true>(); break;
    default: return -1;
  }
  max_pairs = max_pairs < num_sms / 2 ? max_pairs : num_sms / 2;
  if (max_pairs < 1 || p.N % 256 != 0 || p.K % 256 != 0 || (epi == EPI_QKV && p.H % 256 != 0))
    return -1;
  GemmParams q = p;
  const int m_tiles = (p.M + 2 * GEMM_BM - 1) / (2 * GEMM_BM);
  q.group_m = m_tiles;   // B is small (4.25 bits per weight); A stays in L2
  CUtensorMap ta, tc;
  if (!make_tmap_2d(&ta, A, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<uint64_t>(p.K),
                    static_cast<uint64_t>(p.M), static_cast<uint64_t>(lda) * 2, 64, GEMM_BM))
    return -2;
  // the packed codes [N, K/2] bytes: a box of 32 bytes (one stage) x 128 rows, unswizzled
  if (!make_tmap_2d(&tc, p.b_packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<uint64_t>(p.K) / 2,
                    static_cast<uint64_t>(p.N), static_cast<uint64_t>(p.K) / 2, 32, 128, false))
    return -2;
  switch (epi) {
    case EPI_BF16: return launch_gemm_pair<false, EPI_BF16, true>(ta, tc, q, max_pairs, st);
    case EPI_GELU: return launch_gemm_pair<false, EPI_GELU, true>(ta, tc, q, max_pairs, st);
    case EPI_GATED: return launch_gemm_pair<false, EPI_GATED, true>(ta, tc, q, max_pairs, st);
    case EPI_QKV: return launch_gemm_pair<false, EPI_QKV, true>(ta, tc, q, max_pairs, st);
  }
  return -1;
}

template <bool I8, int EPI>
static int launch_gemm_bn(int bn, const CUtensorMap& ta, const CUtensorMap& tb,
                          const GemmParams& p, int num_sms, cudaStream_t st) {
  switch (bn) {
    case 256: return launch_gemm_t<I8, 256, EPI>(ta, tb, p, num_sms, st);
    case 128: return launch_gemm_t<I8, 128, EPI>(ta, tb, p, num_sms, st);
    case 64: return launch_gemm_t<I8, 64, EPI>(ta, tb, p, num_sms, st);
  }
  return -1;
}

int pick_block_n(int N) {
  if (N % 256 == 0 || N > 1024) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

int launch_gemm(bool int8, int epi, const void* A, int lda, const void* B, int ldb,
                const GemmParams& p, int num_sms, cudaStream_t st) {
  if (p.b_packed) return int8 ? -1 : launch_gemm_mx(epi, A, lda, p, num_sms, st);
  const int bn = pick_block_n(p.N);
  const CUtensorMapDataType dt =
      int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int esz = int8 ? 1 : 2;
  const uint32_t box_inner = GEMM_BK_BYTES / esz;
  // GEMMs with 256-wide tiles and a block-Linear epilogue run on CTA pairs
  // (each CTA loads 128 rows of A and 128 of B); the rest on single CTAs.
  int max_pairs = 0;
  if (bn == 256 && !(epi == EPI_QKV && p.H % 256 != 0)) {
    if (int8) {
      switch (epi) {
        case EPI_BF16: max_pairs = pair_capacity<true, EPI_BF16>(); break;
        case EPI_GELU: max_pairs = pair_capacity<true, EPI_GELU>(); break;
        case EPI_GATED: max_pairs = pair_capacity<true, EPI_GATED>(); break;
        case EPI_QKV: max_pairs = pair_capacity<true, EPI_QKV>(); break;
      }
    } else {
      switch (epi) {
        case EPI_BF16: max_pairs = pair_capacity<false, EPI_BF16>(); break;
        case EPI_GELU: max_pairs = pair_capacity<false, EPI_GELU>(); break;
        case EPI_GATED: max_pairs = pair_capacity<false, EPI_GATED>(); break;
        case EPI_QKV: max_pairs = pair_capacity<false, EPI_QKV>(); break;
      }
    }
    max_pairs = max_pairs < num_sms / 2 ? max_pairs : num_sms / 2;
  }
  const bool use_pair = max_pairs > 0;
  // Tile order: when A (M x K) is too large to stay in L2 next to the B
  // panels in flight, walk the tiles in two bands of M tiles so that each
  // wave of tiles reads half of A instead of all of it.
  GemmParams q = p;
  {
    const int bm = use_pair ? 2 * GEMM_BM : GEMM_BM;
    const int m_tiles = (p.M + bm - 1) / bm;
    const double a_bytes = static_cast<double>(p.M) * p.K * esz;
    q.group_m = (a_bytes > 48.0 * (1 << 20) && m_tiles >= 4) ? (m_tiles + 1) / 2 : m_tiles;
  }
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, dt, static_cast<uint64_t>(p.K), static_cast<uint64_t>(p.M),
                    static_cast<uint64_t>(lda) * esz, box_inner, GEMM_BM))
    return -2;
  if (!make_tmap_2d(&tb, B, dt, static_cast<uint64_t>(p.K), static_cast<uint64_t>(p.N),
                    static_cast<uint64_t>(ldb) * esz, box_inner,
                    static_cast<uint32_t>(use_pair ? bn / 2 : bn)))
    return -2;
  if (use_pair) {
    if (int8) {
      switch (epi) {
        case EPI_BF16: return launch_gemm_pair<true, EPI_BF16>(ta, tb, q, max_pairs, st);
        case EPI_GELU: return launch_gemm_pair<true, EPI_GELU>(ta, tb, q, max_pairs, st);
        case EPI_GATED: return launch_gemm_pair<true, EPI_GATED>(ta, tb, q, max_pairs, st);
        case EPI_QKV: return launch_gemm_pair<true, EPI_QKV>(ta, tb, q, max_pairs, st);
      }
    } else {
      switch (epi) {
        case EPI_BF16: return launch_gemm_pair<false, EPI_BF16>(ta, tb, q, max_pairs, st);
        case EPI_GELU: return launch_gemm_pair<false, EPI_GELU>(ta, tb, q, max_pairs, st);
        case EPI_GATED: return launch_gemm_pair<false, EPI_GATED>(ta, tb, q, max_pairs, st);
        case EPI_QKV: return launch_gemm_pair<false, EPI_QKV>(ta, tb, q, max_pairs, st);
      }
    }
    return -1;
  }
  if (int8) {
    switch (epi) {
      case EPI_BF16: return launch_gemm_bn<true, EPI_BF16>(bn, ta, tb, q, num_sms, st);
      case EPI_GELU: return launch_gemm_bn<true, EPI_GELU>(bn, ta, tb, q, num_sms, st);
      case EPI_GATED: return launch_gemm_bn<true, EPI_GATED>(bn, ta, tb, q, num_sms, st);
      case EPI_QKV:   // each epilogue half-tile must hold a whole head of one of q, k, v
        if (bn == 256 && p.H % 256 == 0) return launch_gemm_t<true, 256, EPI_QKV>(ta, tb, q, num_sms, st);
        return -1;
    }
  } else {
    switch (epi) {
      case EPI_BF16: return launch_gemm_bn<false, EPI_BF16>(bn, ta, tb, q, num_sms, st);
      case EPI_GELU: return launch_gemm_bn<false, EPI_GELU>(bn, ta, tb, q, num_sms, st);
      case EPI_GATED: return launch_gemm_bn<false, EPI_GATED>(bn, ta, tb, q, num_sms, st);
      case EPI_F32: return launch_gemm_bn<false, EPI_F32>(bn, ta, tb, q, num_sms, st);
      case EPI_EULER: return launch_gemm_bn<false, EPI_EULER>(bn, ta, tb, q, num_sms, st);
      case EPI_QKV:
        if (bn == 256 && p.H % 256 == 0) return launch_gemm_t<false, 256, EPI_QKV>(ta, tb, q, num_sms, st);
        return -1;
    }
  }
  return -1;
}

}  // namespace qi
