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
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256;
  static_assert(2 * STAGES + 5 <= 31, "barrier area");
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

// W8A8 dequantization of 32 accumulator columns starting at column nb,
// rounded to bf16 (the Linear's output dtype).
__device__ __forceinline__ void dequant32_bf16(const GemmParams& p, const uint32_t (&r)[32], int nb,
                                               float sa, int32_t zp, float (&y)[32]) {
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const int n = nb + j;
    const float b = p.bias ? bf16_bits_to_float(__ldg(p.bias + n)) : 0.f;
    const int32_t corr = static_cast<int32_t>(r[j]) - zp * __ldg(p.rowsum + n);
    y[j] = bf16_round_f(fmaf(static_cast<float>(corr) * sa, __ldg(p.s_w + n), b));
  }
}

// Fused epilogue of the QKV projection: the W columns handled by one epilogue
// warp are W/128 whole heads of q, k or v.  For q and k each head row is read from TMEM
// twice: once for the sum of squares of its bf16 values, once to apply
//   r = 1/sqrt(mean + eps), n = bf16(y r), y' = bf16(n w)     (cast before scale)
//   (a, b) -> (bf16(a c - b s), bf16(a s + b c))              (RoPE, pair = column/2)
// with explicitly rounded fp32 operations; v is stored as bf16(y).
template <int W>
__device__ __forceinline__ void qkv_epilogue(const GemmParams& p, uint32_t t_row, int m,
                                             bool row_ok, float sa, int32_t zp, int n0, int lane,
                                             uint64_t* tempty_bar) {
  const int which = n0 / p.H;
  const int col0 = n0 - which * p.H;
  uint16_t* out = which == 0 ? p.q_out : (which == 1 ? p.k_out : p.v_out_bf16);
  const uint16_t* w = which == 0 ? p.wq : p.wk;
#pragma unroll 1
  for (int hh = 0; hh < W / 128; ++hh) {
    float rs = 1.0f;
    if (which < 2) {
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + hh * 128 + c * 32, r);
        if (row_ok) {
          float y[32];
          dequant32_bf16(p, r, n0 + hh * 128 + c * 32, sa, zp, y);
#pragma unroll
          for (int j = 0; j < 32; ++j) ss = __fadd_rn(ss, __fmul_rn(y[j], y[j]));
        }
      }
      rs = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, 128.0f), p.eps)));
    }
#pragma unroll 1
    for (int c = 0; c < 4; ++c) {
      uint32_t r[32];
      tmem_ld32(t_row + hh * 128 + c * 32, r);
      if (hh == W / 128 - 1 && c == 3) {   // this warp's last TMEM read of the accumulator
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar);
      }
      if (!row_ok) continue;
      float y[32];
      dequant32_bf16(p, r, n0 + hh * 128 + c * 32, sa, zp, y);
      uint32_t pk[16];
      if (which < 2) {
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
            const float a = bf16_round_f(__fmul_rn(bf16_round_f(__fmul_rn(y[2 * i], rs)),
                                                   __uint_as_float(ww[t] << 16)));
            const float b = bf16_round_f(__fmul_rn(bf16_round_f(__fmul_rn(y[2 * i + 1], rs)),
                                                   __uint_as_float(ww[t] & 0xFFFF0000u)));
            pk[i] = pack_bf16x2(__fsub_rn(__fmul_rn(a, cs[t]), __fmul_rn(b, si[t])),
                                __fadd_rn(__fmul_rn(a, si[t]), __fmul_rn(b, cs[t])));
          }
        }
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_bf16x2(y[2 * i], y[2 * i + 1]);
      }
      uint4* dst = reinterpret_cast<uint4*>(out + static_cast<size_t>(m) * p.ldo + col0 +
                                            hh * 128 + c * 32);
#pragma unroll
      for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
  }
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

  constexpr int ELEMS_PER_KB = I8 ? 128 : 64;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * GEMM_BM;
        const int n0 = (tile / m_tiles) * BN;
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
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * GEMM_BM;
      const int n0 = (tile / m_tiles) * BN;
      if (!mbar_wait_warp(&tfull[acc], acc_phase, p.status)) break;
      tc_fence_after();
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
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      if constexpr (EPI == EPI_QKV) {
        qkv_epilogue<BN / 2>(p, t_row + half * (BN / 2), m, row_ok, sa, zp, n0 + half * (BN / 2),
                             lane, &tempty[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        continue;
      }
      float rlo = 0.f, rhi = 0.f;   // GELU: row range of this warp's half tile
#pragma unroll 1
      for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
        uint32_t r[32];
        tmem_ld32(t_row + c * 32, r);
        if (c == (half + 1) * (BN / 64) - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
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
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int n = nb + j;
          const int nn = n < p.N ? n : p.N - 1;
          const float b = p.bias ? bf16_bits_to_float(__ldg(p.bias + nn)) : 0.f;
          if (I8) {
            const int32_t corr = static_cast<int32_t>(r[j]) - zp * __ldg(p.rowsum + nn);
            v[j] = fmaf(static_cast<float>(corr) * sa, __ldg(p.s_w + nn), b);
          } else {
            v[j] = __uint_as_float(r[j]) + b;
          }
        }
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
          // x += gate * bf16(y)  (fp32 residual stream)
          float4* dst = reinterpret_cast<float4*>(p.yf + static_cast<size_t>(m) * p.ldyf + nb);
          const uint4* g4 =
              reinterpret_cast<const uint4*>(p.gate + static_cast<size_t>(rs) * p.gate_ld + nb);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (8 * j >= ncols) break;
            const uint4 gr = __ldg(g4 + j);
            const uint32_t gw[4] = {gr.x, gr.y, gr.z, gr.w};
            float4 a = dst[2 * j], b = dst[2 * j + 1];
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
  kern<<<grid, GEMM_THREADS, C::SMEM_BYTES, st>>>(ta, tb, p);
  return launch_result();
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
  const int bn = pick_block_n(p.N);
  const CUtensorMapDataType dt =
      int8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int esz = int8 ? 1 : 2;
  const uint32_t box_inner = GEMM_BK_BYTES / esz;
  CUtensorMap ta, tb;
  if (!make_tmap_2d(&ta, A, dt, static_cast<uint64_t>(p.K), static_cast<uint64_t>(p.M),
                    static_cast<uint64_t>(lda) * esz, box_inner, GEMM_BM))
    return -2;
  if (!make_tmap_2d(&tb, B, dt, static_cast<uint64_t>(p.K), static_cast<uint64_t>(p.N),
                    static_cast<uint64_t>(ldb) * esz, box_inner, static_cast<uint32_t>(bn)))
    return -2;
  if (int8) {
    switch (epi) {
      case EPI_BF16: return launch_gemm_bn<true, EPI_BF16>(bn, ta, tb, p, num_sms, st);
      case EPI_GELU: return launch_gemm_bn<true, EPI_GELU>(bn, ta, tb, p, num_sms, st);
      case EPI_GATED: return launch_gemm_bn<true, EPI_GATED>(bn, ta, tb, p, num_sms, st);
      case EPI_QKV:   // each epilogue half-tile must hold a whole head of one of q, k, v
        if (bn == 256 && p.H % 256 == 0) return launch_gemm_t<true, 256, EPI_QKV>(ta, tb, p, num_sms, st);
        return -1;
    }
  } else {
    switch (epi) {
      case EPI_BF16: return launch_gemm_bn<false, EPI_BF16>(bn, ta, tb, p, num_sms, st);
      case EPI_F32: return launch_gemm_bn<false, EPI_F32>(bn, ta, tb, p, num_sms, st);
      case EPI_EULER: return launch_gemm_bn<false, EPI_EULER>(bn, ta, tb, p, num_sms, st);
    }
  }
  return -1;
}

}  // namespace qi
