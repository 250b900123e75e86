// Bandwidth-bound kernels of the step:
//  * Q/K RMSNorm with the cast ordering of "Qwen Image 2.1 native qualification"
//    (Numerical checks: the normalized activation is cast to the scale's dtype
//    before the scale multiplies) fused with 3-axis RoPE ("RGBA-Image-2.1 - Core
//    AI port of Qwen-Image-2.1", Graph contracts / RoPE: 64 rotation pairs per
//    128-wide head from per-token cos/sin tables);
//  * the thin GEMV behind the timestep MLP and the adaLN modulation rows
//    (qwen-image-mnn, "What runs where": modulation rows), M <= 2 rows;
//  * the sinusoidal timestep embedding, fp32 -> bf16 casts and the FlowMatch
//    Euler update x += (sigma_next - sigma) * v (Core AI port, Sampler).
#include <math.h>

#include "qi_common.cuh"
#include "qi_mx.cuh"
#include "qi_internal.h"

namespace qi {

// ---------------------------------------------------------------- Q/K norm + RoPE

// One CTA per token, 8 warps; warp w handles head slots w, w+8, ... of the
// 3*heads slots (q heads, k heads, v heads).  Lane l holds elements 4l..4l+3
// of the 128-wide head, i.e. rotation pairs 2l and 2l+1.
// Arithmetic is fp32 with explicitly rounded operations (no contraction):
//   r = 1 / sqrt(sum(x^2)/128 + eps);  n = bf16(x * r);  y = bf16(n * w)
//   (a, b) -> (bf16(a c - b s), bf16(a s + b c))
__global__ void __launch_bounds__(256) qk_norm_rope_kernel(const QkNormRopeParams p) {
  const int t = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int H = p.heads * p.d;
  const uint16_t* row = p.qkv + static_cast<int64_t>(t) * p.ldqkv;
  const float2 cs = *reinterpret_cast<const float2*>(p.cos + static_cast<int64_t>(t) * (p.d / 2) + 2 * lane);
  const float2 sn = *reinterpret_cast<const float2*>(p.sin + static_cast<int64_t>(t) * (p.d / 2) + 2 * lane);
  for (int hs = warp; hs < 3 * p.heads; hs += 8) {
    const int which = hs / p.heads, h = hs - which * p.heads;
    const uint2 raw = *reinterpret_cast<const uint2*>(row + which * H + h * p.d + lane * 4);
    uint16_t* dst = (which == 0 ? p.q_out : (which == 1 ? p.k_out : p.v_out)) +
                    static_cast<int64_t>(t) * p.ldo + h * p.d + lane * 4;
    if (which == 2) {
      *reinterpret_cast<uint2*>(dst) = raw;
      continue;
    }
    float x[4] = {__uint_as_float(raw.x << 16), __uint_as_float(raw.x & 0xFFFF0000u),
                  __uint_as_float(raw.y << 16), __uint_as_float(raw.y & 0xFFFF0000u)};
    float ss = __fadd_rn(__fadd_rn(__fmul_rn(x[0], x[0]), __fmul_rn(x[1], x[1])),
                         __fadd_rn(__fmul_rn(x[2], x[2]), __fmul_rn(x[3], x[3])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, o));
    const float ms = __fdiv_rn(ss, static_cast<float>(p.d));
    const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.eps)));
    const uint2 wraw = *reinterpret_cast<const uint2*>((which == 0 ? p.wq : p.wk) + lane * 4);
    const float w[4] = {__uint_as_float(wraw.x << 16), __uint_as_float(wraw.x & 0xFFFF0000u),
                        __uint_as_float(wraw.y << 16), __uint_as_float(wraw.y & 0xFFFF0000u)};
    float y[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = bf16_round_f(__fmul_rn(bf16_round_f(__fmul_rn(x[i], r)), w[i]));
    const float c0 = cs.x, c1 = cs.y, s0 = sn.x, s1 = sn.y;
    const float o0 = __fsub_rn(__fmul_rn(y[0], c0), __fmul_rn(y[1], s0));
    const float o1 = __fadd_rn(__fmul_rn(y[0], s0), __fmul_rn(y[1], c0));
    const float o2 = __fsub_rn(__fmul_rn(y[2], c1), __fmul_rn(y[3], s1));
    const float o3 = __fadd_rn(__fmul_rn(y[2], s1), __fmul_rn(y[3], c1));
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(o0, o1), pack_bf16x2(o2, o3));
  }
}

int launch_qk_norm_rope(const QkNormRopeParams& p, cudaStream_t st) {
  if (p.T == 0) return 0;
  if (p.d != 128) return -1;
  qk_norm_rope_kernel<<<p.T, 256, 0, st>>>(p);
  return launch_result();
}

// ---------------------------------------------------------------- GEMV

// y[r][j] = sum_k act(x[r][k]) * W[j][k] + b[j] for every row j of every job.
// x (R <= 2 rows) is staged in shared memory as fp32 (SiLU applied on load
// when requested).  One warp handles 8 consecutive weight rows at a time:
// every lane streams 8 x 16 bytes of weights per step and reuses the x values
// it read from shared memory for all 8 rows; 16 independent accumulators keep
// the FMA chains short.  The weights are read once: the kernel is bound by
// HBM bandwidth (6.4 GB of adaLN weights per 32-block step).  8 rows a warp
// keep 128 bytes a lane in flight: 1.08 ms per 1024^2 step against 1.18 with
// 4 rows (each row's sum is the same sequence of operations either way).
constexpr int GEMV_THREADS = 256;
constexpr int GEMV_ROWS = 8;

__device__ __forceinline__ float dot8(const uint4 w, const float4 a, const float4 b, float acc) {
  acc = fmaf(__uint_as_float(w.x << 16), a.x, acc);
  acc = fmaf(__uint_as_float(w.x & 0xFFFF0000u), a.y, acc);
  acc = fmaf(__uint_as_float(w.y << 16), a.z, acc);
  acc = fmaf(__uint_as_float(w.y & 0xFFFF0000u), a.w, acc);
  acc = fmaf(__uint_as_float(w.z << 16), b.x, acc);
  acc = fmaf(__uint_as_float(w.z & 0xFFFF0000u), b.y, acc);
  acc = fmaf(__uint_as_float(w.w << 16), b.z, acc);
  acc = fmaf(__uint_as_float(w.w & 0xFFFF0000u), b.w, acc);
  return acc;
}

__global__ void __launch_bounds__(GEMV_THREADS) gemv_kernel(const GemvParams p) {
  extern __shared__ float4 xs4[];
  pdl_wait();
  pdl_trigger();
  float* xs = reinterpret_cast<float*>(xs4);
  const int total_in = p.R * p.k;
  for (int i = threadIdx.x; i < total_in; i += GEMV_THREADS) {
    float v = p.x[i];
    if (p.silu_in) v = v / (1.0f + expf(-v));
    xs[i] = v;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int gwarp = (blockIdx.x * GEMV_THREADS + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * GEMV_THREADS) >> 5;
  int total = 0;
  for (int j = 0; j < p.n_jobs; ++j) total += p.jobs[j].n / GEMV_ROWS;
  const int k4 = p.k / 4;
  for (int g = gwarp; g < total; g += nwarps) {
    int job = 0, grp = g;
    while (grp >= p.jobs[job].n / GEMV_ROWS) {
      grp -= p.jobs[job].n / GEMV_ROWS;
      ++job;
    }
    const GemvJob& J = p.jobs[job];
    const int row0 = grp * GEMV_ROWS;
    const uint16_t* w0 = J.w + static_cast<int64_t>(row0) * p.k;
    float a0[GEMV_ROWS] = {}, a1[GEMV_ROWS] = {};
#pragma unroll 2
    for (int kk = lane * 8; kk < p.k; kk += 256) {
      uint4 w[GEMV_ROWS];
#pragma unroll
      for (int i = 0; i < GEMV_ROWS; ++i)
        w[i] = __ldg(reinterpret_cast<const uint4*>(w0 + static_cast<int64_t>(i) * p.k + kk));
      const float4 xa = xs4[kk / 4], xb = xs4[kk / 4 + 1];
#pragma unroll
      for (int i = 0; i < GEMV_ROWS; ++i) a0[i] = dot8(w[i], xa, xb, a0[i]);
      if (p.R > 1) {
        const float4 ya = xs4[k4 + kk / 4], yb = xs4[k4 + kk / 4 + 1];
#pragma unroll
        for (int i = 0; i < GEMV_ROWS; ++i) a1[i] = dot8(w[i], ya, yb, a1[i]);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < GEMV_ROWS; ++i) {
        a0[i] += __shfl_xor_sync(0xffffffffu, a0[i], o);
        a1[i] += __shfl_xor_sync(0xffffffffu, a1[i], o);
      }
    }
    if (lane < GEMV_ROWS * p.R) {
      const int i = lane % GEMV_ROWS, r = lane / GEMV_ROWS;
      float out = 0.f;
#pragma unroll
      for (int t = 0; t < GEMV_ROWS; ++t)
        if (t == i) out = r == 0 ? a0[t] : a1[t];
      const int row = row0 + i;
      out += J.b ? bf16_bits_to_float(J.b[row]) : 0.f;
      if (p.y_bf16) {
        __nv_bfloat16 hv = __float2bfloat16_rn(out);
        static_cast<uint16_t*>(J.y)[static_cast<int64_t>(r) * J.ldy + row] =
            *reinterpret_cast<uint16_t*>(&hv);
      } else {
        static_cast<float*>(J.y)[static_cast<int64_t>(r) * J.ldy + row] = out;
      }
    }
  }
}

int launch_gemv(const GemvParams& p, cudaStream_t st) {
  if (p.R < 1 || p.R > 2 || p.k % 256 != 0 || p.n_jobs > GEMV_MAX_JOBS) return -1;
  int total = 0;
  for (int j = 0; j < p.n_jobs; ++j) {
    if (p.jobs[j].n % GEMV_ROWS != 0) return -1;
    total += p.jobs[j].n / GEMV_ROWS;
  }
  if (total == 0) return 0;
  const size_t smem = static_cast<size_t>(p.R) * p.k * sizeof(float);
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024) != cudaSuccess) {
      launch_result();
      return -1;
    }
    attr = true;
  }
  if (smem > 64 * 1024) return -1;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_cta = GEMV_THREADS / 32;
  int grid = (total + per_cta - 1) / per_cta;
  const int max_grid = sms * 8;
  if (grid > max_grid) grid = max_grid;
  launch_pdl(gemv_kernel, dim3(grid), dim3(GEMV_THREADS), smem, st, 1, p);
  return launch_result();
}

// ---------------------------------------------------------------- small kernels

// out[r] = [cos(1000 t_r f_i), sin(1000 t_r f_i)], f_i = exp(-ln(1e4) i / 128), i < 128,
// for the two timesteps t_0 (row 0) and t_1 (row 1).  Evaluated in double.
__global__ void timestep_embedding_kernel(float t0, float t1, float* out) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  const int i = threadIdx.x;   // 0..127
  const double f = exp(-log(10000.0) * static_cast<double>(i) / 128.0);
  const double a = 1000.0 * static_cast<double>(r == 0 ? t0 : t1) * f;
  out[r * 256 + i] = static_cast<float>(cos(a));
  out[r * 256 + 128 + i] = static_cast<float>(sin(a));
}

int launch_timestep_embedding(float t0, float t1, float* out, cudaStream_t st) {
  launch_pdl(timestep_embedding_kernel, dim3(2), dim3(128), 0, st, 1, t0, t1, out);
  return launch_result();
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ x, uint16_t* __restrict__ y, int64_t n) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    __nv_bfloat16 h = __float2bfloat16_rn(x[i]);
    y[i] = *reinterpret_cast<uint16_t*>(&h);
  }
}

int launch_f32_to_bf16(const float* x, uint16_t* y, int64_t n, cudaStream_t st) {
  if (n == 0) return 0;
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  launch_pdl(f32_to_bf16_kernel, dim3(static_cast<unsigned>(g)), dim3(256), 0, st, 1, x, y, n);
  return launch_result();
}

// x += dt * v in fp32, one rounding per operation (no fused multiply-add).
__global__ void euler_kernel(float* __restrict__ x, const float* __restrict__ v, int64_t n, float dt) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    x[i] = __fadd_rn(x[i], __fmul_rn(dt, v[i]));
}

int launch_euler(float* x, const float* v, int64_t n, float dt, cudaStream_t st) {
  if (n == 0) return 0;
  int64_t g = (n + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  launch_pdl(euler_kernel, dim3(static_cast<unsigned>(g)), dim3(256), 0, st, 1, x, v, n, dt);
  return launch_result();
}

// MXFP4 weights -> fp32: w[n, k] = e2m1(code) * 2^(scale[n, k / 32] - 127).
// E2M1 codes (1 sign, 2 exponent, 1 mantissa bit): magnitudes 0, 0.5, 1, 1.5,
// 2, 3, 4, 6; two codes per byte, the lower column in the low nibble; one
// E8M0 scale byte per 32 columns (255 = NaN).  One thread per packed byte.
__global__ void mxfp4_decode_kernel(const uint8_t* __restrict__ packed,
                                    const uint8_t* __restrict__ scales, int n, int k_stored, int k,
                                    float* __restrict__ w) {
  const int bytes_per_row = k_stored / 2;
  const int64_t total = static_cast<int64_t>(n) * bytes_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int row = static_cast<int>(i / bytes_per_row);
    const int col = static_cast<int>(i % bytes_per_row) * 2;
    if (col >= k) continue;
    const uint8_t b = packed[i];
    const uint8_t e8 = scales[static_cast<int64_t>(row) * (k_stored / 32) + col / 32];
    // 2^(e8 - 127) built from its bits: exponent field e8 for e8 >= 1, the
    // denormal 2^-127 for e8 = 0; 255 encodes NaN
    const float scale = e8 == 255 ? __int_as_float(0x7FC00000)
                                  : __int_as_float(e8 == 0 ? 0x00400000 : static_cast<int>(e8) << 23);
    float out[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = (b >> (4 * h)) & 15;
      const int e = (c >> 1) & 3, m = c & 1;
      float mag = e == 0 ? 0.5f * m : (1.0f + 0.5f * m) * static_cast<float>(1 << (e - 1));
      out[h] = (c & 8) ? -mag * scale : mag * scale;
    }
    float* dst = w + static_cast<int64_t>(row) * k + col;
    dst[0] = out[0];
    if (col + 1 < k) dst[1] = out[1];
  }
}

int launch_mxfp4_decode(const uint8_t* packed, const uint8_t* scales, int n, int k_stored, int k,
                        float* w, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(n) * (k_stored / 2);
  if (total == 0) return 0;
  int64_t g = (total + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  mxfp4_decode_kernel<<<static_cast<int>(g), 256, 0, st>>>(packed, scales, n, k_stored, k, w);
  return launch_result();
}

// MXFP4 weights -> bf16, for k % 32 == 0 (no padding): the same values as the
// fp32 decode, each exact in bf16, by the GEMM's byte-table decoder
// (qi_mx.cuh).  One thread per 32-bit word of codes (8 columns): a warp reads
// 128 contiguous bytes of codes and writes 512 contiguous bytes of bf16 per
// instruction; two words per thread are in flight at once.  (The writes are
// 80% of the traffic; on B200 the kernel moves ~3.2 TB/s, about where a
// write-dominated stream levels off; 4 or 8 words per thread, fewer CTAs or
// streaming stores measured 3-15% slower.)
//
// early: the kernel reads only the weights, which no kernel writes, and
// writes a scratch buffer that the caller guarantees no earlier kernel still
// reads; it then expands while the previous kernel of the stream is still
// running (programmatic dependent launch) and waits for that kernel only at
// its end, so that a kernel waiting on this one still finds every earlier
// kernel complete.
__global__ void mxfp4_expand_bf16_kernel(const uint32_t* __restrict__ packed,
                                         const uint8_t* __restrict__ scales, int64_t words,
                                         uint4* __restrict__ w, int early) {
  constexpr int U = 2;
  if (!early) pdl_wait();
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i0 = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i0 < words;
       i0 += U * stride) {
    uint32_t c[U], e[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      c[u] = i < words ? packed[i] : 0u;
      e[u] = i < words ? scales[i >> 2] : 127u;   // four words per scale group
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t i = i0 + u * stride;
      if (i >= words) break;
      uint32_t o[4];
      if (e[u] >= 2u && e[u] <= 252u)
        mx_decode8(mx_table(e[u]), c[u], o);
      else
        mx_decode8_general(e[u], c[u], o);
      w[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  if (early) pdl_wait();
}

int launch_mxfp4_expand_bf16(const uint8_t* packed, const uint8_t* scales, int n, int k,
                             uint16_t* w, cudaStream_t st, bool early) {
  const int64_t words = static_cast<int64_t>(n) * (k / 8);
  if (words == 0) return 0;
  int64_t g = (words + 255) / 256;
  if (g > 148 * 32) g = 148 * 32;
  launch_pdl(mxfp4_expand_bf16_kernel, dim3(static_cast<unsigned>(g)), dim3(256), 0, st, 1,
             reinterpret_cast<const uint32_t*>(packed), scales, words, reinterpret_cast<uint4*>(w),
             early ? 1 : 0);
  return launch_result();
}


// bf16 -> e4m3 (nearest, ties to even, saturating at +-448), 8 values per
// thread step: the operands of the fp8 attention.
__global__ void bf16_to_e4m3_kernel(const uint4* __restrict__ x, uint2* __restrict__ y, int64_t n8) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 v = x[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint16_t h[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;"
          : "=h"(h[j])
          : "f"(__uint_as_float(w[j] & 0xFFFF0000u)), "f"(__uint_as_float(w[j] << 16)));
    y[i] = make_uint2(static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16),
                      static_cast<uint32_t>(h[2]) | (static_cast<uint32_t>(h[3]) << 16));
  }
}

int launch_bf16_to_e4m3(const uint16_t* x, uint8_t* y, int64_t n, cudaStream_t st) {
  if (n == 0) return 0;
  if (n % 8) return -1;
  const int64_t n8 = n / 8;
  int64_t g = (n8 + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  launch_pdl(bf16_to_e4m3_kernel, dim3(static_cast<unsigned>(g)), dim3(256), 0, st, 1,
             reinterpret_cast<const uint4*>(x), reinterpret_cast<uint2*>(y), n8);
  return launch_result();
}

// Classifier-free guidance (true CFG: the conditional and the unconditional
// velocities of one step) followed by the FlowMatch Euler update, element-wise
// in fp32 with one rounding per operation and no fused multiply-add:
//   v = v_u + g (v_c - v_u),  x = x + (sigma_next - sigma) v
__global__ void cfg_euler_kernel(float* __restrict__ x, const float* __restrict__ vc,
                                 const float* __restrict__ vu, int64_t n, float g, float dt,
                                 float* __restrict__ vout) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float u = vu[i];
    const float v = __fadd_rn(u, __fmul_rn(g, __fsub_rn(vc[i], u)));
    if (vout) vout[i] = v;
    x[i] = __fadd_rn(x[i], __fmul_rn(dt, v));
  }
}

int launch_cfg_euler(float* x, const float* v_c, const float* v_u, int64_t n, float g, float dt,
                     float* v_out, cudaStream_t st) {
  if (n == 0) return 0;
  int64_t gr = (n + 255) / 256;
  if (gr > 148 * 16) gr = 148 * 16;
  launch_pdl(cfg_euler_kernel, dim3(static_cast<unsigned>(gr)), dim3(256), 0, st, 1, x, v_c, v_u, n, g, dt, v_out);
  return launch_result();
}

// Failure-detection probe: wait on an mbarrier that nothing ever arrives on,
// bounded by limit_ns; the expiry is recorded in the status word.
__global__ void timeout_probe_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > limit_ns) {
        set_error(status, QI_DEV_ERR_TIMEOUT);
        break;
      }
    }
  }
}

int launch_timeout_probe(uint64_t limit_ns, int* status, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(limit_ns, status);
  return launch_result();
}

// ---------------------------------------------------------------- tensor-pipe probe
//
// Back-to-back tcgen05.mma (M = 128, N = 256, one 128-byte K row = 4 MMAs per
// iteration) on operands resident in shared memory: no loads, no epilogue, so
// the launch measures the tensor pipe's own rate at the clock the GPU holds
// while it runs.  The operands are pseudo-random (int8 bytes, or bf16 values
// of magnitude [1, 2) with random signs), so the switching activity, and with
// it the power drawn, is that of real data.  One CTA per SM.
constexpr int PROBE_A_BYTES = 128 * 128;
constexpr int PROBE_B_BYTES = 256 * 128;
constexpr int PROBE_SMEM = 1024 + PROBE_A_BYTES + PROBE_B_BYTES;

template <bool I8>
__global__ void __launch_bounds__(128, 1) mma_probe_kernel(int iters, int* status) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t done;
  __shared__ uint32_t tslot;
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint32_t* w = reinterpret_cast<uint32_t*>(sm);
  for (int i = threadIdx.x; i < (PROBE_A_BYTES + PROBE_B_BYTES) / 4; i += blockDim.x) {
    uint32_t h = static_cast<uint32_t>(i) * 2654435761u + blockIdx.x * 40503u;
    h ^= h >> 15;
    h *= 2246822519u;
    h ^= h >> 13;
    // bf16: exponent of 1.0 with a random mantissa and sign in each half
    w[i] = I8 ? h : ((h & 0x807F807Fu) | 0x3F803F80u);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (threadIdx.x < 32) {
    tmem_alloc(&tslot, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    mbar_init(&done, 1);
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tslot;
  if (threadIdx.x == 0) {
    constexpr uint32_t idesc = umma_idesc(I8, 128, 256);
    const uint64_t a = umma_desc_kmajor_sw128(smem_u32(sm));
    const uint64_t b = umma_desc_kmajor_sw128(smem_u32(sm + PROBE_A_BYTES));
    for (int it = 0; it < iters; ++it) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint64_t off = static_cast<uint64_t>(k * 32) >> 4;
        if (I8)
          umma_i8(tmem, a + off, b + off, idesc, (it | k) != 0);
        else
          umma_f16(tmem, a + off, b + off, idesc, (it | k) != 0);
      }
    }
    umma_commit(&done);
    if (!mbar_wait(&done, 0, status)) {
      // the MMAs must be finished before their TMEM is released
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(&done, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x < 32) tmem_dealloc(tmem, 256);
}

int launch_mma_probe(bool i8, int iters, int num_sms, int* status, cudaStream_t st) {
  static bool attr[2] = {false, false};
  auto kern = i8 ? mma_probe_kernel<true> : mma_probe_kernel<false>;
  if (!attr[i8]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, PROBE_SMEM) !=
        cudaSuccess) {
      launch_result();
      return -1;
    }
    attr[i8] = true;
  }
  kern<<<num_sms, 128, PROBE_SMEM, st>>>(iters, status);
  return launch_result();
}

}  // namespace qi
