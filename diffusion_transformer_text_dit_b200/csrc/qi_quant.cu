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
// One CTA per row; the row lives in registers (one thread per 32 values), so
// the input is read once from HBM and the int8 codes are written once.
#include "qi_common.cuh"
#include "qi_internal.h"

namespace qi {

constexpr int QT = 256;        // threads per row of the weight-preparation kernel
constexpr int QCH = 4;         // chunks of 8 elements per thread (32 values)

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

template <bool XBF16>
__device__ __forceinline__ void load8(const void* base, int64_t off, float* v) {
  if (XBF16) {
    const uint4 raw = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

// One CTA per row with blockDim.x = max(32, K / 32) threads, each holding up
// to QCH chunks of 8 consecutive elements: chunk c of thread t covers
// [8 (t + c blockDim), +8), so each load instruction of a warp reads one
// contiguous segment of the row.
template <bool XBF16, bool LN, bool RANGE>
__global__ void __launch_bounds__(1024) quant_kernel(const QuantParams p) {
  __shared__ float red[64];
  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int nt = blockDim.x;
  const int nchunk = p.K >> 3;
  float v[QCH][8];

#pragma unroll
  for (int c = 0; c < QCH; ++c) {
    const int ch = tid + c * nt;
    if (ch < nchunk) load8<XBF16>(p.x, static_cast<int64_t>(row) * p.ldx + ch * 8, v[c]);
  }

  if (LN && p.zero_range && tid == 0) {
    p.zero_range[2 * static_cast<int64_t>(row)] = 0u;
    p.zero_range[2 * static_cast<int64_t>(row) + 1] = 0u;
  }

  if (LN) {
    if (p.res_y) {
      // residual add of the previous Linear: x = x + gate[row set] * y (fp32),
      // written back so the residual stream carries it
      const int rs0 = p.groups.row_set[group_of(p.groups, p.row0 + row)];
      const uint16_t* gt = p.res_gate + static_cast<int64_t>(rs0) * p.mod_ld;
      float* xw = const_cast<float*>(static_cast<const float*>(p.x)) + static_cast<int64_t>(row) * p.ldx;
#pragma unroll
      for (int c = 0; c < QCH; ++c) {
        const int ch = tid + c * nt;
        if (ch < nchunk) {
          float fy[8], fg[8];
          load8<true>(p.res_y, static_cast<int64_t>(row) * p.K + ch * 8, fy);
          load8<true>(gt, ch * 8, fg);
#pragma unroll
          for (int i = 0; i < 8; ++i) v[c][i] = fmaf(fg[i], fy[i], v[c][i]);
          float4* o4 = reinterpret_cast<float4*>(xw + ch * 8);
          o4[0] = make_float4(v[c][0], v[c][1], v[c][2], v[c][3]);
          o4[1] = make_float4(v[c][4], v[c][5], v[c][6], v[c][7]);
        }
      }
    }
    float s = 0.f, ss = 0.f;
#pragma unroll
    for (int c = 0; c < QCH; ++c)
      if (tid + c * nt < nchunk)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          s += v[c][i];
          ss = fmaf(v[c][i], v[c][i], ss);
        }
    const float2 t = block_reduce2<false>(s, ss, red);
    const float inv_k = 1.0f / static_cast<float>(p.K);
    const float mean = t.x * inv_k;
    const float var = fmaxf(t.y * inv_k - mean * mean, 0.0f);
    const float rstd = 1.0f / sqrtf(var + p.eps);
    const int rs = p.groups.row_set[group_of(p.groups, p.row0 + row)];
    const uint16_t* sh = p.shift + static_cast<int64_t>(rs) * p.mod_ld;
    const uint16_t* sc = p.scale + static_cast<int64_t>(rs) * p.mod_ld;
#pragma unroll
    for (int c = 0; c < QCH; ++c) {
      const int ch = tid + c * nt;
      if (ch < nchunk) {
        float fsh[8], fsc[8];
        load8<true>(sh, ch * 8, fsh);
        load8<true>(sc, ch * 8, fsc);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          v[c][i] = fmaf((v[c][i] - mean) * rstd, 1.0f + fsc[i], fsh[i]);
      }
    }
    if (p.u_bf16) {   // modulated activation for a BF16 Linear
#pragma unroll
      for (int c = 0; c < QCH; ++c) {
        const int ch = tid + c * nt;
        if (ch < nchunk) {
          uint4 o;
          o.x = pack_bf16x2(v[c][0], v[c][1]);
          o.y = pack_bf16x2(v[c][2], v[c][3]);
          o.z = pack_bf16x2(v[c][4], v[c][5]);
          o.w = pack_bf16x2(v[c][6], v[c][7]);
          *reinterpret_cast<uint4*>(p.u_bf16 + static_cast<int64_t>(row) * p.ldq + ch * 8) = o;
        }
      }
      return;
    }
  }

  float lo = 0.f, hi = 0.f;
  if (RANGE) {
    // range published by the producer: [-min, max] as float bit patterns
    lo = -__uint_as_float(p.range[2 * static_cast<int64_t>(row)]);
    hi = __uint_as_float(p.range[2 * static_cast<int64_t>(row) + 1]);
  } else {
#pragma unroll
    for (int c = 0; c < QCH; ++c)
      if (tid + c * nt < nchunk)
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          lo = fminf(lo, v[c][i]);
          hi = fmaxf(hi, v[c][i]);
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
  // rint(u / s) with the IEEE quotient, computed as u * (1/s): |u/s| <= 255, so
  // the product is within ~3e-5 of the exact quotient and rounds the same way
  // unless its fraction is within 1e-4 of one half; those rare elements take
  // the exact division.
  const float inv_s = __fdiv_rn(1.0f, s);
#pragma unroll
  for (int c = 0; c < QCH; ++c) {
    const int ch = tid + c * nt;
    if (ch < nchunk) {
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float t = v[c][i] * inv_s;
        float rq = rintf(t);
        if (fabsf(fabsf(t - rq) - 0.5f) < 1e-4f) rq = rintf(__fdiv_rn(v[c][i], s));
        int qv = static_cast<int>(rq) + zp;
        qv = max(-128, min(127, qv));
        packed[i >> 2] |= (static_cast<uint32_t>(qv) & 0xFFu) << (8 * (i & 3));
      }
      *reinterpret_cast<uint2*>(p.q + static_cast<int64_t>(row) * p.ldq + ch * 8) =
          make_uint2(packed[0], packed[1]);
    }
  }
  if (tid == 0) {
    p.s[row] = s;
    p.zp[row] = zp;
  }
}

int launch_quant(const QuantParams& p, cudaStream_t st) {
  if (p.M == 0) return 0;
  if (p.K % 8 != 0 || p.K > 1024 * 8 * QCH) return -1;
  int nt = (p.K / 8 + QCH - 1) / QCH;   // threads so that each holds <= QCH chunks
  nt = ((nt + 31) / 32) * 32;
  if (nt < 32) nt = 32;
  dim3 grid(p.M), block(nt);
  if (p.ln && p.range) return -1;                 // LN computes its own range
  if (p.res_y && (!p.ln || p.x_bf16)) return -1;  // the residual add writes the fp32 stream
  if (p.x_bf16) {
    if (p.ln) quant_kernel<true, true, false><<<grid, block, 0, st>>>(p);
    else if (p.range) quant_kernel<true, false, true><<<grid, block, 0, st>>>(p);
    else quant_kernel<true, false, false><<<grid, block, 0, st>>>(p);
  } else {
    if (p.ln) quant_kernel<false, true, false><<<grid, block, 0, st>>>(p);
    else quant_kernel<false, false, false><<<grid, block, 0, st>>>(p);
  }
  return launch_result();
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
