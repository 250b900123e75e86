// Block-causal flash attention, head_dim 128, bf16 in / bf16 out, fp32 softmax.
//
// Mask (RGBA-Image-2.1 Core AI port: "block-causal attention"; qwen-image-mnn:
// "block-causal mask"): the joint sequence is split into contiguous groups
// [text | (reference) | target]; a token sees every token of its own group and
// of all earlier groups.  Because the groups are contiguous and ordered, the
// keys a query at global position t may see are exactly [0, end(group(t))):
// a per-query key limit.  Key tiles at or past the largest limit of a query
// tile are never loaded (skipped); tiles below the smallest limit need no mask.
//
// Queries may be a suffix of the sequence (q_offset > 0): the cached-prefix
// step processes only the target rows while the keys/values cover the whole
// sequence, the prefix part written by an earlier step.
//
// Tiling: a CTA owns 64 queries of one head (4 warps x 16 rows); key/value
// tiles of 64 rows stream through a 2-stage cp.async ring in shared memory
// (rows of 256 bytes, 16-byte chunks XOR-swizzled by row).  S = Q K^T and
// O += P V run on mma.sync m16n8k16 (bf16, fp32 accumulate); the running max
// and sum follow the online-softmax recurrence in base 2.
#include <float.h>

#include "qi_common.cuh"
#include "qi_internal.h"

namespace qi {

constexpr int AT_BM = 64;
constexpr int AT_BN = 64;
constexpr int AT_D = 128;
constexpr int AT_THREADS = 128;
constexpr int AT_TILE_BYTES = 64 * AT_D * 2;      // 16 KB
constexpr int AT_SMEM = AT_TILE_BYTES * 5;          // Q + 2 x (K, V)

__device__ __forceinline__ uint32_t swz(int row, int chunk) {   // byte offset in a tile
  return static_cast<uint32_t>(row * 256 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Load a 64 x 128 bf16 tile (rows [row0, row0+64) of a row-major matrix with
// leading dimension ld, columns [col0, col0+128)) into swizzled shared memory;
// rows >= nrows are zero-filled.
__device__ __forceinline__ void load_tile(uint32_t sbase, const uint16_t* g, int ld, int row0,
                                          int col0, int nrows) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int i = threadIdx.x + j * AT_THREADS;   // 0..1023
    const int r = i >> 4, c = i & 15;
    const int gr = row0 + r;
    const bool valid = gr < nrows;
    const uint16_t* src = g + static_cast<int64_t>(valid ? gr : 0) * ld + col0 + c * 8;
    cp_async16(sbase + swz(r, c), src, valid);
  }
}

__device__ __forceinline__ int key_limit(const GroupTable& g, int t) {
  return g.end[group_of(g, t)];
}

__global__ void __launch_bounds__(AT_THREADS, 2) attn_kernel(const AttnParams p) {
  extern __shared__ __align__(128) uint8_t at_smem[];
  // layout: Q | K0 | V0 | K1 | V1  (5 x 16 KB); stage b: K at 16K + 32K b, V at 32K + 32K b
  const uint32_t sQ = smem_u32(at_smem);
  const uint32_t sK0 = sQ + AT_TILE_BYTES;
  const uint32_t sV0 = sQ + 2 * AT_TILE_BYTES;

  const int n_qtiles = (p.Sq + AT_BM - 1) / AT_BM;
  const int qt = n_qtiles - 1 - static_cast<int>(blockIdx.x);   // heavy tiles first
  const int h = blockIdx.y;
  const int q0 = qt * AT_BM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g8 = lane >> 2, t4 = lane & 3;

  // key range of this query tile
  const int q_last = min(q0 + AT_BM, p.Sq) - 1;
  const int kv_end = min(key_limit(p.groups, p.q_offset + q_last), p.Sk);
  const int kv_min = min(key_limit(p.groups, p.q_offset + q0), p.Sk);
  const int n_ktiles = (kv_end + AT_BN - 1) / AT_BN;

  // per-row limits of this thread's two rows
  const int ra = q0 + warp * 16 + g8, rb = ra + 8;
  const int lim_a = ra < p.Sq ? min(key_limit(p.groups, p.q_offset + ra), p.Sk) : p.Sk;
  const int lim_b = rb < p.Sq ? min(key_limit(p.groups, p.q_offset + rb), p.Sk) : p.Sk;

  const int hc = h * AT_D;
  load_tile(sQ, p.q, p.ldq, q0, hc, p.Sq);
  load_tile(sK0, p.k, p.ldkv, 0, hc, p.Sk);
  load_tile(sV0, p.v, p.ldkv, 0, hc, p.Sk);
  cp_async_commit();

  uint32_t qf[8][4];
  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
  const float sl2 = p.sm_scale * 1.4426950408889634f;

  for (int kt = 0; kt < n_ktiles; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < n_ktiles) {
      const int nb = buf ^ 1;
      load_tile(sK0 + nb * 2 * AT_TILE_BYTES, p.k, p.ldkv, (kt + 1) * AT_BN, hc, p.Sk);
      load_tile(sV0 + nb * 2 * AT_TILE_BYTES, p.v, p.ldkv, (kt + 1) * AT_BN, hc, p.Sk);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (kt == 0) {
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int row = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * kk + (lane >> 4);
        ldsm_x4(sQ + swz(row, chunk), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t sK = sK0 + buf * 2 * AT_TILE_BYTES;
    const uint32_t sV = sV0 + buf * 2 * AT_TILE_BYTES;

    // S = Q K^T for 16 rows x 64 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {   // pairs of 8-key tiles
        const int key = jp * 16 + (lane & 7) + (lane >> 4) * 8;
        const int chunk = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(key, chunk), b0, b1, b2, b3);
        mma_bf16(s[2 * jp], qf[kk], b0, b1);
        mma_bf16(s[2 * jp + 1], qf[kk], b2, b3);
      }
    }

    // mask, scale to base 2
    const int k0 = kt * AT_BN;
    const bool need_mask = (k0 + AT_BN > kv_min);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int kc = k0 + j * 8 + 2 * t4;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float va = s[j][e] * sl2, vb = s[j][2 + e] * sl2;
        if (need_mask) {
          if (kc + e >= lim_a) va = -INFINITY;
          if (kc + e >= lim_b) vb = -INFINITY;
        }
        s[j][e] = va;
        s[j][2 + e] = vb;
      }
    }
    float mx_a = m_a, mx_b = m_b;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      mx_a = fmaxf(mx_a, fmaxf(s[j][0], s[j][1]));
      mx_b = fmaxf(mx_b, fmaxf(s[j][2], s[j][3]));
    }
#pragma unroll
    for (int o_ = 1; o_ <= 2; o_ <<= 1) {
      mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, o_));
      mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, o_));
    }
    // every row sees key 0 in tile 0, so the running max is finite from here on
    const float corr_a = exp2f(m_a - mx_a), corr_b = exp2f(m_b - mx_b);
    m_a = mx_a;
    m_b = mx_b;
    float sum_a = 0.f, sum_b = 0.f;
    uint32_t pf[4][4];   // P as bf16 A fragments, one per 16-key step
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = exp2f(s[j][0] - m_a), p1 = exp2f(s[j][1] - m_a);
      const float p2 = exp2f(s[j][2] - m_b), p3 = exp2f(s[j][3] - m_b);
      sum_a += p0 + p1;
      sum_b += p2 + p3;
      const int kk = j >> 1, hi = j & 1;
      pf[kk][hi * 2 + 0] = pack_bf16x2(p0, p1);
      pf[kk][hi * 2 + 1] = pack_bf16x2(p2, p3);
    }
    l_a = l_a * corr_a + sum_a;
    l_b = l_b * corr_b + sum_b;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= corr_a;
      o[i][1] *= corr_a;
      o[i][2] *= corr_b;
      o[i][3] *= corr_b;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const uint32_t a[4] = {pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3]};
#pragma unroll
      for (int dp = 0; dp < 8; ++dp) {   // pairs of 8-wide d tiles
        const int key = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * dp + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(key, chunk), b0, b1, b2, b3);
        mma_bf16(o[2 * dp], a, b0, b1);
        mma_bf16(o[2 * dp + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

  cp_async_wait<0>();

  // full row sums across the quad, normalise, store
#pragma unroll
  for (int o_ = 1; o_ <= 2; o_ <<= 1) {
    l_a += __shfl_xor_sync(0xffffffffu, l_a, o_);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, o_);
  }
  const float inv_a = l_a > 0.f ? 1.0f / l_a : 0.f;
  const float inv_b = l_b > 0.f ? 1.0f / l_b : 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int col = hc + i * 8 + 2 * t4;
    if (ra < p.Sq)
      *reinterpret_cast<uint32_t*>(p.o + static_cast<int64_t>(ra) * p.ldo + col) =
          pack_bf16x2(o[i][0] * inv_a, o[i][1] * inv_a);
    if (rb < p.Sq)
      *reinterpret_cast<uint32_t*>(p.o + static_cast<int64_t>(rb) * p.ldo + col) =
          pack_bf16x2(o[i][2] * inv_b, o[i][3] * inv_b);
  }
}

int launch_attention(const AttnParams& p, cudaStream_t st) {
  if (p.Sq == 0) return 0;
  static bool attr = false;
  if (!attr) {
    if (cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, AT_SMEM) !=
        cudaSuccess)
      return -1;
    attr = true;
  }
  dim3 grid((p.Sq + AT_BM - 1) / AT_BM, p.heads);
  attn_kernel<<<grid, AT_THREADS, AT_SMEM, st>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace qi
