// Internal (non-exported) declarations shared by the kernel files and the
// C-ABI layer.  Nothing here is part of the public interface in include/qi.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qi_common.cuh"

namespace qi {

// The CUDA error of the last failed launch on this thread (launchers return -1
// after reading and clearing cudaGetLastError; the C ABI reports this one).
inline cudaError_t& last_launch_error() {
  static thread_local cudaError_t e = cudaSuccess;
  return e;
}
inline int launch_result() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return 0;
  last_launch_error() = e;
  return -1;
}

// Launch `kern` with programmatic stream serialization (and, for
// cluster_x > 1, clusters of cluster_x CTAs): the kernel may be scheduled
// while the previous kernel of the stream drains; it calls pdl_wait() before
// its first access to memory that kernel touches.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, unsigned cluster_x, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  unsigned na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (cluster_x > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster_x;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

enum GemmEpilogue {
  EPI_BF16 = 0,    // y (bf16) = value
  EPI_GELU = 1,    // y (bf16) = GELU_tanh(bf16(value))
  EPI_GATED = 2,   // yf (fp32) += gate[row set] * bf16(value)
  EPI_F32 = 3,     // yf (fp32) = value
  EPI_EULER = 4,   // v = value; yf (fp32 latents) += dt * v
  EPI_QKV = 5,     // q, k: RMSNorm (cast first) + RoPE of bf16(value); v: bf16(value)
};

struct GemmParams {
  int M, N, K;       // K in elements
  int num_kb;        // K / (128 bytes / element size)
  // W8A8 dequantization
  const float* s_a;
  const int32_t* zp_a;
  const float* s_w;
  const int32_t* rowsum;
  const uint16_t* bias;   // bf16 [N] or null
  // outputs
  uint16_t* y;            // bf16 [M, ldy]
  int ldy;
  float* yf;              // fp32 [M, ldyf]: output, residual or latents
  int ldyf;
  const uint16_t* gate;   // bf16: gate of row set r at gate + r * gate_ld
  int gate_ld;
  // EPI_GATED: if res_y is set, each residual value x first becomes
  // x + gate1 * res_y (one rounding; gate1 rows like gate's): the mid-block
  // residual the LayerNorm before this Linear used without storing it
  const uint16_t* res_y;  // bf16 [M, ld_res_y] or null
  int ld_res_y;
  const uint16_t* gate1;
  GroupTable groups;      // row sets of global tokens
  int row0;               // global token index of row 0
  int32_t* acc_debug;     // optional raw int32 accumulators [M, N]
  float dt;               // Euler: sigma_next - sigma
  float* v_out;           // Euler: optional velocity [M, ldyf]
  // fused QKV epilogue (a tile holds whole heads of one of q, k, v): column
  // n of this GEMM is column n_base + n of the [q | k | v] projection (N = 3H
  // with n_base 0, or a part: the q, k columns, or the v columns at n_base 2H)
  int H;
  int n_base;
  float eps;
  const uint16_t* wq;     // [128] bf16 RMSNorm scales
  const uint16_t* wk;
  const float* rcos;      // [M, 64] tables of the rows of this GEMM
  const float* rsin;
  uint16_t* q_out;        // [M, H] rows of this GEMM
  uint16_t* k_out;        // K/V rows m < kv_split (all rows if k_out2 is null)
  uint16_t* v_out_bf16;
  uint16_t* k_out2;       // K/V rows m >= kv_split go to k_out2/v_out2 row m - kv_split
  uint16_t* v_out2;       // (a batch of two sequences with separate K/V buffers)
  int kv_split;
  // optional e4m3 copies of the q / k / v rows above (same rows and ldo, one
  // byte per element: round to nearest even, saturating), for fp8 attention
  uint8_t* q8_out;
  uint8_t* k8_out;
  uint8_t* v8_out;
  uint8_t* k8_out2;
  uint8_t* v8_out2;
  int ldo;
  uint32_t* row_range;    // GELU: optional per-row [-min, max] bit patterns of the bf16 output
  int group_m;            // tile order: bands of group_m M tiles (set by launch_gemm)
  // MXFP4 B operand (BF16 GEMM only): E2M1 codes [N, K/2] (low nibble first)
  // and E8M0 scales [N, K/32], decoded to bf16 in the load path; B is unused
  const uint8_t* b_packed;
  const uint8_t* b_scales;
  int* status;            // device status word
};

// TMA descriptor for a row-major 2-D tensor [outer, inner] with a box of
// box_inner x box_outer elements, 128-byte swizzled unless swizzle128 is false.
bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner,
                  uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128 = true);

int pick_block_n(int N);
int launch_gemm(bool int8, int epi, const void* A, int lda, const void* B, int ldb,
                const GemmParams& p, int num_sms, cudaStream_t st);

// Per-row quantization (optionally fused with LayerNorm + adaLN modulate).
struct QuantParams {
  const void* x;          // [M, ldx], fp32 or bf16
  int x_bf16;
  int M, K, ldx;
  int ln;                 // 1: LayerNorm + modulate before quantizing
  const uint16_t* shift;  // bf16 row of set r at shift + r * mod_ld
  const uint16_t* scale;
  int mod_ld;
  GroupTable groups;
  int row0;
  float eps;
  int8_t* q;              // [M, ldq]
  int ldq;
  float* s;               // [M]
  int32_t* zp;            // [M]
  uint16_t* u_bf16;       // if non-null: write bf16(u) [M, ldq] instead of quantizing ...
  int quant_too;          // ... or as well as quantizing (LN variant)
  // LN variant: residual add before the LayerNorm, x + gate[row set] * y,
  // written to res_out (fp32 [M, ldx]) if that is set
  const uint16_t* res_y;  // bf16 [M, K] or null
  const uint16_t* res_gate;   // gate row of set r at res_gate + r * mod_ld
  float* res_out;
  uint32_t* zero_range;   // if non-null: rows' [2] range words set to 0 (for a later producer)
  uint32_t* zero_words;   // LN variant, if non-null: n_zero_words words set to 0 (by the first row)
  int n_zero_words;
  float* u_f32;           // LN variant, if non-null: also write u (the quantized value) [M, ldq] fp32
  // plain variant: the row's range was published by the producer as
  // [float bits of -min, float bits of max] (both >= 0); no reduction needed
  const uint32_t* range;
  int* status;            // device status word (bounded wait for the row copy)
};
int launch_quant(const QuantParams& p, cudaStream_t st);

int launch_prepare_w8(const float* w, int n, int k, int8_t* q, float* s, int32_t* rowsum,
                      cudaStream_t st);

// Q/K RMSNorm (cast before scale) + 3-axis RoPE on a fused QKV row block.
struct QkNormRopeParams {
  const uint16_t* qkv;    // [T, ldqkv] bf16: q | k | v, each heads*d wide
  int ldqkv;
  int T, heads, d;
  const uint16_t* wq;     // [d] bf16
  const uint16_t* wk;
  const float* cos;       // [T, d/2]
  const float* sin;
  float eps;
  uint16_t* q_out;        // [T, ldo]
  uint16_t* k_out;        // [T, ldo]
  uint16_t* v_out;        // [T, ldo]
  int ldo;
};
int launch_qk_norm_rope(const QkNormRopeParams& p, cudaStream_t st);

// Block-causal attention.
struct AttnParams {
  const void* q;          // [Sq, ldq] bf16, or e4m3 bytes when fp8
  const void* k;          // [Sk, ldkv]
  const void* v;
  int fp8;                // 1: q, k, v are e4m3 (tcgen05 kind::f8f6f4, P as e4m3)
  uint16_t* o;            // [Sq, ldo] bf16
  int ldq, ldkv, ldo;
  int Sq, Sk, heads, q_offset;
  float sm_scale;
  GroupTable groups;
  uint32_t* row_range;    // optional per-query-row [-min, max] bit patterns of the bf16 output
  // Key-range split of whole heads.  The query tiles with the longest key
  // range (ceil(Sk / 128) key tiles) of the last `split_heads` heads run as
  // two CTAs each, over key tiles [0, n/2) and [n/2, n); each half writes its
  // unnormalised O, reference maximum and row sum to the scratch, and the
  // half that finishes second combines the two.  launch_attention chooses
  // split_heads from Sk, the group table, heads, the SM count and
  // split_bytes alone, so two launches over the same sequence split the same
  // rows whatever their query rows (a cached-prefix launch and the uncached
  // one give identical target rows).  Scratch layout: counters [units]
  // (must be zero at launch; the combining CTA sets its counter back to 0),
  // then part_ml [units][2][256 rows][2] and part_o [units][2][32 column
  // quads][256 rows][4] fp32.
  void* split_scratch;    // 256-byte aligned device scratch, or null (no split)
  size_t split_bytes;     // bytes the plan may assume (the same for every launch of a sequence)
  size_t split_have;      // bytes split_scratch holds in this launch (a launch needing more
                          // than this does not split)
  int num_sms;
  // filled in by launch_attention
  int n_ctiles, ct_heavy, split_heads;
  int* status;            // device status word
};
// Split plan of a launch (reads Sk, groups, heads, num_sms, split_bytes):
// heads split (0: none), the scratch bytes it may use and, at their start,
// the bytes of counters that must be zero when the kernel starts.
void attention_split_plan(const AttnParams& p, int* split_heads, size_t* bytes,
                          size_t* counter_bytes);
int launch_attention(const AttnParams& p, cudaStream_t st);

// Thin GEMV for M <= 2 rows (timestep MLP, adaLN rows).
struct GemvJob {
  const uint16_t* w;      // [n, k] bf16
  const uint16_t* b;      // [n] bf16 or null
  void* y;                // [R, ldy] (fp32 or bf16)
  int n;
  int ldy;
};
constexpr int GEMV_MAX_JOBS = 80;
struct GemvParams {
  const float* x;         // [R, k] fp32 input rows
  int R, k;
  int silu_in;            // apply SiLU to x
  int y_bf16;
  int n_jobs;
  GemvJob jobs[GEMV_MAX_JOBS];
};
int launch_gemv(const GemvParams& p, cudaStream_t st);

int launch_timestep_embedding(float t0, float t1, float* out, cudaStream_t st);
int launch_timeout_probe(uint64_t limit_ns, int* status, cudaStream_t st);
// Back-to-back tcgen05.mma (kind::i8 or kind::f16, M = 128, N = 256) on
// shared-memory operands, `iters` x 4 MMAs per CTA, one CTA per SM.
int launch_mma_probe(bool i8, int iters, int num_sms, int* status, cudaStream_t st);
int launch_f32_to_bf16(const float* x, uint16_t* y, int64_t n, cudaStream_t st);
int launch_euler(float* x, const float* v, int64_t n, float dt, cudaStream_t st);
// MXFP4 (E2M1 codes, low nibble first; E8M0 scale per 32 columns) -> fp32 [n, k].
// MXFP4 -> bf16 [n, k] (k % 32 == 0; packed and w 16-byte aligned).  early:
// overlap the previous kernel of the stream (w must be free of readers).
int launch_mxfp4_expand_bf16(const uint8_t* packed, const uint8_t* scales, int n, int k,
                             uint16_t* w, cudaStream_t st, bool early = false);
int launch_mxfp4_decode(const uint8_t* packed, const uint8_t* scales, int n, int k_stored, int k,
                        float* w, cudaStream_t st);
// bf16 -> e4m3 (round to nearest, ties to even, saturating), n % 8 == 0.
int launch_bf16_to_e4m3(const uint16_t* x, uint8_t* y, int64_t n, cudaStream_t st);
// Classifier-free guidance + Euler: v = v_u + g (v_c - v_u), x += dt v, fp32,
// one rounding per operation; v_out (optional) receives v.
int launch_cfg_euler(float* x, const float* v_c, const float* v_u, int64_t n, float g, float dt,
                     float* v_out, cudaStream_t st);

}  // namespace qi
