/*
 * qi.h - C ABI of libqi: one denoising step of the Qwen-Image-2.1
 * single-stream diffusion transformer with W8A8 Linears, for NVIDIA B200
 * (sm_100a).
 *
 * Sources (cited by page title and section):
 *   [W8]   FlagRelease "Qwen-Image-2.1-W8A8-arm-FlagOS", "Quantization and
 *          validation": symmetric INT8 weights per output channel (zero point 0,
 *          FP32 scales); dynamic asymmetric INT8 activations per token/row
 *          (FP32 scales); INT32 accumulation, FP32 scaling, BF16 output.
 *   [QN]   "Qwen Image 2.1 native qualification", "Numerical checks": Q/K
 *          RMSNorm casts the normalized activation to the scale's dtype
 *          before scaling.
 *   [GC]   "RGBA-Image-2.1 - Core AI port of Qwen-Image-2.1", intro and
 *          "Graph contracts": 32-block single-stream DiT with block-causal
 *          attention; joint sequence [text | image] with one image token per
 *          16x16 px tile; 3-axis RoPE positions; 64 rotation pairs per head;
 *          shifted sigmas and the Euler update x += (sigma_next - sigma) * v.
 *   [MNN]  qwen-image-mnn, "What runs where": 3-axis RoPE, block-causal mask
 *          and modulation rows as the joint-sequence bookkeeping; "Install /
 *          run": a true CFG scale > 1 with a negative prompt enables
 *          classifier-free guidance.
 *   [QC]   "Qwen Image 2.1 native qualification", "Native CLI cases": CFG,
 *          single- and multi-reference edit (up to ten references) cases.
 *   [PX]   EliovpAI "Qwen_Image-2.1-MXFP4-Paiton-RDNA4", "Runtime precision and
 *          quality" / "Tested operating limits": cached text-prefix pass
 *          (prefix KV reuse); unsupported settings rejected before GPU work.
 *
 * Conventions (all entry points):
 *   - Every call returns a qi_status.  Arguments are validated on the host
 *     before anything is launched; a rejected call launches nothing.
 *     qi_last_error() returns a text description of the last failure on the
 *     calling thread.
 *   - Tensor pointers are device pointers owned by the caller unless stated
 *     otherwise; all must be 16-byte aligned.  A call on zero rows
 *     (qi_quantize_act, qi_w8a8_linear, qi_bf16_linear with M = 0; the
 *     attention calls with Sq = 0) checks its other arguments (weights,
 *     shapes, epilogue, groups) like any call, then returns QI_OK and touches
 *     nothing; its row pointers may be NULL.  Matrices are row-major
 *     [rows, ld] with ld in elements.  bf16 values are passed as uint16_t bit
 *     patterns.  Weights are [out, in] (K-major).
 *   - Every device call is asynchronous on the given CUDA stream
 *     (cudaStream_t passed as void*; NULL = the legacy default stream).
 *     Nothing synchronizes except qi_ctx_check() (and
 *     qi_ctx_reserve_attention() when it replaces a smaller scratch).
 *   - The library never allocates device memory in a compute call.  Scratch
 *     comes from a caller-owned workspace whose size the *_workspace_bytes
 *     functions return; qi_ctx_create() allocates only a 256-byte device
 *     status word, and qi_ctx_reserve_attention() the optional scratch of
 *     the standalone attention calls.
 *   - Kernels never trap.  A pipeline wait that does not complete within 2 s
 *     records QI_ERR_TIMEOUT in the context's status word and the kernel
 *     returns; qi_ctx_check() reports it.
 */
#ifndef QI_H_
#define QI_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct qi_ctx qi_ctx;

typedef enum {
  QI_OK = 0,
  QI_ERR_INVALID_ARG = 1,       /* null pointer, negative size, bad enum, bad group table */
  QI_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside what the kernels support (see each call) */
  QI_ERR_ALIGNMENT = 3,         /* pointer or leading dimension not 16-byte aligned */
  QI_ERR_CUDA = 4,              /* a CUDA runtime / driver call failed */
  QI_ERR_TIMEOUT = 5,           /* a kernel's bounded wait expired (device status word) */
  QI_ERR_WORKSPACE = 6          /* workspace smaller than the *_workspace_bytes size */
} qi_status;

typedef enum { QI_F32 = 0, QI_BF16 = 1 } qi_dtype;

/* Joint-sequence groups ([MNN] "block-causal mask"; [GC] Sequence).
 * Groups are contiguous and ordered: group g holds global tokens
 * [end[g-1], end[g]) (end[-1] = 0).  A token attends to every token of its
 * own group and of all earlier groups.  row_set[g] selects which modulation
 * row set (adaLN rows) the group's tokens use.  Passed by host pointer. */
#define QI_MAX_GROUPS 16
typedef struct qi_groups {
  int32_t n;                        /* 1..QI_MAX_GROUPS */
  int32_t end[QI_MAX_GROUPS];       /* strictly ascending; end[n-1] = sequence length */
  int32_t row_set[QI_MAX_GROUPS];   /* >= 0 */
} qi_groups;

/* One W8A8 Linear prepared by qi_prepare_w8 ([W8]). */
typedef struct qi_w8 {
  const int8_t* q;         /* [n, k] int8 codes, K-major */
  const float* s;          /* [n] per-output-channel scale */
  const int32_t* rowsum;   /* [n] sum_k q[n, k] (zero-point correction) */
  const uint16_t* bias;    /* [n] bf16, or NULL */
  int32_t n, k;
} qi_w8;

/* One BF16 Linear: y = x W^T + b. */
typedef struct qi_linear_bf16 {
  const uint16_t* w;       /* [n, k] bf16 */
  const uint16_t* bias;    /* [n] bf16, or NULL */
  int32_t n, k;
} qi_linear_bf16;

typedef enum {
  QI_EPI_STORE = 0,           /* y = bf16(Linear(x)) */
  QI_EPI_GELU_TANH = 1,       /* y = bf16(GELU_tanh(bf16(Linear(x)))) */
  QI_EPI_GATED_RESIDUAL = 2,  /* residual += gate[row set] * bf16(Linear(x)), fp32 */
  QI_EPI_QKV_NORM_ROPE = 3    /* fused QKV projection: y = bf16(Linear(x)) split into q | k | v
                                 (n = 3 * hidden); q and k get the Q/K RMSNorm (cast before
                                 scale) and RoPE of qi_qk_norm_rope, v is stored as is */
} qi_epilogue_kind;

typedef struct qi_epilogue {
  int32_t kind;                /* qi_epilogue_kind */
  float* residual;             /* GATED_RESIDUAL: fp32 [M, ld_residual], updated in place */
  int32_t ld_residual;
  const uint16_t* gate;        /* GATED_RESIDUAL: bf16 gate row of set r at gate + r * gate_ld */
  int32_t gate_ld;
  const qi_groups* groups;     /* GATED_RESIDUAL: row set of each row (host pointer) */
  int32_t row0;                /* global token index of row 0 */
  /* QKV_NORM_ROPE: hidden % 128 == 0 (a GEMM tile holds whole heads), head_dim 128 */
  int32_t hidden;
  float eps;
  const uint16_t* norm_q;      /* [128] bf16 */
  const uint16_t* norm_k;
  const float* rope_cos;       /* [M, 64] fp32 tables of the M rows */
  const float* rope_sin;
  uint16_t* q_out;             /* [M, ld_out] bf16 */
  uint16_t* k_out;
  uint16_t* v_out;
  int32_t ld_out;
} qi_epilogue;

typedef struct qi_dims {
  int32_t hidden;     /* H = heads * head_dim */
  int32_t heads;
  int32_t head_dim;   /* must be 128 */
  int32_t mlp;        /* F */
  int32_t patch;      /* P: latent token width (64, or 256 with 2x2 packing) */
  int32_t blocks;
  float eps;          /* LayerNorm / RMSNorm epsilon (1e-6) */
} qi_dims;

/* One Linear stored as MXFP4 ([PX] What was quantized: E2M1 values packed two
 * per byte, low nibble first; one E8M0 scale per 32 input columns), used with
 * bf16 activations ([PX] Runtime precision and quality: the exact profile runs
 * MXFP4 weights with BF16 activation arithmetic).  The GEMM decodes the codes
 * to bf16 tile by tile in shared memory (every E2M1 x 2^(e-127) value is
 * exact in bf16; E8M0 255 decodes to NaN) and accumulates in fp32 on tcgen05
 * kind::f16, so HBM holds 4.25 bits per weight and no decoded copy exists.
 *   packed [n, k/2] bytes, scales [n, k/32] bytes, bias [n] bf16 or NULL;
 *   k % 256 == 0, n % 256 == 0; packed and scales 16-byte aligned. */
typedef struct qi_mxfp4 {
  const uint8_t* packed;
  const uint8_t* scales;
  const uint16_t* bias;
  int32_t n, k;
} qi_mxfp4;

/* One block's weights.  Each of the four Linears is W8A8 ([W8]) or BF16: the
 * pages' deployed layout keeps some Linears in BF16 ([W8] "Scope": only the
 * attention q/k and the MLP Linears of blocks 2-29 are W8A8, everything else
 * stays BF16).  A Linear whose W8A8 codes are NULL (q == NULL) uses the BF16
 * weight of the same name.  The fused q | k | v projection comes in three
 * forms: qkv.n == 3H (all W8A8); qkv.n == 2H (q, k W8A8) with qkv_bf16 holding
 * the v rows (n = H); or qkv.q == NULL with qkv_bf16.n == 3H (all BF16).  A
 * BF16 Linear takes the bf16-rounded activation (the LayerNorm + modulate
 * value, the attention output or the GELU output) and accumulates in fp32 on
 * tcgen05 kind::f16; its output is rounded to bf16 like a W8A8 Linear's. */
typedef struct qi_block_weights {
  qi_w8 qkv;               /* n = 3H: rows [0,H) = q, [H,2H) = k, [2H,3H) = v (or n = 2H, see above) */
  qi_w8 out;               /* n = H, k = H */
  qi_w8 up;                /* n = F, k = H */
  qi_w8 down;              /* n = H, k = F */
  const uint16_t* norm_q;  /* [head_dim] bf16 RMSNorm scale */
  const uint16_t* norm_k;
  qi_linear_bf16 mod;      /* adaLN: n = 6H, k = H (used by the step-level calls) */
  qi_linear_bf16 qkv_bf16; /* BF16 forms, used where the W8A8 codes are NULL (qkv: see above) */
  qi_linear_bf16 out_bf16;
  qi_linear_bf16 up_bf16;
  qi_linear_bf16 down_bf16;
  qi_mxfp4 qkv_mx;         /* MXFP4 forms, used where the W8A8 codes are NULL and packed != NULL */
  qi_mxfp4 out_mx;         /*   (qkv_mx: all of q | k | v, n = 3H); bf16 activations as for BF16 */
  qi_mxfp4 up_mx;
  qi_mxfp4 down_mx;
  /* Optional device scratch for the MXFP4 Linears (16-byte aligned).  Where it
   * holds n x k bf16 values, an MXFP4 Linear is expanded into it (the exact
   * bf16 weights, qi_mxfp4_expand_bf16) right before its GEMM, which then
   * reads them as a BF16 Linear; otherwise the GEMM decodes the codes tile by
   * tile in shared memory.  Both give the same outputs bit for bit.  HBM
   * keeps the 4.25-bit weights either way.  With room for two of the largest
   * Linears (2 x max(3H, F) x H bf16) the Linears alternate between two
   * halves and each expansion overlaps the kernel before it; with room for
   * one, they take turns in it.  Blocks may share one scratch (their calls
   * are ordered on the stream).  NULL / 0: no expansion. */
  uint16_t* mx_expand;
  size_t mx_expand_bytes;
} qi_block_weights;

typedef struct qi_model {
  qi_dims dims;
  const qi_block_weights* blocks;   /* host array of dims.blocks entries */
  qi_linear_bf16 t1;                /* timestep MLP 1: n = H, k = 256 */
  qi_linear_bf16 t2;                /* timestep MLP 2: n = H, k = H */
  qi_linear_bf16 img_in;            /* n = H, k = P */
  qi_linear_bf16 txt_in;            /* n = H, k = H */
  qi_linear_bf16 final_mod;         /* final adaLN: n = 2H (shift, scale), k = H */
  qi_linear_bf16 proj_out;          /* n = P, k = H */
} qi_model;

typedef enum {
  QI_KV_NONE = 0,          /* every token processed; K/V buffers are scratch */
  QI_KV_WRITE_PREFIX = 1,  /* every token processed; the prefix K/V stay in the buffers */
  QI_KV_READ_PREFIX = 2    /* only the target rows processed; prefix K/V read from the buffers */
} qi_kv_mode;

/* ------------------------------------------------------------------ context */

/* Create a context on CUDA device `device`.  Allocates one 256-byte device
 * status word (cudaMalloc, outside any compute call).  *out is owned by the
 * caller and released with qi_ctx_destroy. */
int qi_ctx_create(int device, qi_ctx** out);
int qi_ctx_destroy(qi_ctx* ctx);

/* Synchronize `stream`, then read and clear the device status word.
 * Returns QI_ERR_TIMEOUT if a kernel recorded an expired wait, QI_ERR_CUDA if
 * the stream reported an error, else QI_OK. */
int qi_ctx_check(qi_ctx* ctx, void* stream);

/* Reserve `bytes` of device scratch in the context for the attention's
 * key-range split in qi_attn_block_causal(_fp8) (qi_attn_split_plan gives the
 * bytes a sequence needs).  Grows the scratch if it is smaller (the device is
 * synchronised when an old scratch is freed); freed by qi_ctx_destroy.
 * Without it the standalone attention calls do not split. */
int qi_ctx_reserve_attention(qi_ctx* ctx, size_t bytes);

/* Copy the calling thread's last error text into buf (NUL-terminated). */
int qi_last_error(char* buf, size_t n);

/* Kernel classes counted (and optionally timed) per context. */
typedef enum {
  QI_KCLASS_GEMM_I8 = 0,    /* tcgen05 kind::i8 W8A8 GEMMs */
  QI_KCLASS_GEMM_BF16 = 1,  /* tcgen05 kind::f16 BF16 GEMMs */
  QI_KCLASS_ATTN = 2,       /* block-causal attention */
  QI_KCLASS_QUANT = 3,      /* LayerNorm/modulate/int8 quantization */
  QI_KCLASS_QKNORM = 4,     /* Q/K RMSNorm + RoPE */
  QI_KCLASS_GEMV = 5,       /* timestep MLP / adaLN rows */
  QI_KCLASS_OTHER = 6       /* embeddings, casts */
} qi_kernel_class;

/* Reset the per-class launch counters and switch per-launch timing on or off.
 * When on, every launch is bracketed by two CUDA events recorded on its
 * stream (at most 16384 launches are timed until the next reset).  The first
 * call with enable != 0 creates the events (host-side, not in a compute call). */
int qi_ctx_profile(qi_ctx* ctx, int enable);

/* Launches of `kernel_class` since the last qi_ctx_profile() call, how many of
 * them were timed, and their summed device duration in milliseconds (waits for
 * the recorded events). */
int qi_ctx_profile_read(qi_ctx* ctx, int kernel_class, long long* launches, int* timed,
                        double* total_ms);

/* ------------------------------------------------------------------ W8A8 ([W8]) */

/* Quantize fp32 weights w [n, k] symmetrically per output channel:
 * s[n] = max|w[n,:]| / 127 (1 for an all-zero row), q = clamp(rint(w / s), -127, 127),
 * rowsum[n] = sum_k q[n, k].  Requires k % 8 == 0 (8 <= k). */
int qi_prepare_w8(qi_ctx* ctx, const float* w, int n, int k, int8_t* q, float* s,
                  int32_t* rowsum, void* stream);

/* Per-token dynamic asymmetric int8 quantization of x [M, K] (ld ldx):
 *   lo = min(min_k u, 0), hi = max(max_k u, 0), s = (hi - lo)/255,
 *   zp = clamp(rint(-128 - lo/s), -128, 127), q = clamp(rint(u/s) + zp, -128, 127)
 * (fp32 IEEE operations; an all-zero row gets s = 1, zp = 0).
 * If shift != NULL the quantized value is u = LN(x)(1 + scale) + shift, with a
 * non-affine LayerNorm (eps) and the bf16 shift/scale row of the token's row
 * set (shift + r * mod_ld, scale + r * mod_ld; groups/row0 map rows to global
 * tokens); else u = x.  x_dtype is QI_F32 or QI_BF16.
 * Outputs: q [M, K] int8 (ld K), s_a [M] fp32, zp_a [M] int32.
 * Requires K % 8 == 0 and K <= 16384; ldx % 8 == 0. */
int qi_quantize_act(qi_ctx* ctx, const void* x, int x_dtype, int M, int K, int ldx,
                    const uint16_t* shift, const uint16_t* scale, int mod_ld,
                    const qi_groups* groups, int row0, float eps, int8_t* q, float* s_a,
                    int32_t* zp_a, void* stream);

/* W8A8 Linear on tcgen05 tensor cores (int8 x int8 -> int32 in TMEM):
 *   acc[m, n] = sum_k qa[m, k] w.q[n, k]
 *   val = (acc - zp_a[m] * w.rowsum[n]) * s_a[m] * w.s[n] + w.bias[n]   (fp32)
 * then the epilogue ep (NULL = QI_EPI_STORE) writes y [M, w.n] bf16 (ld ldy) or
 * updates ep->residual.  acc_debug, if not NULL, receives the raw int32
 * accumulators [M, w.n] (not written by the QKV_NORM_ROPE epilogue).  Requires w.k % 128 == 0, w.n % 16 == 0, ldy % 8 == 0. */
int qi_w8a8_linear(qi_ctx* ctx, const int8_t* qa, const float* s_a, const int32_t* zp_a, int M,
                   const qi_w8* w, const qi_epilogue* ep, uint16_t* y, int ldy,
                   int32_t* acc_debug, void* stream);

/* Linear with MXFP4 weights (qi_mxfp4) on bf16 activations:
 *   y [M, w.n] bf16 (ld ldy) = bf16(a [M, w.k] decode(w)^T + bias)
 * the weights decoded to bf16 in shared memory inside the GEMM (fp32
 * accumulation on tcgen05 kind::f16, CTA pairs).  lda % 8 == 0, ldy % 8 == 0. */
int qi_mxfp4_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_mxfp4* w,
                    uint16_t* y, int ldy, void* stream);

/* BF16 Linear on tcgen05 tensor cores: y [M, w.n] fp32 (ld ldy) = a [M, w.k] W^T + b.
 * Requires w.k % 64 == 0, w.n % 16 == 0, lda % 8 == 0. */
int qi_bf16_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_linear_bf16* w,
                   float* y, int ldy, void* stream);

/* ------------------------------------------------------------------ attention path */

/* Q/K RMSNorm + 3-axis RoPE on a fused QKV block qkv [T, 3H] bf16 ([QN], [GC] RoPE):
 *   r = 1/sqrt(mean(x^2) + eps); n = bf16(x r); y = bf16(n w)   (cast BEFORE the scale)
 *   pair j = (y[2j], y[2j+1]) -> (bf16(a c - b s), bf16(a s + b c)), c/s = cos/sin[t, j]
 * applied per head to q (wq) and k (wk); v is copied.  Outputs q_out, k_out,
 * v_out [T, ldo] bf16.  cos/sin: [T, head_dim/2] fp32.  head_dim must be 128. */
int qi_qk_norm_rope(qi_ctx* ctx, const uint16_t* qkv, int T, int heads, int head_dim,
                    const uint16_t* wq, const uint16_t* wk, const float* rope_cos,
                    const float* rope_sin, float eps, uint16_t* q_out, uint16_t* k_out,
                    uint16_t* v_out, int ldo, void* stream);

/* Block-causal attention ([GC], [MNN]):  O = softmax(Q K^T sm_scale + M) V per head,
 * M(i, j) = 0 iff group(j) <= group(q_offset + i), else -inf.
 * q [Sq, ldq], k/v [Sk, ldkv], o [Sq, ldo] bf16; head h occupies columns
 * [h*128, (h+1)*128).  Queries are global tokens q_offset .. q_offset+Sq-1;
 * keys are global tokens 0 .. Sk-1 (Sk = groups->end[n-1]).  Key tiles that
 * no query of a tile may see are skipped.  head_dim must be 128. */
int qi_attn_block_causal(qi_ctx* ctx, const uint16_t* q, int ldq, int Sq, int q_offset,
                         const uint16_t* k, const uint16_t* v, int ldkv, int Sk, int heads,
                         int head_dim, const qi_groups* groups, float sm_scale, uint16_t* o,
                         int ldo, void* stream);

/* The attention calls above and the block and step calls below schedule one
 * CTA per (256 query rows, head), longest key range first.  When that leaves
 * the SMs' last round of CTAs mostly idle, the longest-range query tiles of
 * the last `split_heads` heads are split over the key range: two CTAs take
 * key tiles [0, n/2) and [n/2, n), each writes its unnormalised O, running
 * maximum and row sum to device scratch, and the one that finishes second
 * combines them (same softmax, rounding of those rows changes by about one
 * bf16 step).  The choice depends on Sk, the groups, heads, the SM count and
 * the scratch available only -- not on Sq or q_offset -- so a cached-prefix
 * call computes the target rows bit for bit as the uncached call does.
 * Scratch: qi_attn_block_causal(_fp8) split only into scratch the context
 * holds (qi_ctx_reserve_attention; they allocate nothing, and calls sharing a
 * context must not run concurrently on different streams); the block and
 * step calls use
 * the block workspace's MLP activation buffer, up to T_last x mlp x 2 bytes
 * (T_last = tokens of the last group).  A block call on fewer rows than the
 * last group whose buffer cannot hold the split's partials runs unsplit
 * (its rows then differ from the uncached call's by rounding only).
 *
 * qi_attn_split_plan reports that choice (host only, no device work):
 * split_heads (0: no split) and the scratch bytes it uses, for a sequence of
 * Sk tokens in `groups`, `heads` heads, num_sms SMs and scratch_bytes of
 * scratch (SIZE_MAX: unbounded). */
int qi_attn_split_plan(int Sk, int heads, const qi_groups* groups, int num_sms,
                       size_t scratch_bytes, int* split_heads, size_t* bytes);

/* ------------------------------------------------------------------ block */

/* Block-causal attention with e4m3 operands (the pages' reduced-precision
 * attention for later denoising steps: [PX] Runtime precision and quality,
 * "int8/fp8 attention for steps 8-40").  q, k, v are e4m3 bytes (ld in
 * elements = bytes; see qi_to_e4m3); S = Q K^T accumulates in fp32 on
 * tcgen05.mma kind::f8f6f4, the softmax runs in fp32 as in
 * qi_attn_block_causal, P is rounded to e4m3 (nearest, ties to even,
 * saturating) before P.V, the row sum uses the unrounded fp32 P values, and O
 * is written as bf16.  No scale factors: e4m3 covers +-448, which the
 * RMS-normalised q and k and the attention weights P <= 256 stay within.
 * Other arguments and checks as qi_attn_block_causal; ldq and ldkv must be
 * multiples of 16. */
int qi_attn_block_causal_fp8(qi_ctx* ctx, const uint8_t* q, int ldq, int Sq, int q_offset,
                             const uint8_t* k, const uint8_t* v, int ldkv, int Sk, int heads,
                             int head_dim, const qi_groups* groups, float sm_scale, uint16_t* o,
                             int ldo, void* stream);

/* y = e4m3(x) for n bf16 values (round to nearest, ties to even, saturating at
 * +-448); n % 16 == 0. */
int qi_to_e4m3(qi_ctx* ctx, const uint16_t* x, int64_t n, uint8_t* y, void* stream);

/* MXFP4 weights -> bf16 w [n, k] (k % 32 == 0, no padding; packed, scales
 * and w 16-byte aligned), the same values as qi_mxfp4_decode, each exact in
 * bf16.  One thread per 32-column scale group.  The block calls use it to
 * expand an MXFP4 Linear into qi_block_weights.mx_expand. */
int qi_mxfp4_expand_bf16(qi_ctx* ctx, const uint8_t* packed, const uint8_t* scales, int n, int k,
                         uint16_t* w, void* stream);

/* MXFP4 checkpoint weights -> fp32 ([PX] Runtime precision and quality /
 * What was quantized: E2M1 values packed low nibble first, an E8M0 scale per
 * group of 32 input columns; rows zero-padded to a multiple of 32 columns,
 * the padding removed on load).  packed [n, k_stored/2] bytes, scales
 * [n, k_stored/32] bytes, w [n, k] fp32 with k <= k_stored:
 *   w[r, c] = e2m1(code) * 2^(scale[r, c/32] - 127)   (E8M0 255 -> NaN)
 * E2M1 magnitudes (exponent bias 1, one mantissa bit): 0, 0.5, 1, 1.5, 2, 3,
 * 4, 6.  The result feeds qi_prepare_w8 like any fp32 weight.  The runtime
 * keeps the W8A8 int8 codes: the pages' MXFP4 is a storage format that a
 * loader reconstructs for computation. */
int qi_mxfp4_decode(qi_ctx* ctx, const uint8_t* packed, const uint8_t* scales, int n,
                    int k_stored, int k, float* w, void* stream);

/* Attention precision of the steps run on this context (qi_denoise_step,
 * qi_denoise_step_cfg): enable != 0 -> in every block the QKV projection
 * also writes e4m3 (round to nearest even, saturating) copies of the q, k, v
 * rows it produces, cached prefix K/V rows are converted the same way, and
 * qi_attn_block_causal_fp8's kernel runs on them
 * (the pages' schedule: the prefix pass and the first seven steps at full
 * precision, later steps with fp8 attention - the caller switches between
 * steps).  Block-level calls are not affected.  Default 0. */
int qi_ctx_set_attention_fp8(qi_ctx* ctx, int enable);

/* Copies of what each activation quantizer of a block reads and writes, for
 * checking those quantizers bit for bit at their own inputs ([W8]: dynamic
 * asymmetric INT8 per token with FP32 scales).  Every pointer is a caller-owned
 * device buffer for the block's T processed rows, or NULL to skip that tap.
 *   u1, u2     [T, H] fp32: LN(x)(1 + scale) + shift as the two LayerNorm
 *              quantizers computed and quantized it (written by those kernels)
 *   x_mid      [T, H] fp32: the residual stream after the attention half
 *              (x + gate1 * out), the input of the second LayerNorm
 *   o          [T, H] bf16: attention output, the input of the third quantizer
 *   g          [T, F] bf16: GELU output, the input of the fourth quantizer
 *   o_range, g_range [T, 2] uint32: the range the attention / GELU epilogue
 *              published for each row, as float bits of (-min(min, 0), max(max, 0))
 *   q*, s*, zp* codes [T, H or F] int8, scales [T] fp32, zero points [T] int32
 *              of quantizer 1 (u1), o (o), 2 (u2) and g (g).
 * The taps are copied with stream-ordered device copies after the kernels that
 * produce them; they cost time and are meant for tests. */
typedef struct qi_block_taps {
  float* u1;
  int8_t* q1;
  float* s1;
  int32_t* zp1;
  uint16_t* o;
  uint32_t* o_range;
  int8_t* qo;
  float* so;
  int32_t* zpo;
  float* x_mid;
  float* u2;
  int8_t* q2;
  float* s2;
  int32_t* zp2;
  uint16_t* g;
  uint32_t* g_range;
  int8_t* qg;
  float* sg;
  int32_t* zpg;
  float* x_layers;   /* qi_denoise_step only: [blocks + 1][T][H] fp32, the residual stream
                        before the first block and after each block */
} qi_block_taps;

/* Take the taps above in every block this context runs from now on (each block
 * overwrites them), or stop with taps = NULL.  The struct is copied; the
 * buffers must hold the T rows of the blocks run.  Host-side, no launch. */
int qi_ctx_set_block_taps(qi_ctx* ctx, const qi_block_taps* taps);

/* Workspace bytes needed by qi_dit_block_forward for T processed rows. */
int qi_block_workspace_bytes(const qi_dims* dims, int T, size_t* bytes);

/* One single-stream block on rows row0 .. row0+T-1 of the joint sequence:
 *   u1 = LN(x)(1 + scale1) + shift1 -> W8A8 QKV -> Q/K RMSNorm + RoPE
 *   x += gate1 * W8A8_out(attention)          (block-causal, keys 0 .. end of row's group)
 *   u2 = LN(x)(1 + scale2) + shift2 -> W8A8 up -> GELU-tanh -> W8A8 down
 *   x += gate2 * down
 * x: fp32 residual rows [T, H] (in/out).  mod: bf16 [R, 6, H] rows
 * (shift1, scale1, gate1, shift2, scale2, gate2) per row set.  rope_cos/sin:
 * [T, 64] fp32 tables of the processed rows.  k_layer / v_layer: this layer's
 * bf16 [S, H] key and value buffers (S = groups->end[n-1]); the call writes
 * rows row0 .. row0+T-1 and attends over rows 0 .. S-1 within the mask.
 * kv_mode NONE / WRITE_PREFIX need row0 == 0 and T == S; READ_PREFIX needs
 * row0 + T == S with rows 0 .. row0-1 already written by an earlier call
 * ([PX] cached prefix pass). */
int qi_dit_block_forward(qi_ctx* ctx, const qi_dims* dims, const qi_block_weights* w, float* x,
                         int T, int row0, const uint16_t* mod, const qi_groups* groups,
                         const float* rope_cos, const float* rope_sin, uint16_t* k_layer,
                         uint16_t* v_layer, int kv_mode, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Same block as qi_dit_block_forward, for callers that cannot allocate device
 * memory: a program that only receives input and output buffers from its host
 * framework, or one that runs under a fixed device-memory budget and must not
 * grow it at an unpredictable moment.  It takes no workspace argument and calls
 * no cudaMalloc, cudaFree or other allocating routine; its scratch is a fixed
 * 16 MiB array inside the library (every GPU that loads the library holds it
 * until the process exits).  The pages describe no such call; it has no
 * counterpart there.
 *   - Sizes whose scratch (qi_block_workspace_bytes) exceeds 16 MiB are rejected
 *     with QI_ERR_WORKSPACE before anything is launched (at hidden 256 / mlp
 *     1024 up to 4,071 rows fit; at hidden 4096 / mlp 16384 up to 255 rows).
 *   - The first call on a device looks up the array's device address (with
 *     that device current; the current device must be the context's) and
 *     caches it with the CUDA context it belongs to; a call in a new context
 *     (after a device reset) looks it up again.  Make the first call on a
 *     device, and the first after a reset, before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     The block writes each region before reading it; the per-row range
 *     tables that the attention and GELU epilogues fill with atomic maxima
 *     are cleared by the LayerNorm quantizers that run before them in the
 *     same call, so nothing needs clearing between calls.
 *     Calls whose kernels overlap on the GPU (different streams, or several
 *     host threads) race on it: serialize them.
 * Arguments and results are those of qi_dit_block_forward. */
int qi_dit_block_forward_noalloc(qi_ctx* ctx, const qi_dims* dims, const qi_block_weights* w,
                                 float* x, int T, int row0, const uint16_t* mod,
                                 const qi_groups* groups, const float* rope_cos,
                                 const float* rope_sin, uint16_t* k_layer, uint16_t* v_layer,
                                 int kv_mode, void* stream);

/* ------------------------------------------------------------------ step */

/* Timestep conditioning of a step: temb_r = t2(SiLU(t1(sinusoid(1000 t_r))))
 * for t_0 = 0 (conditioning prefix rows) and t_1 = sigma (target rows);
 * block_mod [blocks][2][6H] bf16 = mod_l(SiLU(temb_r)); final_mod [2H] bf16 =
 * final_mod(SiLU(temb_1)) as (shift, scale).  Workspace: qi_step_workspace_bytes. */
int qi_time_conditioning(qi_ctx* ctx, const qi_model* model, float sigma, uint16_t* block_mod,
                         uint16_t* final_mod, void* workspace, size_t workspace_bytes,
                         void* stream);

/* Workspace bytes needed by qi_denoise_step for a sequence of S tokens. */
int qi_step_workspace_bytes(const qi_dims* dims, int S, size_t* bytes);

/* One FlowMatch Euler denoising step ([GC] Graph contracts / Sampler):
 *   x = [txt_in(txt) | img_in(ref_latents) | img_in(latents)]
 *   x = blocks(x) with the time conditioning above
 *   v = proj_out(LN(x_target)(1 + scale) + shift);   latents += (sigma_next - sigma) v
 * latents [N, P] fp32 (in/out); txt [L, H] bf16 with L = text_tokens (NULL in
 * READ_PREFIX mode); ref_latents [R, P] fp32 for an edit sequence (NULL if
 * none; R = prefix tokens - L).  groups: the joint sequence, target last.
 * rope_cos/sin [S, 64] fp32 for the whole sequence.  kv_cache: bf16
 * [blocks][2][S][H] (K then V per block) holding the prefix K/V across steps;
 * may be NULL in QI_KV_NONE mode (workspace used).  v_out [N, P] fp32 gets the
 * velocity if not NULL. */
int qi_denoise_step(qi_ctx* ctx, const qi_model* model, float* latents, const uint16_t* txt,
                    int text_tokens, const float* ref_latents, const qi_groups* groups,
                    const float* rope_cos, const float* rope_sin, float sigma, float sigma_next,
                    int kv_mode, uint16_t* kv_cache, float* v_out, void* workspace,
                    size_t workspace_bytes, void* stream);

/* One sequence of a classifier-free-guidance step (qi_denoise_step_cfg);
 * the fields mean what the arguments of the same names of qi_denoise_step do. */
typedef struct qi_seq {
  const uint16_t* txt;        /* [text_tokens, H] bf16; may be NULL in READ_PREFIX mode */
  int text_tokens;
  const float* ref_latents;   /* [R, P] fp32 reference latents, NULL if none */
  const qi_groups* groups;    /* the joint sequence, target last */
  const float* rope_cos;      /* [S, 64] fp32 */
  const float* rope_sin;
  uint16_t* kv_cache;         /* [blocks][2][S][H] bf16; may be NULL in QI_KV_NONE mode */
} qi_seq;

/* Workspace bytes needed by qi_denoise_step_cfg for a conditional sequence of
 * S_cond tokens and an unconditional one of S_uncond, both ending in a target
 * group of target_tokens. */
int qi_step_cfg_workspace_bytes(const qi_dims* dims, int S_cond, int S_uncond, int target_tokens,
                                size_t* bytes);

/* One denoising step with true classifier-free guidance ([MNN] Install / run;
 * [QC] Native CLI cases).  The conditional sequence and the unconditional one
 * (a negative prompt of any text length, the same target and usually the same
 * references) run as one batch: every Linear, quantizer and norm runs once over
 * the rows of both (shared weights, twice the GEMM rows), attention runs per
 * sequence with its own mask and K/V.  Each sequence's velocity is
 * bit-identical to what qi_denoise_step computes for it alone.  Then
 *   v = v_u + guidance (v_c - v_u),   latents += (sigma_next - sigma) v
 * in fp32 with one rounding per operation and no fused multiply-add (the pages
 * give the guidance scale but no formula; this is the plain reading, with no
 * renormalization).  latents [N, P] fp32 (in/out); v_out [N, P] fp32 gets the
 * guided v if not NULL.  Both target groups must hold N tokens; each sequence
 * may have up to QI_MAX_GROUPS groups (its prefix groups use row set 0 and its
 * target row set 1, as for qi_denoise_step, so the batch's table of row sets
 * holds two runs per sequence whatever the number of references).
 * kv_mode applies to both sequences (each with its own kv_cache). */
int qi_denoise_step_cfg(qi_ctx* ctx, const qi_model* model, float* latents, const qi_seq* cond,
                        const qi_seq* uncond, float guidance, float sigma, float sigma_next,
                        int kv_mode, float* v_out, void* workspace, size_t workspace_bytes,
                        void* stream);

/* x += (sigma_next - sigma) * v over n fp32 values, one rounding per operation
 * (no fused multiply-add); sigma_next - sigma is rounded to fp32 first ([GC] Sampler). */
int qi_euler_update(qi_ctx* ctx, float* x, const float* v, int64_t n, float sigma,
                    float sigma_next, void* stream);

/* ------------------------------------------------------------------ host helpers */

/* RoPE tables ([GC] RoPE): text token i at (i, i, i); image token (y, x) of the
 * k-th image group (h x w grid, raster order) at (L + k, y - (h - h/2), x - (w - w/2)),
 * L = number of text tokens.  Rotation pairs 0..7 use the frame axis, 8..35 the
 * h axis, 36..63 the w axis; pair i of an axis with n pairs has frequency
 * 10000^(-i/n).  kinds[g]: 0 text, 1 image.  Writes HOST arrays cos/sin [S, 64]. */
int qi_rope_tables(int n_groups, const int32_t* kinds, const int32_t* tokens,
                   const int32_t* grid_h, const int32_t* grid_w, float* rope_cos,
                   float* rope_sin);

/* Shifted FlowMatch sigmas ([GC] Sampler): linspace(1, 1/steps, steps) shifted by
 * e^mu / (e^mu + 1/sigma - 1), mu linear in image_tokens (0.5 at 256 tokens,
 * 0.9 at 8192), tail stretched to 0.02, then 0 appended.  Writes HOST sigmas[steps+1]. */
int qi_sigma_schedule(int steps, int image_tokens, float* sigmas);

/* Tensor-pipe probe (measurement support): one CTA per SM issues iters x 4
 * back-to-back tcgen05.mma (M = 128, N = 256, K = 32 int8 bytes for
 * int8 != 0, else K = 16 bf16 values) on pseudo-random operands held in shared
 * memory, with no memory traffic and no epilogue.  Work per launch:
 * num_SMs * iters * 4 * 2 * 128 * 256 * K operations.  Time it with CUDA events
 * on `stream`; the result is the tensor pipe's dense rate at the clock the GPU
 * holds meanwhile.  iters in 1 .. 100000. */
int qi_debug_mma_probe(qi_ctx* ctx, int int8, int iters, void* stream);

/* Failure-detection probe: launch one CTA that waits on an mbarrier nothing
 * arrives on, bounded by limit_ns (1e3 .. 5e9).  The wait expires, the kernel
 * records QI_ERR_TIMEOUT in the status word and returns; the context stays
 * usable.  Read the result with qi_ctx_check(). */
int qi_debug_timeout_probe(qi_ctx* ctx, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QI_H_ */
