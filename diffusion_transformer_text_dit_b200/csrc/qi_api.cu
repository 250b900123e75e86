// C ABI of libqi (declared in include/qi.h): host-side validation, workspace
// carving and the orchestration of the block and of the denoising step.
// Every argument check runs before the first launch of a call.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <string>

#include "qi.h"
#include "qi_common.cuh"
#include "qi_internal.h"

// Optional per-launch timing: when enabled, every kernel launch of the library
// is bracketed by a pair of CUDA events on its stream; durations are summed per
// kernel class when read back.  Launches are counted per class either way.
constexpr int QI_PROF_CLASSES = 8;
constexpr int QI_PROF_MAX_PAIRS = 16384;

struct qi_ctx {
  int device;
  int num_sms;
  int* status;   // device status word
  bool prof_on;
  int prof_used;
  cudaEvent_t* prof_ev;          // [2 * QI_PROF_MAX_PAIRS]
  int* prof_cls;                 // [QI_PROF_MAX_PAIRS]
  long long launches[QI_PROF_CLASSES];
  int attn_fp8;                  // steps run e4m3 attention (qi_ctx_set_attention_fp8)
  bool taps_on;                  // copy the quantizers' inputs and outputs (qi_ctx_set_block_taps)
  qi_block_taps taps;
  void* attn_scratch;            // key-range split scratch of qi_attn_block_causal(_fp8)
  size_t attn_scratch_bytes;
};

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) {   // already read by the launcher
    e = qi::last_launch_error();
    qi::last_launch_error() = cudaSuccess;
  }
  return fail(QI_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }

struct Prof {
  qi_ctx* c;
  int slot;
  cudaStream_t st;
  Prof(qi_ctx* ctx, int cls, cudaStream_t s) : c(ctx), slot(-1), st(s) {
    if (!c) return;
    c->launches[cls] += 1;
    if (c->prof_on && c->prof_used < QI_PROF_MAX_PAIRS) {
      slot = c->prof_used++;
      c->prof_cls[slot] = cls;
      cudaEventRecord(c->prof_ev[2 * slot], st);
    }
  }
  ~Prof() {
    if (slot >= 0) cudaEventRecord(c->prof_ev[2 * slot + 1], st);
  }
};

// Validate a group table against a sequence length; fill the device-side copy.
int check_groups(const qi_groups* g, int total, qi::GroupTable* out) {
  if (!g) return fail(QI_ERR_INVALID_ARG, "groups is NULL");
  if (g->n < 1 || g->n > QI_MAX_GROUPS)
    return fail(QI_ERR_INVALID_ARG, "groups->n = %d outside 1..%d", g->n, QI_MAX_GROUPS);
  int prev = 0;
  for (int i = 0; i < g->n; ++i) {
    if (g->end[i] <= prev)
      return fail(QI_ERR_INVALID_ARG, "group ends must be strictly ascending and positive");
    if (g->row_set[i] < 0) return fail(QI_ERR_INVALID_ARG, "negative row set");
    prev = g->end[i];
  }
  if (total >= 0 && prev != total)
    return fail(QI_ERR_INVALID_ARG, "groups->end[n-1] = %d but the sequence has %d tokens", prev,
                total);
  if (out) {
    memset(out, 0, sizeof(*out));
    out->n = g->n;
    for (int i = 0; i < g->n; ++i) {
      out->end[i] = g->end[i];
      out->row_set[i] = g->row_set[i];
    }
  }
  return QI_OK;
}

int check_dims(const qi_dims* d) {
  if (!d) return fail(QI_ERR_INVALID_ARG, "dims is NULL");
  if (d->head_dim != 128) return fail(QI_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (d->heads < 1 || d->hidden != d->heads * d->head_dim)
    return fail(QI_ERR_INVALID_ARG, "hidden must equal heads * head_dim");
  if (d->hidden % 256 != 0 || d->hidden > 16384)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "hidden must be a multiple of 256, at most 16384");
  if (d->mlp % 128 != 0 || d->mlp < 128 || d->mlp > 16384)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "mlp must be a multiple of 128 in 128..16384");
  if (d->patch % 64 != 0 || d->patch < 64)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "patch must be a positive multiple of 64");
  if (d->blocks < 1 || d->blocks > 64)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "blocks must be in 1..64");
  if (!(d->eps >= 0.f)) return fail(QI_ERR_INVALID_ARG, "eps must be >= 0");
  return QI_OK;
}

int check_w8(const qi_w8* w, const char* name, int n, int k) {
  if (!w || !w->q || !w->s || !w->rowsum)
    return fail(QI_ERR_INVALID_ARG, "W8A8 weight %s has a NULL pointer", name);
  if ((n >= 0 && w->n != n) || (k >= 0 && w->k != k))
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "W8A8 weight %s is [%d, %d], expected [%d, %d]", name,
                w->n, w->k, n, k);
  if (w->k % 128 != 0 || w->k < 128)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "W8A8 weight %s: k = %d is not a multiple of 128", name,
                w->k);
  if (w->n % 16 != 0 || w->n < 16)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "W8A8 weight %s: n = %d is not a multiple of 16", name,
                w->n);
  if (!aligned16(w->q) || !aligned16(w->s) || !aligned16(w->rowsum) ||
      (w->bias && !aligned16(w->bias)))
    return fail(QI_ERR_ALIGNMENT, "W8A8 weight %s: pointers must be 16-byte aligned", name);
  return QI_OK;
}

int check_bf16_linear(const qi_linear_bf16* w, const char* name, int n, int k) {
  if (!w || !w->w) return fail(QI_ERR_INVALID_ARG, "BF16 weight %s is NULL", name);
  if ((n >= 0 && w->n != n) || (k >= 0 && w->k != k))
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "BF16 weight %s is [%d, %d], expected [%d, %d]", name,
                w->n, w->k, n, k);
  if (!aligned16(w->w) || (w->bias && !aligned16(w->bias)))
    return fail(QI_ERR_ALIGNMENT, "BF16 weight %s: pointers must be 16-byte aligned", name);
  return QI_OK;
}

// Bump allocator over the caller's workspace (256-byte aligned pieces).
struct Carve {
  uint8_t* base;
  size_t cap, off;
  template <class T>
  T* take(size_t count) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = reinterpret_cast<T*>(base ? base + off : nullptr);
    off += count * sizeof(T);
    return p;
  }
};

struct BlockBufs {
  int8_t* uq;       // [T, max(H, F)]
  float* sa;        // [T]
  int32_t* zp;      // [T]
  uint16_t* q;      // [T, H]
  uint16_t* o;      // [T, H]
  uint16_t* g;      // [T, F]
  uint32_t* o_range;   // [T][2] row ranges of the attention output
  uint32_t* g_range;   // [T][2] row ranges of the GELU output
};

BlockBufs carve_block(Carve& c, const qi_dims& d, int T) {
  BlockBufs b;
  const size_t H = d.hidden, F = d.mlp, W = H > F ? H : F;
  b.uq = c.take<int8_t>(static_cast<size_t>(T) * W);
  b.sa = c.take<float>(T);
  b.zp = c.take<int32_t>(T);
  b.q = c.take<uint16_t>(static_cast<size_t>(T) * H);
  b.o = c.take<uint16_t>(static_cast<size_t>(T) * H);
  b.g = c.take<uint16_t>(static_cast<size_t>(T) * F);
  b.o_range = c.take<uint32_t>(static_cast<size_t>(T) * 2);
  b.g_range = c.take<uint32_t>(static_cast<size_t>(T) * 2);
  return b;
}

size_t block_bytes(const qi_dims& d, int T) {
  Carve c{nullptr, 0, 0};
  carve_block(c, d, T);
  return c.off + 256;
}

// e4m3 copies of the attention operands of one block (fp8 attention): q for
// the batch's processed rows, then per sequence its K rows and its V rows.
struct Fp8Bufs {
  uint8_t* q;
  uint8_t* kv;
};

struct StepBufs {
  float* x;             // [S, H] fp32 residual stream
  float* emb;           // [2, 256]
  float* h1;            // [2, H]
  float* temb;          // [2, H]
  uint16_t* block_mod;  // [blocks][2][6H]
  uint16_t* final_mod;  // [2][2H]
  uint16_t* lat_bf16;   // [S, P] bf16 copies of the latents fed to img_in
  uint16_t* u_final;    // [S, H]
  uint16_t* kv;         // [blocks][2][S][H] when the caller passes no cache
  Fp8Bufs f8;           // e4m3 attention operands (fp8 attention)
  uint8_t* block_ws;
  size_t block_ws_bytes;
};

StepBufs carve_step(Carve& c, const qi_dims& d, int Sq, int S, bool own_kv) {
  StepBufs b;
  const size_t H = d.hidden, P = d.patch;
  b.x = c.take<float>(static_cast<size_t>(Sq) * H);
  b.emb = c.take<float>(2 * 256);
  b.h1 = c.take<float>(2 * H);
  b.temb = c.take<float>(2 * H);
  b.block_mod = c.take<uint16_t>(static_cast<size_t>(d.blocks) * 2 * 6 * H);
  b.final_mod = c.take<uint16_t>(2 * 2 * H);
  b.lat_bf16 = c.take<uint16_t>(static_cast<size_t>(S) * P);
  b.u_final = c.take<uint16_t>(static_cast<size_t>(S) * H);
  b.kv = own_kv ? c.take<uint16_t>(static_cast<size_t>(d.blocks) * 2 * S * H) : nullptr;
  b.f8.q = c.take<uint8_t>(static_cast<size_t>(Sq) * H);
  b.f8.kv = c.take<uint8_t>(static_cast<size_t>(2) * S * H);
  b.block_ws_bytes = block_bytes(d, Sq);
  b.block_ws = c.take<uint8_t>(b.block_ws_bytes);
  return b;
}

}  // namespace

// ---------------------------------------------------------------- TMA encode

namespace qi {

bool make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, uint64_t inner,
                  uint64_t outer, uint64_t row_stride_bytes, uint32_t box_inner,
                  uint32_t box_outer, bool swizzle128) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE,
                            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace qi

// ---------------------------------------------------------------- internal ops

namespace {

struct QuantExtras {
  const uint16_t* res_y = nullptr;     // LN: residual add x + gate * y first ...
  const uint16_t* res_gate = nullptr;
  float* res_out = nullptr;            // ... written here if set
  uint32_t* zero_range = nullptr;      // LN: clear these row ranges
  uint32_t* zero_words = nullptr;      // LN: clear these words (n_zero_words of them)
  int n_zero_words = 0;
  const uint32_t* range = nullptr;     // plain: producer-published row ranges
  float* u_f32 = nullptr;              // LN: also write the quantized value u (fp32 tap)
  bool quant_too = false;              // LN with u_bf16: quantize as well as write bf16(u)
};

// Stream-ordered device copy of a tap (skipped when the tap is NULL).
int tap_copy(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  if (!dst || bytes == 0) return QI_OK;
  if (cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
    return cuda_fail("tap copy");
  return QI_OK;
}

// Copy one quantizer's codes, scales and zero points into the taps.
int tap_codes(int8_t* q_dst, float* s_dst, int32_t* zp_dst, const int8_t* q, const float* s,
              const int32_t* zp, int T, int K, cudaStream_t st) {
  int r;
  if ((r = tap_copy(q_dst, q, static_cast<size_t>(T) * K, st))) return r;
  if ((r = tap_copy(s_dst, s, static_cast<size_t>(T) * sizeof(float), st))) return r;
  return tap_copy(zp_dst, zp, static_cast<size_t>(T) * sizeof(int32_t), st);
}

int run_quant(qi_ctx* ctx, const void* x, bool xbf16, int M, int K, int ldx,
              const uint16_t* shift, const uint16_t* scale, int mod_ld, const qi::GroupTable& gt,
              int row0, float eps, int8_t* q, float* s, int32_t* zp, uint16_t* u_bf16,
              cudaStream_t st, const QuantExtras& ex = QuantExtras()) {
  qi::QuantParams p;
  memset(&p, 0, sizeof(p));
  p.res_y = ex.res_y;
  p.res_gate = ex.res_gate;
  p.res_out = ex.res_out;
  p.zero_range = ex.zero_range;
  p.zero_words = ex.n_zero_words > 0 ? ex.zero_words : nullptr;
  p.n_zero_words = ex.n_zero_words;
  p.range = ex.range;
  p.u_f32 = ex.u_f32;
  p.quant_too = ex.quant_too ? 1 : 0;
  p.x = x;
  p.x_bf16 = xbf16 ? 1 : 0;
  p.M = M;
  p.K = K;
  p.ldx = ldx;
  p.ln = shift ? 1 : 0;
  p.shift = shift;
  p.scale = scale;
  p.mod_ld = mod_ld;
  p.groups = gt;
  p.row0 = row0;
  p.eps = eps;
  p.q = q;
  p.ldq = K;
  p.s = s;
  p.zp = zp;
  p.u_bf16 = u_bf16;
  p.status = ctx->status;
  Prof pr(ctx, QI_KCLASS_QUANT, st);
  if (qi::launch_quant(p, st) != 0) return cuda_fail("quantize launch");
  return QI_OK;
}

int run_w8a8(qi_ctx* ctx, const int8_t* qa, const float* sa, const int32_t* zp, int M,
             const qi_w8& w, int epi, uint16_t* y, int ldy, float* res, int ldr,
             const uint16_t* gate, int gate_ld, const qi::GroupTable& gt, int row0,
             int32_t* acc_debug, cudaStream_t st, uint32_t* row_range = nullptr,
             const uint16_t* res_y = nullptr, int ld_res_y = 0, const uint16_t* gate1 = nullptr) {
  if (M == 0) return QI_OK;
  qi::GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = w.n;
  p.K = w.k;
  p.num_kb = w.k / 128;
  p.s_a = sa;
  p.zp_a = zp;
  p.s_w = w.s;
  p.rowsum = w.rowsum;
  p.bias = w.bias;
  p.y = y;
  p.ldy = ldy;
  p.yf = res;
  p.ldyf = ldr;
  p.gate = gate;
  p.gate_ld = gate_ld;
  p.res_y = res_y;
  p.ld_res_y = ld_res_y;
  p.gate1 = gate1;
  p.groups = gt;
  p.row0 = row0;
  p.acc_debug = acc_debug;
  p.row_range = row_range;
  p.status = ctx->status;
  Prof pr(ctx, QI_KCLASS_GEMM_I8, st);
  const int r = qi::launch_gemm(true, epi, qa, w.k, w.q, w.k, p, ctx->num_sms, st);
  if (r == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (W8A8 operands)");
  if (r != 0) return cuda_fail("W8A8 GEMM launch");
  return QI_OK;
}

int run_bf16_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_linear_bf16& w,
                    int epi, float* yf, int ldyf, float dt, float* v_out, cudaStream_t st) {
  if (M == 0) return QI_OK;
  qi::GemmParams p;
  memset(&p, 0, sizeof(p));
  p.M = M;
  p.N = w.n;
  p.K = w.k;
  p.num_kb = w.k / 64;
  p.bias = w.bias;
  p.yf = yf;
  p.ldyf = ldyf;
  p.dt = dt;
  p.v_out = v_out;
  p.status = ctx->status;
  Prof pr(ctx, QI_KCLASS_GEMM_BF16, st);
  const int r = qi::launch_gemm(false, epi, a, lda, w.w, w.k, p, ctx->num_sms, st);
  if (r == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (BF16 operands)");
  if (r != 0) return cuda_fail("BF16 GEMM launch");
  return QI_OK;
}

// One sequence of a block batch: its processed rows are rows off .. off+T-1 of
// the batch; they are rows row0 .. row0+T-1 of the sequence, whose S keys and
// values live in kl / vl ([S, H] bf16 each) and whose groups define the mask.
struct SeqAttn {
  int off, T, row0, S;
  qi::GroupTable gt;
  uint16_t* kl;
  uint16_t* vl;
};

// Which Linears of a block are W8A8 and which BF16 (qi_block_weights).
struct BlockPrecision {
  int qkv_w8_cols;   // columns of q | k | v computed by the W8A8 GEMM: 3H, 2H (v BF16) or 0
  bool out_w8, up_w8, down_w8;
};

BlockPrecision block_precision(const qi_dims& d, const qi_block_weights& w) {
  BlockPrecision bp;
  bp.qkv_w8_cols = w.qkv.q ? w.qkv.n : 0;
  bp.out_w8 = w.out.q != nullptr;
  bp.up_w8 = w.up.q != nullptr;
  bp.down_w8 = w.down.q != nullptr;
  (void)d;
  return bp;
}

// A BF16 block Linear on tcgen05 kind::f16 (CTA pairs for 256-wide tiles)
// with one of the block epilogues; `p` carries the epilogue fields.
// Where an MXFP4 Linear is expanded to bf16 before its GEMM (MxExpand::buf
// null: decoded inside the GEMM).  early: the expansion may overlap the
// kernel before it (the buffer's previous reader is at least two kernels
// back).
struct MxExpand {
  uint16_t* buf = nullptr;
  size_t bytes = 0;
  bool early = false;
};

int run_bf16_block_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_linear_bf16& w,
                          const qi_mxfp4& mx, int epi, qi::GemmParams p, cudaStream_t st,
                          const MxExpand& ex = MxExpand()) {
  if (M == 0) return QI_OK;
  if (mx.packed && ex.buf &&
      ex.bytes >= static_cast<size_t>(mx.n) * static_cast<size_t>(mx.k) * sizeof(uint16_t)) {
    // expand the MXFP4 weights into the scratch, then run them as BF16
    uint16_t* expand = ex.buf;
    {
      Prof pr(ctx, QI_KCLASS_OTHER, st);
      if (qi::launch_mxfp4_expand_bf16(mx.packed, mx.scales, mx.n, mx.k, expand, st, ex.early))
        return cuda_fail("MXFP4 expansion launch");
    }
    qi_linear_bf16 wb;
    memset(&wb, 0, sizeof(wb));
    wb.w = expand;
    wb.bias = mx.bias;
    wb.n = mx.n;
    wb.k = mx.k;
    qi_mxfp4 none;
    memset(&none, 0, sizeof(none));
    return run_bf16_block_linear(ctx, a, M, lda, wb, none, epi, p, st);
  }
  const bool is_mx = mx.packed != nullptr;
  p.M = M;
  p.N = is_mx ? mx.n : w.n;
  p.K = is_mx ? mx.k : w.k;
  p.num_kb = p.K / 64;
  p.s_a = nullptr;
  p.zp_a = nullptr;
  p.s_w = nullptr;
  p.rowsum = nullptr;
  p.bias = is_mx ? mx.bias : w.bias;
  p.b_packed = is_mx ? mx.packed : nullptr;
  p.b_scales = is_mx ? mx.scales : nullptr;
  p.status = ctx->status;
  Prof pr(ctx, QI_KCLASS_GEMM_BF16, st);
  const int r = qi::launch_gemm(false, epi, a, lda, is_mx ? nullptr : w.w, p.K, p, ctx->num_sms, st);
  if (r == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (BF16 block Linear)");
  if (r != 0) return cuda_fail("BF16 block Linear launch");
  return QI_OK;
}

// One block over the processed rows of up to two sequences (a true-CFG batch):
// every Linear, quantizer and norm runs once over all T rows (rows_gt maps a
// row, offset by rows_row0, to its modulation row set; cs/sn hold the RoPE
// tables of the T rows); attention runs per sequence.  Each Linear is W8A8 or
// BF16 as the weights say; a BF16 Linear reads the bf16 activation (for the
// LayerNorm values, the LN kernel writes it into the attention-output buffer,
// which is free at that point).
int run_block_multi(qi_ctx* ctx, const qi_dims& d, const qi_block_weights& w, float* x, int T,
                    const qi::GroupTable& rows_gt, int rows_row0, const uint16_t* mod,
                    const float* cs, const float* sn, const SeqAttn* seqs, int nseq, uint8_t* ws,
                    size_t ws_bytes, cudaStream_t st, const Fp8Bufs* f8 = nullptr) {
  const int H = d.hidden, F = d.mlp;
  const qi::GroupTable& gt = rows_gt;
  const int row0 = rows_row0;
  Carve c{ws, ws_bytes, 0};
  BlockBufs b = carve_block(c, d, T);
  const BlockPrecision bp = block_precision(d, w);
  const int mld = 6 * H;
  int r;
  // attention half.  LN1 + modulate + quantize (and/or the bf16 value for a
  // BF16 q | k | v part); it also clears the row ranges that the attention
  // epilogue will publish for the next quantizer.
  const qi_block_taps* tp = ctx->taps_on ? &ctx->taps : nullptr;
  const bool qkv_bf16 = bp.qkv_w8_cols < 3 * H;
  // MXFP4 expansion scratch.  With room for two of the largest Linears the
  // Linears alternate between two halves (q | k | v and up in the first, out
  // and down in the second): a half's previous reader is then at least two
  // kernels before its next expansion, which may start early.  Otherwise all
  // share the one buffer and each expansion waits for the kernel before it.
  MxExpand mxa, mxb;
  if (w.mx_expand) {
    const size_t lin = static_cast<size_t>(std::max(3 * H, F)) * H * sizeof(uint16_t);
    mxa.buf = mxb.buf = w.mx_expand;
    mxa.bytes = mxb.bytes = w.mx_expand_bytes;
    if (w.mx_expand_bytes >= 2 * lin) {
      mxb.buf = w.mx_expand + lin / sizeof(uint16_t);
      mxa.bytes = mxb.bytes = lin;
      mxa.early = mxb.early = true;
    }
  }
  // The attention's key-range split uses the GELU buffer b.g as scratch (free
  // until the up projection).  The plan assumes the bytes of the sequence's
  // last group (T_last x F bf16), a bound that does not depend on which rows
  // this call processes; the launch checks its own need against the T x F
  // bf16 the buffer holds.  LN1 clears the split counters.
  const size_t g_bytes = static_cast<size_t>(T) * F * sizeof(uint16_t);
  auto split_setup = [&](const SeqAttn& q, qi::AttnParams& ap) {
    const int start_last = q.gt.n >= 2 ? q.gt.end[q.gt.n - 2] : 0;
    ap.Sk = q.S;
    ap.heads = d.heads;
    ap.groups = q.gt;
    ap.num_sms = ctx->num_sms;
    ap.split_scratch = b.g;
    ap.split_bytes = static_cast<size_t>(q.S - start_last) * F * sizeof(uint16_t);
    ap.split_have = g_bytes;
  };
  size_t split_counters = 0;
  for (int sq = 0; sq < nseq; ++sq) {
    qi::AttnParams ap;
    memset(&ap, 0, sizeof(ap));
    split_setup(seqs[sq], ap);
    int kh = 0;
    size_t need = 0, counters = 0;
    qi::attention_split_plan(ap, &kh, &need, &counters);
    if (counters > split_counters) split_counters = counters;
  }
  {
    QuantExtras ex;
    ex.zero_words = reinterpret_cast<uint32_t*>(b.g);
    ex.n_zero_words = static_cast<int>(std::min(split_counters, g_bytes) / 4);
    ex.zero_range = b.o_range;
    ex.u_f32 = tp ? tp->u1 : nullptr;
    ex.quant_too = bp.qkv_w8_cols > 0;
    if ((r = run_quant(ctx, x, false, T, H, H, mod + 0 * H, mod + 1 * H, mld, gt, row0, d.eps,
                       b.uq, b.sa, b.zp, qkv_bf16 ? b.o : nullptr, st, ex)))
      return r;
    if (tp && bp.qkv_w8_cols > 0 &&
        (r = tap_codes(tp->q1, tp->s1, tp->zp1, b.uq, b.sa, b.zp, T, H, st)))
      return r;
  }
  // QKV projection with Q/K RMSNorm + RoPE fused into its epilogue: q goes to
  // the block's q buffer, k and v straight into this layer's K/V rows.
  {
    qi::GemmParams p;
    memset(&p, 0, sizeof(p));
    p.H = H;
    p.eps = d.eps;
    p.wq = w.norm_q;
    p.wk = w.norm_k;
    p.rcos = cs;
    p.rsin = sn;
    p.q_out = b.q;
    p.k_out = seqs[0].kl + static_cast<size_t>(seqs[0].row0) * H;
    p.v_out_bf16 = seqs[0].vl + static_cast<size_t>(seqs[0].row0) * H;
    if (nseq > 1) {
      p.kv_split = seqs[1].off;
      p.k_out2 = seqs[1].kl + static_cast<size_t>(seqs[1].row0) * H;
      p.v_out2 = seqs[1].vl + static_cast<size_t>(seqs[1].row0) * H;
    }
    if (f8) {
      // e4m3 copies for fp8 attention, written by the same epilogue: q rows,
      // and each sequence's K/V rows at their place in its e4m3 K | V block
      p.q8_out = f8->q;
      const size_t n0 = static_cast<size_t>(seqs[0].S) * H;
      p.k8_out = f8->kv + static_cast<size_t>(seqs[0].row0) * H;
      p.v8_out = f8->kv + n0 + static_cast<size_t>(seqs[0].row0) * H;
      if (nseq > 1) {
        const size_t n1 = static_cast<size_t>(seqs[1].S) * H;
        p.k8_out2 = f8->kv + 2 * n0 + static_cast<size_t>(seqs[1].row0) * H;
        p.v8_out2 = f8->kv + 2 * n0 + n1 + static_cast<size_t>(seqs[1].row0) * H;
      }
    }
    p.ldo = H;
    p.status = ctx->status;
    if (bp.qkv_w8_cols > 0) {
      qi::GemmParams pw = p;
      pw.M = T;
      pw.N = w.qkv.n;
      pw.K = w.qkv.k;
      pw.num_kb = w.qkv.k / 128;
      pw.s_a = b.sa;
      pw.zp_a = b.zp;
      pw.s_w = w.qkv.s;
      pw.rowsum = w.qkv.rowsum;
      pw.bias = w.qkv.bias;
      pw.n_base = 0;
      Prof pr(ctx, QI_KCLASS_GEMM_I8, st);
      const int rr = qi::launch_gemm(true, qi::EPI_QKV, b.uq, w.qkv.k, w.qkv.q, w.qkv.k, pw,
                                     ctx->num_sms, st);
      if (rr == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (QKV operands)");
      if (rr != 0) return cuda_fail("QKV GEMM launch");
    }
    if (qkv_bf16) {
      p.n_base = bp.qkv_w8_cols;   // the v rows (2H) or all of q | k | v (0)
      if ((r = run_bf16_block_linear(ctx, b.o, T, H, w.qkv_bf16, w.qkv_mx, qi::EPI_QKV, p, st, mxa)))
        return r;
    }
  }
  if (f8) {
    // fp8 attention: the QKV epilogue wrote e4m3 q and the e4m3 K/V rows it
    // produced; the K/V rows this call did not produce (a cached prefix) are
    // cast from their bf16 rows
    size_t o = 0;
    for (int sq = 0; sq < nseq; ++sq) {
      const size_t n = static_cast<size_t>(seqs[sq].S) * H;
      const int lo = seqs[sq].row0, hi = seqs[sq].row0 + seqs[sq].T;   // rows written above
      const int spans[2][2] = {{0, lo}, {hi, seqs[sq].S}};
      for (const auto& sp : spans) {
        if (sp[1] <= sp[0]) continue;
        Prof pr(ctx, QI_KCLASS_OTHER, st);
        const size_t r0 = static_cast<size_t>(sp[0]) * H;
        const int64_t cnt = static_cast<int64_t>(sp[1] - sp[0]) * H;
        if (qi::launch_bf16_to_e4m3(seqs[sq].kl + r0, f8->kv + o + r0, cnt, st) ||
            qi::launch_bf16_to_e4m3(seqs[sq].vl + r0, f8->kv + o + n + r0, cnt, st))
          return cuda_fail("e4m3 cast launch");
      }
      o += 2 * n;
    }
  }
  size_t kv8 = 0;
  for (int sq = 0; sq < nseq; ++sq) {
    const SeqAttn& q = seqs[sq];
    qi::AttnParams ap;
    memset(&ap, 0, sizeof(ap));
    if (f8) {
      const size_t n = static_cast<size_t>(q.S) * H;
      ap.q = f8->q + static_cast<size_t>(q.off) * H;
      ap.k = f8->kv + kv8;
      ap.v = f8->kv + kv8 + n;
      ap.fp8 = 1;
      kv8 += 2 * n;
    } else {
      ap.q = b.q + static_cast<size_t>(q.off) * H;
      ap.k = q.kl;
      ap.v = q.vl;
    }
    ap.o = b.o + static_cast<size_t>(q.off) * H;
    ap.ldq = H;
    ap.ldkv = H;
    ap.ldo = H;
    ap.Sq = q.T;
    ap.Sk = q.S;
    ap.heads = d.heads;
    ap.q_offset = q.row0;
    ap.sm_scale = 1.0f / sqrtf(static_cast<float>(d.head_dim));
    ap.groups = q.gt;
    ap.row_range = bp.out_w8 ? b.o_range + 2 * static_cast<size_t>(q.off) : nullptr;
    split_setup(q, ap);
    ap.status = ctx->status;
    Prof pr(ctx, QI_KCLASS_ATTN, st);
    const int r2 = qi::launch_attention(ap, st);
    if (r2 == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (attention operands)");
    if (r2 != 0) return cuda_fail("attention launch");
  }
  if (tp && ((r = tap_copy(tp->o, b.o, static_cast<size_t>(T) * H * 2, st)) ||
             (bp.out_w8 && (r = tap_copy(tp->o_range, b.o_range, static_cast<size_t>(T) * 8, st)))))
    return r;
  // output projection stored as bf16 into the q buffer (consumed by the
  // attention); its gated residual is applied by the LN2 kernel below, which
  // reads the residual stream anyway
  uint16_t* y_out = b.q;
  if (bp.out_w8) {
    {
      QuantExtras ex;   // the attention epilogue published each row's range
      ex.range = b.o_range;
      if ((r = run_quant(ctx, b.o, true, T, H, H, nullptr, nullptr, 0, gt, row0, d.eps, b.uq,
                         b.sa, b.zp, nullptr, st, ex)))
        return r;
      if (tp && (r = tap_codes(tp->qo, tp->so, tp->zpo, b.uq, b.sa, b.zp, T, H, st))) return r;
    }
    if ((r = run_w8a8(ctx, b.uq, b.sa, b.zp, T, w.out, qi::EPI_BF16, y_out, H, nullptr, 0, nullptr,
                      0, gt, row0, nullptr, st)))
      return r;
  } else {
    qi::GemmParams p;
    memset(&p, 0, sizeof(p));
    p.y = y_out;
    p.ldy = H;
    if ((r = run_bf16_block_linear(ctx, b.o, T, H, w.out_bf16, w.out_mx, qi::EPI_BF16, p, st, mxb)))
      return r;
  }
  // MLP half: LN2 + modulate + quantize of x + gate1 * out (and/or the
  // bf16 value for a BF16 up projection, into the attention-output buffer,
  // now consumed); clears the GELU ranges.  The stream itself is not written
  // here: the down projection's epilogue adds gate1 * out (y_out, untouched
  // until the next block's QKV projection) along with its own term.
  {
    QuantExtras ex;
    ex.res_y = y_out;
    ex.res_gate = mod + 2 * H;
    ex.res_out = tp ? tp->x_mid : nullptr;
    ex.zero_range = b.g_range;
    ex.u_f32 = tp ? tp->u2 : nullptr;
    ex.quant_too = bp.up_w8;
    if ((r = run_quant(ctx, x, false, T, H, H, mod + 3 * H, mod + 4 * H, mld, gt, row0, d.eps,
                       b.uq, b.sa, b.zp, bp.up_w8 ? nullptr : b.o, st, ex)))
      return r;
    if (tp && bp.up_w8 && (r = tap_codes(tp->q2, tp->s2, tp->zp2, b.uq, b.sa, b.zp, T, H, st)))
      return r;
  }
  uint32_t* g_range = bp.down_w8 ? b.g_range : nullptr;
  if (bp.up_w8) {
    if ((r = run_w8a8(ctx, b.uq, b.sa, b.zp, T, w.up, qi::EPI_GELU, b.g, F, nullptr, 0, nullptr, 0,
                      gt, row0, nullptr, st, g_range)))
      return r;
  } else {
    qi::GemmParams p;
    memset(&p, 0, sizeof(p));
    p.y = b.g;
    p.ldy = F;
    p.row_range = g_range;
    if ((r = run_bf16_block_linear(ctx, b.o, T, H, w.up_bf16, w.up_mx, qi::EPI_GELU, p, st, mxa)))
      return r;
  }
  if (tp && ((r = tap_copy(tp->g, b.g, static_cast<size_t>(T) * F * 2, st)) ||
             (bp.down_w8 && (r = tap_copy(tp->g_range, b.g_range, static_cast<size_t>(T) * 8, st)))))
    return r;
  if (bp.down_w8) {
    {
      QuantExtras ex;   // the GELU epilogue published each row's range
      ex.range = b.g_range;
      if ((r = run_quant(ctx, b.g, true, T, F, F, nullptr, nullptr, 0, gt, row0, d.eps, b.uq,
                         b.sa, b.zp, nullptr, st, ex)))
        return r;
      if (tp && (r = tap_codes(tp->qg, tp->sg, tp->zpg, b.uq, b.sa, b.zp, T, F, st))) return r;
    }
    if ((r = run_w8a8(ctx, b.uq, b.sa, b.zp, T, w.down, qi::EPI_GATED, nullptr, 0, x, H,
                      mod + 5 * H, mld, gt, row0, nullptr, st, nullptr, y_out, H, mod + 2 * H)))
      return r;
  } else {
    qi::GemmParams p;
    memset(&p, 0, sizeof(p));
    p.yf = x;
    p.ldyf = H;
    p.gate = mod + 5 * H;
    p.gate_ld = mld;
    p.res_y = y_out;
    p.ld_res_y = H;
    p.gate1 = mod + 2 * H;
    p.groups = gt;
    p.row0 = row0;
    if ((r = run_bf16_block_linear(ctx, b.g, T, F, w.down_bf16, w.down_mx, qi::EPI_GATED, p,
                                   st, mxb)))
      return r;
  }
  return QI_OK;
}

int run_block(qi_ctx* ctx, const qi_dims& d, const qi_block_weights& w, float* x, int T, int row0,
              const uint16_t* mod, const qi::GroupTable& gt, int S, const float* cs,
              const float* sn, uint16_t* kl, uint16_t* vl, uint8_t* ws, size_t ws_bytes,
              cudaStream_t st, const Fp8Bufs* f8 = nullptr) {
  SeqAttn one;
  one.off = 0;
  one.T = T;
  one.row0 = row0;
  one.S = S;
  one.gt = gt;
  one.kl = kl;
  one.vl = vl;
  return run_block_multi(ctx, d, w, x, T, gt, row0, mod, cs, sn, &one, 1, ws, ws_bytes, st, f8);
}

int check_mx(const qi_mxfp4* w, const char* name, int n, int k) {
  if (!w || !w->packed || !w->scales)
    return fail(QI_ERR_INVALID_ARG, "MXFP4 weight %s has a NULL pointer", name);
  if ((n >= 0 && w->n != n) || (k >= 0 && w->k != k))
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "MXFP4 weight %s is [%d, %d], expected [%d, %d]", name,
                w->n, w->k, n, k);
  if (w->k < 256 || w->k % 256 != 0 || w->n < 256 || w->n % 256 != 0)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "MXFP4 weight %s: need k %% 256 == 0 and n %% 256 == 0",
                name);
  if (!aligned16(w->packed) || !aligned16(w->scales) || (w->bias && !aligned16(w->bias)))
    return fail(QI_ERR_ALIGNMENT, "MXFP4 weight %s: pointers must be 16-byte aligned", name);
  return QI_OK;
}

// A block Linear given as W8A8 codes, MXFP4 codes or a BF16 weight.
int check_linear(const qi_w8* w8, const qi_linear_bf16* bf, const qi_mxfp4* mx, const char* name,
                 int n, int k) {
  if (w8->q) return check_w8(w8, name, n, k);
  if (mx->packed) return check_mx(mx, name, n, k);
  int r;
  if ((r = check_bf16_linear(bf, name, n, k))) return r;
  if (k % 64 != 0) return fail(QI_ERR_UNSUPPORTED_SHAPE, "BF16 weight %s: k %% 64 != 0", name);
  return QI_OK;
}

int check_block_weights(const qi_dims& d, const qi_block_weights* w) {
  if (!w) return fail(QI_ERR_INVALID_ARG, "block weights are NULL");
  const int H = d.hidden, F = d.mlp;
  int r;
  if (!w->qkv.q) {
    if ((r = check_linear(&w->qkv, &w->qkv_bf16, &w->qkv_mx, "qkv", 3 * H, H))) return r;
  } else if (w->qkv.n == 2 * H) {   // q, k W8A8; v BF16
    if ((r = check_w8(&w->qkv, "qkv (q, k rows)", 2 * H, H))) return r;
    if ((r = check_bf16_linear(&w->qkv_bf16, "qkv_bf16 (v rows)", H, H))) return r;
  } else if ((r = check_w8(&w->qkv, "qkv", 3 * H, H))) {
    return r;
  }
  if ((r = check_linear(&w->out, &w->out_bf16, &w->out_mx, "out", H, H))) return r;
  if ((r = check_linear(&w->up, &w->up_bf16, &w->up_mx, "up", F, H))) return r;
  if ((r = check_linear(&w->down, &w->down_bf16, &w->down_mx, "down", H, F))) return r;
  if (w->mx_expand && !aligned16(w->mx_expand))
    return fail(QI_ERR_ALIGNMENT, "mx_expand must be 16-byte aligned");
  if (!w->norm_q || !w->norm_k) return fail(QI_ERR_INVALID_ARG, "norm_q / norm_k is NULL");
  if (!aligned16(w->norm_q) || !aligned16(w->norm_k))
    return fail(QI_ERR_ALIGNMENT, "norm_q / norm_k must be 16-byte aligned");
  return QI_OK;
}

int run_time_conditioning(qi_ctx* ctx, const qi_model& m, float sigma, uint16_t* block_mod,
                          uint16_t* final_mod, StepBufs& b, cudaStream_t st) {
  const qi_dims& d = m.dims;
  const int H = d.hidden;
  // t = 0 for the conditioning prefix, t = sigma for the target.
  {
    Prof pr(ctx, QI_KCLASS_OTHER, st);
    if (qi::launch_timestep_embedding(0.0f, sigma, b.emb, st) != 0)
      return cuda_fail("timestep embedding launch");
  }
  qi::GemvParams g;
  memset(&g, 0, sizeof(g));
  g.x = b.emb;
  g.R = 2;
  g.k = 256;
  g.silu_in = 0;
  g.y_bf16 = 0;
  g.n_jobs = 1;
  g.jobs[0] = {m.t1.w, m.t1.bias, b.h1, H, H};
  {
    Prof pr(ctx, QI_KCLASS_GEMV, st);
    if (qi::launch_gemv(g, st) != 0) return cuda_fail("timestep MLP 1 launch");
  }
  g.x = b.h1;
  g.k = H;
  g.silu_in = 1;
  g.jobs[0] = {m.t2.w, m.t2.bias, b.temb, H, H};
  {
    Prof pr(ctx, QI_KCLASS_GEMV, st);
    if (qi::launch_gemv(g, st) != 0) return cuda_fail("timestep MLP 2 launch");
  }
  g.x = b.temb;
  g.silu_in = 1;
  g.y_bf16 = 1;
  g.n_jobs = 0;
  for (int l = 0; l < d.blocks; ++l)
    g.jobs[g.n_jobs++] = {m.blocks[l].mod.w, m.blocks[l].mod.bias,
                          block_mod + static_cast<size_t>(l) * 2 * 6 * H, 6 * H, 6 * H};
  g.jobs[g.n_jobs++] = {m.final_mod.w, m.final_mod.bias, final_mod, 2 * H, 2 * H};
  {
    Prof pr(ctx, QI_KCLASS_GEMV, st);
    if (qi::launch_gemv(g, st) != 0) return cuda_fail("adaLN rows launch");
  }
  return QI_OK;
}

int check_model(const qi_model* m) {
  if (!m) return fail(QI_ERR_INVALID_ARG, "model is NULL");
  int r;
  if ((r = check_dims(&m->dims))) return r;
  const qi_dims& d = m->dims;
  const int H = d.hidden, P = d.patch;
  if (!m->blocks) return fail(QI_ERR_INVALID_ARG, "model->blocks is NULL");
  for (int l = 0; l < d.blocks; ++l) {
    if ((r = check_block_weights(d, &m->blocks[l]))) return r;
    if ((r = check_bf16_linear(&m->blocks[l].mod, "block mod", 6 * H, H))) return r;
  }
  if ((r = check_bf16_linear(&m->t1, "t1", H, 256))) return r;
  if ((r = check_bf16_linear(&m->t2, "t2", H, H))) return r;
  if ((r = check_bf16_linear(&m->img_in, "img_in", H, P))) return r;
  if ((r = check_bf16_linear(&m->txt_in, "txt_in", H, H))) return r;
  if ((r = check_bf16_linear(&m->final_mod, "final_mod", 2 * H, H))) return r;
  if ((r = check_bf16_linear(&m->proj_out, "proj_out", P, H))) return r;
  return QI_OK;
}

}  // namespace

// ================================================================= fixed scratch

// Scratch for qi_dit_block_forward_noalloc: a fixed array inside the library,
// so that callers which may not allocate device memory can still run a block.
// Every GPU that loads the library holds these bytes until the process exits.
#define QI_NOALLOC_SCRATCH_BYTES (16u << 20)
static __device__ __align__(256) uint8_t qi_noalloc_scratch[QI_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int QI_NOALLOC_MAX_DEVICES = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[QI_NOALLOC_MAX_DEVICES] = {};
CUcontext g_noalloc_cuctx[QI_NOALLOC_MAX_DEVICES] = {};

// The CUDA context current on this thread (driver entry point looked up once).
int current_cu_context(CUcontext* out) {
  static PFN_cuCtxGetCurrent_v4000 get = nullptr;
  if (!get) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return fail(QI_ERR_CUDA, "cuCtxGetCurrent is not available");
    get = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  }
  if (get(out) != CUDA_SUCCESS || !*out) return fail(QI_ERR_CUDA, "no current CUDA context");
  return QI_OK;
}

// Device address of the scratch array on the current device.  The array's
// name is only a host-side stand-in, so the address is looked up with the
// device current and cached per device together with the CUDA context it was
// found in: after a device reset the module is loaded again into a new
// context, and the address is looked up again instead of reusing a stale one.
int noalloc_scratch(int device, void** out) {
  if (device < 0 || device >= QI_NOALLOC_MAX_DEVICES)
    return fail(QI_ERR_INVALID_ARG, "device %d outside 0..%d", device, QI_NOALLOC_MAX_DEVICES - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  CUcontext cur = nullptr;
  int r;
  if ((r = current_cu_context(&cur))) return r;
  if (!g_noalloc_addr[device] || g_noalloc_cuctx[device] != cur) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, qi_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(QI_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_addr[device] = p;
    g_noalloc_cuctx[device] = cur;
  }
  *out = g_noalloc_addr[device];
  return QI_OK;
}

}  // namespace

// ================================================================= C ABI

extern "C" {

int qi_ctx_create(int device, qi_ctx** out) {
  if (!out) return fail(QI_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (cudaSetDevice(device) != cudaSuccess) return cuda_fail("cudaSetDevice");
  int major = 0, minor = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (major != 10 || minor != 0)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "device %d is sm_%d%d; libqi is built for sm_100a",
                device, major, minor);
  qi_ctx* c = new qi_ctx;
  c->device = device;
  c->num_sms = sms;
  c->status = nullptr;
  c->prof_on = false;
  c->prof_used = 0;
  c->prof_ev = nullptr;
  c->prof_cls = nullptr;
  c->attn_fp8 = 0;
  c->taps_on = false;
  memset(&c->taps, 0, sizeof(c->taps));
  c->attn_scratch = nullptr;
  c->attn_scratch_bytes = 0;
  for (int i = 0; i < QI_PROF_CLASSES; ++i) c->launches[i] = 0;
  if (cudaMalloc(&c->status, 256) != cudaSuccess) {
    delete c;
    return cuda_fail("cudaMalloc(status)");
  }
  if (cudaMemset(c->status, 0, 256) != cudaSuccess) {
    cudaFree(c->status);
    delete c;
    return cuda_fail("cudaMemset(status)");
  }
  *out = c;
  return QI_OK;
}

int qi_ctx_destroy(qi_ctx* ctx) {
  if (!ctx) return QI_OK;
  if (ctx->prof_ev) {
    for (int i = 0; i < 2 * QI_PROF_MAX_PAIRS; ++i) cudaEventDestroy(ctx->prof_ev[i]);
    delete[] ctx->prof_ev;
    delete[] ctx->prof_cls;
  }
  cudaFree(ctx->status);
  if (ctx->attn_scratch) cudaFree(ctx->attn_scratch);
  delete ctx;
  return QI_OK;
}

int qi_ctx_reserve_attention(qi_ctx* ctx, size_t bytes) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  if (bytes <= ctx->attn_scratch_bytes) return QI_OK;
  if (ctx->attn_scratch) cudaFree(ctx->attn_scratch);   // synchronises the device
  ctx->attn_scratch = nullptr;
  ctx->attn_scratch_bytes = 0;
  if (cudaMalloc(&ctx->attn_scratch, bytes) != cudaSuccess)
    return cuda_fail("cudaMalloc(attention split scratch)");
  ctx->attn_scratch_bytes = bytes;
  return QI_OK;
}

int qi_ctx_check(qi_ctx* ctx, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return cuda_fail("stream synchronize");
  int st = 0;
  if (cudaMemcpy(&st, ctx->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_fail("status read");
  if (st != 0) {
    cudaMemset(ctx->status, 0, sizeof(int));
    return fail(QI_ERR_TIMEOUT, "a kernel recorded device status %d (bounded wait expired)", st);
  }
  return QI_OK;
}

int qi_last_error(char* buf, size_t n) {
  if (!buf || n == 0) return QI_ERR_INVALID_ARG;
  snprintf(buf, n, "%s", g_last_error.c_str());
  return QI_OK;
}

int qi_prepare_w8(qi_ctx* ctx, const float* w, int n, int k, int8_t* q, float* s,
                  int32_t* rowsum, void* stream) {
  if (!ctx || !w || !q || !s || !rowsum) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (n < 0 || k < 8 || k % 8 != 0) return fail(QI_ERR_UNSUPPORTED_SHAPE, "need k %% 8 == 0");
  if (qi::launch_prepare_w8(w, n, k, q, s, rowsum, S(stream)) != 0)
    return cuda_fail("prepare_w8 launch");
  return QI_OK;
}

int qi_quantize_act(qi_ctx* ctx, const void* x, int x_dtype, int M, int K, int ldx,
                    const uint16_t* shift, const uint16_t* scale, int mod_ld,
                    const qi_groups* groups, int row0, float eps, int8_t* q, float* s_a,
                    int32_t* zp_a, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (x_dtype != QI_F32 && x_dtype != QI_BF16) return fail(QI_ERR_INVALID_ARG, "bad x_dtype");
  if (M < 0 || K < 8 || K % 8 != 0 || K > 16384 || ldx < K || ldx % 8 != 0)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "quantize: need 8 <= K <= 16384, K %% 8 == 0, ldx %% 8 == 0");
  if (M > 0 && (!x || !q || !s_a || !zp_a)) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(x) || !aligned16(q)) return fail(QI_ERR_ALIGNMENT, "x / q must be 16-byte aligned");
  qi::GroupTable gt;
  memset(&gt, 0, sizeof(gt));
  gt.n = 1;
  gt.end[0] = 1 << 30;
  if (shift || scale) {
    if (!shift || !scale) return fail(QI_ERR_INVALID_ARG, "shift and scale go together");
    if (!aligned16(shift) || !aligned16(scale) || mod_ld % 8 != 0)
      return fail(QI_ERR_ALIGNMENT, "shift / scale rows must be 16-byte aligned");
    int r;
    if ((r = check_groups(groups, -1, &gt))) return r;
    if (row0 < 0 || row0 + M > gt.end[gt.n - 1])
      return fail(QI_ERR_INVALID_ARG, "rows row0..row0+M-1 fall outside the groups");
  }
  if (M == 0) return QI_OK;   // no rows: nothing to do (the row pointers may be NULL)
  return run_quant(ctx, x, x_dtype == QI_BF16, M, K, ldx, shift, scale, mod_ld, gt, row0, eps, q,
                   s_a, zp_a, nullptr, S(stream));
}

int qi_w8a8_linear(qi_ctx* ctx, const int8_t* qa, const float* s_a, const int32_t* zp_a, int M,
                   const qi_w8* w, const qi_epilogue* ep, uint16_t* y, int ldy,
                   int32_t* acc_debug, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (M < 0) return fail(QI_ERR_INVALID_ARG, "M < 0");
  // Weight, epilogue and layout checks come first, so that a zero-row call
  // with bad arguments is rejected like any other; only the row pointers
  // (qa, s_a, zp_a, y, residual, q/k/v outputs) may be NULL when M == 0.
  if (M > 0 && (!qa || !s_a || !zp_a)) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  int r;
  if ((r = check_w8(w, "w", -1, -1))) return r;
  if (!aligned16(qa)) return fail(QI_ERR_ALIGNMENT, "qa must be 16-byte aligned");
  const int kind = ep ? ep->kind : QI_EPI_STORE;
  qi::GroupTable gt;
  memset(&gt, 0, sizeof(gt));
  gt.n = 1;
  gt.end[0] = 1 << 30;
  if (kind == QI_EPI_STORE || kind == QI_EPI_GELU_TANH) {
    if (!y && M > 0) return fail(QI_ERR_INVALID_ARG, "y is NULL");
    if (!aligned16(y) || ldy < w->n || ldy % 8 != 0)
      return fail(QI_ERR_ALIGNMENT, "y must be 16-byte aligned with ldy %% 8 == 0, ldy >= n");
    if (M == 0) return QI_OK;
    return run_w8a8(ctx, qa, s_a, zp_a, M, *w, kind == QI_EPI_STORE ? qi::EPI_BF16 : qi::EPI_GELU,
                    y, ldy, nullptr, 0, nullptr, 0, gt, 0, acc_debug, S(stream));
  }
  if (kind == QI_EPI_QKV_NORM_ROPE) {
    const int H = ep->hidden;
    if (H < 128 || H % 128 != 0 || w->n != 3 * H)
      return fail(QI_ERR_UNSUPPORTED_SHAPE, "QKV epilogue: need hidden %% 128 == 0 and n == 3 * hidden");
    if (!ep->norm_q || !ep->norm_k ||
        (M > 0 && (!ep->rope_cos || !ep->rope_sin || !ep->q_out || !ep->k_out || !ep->v_out)))
      return fail(QI_ERR_INVALID_ARG, "QKV epilogue: NULL pointer");
    if (ep->ld_out < H || ep->ld_out % 8 != 0 || !aligned16(ep->q_out) || !aligned16(ep->k_out) ||
        !aligned16(ep->v_out) || !aligned16(ep->rope_cos) || !aligned16(ep->rope_sin) ||
        !aligned16(ep->norm_q) || !aligned16(ep->norm_k))
      return fail(QI_ERR_ALIGNMENT, "QKV epilogue: pointers must be 16-byte aligned, ld_out %% 8 == 0");
    if (M == 0) return QI_OK;
    qi::GemmParams p;
    memset(&p, 0, sizeof(p));
    p.M = M;
    p.N = w->n;
    p.K = w->k;
    p.num_kb = w->k / 128;
    p.s_a = s_a;
    p.zp_a = zp_a;
    p.s_w = w->s;
    p.rowsum = w->rowsum;
    p.bias = w->bias;
    p.H = H;
    p.eps = ep->eps;
    p.wq = ep->norm_q;
    p.wk = ep->norm_k;
    p.rcos = ep->rope_cos;
    p.rsin = ep->rope_sin;
    p.q_out = ep->q_out;
    p.k_out = ep->k_out;
    p.v_out_bf16 = ep->v_out;
    p.ldo = ep->ld_out;
    p.status = ctx->status;
    Prof pr(ctx, QI_KCLASS_GEMM_I8, S(stream));
    const int rr = qi::launch_gemm(true, qi::EPI_QKV, qa, w->k, w->q, w->k, p, ctx->num_sms,
                                   S(stream));
    if (rr == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (QKV operands)");
    if (rr != 0) return fail(QI_ERR_UNSUPPORTED_SHAPE, "QKV epilogue launch failed (tile/head layout)");
    return QI_OK;
  }
  if (kind != QI_EPI_GATED_RESIDUAL) return fail(QI_ERR_INVALID_ARG, "bad epilogue kind");
  if ((M > 0 && !ep->residual) || !ep->gate) return fail(QI_ERR_INVALID_ARG, "residual / gate is NULL");
  if (ep->ld_residual < w->n) return fail(QI_ERR_INVALID_ARG, "ld_residual < n");
  if ((r = check_groups(ep->groups, -1, &gt))) return r;
  if (ep->row0 < 0 || ep->row0 + M > gt.end[gt.n - 1])
    return fail(QI_ERR_INVALID_ARG, "rows row0..row0+M-1 fall outside the groups");
  if (M == 0) return QI_OK;
  return run_w8a8(ctx, qa, s_a, zp_a, M, *w, qi::EPI_GATED, nullptr, 0, ep->residual,
                  ep->ld_residual, ep->gate, ep->gate_ld, gt, ep->row0, acc_debug, S(stream));
}

int qi_mxfp4_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_mxfp4* w,
                    uint16_t* y, int ldy, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (M < 0) return fail(QI_ERR_INVALID_ARG, "M < 0");
  if (M > 0 && (!a || !y)) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  int r;
  if ((r = check_mx(w, "w", -1, -1))) return r;
  if (lda < w->k || lda % 8 != 0 || ldy < w->n || ldy % 8 != 0)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "mxfp4 linear: need lda >= k, ldy >= n, both %% 8 == 0");
  if (!aligned16(a) || !aligned16(y)) return fail(QI_ERR_ALIGNMENT, "a / y must be 16-byte aligned");
  if (M == 0) return QI_OK;
  qi::GemmParams p;
  memset(&p, 0, sizeof(p));
  p.y = y;
  p.ldy = ldy;
  qi_linear_bf16 none;
  memset(&none, 0, sizeof(none));
  return run_bf16_block_linear(ctx, a, M, lda, none, *w, qi::EPI_BF16, p, S(stream));
}

int qi_bf16_linear(qi_ctx* ctx, const uint16_t* a, int M, int lda, const qi_linear_bf16* w,
                   float* y, int ldy, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (M > 0 && (!a || !y)) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  int r;
  if ((r = check_bf16_linear(w, "w", -1, -1))) return r;
  if (M < 0 || w->k % 64 != 0 || w->k < 64 || w->n % 16 != 0 || lda < w->k || lda % 8 != 0 ||
      ldy < w->n)
    return fail(QI_ERR_UNSUPPORTED_SHAPE, "bf16 linear: need k %% 64 == 0, n %% 16 == 0, lda %% 8 == 0");
  if (!aligned16(a)) return fail(QI_ERR_ALIGNMENT, "a must be 16-byte aligned");
  if (M == 0) return QI_OK;   // no rows: nothing to do (the row pointers may be NULL)
  return run_bf16_linear(ctx, a, M, lda, *w, qi::EPI_F32, y, ldy, 0.f, nullptr, S(stream));
}

int qi_qk_norm_rope(qi_ctx* ctx, const uint16_t* qkv, int T, int heads, int head_dim,
                    const uint16_t* wq, const uint16_t* wk, const float* rope_cos,
                    const float* rope_sin, float eps, uint16_t* q_out, uint16_t* k_out,
                    uint16_t* v_out, int ldo, void* stream) {
  if (!ctx || !qkv || !wq || !wk || !rope_cos || !rope_sin || !q_out || !k_out || !v_out)
    return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (head_dim != 128) return fail(QI_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (T < 0 || heads < 1 || ldo < heads * head_dim)
    return fail(QI_ERR_INVALID_ARG, "bad T / heads / ldo");
  qi::QkNormRopeParams p;
  p.qkv = qkv;
  p.ldqkv = 3 * heads * head_dim;
  p.T = T;
  p.heads = heads;
  p.d = head_dim;
  p.wq = wq;
  p.wk = wk;
  p.cos = rope_cos;
  p.sin = rope_sin;
  p.eps = eps;
  p.q_out = q_out;
  p.k_out = k_out;
  p.v_out = v_out;
  p.ldo = ldo;
  if (qi::launch_qk_norm_rope(p, S(stream)) != 0) return cuda_fail("qk norm/rope launch");
  return QI_OK;
}

namespace {

int attn_call(qi_ctx* ctx, const void* q, int ldq, int Sq, int q_offset, const void* k,
              const void* v, int ldkv, int Sk, int heads, int head_dim, const qi_groups* groups,
              float sm_scale, uint16_t* o, int ldo, void* stream, bool fp8) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (Sq > 0 && (!q || !k || !v || !o)) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (head_dim != 128) return fail(QI_ERR_UNSUPPORTED_SHAPE, "head_dim must be 128");
  if (Sq < 0 || Sk < 1 || q_offset < 0 || q_offset + Sq > Sk || heads < 1)
    return fail(QI_ERR_INVALID_ARG, "need 0 <= q_offset, q_offset + Sq <= Sk");
  const int W = heads * head_dim;
  const int qa = fp8 ? 16 : 8;   // elements per 16 bytes
  if (ldq < W || ldkv < W || ldo < W || ldq % qa || ldkv % qa || ldo % 8)
    return fail(QI_ERR_ALIGNMENT, "leading dimensions must be >= heads*128 and 16-byte multiples");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(QI_ERR_ALIGNMENT, "q/k/v/o must be 16-byte aligned");
  qi::GroupTable gt;
  int r;
  if ((r = check_groups(groups, Sk, &gt))) return r;
  if (Sq == 0) return QI_OK;   // no query rows: nothing to do (the pointers may be NULL)
  qi::AttnParams p;
  memset(&p, 0, sizeof(p));
  p.q = q;
  p.k = k;
  p.v = v;
  p.fp8 = fp8 ? 1 : 0;
  p.o = o;
  p.ldq = ldq;
  p.ldkv = ldkv;
  p.ldo = ldo;
  p.Sq = Sq;
  p.Sk = Sk;
  p.heads = heads;
  p.q_offset = q_offset;
  p.sm_scale = sm_scale;
  p.groups = gt;
  p.status = ctx->status;
  p.num_sms = ctx->num_sms;
  {
    // key-range split: only into scratch the context already holds
    // (qi_ctx_reserve_attention; this call allocates nothing); its counters
    // are cleared before every launch
    int kh = 0;
    size_t need = 0, counters = 0;
    p.split_bytes = ctx->attn_scratch_bytes;
    if (ctx->attn_scratch) qi::attention_split_plan(p, &kh, &need, &counters);
    if (kh > 0) {
      if (cudaMemsetAsync(ctx->attn_scratch, 0, counters, S(stream)) != cudaSuccess)
        return cuda_fail("attention split counters");
      p.split_scratch = ctx->attn_scratch;
      p.split_have = ctx->attn_scratch_bytes;
    } else {
      p.split_scratch = nullptr;
      p.split_bytes = 0;
    }
  }
  {
    Prof pr(ctx, QI_KCLASS_ATTN, S(stream));
    const int r2 = qi::launch_attention(p, S(stream));
    if (r2 == -2) return fail(QI_ERR_CUDA, "cuTensorMapEncodeTiled failed (attention operands)");
    if (r2 != 0) return cuda_fail("attention launch");
  }
  return QI_OK;
}

}  // namespace

int qi_attn_split_plan(int Sk, int heads, const qi_groups* groups, int num_sms,
                       size_t scratch_bytes, int* split_heads, size_t* bytes) {
  if (!split_heads || !bytes) return fail(QI_ERR_INVALID_ARG, "NULL output");
  if (Sk < 1 || heads < 1 || num_sms < 1) return fail(QI_ERR_INVALID_ARG, "need Sk, heads, num_sms >= 1");
  qi::GroupTable gt;
  int r;
  if ((r = check_groups(groups, Sk, &gt))) return r;
  qi::AttnParams p;
  memset(&p, 0, sizeof(p));
  p.Sk = Sk;
  p.heads = heads;
  p.groups = gt;
  p.num_sms = num_sms;
  p.split_bytes = scratch_bytes;
  size_t counters = 0;
  qi::attention_split_plan(p, split_heads, bytes, &counters);
  return QI_OK;
}

int qi_attn_block_causal(qi_ctx* ctx, const uint16_t* q, int ldq, int Sq, int q_offset,
                         const uint16_t* k, const uint16_t* v, int ldkv, int Sk, int heads,
                         int head_dim, const qi_groups* groups, float sm_scale, uint16_t* o,
                         int ldo, void* stream) {
  return attn_call(ctx, q, ldq, Sq, q_offset, k, v, ldkv, Sk, heads, head_dim, groups, sm_scale,
                   o, ldo, stream, false);
}

int qi_attn_block_causal_fp8(qi_ctx* ctx, const uint8_t* q, int ldq, int Sq, int q_offset,
                             const uint8_t* k, const uint8_t* v, int ldkv, int Sk, int heads,
                             int head_dim, const qi_groups* groups, float sm_scale, uint16_t* o,
                             int ldo, void* stream) {
  return attn_call(ctx, q, ldq, Sq, q_offset, k, v, ldkv, Sk, heads, head_dim, groups, sm_scale,
                   o, ldo, stream, true);
}

int qi_to_e4m3(qi_ctx* ctx, const uint16_t* x, int64_t n, uint8_t* y, void* stream) {
  if (!ctx || !x || !y) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (n < 0 || n % 16) return fail(QI_ERR_INVALID_ARG, "n must be a multiple of 16");
  if (!aligned16(x) || !aligned16(y)) return fail(QI_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
  Prof pr(ctx, QI_KCLASS_OTHER, S(stream));
  if (qi::launch_bf16_to_e4m3(x, y, n, S(stream))) return cuda_fail("e4m3 cast launch");
  return QI_OK;
}

int qi_mxfp4_expand_bf16(qi_ctx* ctx, const uint8_t* packed, const uint8_t* scales, int n, int k,
                         uint16_t* w, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (n < 0 || k < 32 || k % 32) return fail(QI_ERR_INVALID_ARG, "need n >= 0 and k a positive multiple of 32");
  if (n == 0) return QI_OK;
  if (!packed || !scales || !w) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (!aligned16(packed) || !aligned16(w))
    return fail(QI_ERR_ALIGNMENT, "packed / w must be 16-byte aligned");
  Prof pr(ctx, QI_KCLASS_OTHER, S(stream));
  if (qi::launch_mxfp4_expand_bf16(packed, scales, n, k, w, S(stream)))
    return cuda_fail("MXFP4 expansion launch");
  return QI_OK;
}

int qi_mxfp4_decode(qi_ctx* ctx, const uint8_t* packed, const uint8_t* scales, int n,
                    int k_stored, int k, float* w, void* stream) {
  if (!ctx || !packed || !scales || !w) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if (n < 0 || k_stored < 32 || k_stored % 32 || k < 1 || k > k_stored)
    return fail(QI_ERR_INVALID_ARG, "need k_stored a positive multiple of 32 and 1 <= k <= k_stored");
  Prof pr(ctx, QI_KCLASS_OTHER, S(stream));
  if (qi::launch_mxfp4_decode(packed, scales, n, k_stored, k, w, S(stream)))
    return cuda_fail("MXFP4 decode launch");
  return QI_OK;
}

int qi_ctx_set_block_taps(qi_ctx* ctx, const qi_block_taps* taps) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL context");
  if (!taps) {
    ctx->taps_on = false;
    memset(&ctx->taps, 0, sizeof(ctx->taps));
    return QI_OK;
  }
  const void* ptrs[] = {taps->u1, taps->q1, taps->s1, taps->zp1, taps->o, taps->o_range,
                        taps->qo, taps->so, taps->zpo, taps->x_mid, taps->u2, taps->q2,
                        taps->s2, taps->zp2, taps->g, taps->g_range, taps->qg, taps->sg,
                        taps->zpg, taps->x_layers};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(QI_ERR_ALIGNMENT, "tap buffers must be 16-byte aligned");
  ctx->taps = *taps;
  ctx->taps_on = true;
  return QI_OK;
}

int qi_ctx_set_attention_fp8(qi_ctx* ctx, int enable) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "NULL context");
  ctx->attn_fp8 = enable ? 1 : 0;
  return QI_OK;
}

int qi_block_workspace_bytes(const qi_dims* dims, int T, size_t* bytes) {
  int r;
  if ((r = check_dims(dims))) return r;
  if (!bytes || T < 0) return fail(QI_ERR_INVALID_ARG, "bad arguments");
  *bytes = block_bytes(*dims, T);
  return QI_OK;
}

int qi_dit_block_forward(qi_ctx* ctx, const qi_dims* dims, const qi_block_weights* w, float* x,
                         int T, int row0, const uint16_t* mod, const qi_groups* groups,
                         const float* rope_cos, const float* rope_sin, uint16_t* k_layer,
                         uint16_t* v_layer, int kv_mode, void* workspace,
                         size_t workspace_bytes, void* stream) {
  int r;
  if (!ctx || !x || !mod || !rope_cos || !rope_sin || !k_layer || !v_layer || !workspace)
    return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if ((r = check_dims(dims))) return r;
  if ((r = check_block_weights(*dims, w))) return r;
  qi::GroupTable gt;
  if ((r = check_groups(groups, -1, &gt))) return r;
  const int S_total = gt.end[gt.n - 1];
  if (T < 1 || row0 < 0 || row0 + T != S_total)
    return fail(QI_ERR_INVALID_ARG, "rows row0..row0+T-1 must end the sequence (row0 + T == S)");
  if (kv_mode == QI_KV_NONE || kv_mode == QI_KV_WRITE_PREFIX) {
    if (row0 != 0) return fail(QI_ERR_INVALID_ARG, "this kv_mode processes every token (row0 == 0)");
  } else if (kv_mode == QI_KV_READ_PREFIX) {
    if (row0 == 0) return fail(QI_ERR_INVALID_ARG, "READ_PREFIX needs row0 > 0");
  } else {
    return fail(QI_ERR_INVALID_ARG, "bad kv_mode");
  }
  for (int g = 0; g < gt.n; ++g)
    if (gt.row_set[g] > 1) return fail(QI_ERR_INVALID_ARG, "row sets must be 0 or 1");
  if (!aligned16(x) || !aligned16(mod) || !aligned16(k_layer) || !aligned16(v_layer) ||
      !aligned16(workspace) || !aligned16(rope_cos) || !aligned16(rope_sin))
    return fail(QI_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
  if (workspace_bytes < block_bytes(*dims, T))
    return fail(QI_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes,
                block_bytes(*dims, T));
  return run_block(ctx, *dims, *w, x, T, row0, mod, gt, S_total, rope_cos, rope_sin, k_layer,
                   v_layer, static_cast<uint8_t*>(workspace), workspace_bytes, S(stream));
}

int qi_dit_block_forward_noalloc(qi_ctx* ctx, const qi_dims* dims, const qi_block_weights* w,
                                 float* x, int T, int row0, const uint16_t* mod,
                                 const qi_groups* groups, const float* rope_cos,
                                 const float* rope_sin, uint16_t* k_layer, uint16_t* v_layer,
                                 int kv_mode, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  int r;
  if ((r = check_dims(dims))) return r;
  if (T < 1) return fail(QI_ERR_INVALID_ARG, "T must be >= 1");
  const size_t need = block_bytes(*dims, T);
  if (need > QI_NOALLOC_SCRATCH_BYTES)
    return fail(QI_ERR_WORKSPACE,
                "qi_dit_block_forward_noalloc: %d rows at hidden %d / mlp %d need %zu scratch "
                "bytes, more than the library's fixed %u; use qi_dit_block_forward with a "
                "caller-owned workspace",
                T, dims->hidden, dims->mlp, need, QI_NOALLOC_SCRATCH_BYTES);
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return cuda_fail("cudaGetDevice");
  if (cur != ctx->device)
    return fail(QI_ERR_INVALID_ARG, "the current device (%d) is not the context's device (%d)",
                cur, ctx->device);
  void* scratch = nullptr;
  if ((r = noalloc_scratch(cur, &scratch))) return r;
  // The block writes every region of its scratch before reading it, with one
  // ordering to keep: the two row-range tables that the attention and GELU
  // epilogues publish with atomicMax are cleared by the LayerNorm quantizers
  // that run before those producers in the same call.  So nothing left by an
  // earlier call is read, and nothing has to be cleared here.
  return qi_dit_block_forward(ctx, dims, w, x, T, row0, mod, groups, rope_cos, rope_sin, k_layer,
                              v_layer, kv_mode, scratch, QI_NOALLOC_SCRATCH_BYTES, stream);
}

int qi_step_workspace_bytes(const qi_dims* dims, int S_tokens, size_t* bytes) {
  int r;
  if ((r = check_dims(dims))) return r;
  if (!bytes || S_tokens < 1) return fail(QI_ERR_INVALID_ARG, "bad arguments");
  Carve c{nullptr, 0, 0};
  carve_step(c, *dims, S_tokens, S_tokens, true);
  *bytes = c.off + 256;
  return QI_OK;
}

int qi_time_conditioning(qi_ctx* ctx, const qi_model* model, float sigma, uint16_t* block_mod,
                         uint16_t* final_mod, void* workspace, size_t workspace_bytes,
                         void* stream) {
  int r;
  if (!ctx || !block_mod || !final_mod || !workspace) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if ((r = check_model(model))) return r;
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes, 0};
  StepBufs b = carve_step(c, model->dims, 1, 1, false);
  if (c.off > workspace_bytes) return fail(QI_ERR_WORKSPACE, "workspace too small");
  return run_time_conditioning(ctx, *model, sigma, block_mod, final_mod, b, S(stream));
}

int qi_denoise_step(qi_ctx* ctx, const qi_model* model, float* latents, const uint16_t* txt,
                    int text_tokens, const float* ref_latents, const qi_groups* groups,
                    const float* rope_cos, const float* rope_sin, float sigma, float sigma_next,
                    int kv_mode, uint16_t* kv_cache, float* v_out, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int r;
  if (!ctx || !latents || !rope_cos || !rope_sin || !workspace)
    return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if ((r = check_model(model))) return r;
  const qi_dims& d = model->dims;
  qi::GroupTable gt;
  if ((r = check_groups(groups, -1, &gt))) return r;
  if (gt.n < 2) return fail(QI_ERR_INVALID_ARG, "a step needs a conditioning prefix and a target group");
  for (int g = 0; g < gt.n; ++g)
    if (gt.row_set[g] != (g == gt.n - 1 ? 1 : 0))
      return fail(QI_ERR_INVALID_ARG, "row sets must be 0 for prefix groups and 1 for the target");
  const int S_tok = gt.end[gt.n - 1];
  const int P_tok = gt.end[gt.n - 2];
  const int N = S_tok - P_tok;
  const int R_ref = P_tok - text_tokens;
  if (text_tokens < 1 || R_ref < 0) return fail(QI_ERR_INVALID_ARG, "text_tokens outside the prefix");
  if (R_ref > 0 && !ref_latents && kv_mode != QI_KV_READ_PREFIX)
    return fail(QI_ERR_INVALID_ARG, "the prefix holds reference tokens but ref_latents is NULL");
  const int row0 = kv_mode == QI_KV_READ_PREFIX ? P_tok : 0;
  if (kv_mode != QI_KV_NONE && kv_mode != QI_KV_WRITE_PREFIX && kv_mode != QI_KV_READ_PREFIX)
    return fail(QI_ERR_INVALID_ARG, "bad kv_mode");
  if (kv_mode != QI_KV_READ_PREFIX && !txt) return fail(QI_ERR_INVALID_ARG, "txt is NULL");
  if (kv_mode != QI_KV_NONE && !kv_cache)
    return fail(QI_ERR_INVALID_ARG, "kv_cache is required with prefix caching");
  if (!aligned16(latents) || (txt && !aligned16(txt)) || (ref_latents && !aligned16(ref_latents)) ||
      (kv_cache && !aligned16(kv_cache)) || !aligned16(workspace) || (v_out && !aligned16(v_out)))
    return fail(QI_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
  size_t need = 0;
  {
    Carve c{nullptr, 0, 0};
    carve_step(c, d, S_tok, S_tok, kv_cache == nullptr);
    need = c.off + 256;
  }
  if (workspace_bytes < need)
    return fail(QI_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);

  cudaStream_t st = S(stream);
  const int H = d.hidden, P = d.patch, T = S_tok - row0;
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes, 0};
  StepBufs b = carve_step(c, d, S_tok, S_tok, kv_cache == nullptr);
  uint16_t* kv = kv_cache ? kv_cache : b.kv;

  if ((r = run_time_conditioning(ctx, *model, sigma, b.block_mod, b.final_mod, b, st))) return r;

  // residual stream rows row0 .. S-1
  float* x = b.x;
  if (row0 == 0) {
    if ((r = run_bf16_linear(ctx, txt, text_tokens, H, model->txt_in, qi::EPI_F32, x, H, 0.f,
                             nullptr, st)))
      return r;
    if (R_ref > 0) {
      Prof pr(ctx, QI_KCLASS_OTHER, st);
      if (qi::launch_f32_to_bf16(ref_latents, b.lat_bf16, static_cast<int64_t>(R_ref) * P, st))
        return cuda_fail("cast launch");
      if ((r = run_bf16_linear(ctx, b.lat_bf16, R_ref, P, model->img_in, qi::EPI_F32,
                               x + static_cast<size_t>(text_tokens) * H, H, 0.f, nullptr, st)))
        return r;
    }
  }
  uint16_t* lat_t = b.lat_bf16 + static_cast<size_t>(R_ref > 0 ? R_ref : 0) * P;
  {
    Prof pr(ctx, QI_KCLASS_OTHER, st);
    if (qi::launch_f32_to_bf16(latents, lat_t, static_cast<int64_t>(N) * P, st))
      return cuda_fail("cast launch");
  }
  float* x_tgt = x + static_cast<size_t>(P_tok - row0) * H;
  if ((r = run_bf16_linear(ctx, lat_t, N, P, model->img_in, qi::EPI_F32, x_tgt, H, 0.f, nullptr,
                           st)))
    return r;

  float* x_layers = ctx->taps_on ? ctx->taps.x_layers : nullptr;
  const size_t x_bytes = static_cast<size_t>(T) * H * sizeof(float);
  if (x_layers && (r = tap_copy(x_layers, x, x_bytes, st))) return r;
  for (int l = 0; l < d.blocks; ++l) {
    uint16_t* kl = kv + static_cast<size_t>(l) * 2 * S_tok * H;
    uint16_t* vl = kl + static_cast<size_t>(S_tok) * H;
    if ((r = run_block(ctx, d, model->blocks[l], x, T, row0,
                       b.block_mod + static_cast<size_t>(l) * 2 * 6 * H, gt, S_tok,
                       rope_cos + static_cast<size_t>(row0) * 64,
                       rope_sin + static_cast<size_t>(row0) * 64, kl, vl, b.block_ws,
                       b.block_ws_bytes, st, ctx->attn_fp8 ? &b.f8 : nullptr)))
      return r;
    if (x_layers &&
        (r = tap_copy(reinterpret_cast<uint8_t*>(x_layers) + (l + 1) * x_bytes, x, x_bytes, st)))
      return r;
  }

  // final adaLN (row set of the target: row 1 of final_mod) + proj_out + Euler
  qi::GroupTable one;
  memset(&one, 0, sizeof(one));
  one.n = 1;
  one.end[0] = N;
  const uint16_t* fm = b.final_mod + 2 * H;   // row 1 (the step's sigma)
  if ((r = run_quant(ctx, x_tgt, false, N, H, H, fm, fm + H, 0, one, 0, d.eps, nullptr, nullptr,
                     nullptr, b.u_final, st)))
    return r;
  const float dt = sigma_next - sigma;
  if ((r = run_bf16_linear(ctx, b.u_final, N, H, model->proj_out, qi::EPI_EULER, latents, P, dt,
                           v_out, st)))
    return r;
  return QI_OK;
}

int qi_euler_update(qi_ctx* ctx, float* x, const float* v, int64_t n, float sigma,
                    float sigma_next, void* stream) {
  if (!ctx || !x || !v || n < 0) return fail(QI_ERR_INVALID_ARG, "bad arguments");
  const float dt = sigma_next - sigma;
  if (qi::launch_euler(x, v, n, dt, S(stream)) != 0) return cuda_fail("euler launch");
  return QI_OK;
}


// ---------------------------------------------------------------- true CFG step

namespace {

// A validated sequence of a CFG step.
struct SeqPlan {
  qi::GroupTable gt;
  int S, P, N, L, R, row0, T;
};

int plan_seq(const qi_seq* q, int kv_mode, const char* which, SeqPlan* sp) {
  int r;
  if (!q || !q->rope_cos || !q->rope_sin)
    return fail(QI_ERR_INVALID_ARG, "%s sequence: NULL argument", which);
  if ((r = check_groups(q->groups, -1, &sp->gt))) return r;
  const qi::GroupTable& gt = sp->gt;
  if (gt.n < 2) return fail(QI_ERR_INVALID_ARG, "%s sequence needs a prefix and a target group", which);
  for (int g = 0; g < gt.n; ++g)
    if (gt.row_set[g] != (g == gt.n - 1 ? 1 : 0))
      return fail(QI_ERR_INVALID_ARG, "%s sequence: row sets must be 0 for prefix groups and 1 for the target", which);
  sp->S = gt.end[gt.n - 1];
  sp->P = gt.end[gt.n - 2];
  sp->N = sp->S - sp->P;
  sp->L = q->text_tokens;
  sp->R = sp->P - sp->L;
  if (sp->L < 1 || sp->R < 0) return fail(QI_ERR_INVALID_ARG, "%s sequence: text_tokens outside the prefix", which);
  if (kv_mode != QI_KV_READ_PREFIX && !q->txt) return fail(QI_ERR_INVALID_ARG, "%s sequence: txt is NULL", which);
  if (sp->R > 0 && !q->ref_latents && kv_mode != QI_KV_READ_PREFIX)
    return fail(QI_ERR_INVALID_ARG, "%s sequence holds reference tokens but ref_latents is NULL", which);
  if (kv_mode != QI_KV_NONE && !q->kv_cache)
    return fail(QI_ERR_INVALID_ARG, "%s sequence: kv_cache is required with prefix caching", which);
  if ((q->txt && !aligned16(q->txt)) || (q->ref_latents && !aligned16(q->ref_latents)) ||
      (q->kv_cache && !aligned16(q->kv_cache)) || !aligned16(q->rope_cos) || !aligned16(q->rope_sin))
    return fail(QI_ERR_ALIGNMENT, "%s sequence: pointers must be 16-byte aligned", which);
  sp->row0 = kv_mode == QI_KV_READ_PREFIX ? sp->P : 0;
  sp->T = sp->S - sp->row0;
  return QI_OK;
}

struct CfgBufs {
  StepBufs sb;        // x [T, H], time-conditioning buffers, lat_bf16, u_final [2N, H], own K/V
  float* cos;         // [T, 64] RoPE tables of the processed rows of both sequences
  float* sin;
  float* v;           // [2N, P] conditional then unconditional velocity
};

CfgBufs carve_cfg(Carve& c, const qi_dims& d, int T, int S_c, int S_u, int N, bool own_kv) {
  CfgBufs b;
  const size_t H = d.hidden, P = d.patch;
  b.sb.x = c.take<float>(static_cast<size_t>(T) * H);
  b.sb.emb = c.take<float>(2 * 256);
  b.sb.h1 = c.take<float>(2 * H);
  b.sb.temb = c.take<float>(2 * H);
  b.sb.block_mod = c.take<uint16_t>(static_cast<size_t>(d.blocks) * 2 * 6 * H);
  b.sb.final_mod = c.take<uint16_t>(2 * 2 * H);
  b.sb.lat_bf16 = c.take<uint16_t>(static_cast<size_t>(S_c + S_u) * P);
  b.sb.u_final = c.take<uint16_t>(static_cast<size_t>(2 * N) * H);
  b.sb.kv = own_kv ? c.take<uint16_t>(static_cast<size_t>(d.blocks) * 2 * (S_c + S_u) * H) : nullptr;
  b.sb.f8.q = c.take<uint8_t>(static_cast<size_t>(T) * H);
  b.sb.f8.kv = c.take<uint8_t>(static_cast<size_t>(2) * (S_c + S_u) * H);
  b.cos = c.take<float>(static_cast<size_t>(T) * 64);
  b.sin = c.take<float>(static_cast<size_t>(T) * 64);
  b.v = c.take<float>(static_cast<size_t>(2 * N) * P);
  b.sb.block_ws_bytes = block_bytes(d, T);
  b.sb.block_ws = c.take<uint8_t>(b.sb.block_ws_bytes);
  return b;
}

}  // namespace

int qi_step_cfg_workspace_bytes(const qi_dims* dims, int S_cond, int S_uncond, int target_tokens,
                                size_t* bytes) {
  int r;
  if ((r = check_dims(dims))) return r;
  if (!bytes || S_cond < 1 || S_uncond < 1 || target_tokens < 1 || target_tokens > S_cond ||
      target_tokens > S_uncond)
    return fail(QI_ERR_INVALID_ARG, "bad arguments");
  Carve c{nullptr, 0, 0};
  carve_cfg(c, *dims, S_cond + S_uncond, S_cond, S_uncond, target_tokens, true);
  *bytes = c.off + 256;
  return QI_OK;
}

int qi_denoise_step_cfg(qi_ctx* ctx, const qi_model* model, float* latents, const qi_seq* cond,
                        const qi_seq* uncond, float guidance, float sigma, float sigma_next,
                        int kv_mode, float* v_out, void* workspace, size_t workspace_bytes,
                        void* stream) {
  int r;
  if (!ctx || !latents || !cond || !uncond || !workspace) return fail(QI_ERR_INVALID_ARG, "NULL argument");
  if ((r = check_model(model))) return r;
  if (kv_mode != QI_KV_NONE && kv_mode != QI_KV_WRITE_PREFIX && kv_mode != QI_KV_READ_PREFIX)
    return fail(QI_ERR_INVALID_ARG, "bad kv_mode");
  const qi_dims& d = model->dims;
  SeqPlan sp[2];
  if ((r = plan_seq(cond, kv_mode, "conditional", &sp[0]))) return r;
  if ((r = plan_seq(uncond, kv_mode, "unconditional", &sp[1]))) return r;
  if (sp[0].N != sp[1].N)
    return fail(QI_ERR_INVALID_ARG, "both sequences must end in target groups of the same size");
  if (!aligned16(latents) || !aligned16(workspace) || (v_out && !aligned16(v_out)))
    return fail(QI_ERR_ALIGNMENT, "pointers must be 16-byte aligned");
  const int N = sp[0].N, T = sp[0].T + sp[1].T;
  // row -> modulation row set over the processed rows of both sequences
  qi::GroupTable rows;
  memset(&rows, 0, sizeof(rows));
  if (kv_mode == QI_KV_READ_PREFIX) {
    rows.n = 2;
    rows.end[0] = sp[0].T;
    rows.end[1] = T;
    rows.row_set[0] = rows.row_set[1] = 1;
  } else {
    // the table only maps rows to row sets, so neighbouring groups with the
    // same row set become one run: [text | references] of each sequence use
    // the prefix set, so a prompt and a negative prompt with any number of
    // references make four runs
    for (int b = 0; b < 2; ++b)
      for (int g = 0; g < sp[b].gt.n; ++g) {
        const int end = (b ? sp[0].S : 0) + sp[b].gt.end[g];
        if (rows.n > 0 && rows.row_set[rows.n - 1] == sp[b].gt.row_set[g]) {
          rows.end[rows.n - 1] = end;
          continue;
        }
        if (rows.n == QI_MAX_GROUPS)
          return fail(QI_ERR_UNSUPPORTED_SHAPE,
                      "the two sequences hold more than %d runs of equal row sets together",
                      QI_MAX_GROUPS);
        rows.end[rows.n] = end;
        rows.row_set[rows.n] = sp[b].gt.row_set[g];
        ++rows.n;
      }
  }
  const bool own_kv = cond->kv_cache == nullptr || uncond->kv_cache == nullptr;
  size_t need = 0;
  {
    Carve c{nullptr, 0, 0};
    carve_cfg(c, d, T, sp[0].S, sp[1].S, N, own_kv);
    need = c.off + 256;
  }
  if (workspace_bytes < need)
    return fail(QI_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes, need);

  cudaStream_t st = S(stream);
  const int H = d.hidden, P = d.patch;
  Carve c{static_cast<uint8_t*>(workspace), workspace_bytes, 0};
  CfgBufs b = carve_cfg(c, d, T, sp[0].S, sp[1].S, N, own_kv);
  const qi_seq* seq[2] = {cond, uncond};
  uint16_t* kv[2];
  kv[0] = cond->kv_cache ? cond->kv_cache : b.sb.kv;
  kv[1] = uncond->kv_cache ? uncond->kv_cache
                           : b.sb.kv + static_cast<size_t>(d.blocks) * 2 * sp[0].S * H;
  const int off[2] = {0, sp[0].T};

  // RoPE rows of the processed rows, both sequences back to back
  for (int q = 0; q < 2; ++q) {
    const size_t n = static_cast<size_t>(sp[q].T) * 64 * sizeof(float);
    const size_t so = static_cast<size_t>(sp[q].row0) * 64, dof = static_cast<size_t>(off[q]) * 64;
    if (cudaMemcpyAsync(b.cos + dof, seq[q]->rope_cos + so, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess ||
        cudaMemcpyAsync(b.sin + dof, seq[q]->rope_sin + so, n, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return cuda_fail("RoPE row copy");
  }
  if ((r = run_time_conditioning(ctx, *model, sigma, b.sb.block_mod, b.sb.final_mod, b.sb, st)))
    return r;

  // residual streams: text, references (uncached steps) and the shared target
  uint16_t* lat_t = b.sb.lat_bf16 + static_cast<size_t>(sp[0].S + sp[1].S - N) * P;
  {
    Prof pr(ctx, QI_KCLASS_OTHER, st);
    if (qi::launch_f32_to_bf16(latents, lat_t, static_cast<int64_t>(N) * P, st))
      return cuda_fail("cast launch");
  }
  size_t lat_off = 0;
  for (int q = 0; q < 2; ++q) {
    float* xs = b.sb.x + static_cast<size_t>(off[q]) * H;
    if (sp[q].row0 == 0) {
      if ((r = run_bf16_linear(ctx, seq[q]->txt, sp[q].L, H, model->txt_in, qi::EPI_F32, xs, H,
                               0.f, nullptr, st)))
        return r;
      if (sp[q].R > 0) {
        uint16_t* lr = b.sb.lat_bf16 + lat_off;
        lat_off += static_cast<size_t>(sp[q].R) * P;
        {
          Prof pr(ctx, QI_KCLASS_OTHER, st);
          if (qi::launch_f32_to_bf16(seq[q]->ref_latents, lr, static_cast<int64_t>(sp[q].R) * P, st))
            return cuda_fail("cast launch");
        }
        if ((r = run_bf16_linear(ctx, lr, sp[q].R, P, model->img_in, qi::EPI_F32,
                                 xs + static_cast<size_t>(sp[q].L) * H, H, 0.f, nullptr, st)))
          return r;
      }
    }
    if ((r = run_bf16_linear(ctx, lat_t, N, P, model->img_in, qi::EPI_F32,
                             xs + static_cast<size_t>(sp[q].P - sp[q].row0) * H, H, 0.f, nullptr, st)))
      return r;
  }

  for (int l = 0; l < d.blocks; ++l) {
    SeqAttn sa[2];
    for (int q = 0; q < 2; ++q) {
      sa[q].off = off[q];
      sa[q].T = sp[q].T;
      sa[q].row0 = sp[q].row0;
      sa[q].S = sp[q].S;
      sa[q].gt = sp[q].gt;
      sa[q].kl = kv[q] + static_cast<size_t>(l) * 2 * sp[q].S * H;
      sa[q].vl = sa[q].kl + static_cast<size_t>(sp[q].S) * H;
    }
    if ((r = run_block_multi(ctx, d, model->blocks[l], b.sb.x, T, rows, 0,
                             b.sb.block_mod + static_cast<size_t>(l) * 2 * 6 * H, b.cos, b.sin, sa,
                             2, b.sb.block_ws, b.sb.block_ws_bytes, st,
                             ctx->attn_fp8 ? &b.sb.f8 : nullptr)))
      return r;
  }

  // final adaLN of both targets, one proj_out over their 2N rows, then the
  // guided velocity and the Euler update
  qi::GroupTable one;
  memset(&one, 0, sizeof(one));
  one.n = 1;
  one.end[0] = N;
  const uint16_t* fm = b.sb.final_mod + 2 * H;   // row 1 (the step's sigma)
  for (int q = 0; q < 2; ++q) {
    const float* xt = b.sb.x + static_cast<size_t>(off[q] + sp[q].P - sp[q].row0) * H;
    if ((r = run_quant(ctx, xt, false, N, H, H, fm, fm + H, 0, one, 0, d.eps, nullptr, nullptr,
                       nullptr, b.sb.u_final + static_cast<size_t>(q) * N * H, st)))
      return r;
  }
  if ((r = run_bf16_linear(ctx, b.sb.u_final, 2 * N, H, model->proj_out, qi::EPI_F32, b.v, P, 0.f,
                           nullptr, st)))
    return r;
  {
    Prof pr(ctx, QI_KCLASS_OTHER, st);
    if (qi::launch_cfg_euler(latents, b.v, b.v + static_cast<size_t>(N) * P,
                             static_cast<int64_t>(N) * P, guidance, sigma_next - sigma, v_out, st))
      return cuda_fail("guidance launch");
  }
  return QI_OK;
}

int qi_rope_tables(int n_groups, const int32_t* kinds, const int32_t* tokens,
                   const int32_t* grid_h, const int32_t* grid_w, float* rope_cos,
                   float* rope_sin) {
  if (n_groups < 1 || n_groups > QI_MAX_GROUPS || !kinds || !tokens || !rope_cos || !rope_sin)
    return fail(QI_ERR_INVALID_ARG, "bad arguments");
  int L = 0;
  for (int g = 0; g < n_groups; ++g)
    if (kinds[g] == 0) L += tokens[g];
  static const int pairs[3] = {8, 28, 28};
  int t = 0, ti = 0, k = 0;
  for (int g = 0; g < n_groups; ++g) {
    if (kinds[g] != 0 && (!grid_h || !grid_w || grid_h[g] * grid_w[g] != tokens[g]))
      return fail(QI_ERR_INVALID_ARG, "image group %d: grid does not match its token count", g);
    for (int i = 0; i < tokens[g]; ++i, ++t) {
      int pos[3];
      if (kinds[g] == 0) {
        pos[0] = pos[1] = pos[2] = ti++;
      } else {
        const int h = grid_h[g], w = grid_w[g], y = i / w, xx = i % w;
        pos[0] = L + k;
        pos[1] = y - (h - h / 2);
        pos[2] = xx - (w - w / 2);
      }
      int j = 0;
      for (int a = 0; a < 3; ++a)
        for (int p = 0; p < pairs[a]; ++p, ++j) {
          const double f = pow(10000.0, -static_cast<double>(p) / pairs[a]);
          const double ang = pos[a] * f;
          rope_cos[static_cast<size_t>(t) * 64 + j] = static_cast<float>(cos(ang));
          rope_sin[static_cast<size_t>(t) * 64 + j] = static_cast<float>(sin(ang));
        }
    }
    if (kinds[g] != 0) ++k;
  }
  return QI_OK;
}

int qi_sigma_schedule(int steps, int image_tokens, float* sigmas) {
  if (steps < 1 || image_tokens < 1 || !sigmas) return fail(QI_ERR_INVALID_ARG, "bad arguments");
  const double base_len = 256, max_len = 8192, base_shift = 0.5, max_shift = 0.9, terminal = 0.02;
  const double slope = (max_shift - base_shift) / (max_len - base_len);
  const double mu = image_tokens * slope + (base_shift - slope * base_len);
  const double em = exp(mu);
  double* one_minus = new double[steps];
  for (int i = 0; i < steps; ++i) {
    const double base = steps == 1 ? 1.0 : 1.0 + (1.0 / steps - 1.0) * i / (steps - 1);
    const double shifted = em / (em + (1.0 / base - 1.0));
    one_minus[i] = 1.0 - shifted;
  }
  const double stretch = one_minus[steps - 1] / (1.0 - terminal);
  for (int i = 0; i < steps; ++i)
    sigmas[i] = static_cast<float>(stretch > 0 ? 1.0 - one_minus[i] / stretch : 1.0);
  sigmas[steps] = 0.0f;
  delete[] one_minus;
  return QI_OK;
}

int qi_ctx_profile(qi_ctx* ctx, int enable) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  if (enable && !ctx->prof_ev) {
    ctx->prof_ev = new cudaEvent_t[2 * QI_PROF_MAX_PAIRS];
    ctx->prof_cls = new int[QI_PROF_MAX_PAIRS];
    for (int i = 0; i < 2 * QI_PROF_MAX_PAIRS; ++i)
      if (cudaEventCreate(&ctx->prof_ev[i]) != cudaSuccess) return cuda_fail("cudaEventCreate");
  }
  ctx->prof_on = enable != 0;
  ctx->prof_used = 0;
  for (int i = 0; i < QI_PROF_CLASSES; ++i) ctx->launches[i] = 0;
  return QI_OK;
}

int qi_ctx_profile_read(qi_ctx* ctx, int kernel_class, long long* launches, int* timed,
                        double* total_ms) {
  if (!ctx || kernel_class < 0 || kernel_class >= QI_PROF_CLASSES || !launches || !timed ||
      !total_ms)
    return fail(QI_ERR_INVALID_ARG, "bad arguments");
  *launches = ctx->launches[kernel_class];
  *timed = 0;
  *total_ms = 0.0;
  for (int i = 0; i < ctx->prof_used; ++i) {
    if (ctx->prof_cls[i] != kernel_class) continue;
    if (cudaEventSynchronize(ctx->prof_ev[2 * i + 1]) != cudaSuccess)
      return cuda_fail("cudaEventSynchronize");
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, ctx->prof_ev[2 * i], ctx->prof_ev[2 * i + 1]) != cudaSuccess)
      return cuda_fail("cudaEventElapsedTime");
    *total_ms += ms;
    *timed += 1;
  }
  return QI_OK;
}

int qi_debug_mma_probe(qi_ctx* ctx, int int8, int iters, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  if (iters < 1 || iters > 100000) return fail(QI_ERR_INVALID_ARG, "iters outside 1 .. 100000");
  Prof pr(ctx, QI_KCLASS_OTHER, S(stream));
  if (qi::launch_mma_probe(int8 != 0, iters, ctx->num_sms, ctx->status, S(stream)) != 0)
    return cuda_fail("mma probe launch");
  return QI_OK;
}

int qi_debug_timeout_probe(qi_ctx* ctx, uint64_t limit_ns, void* stream) {
  if (!ctx) return fail(QI_ERR_INVALID_ARG, "ctx is NULL");
  if (limit_ns < 1000ull || limit_ns > 5000000000ull)
    return fail(QI_ERR_INVALID_ARG, "limit_ns outside 1e3 .. 5e9");
  if (qi::launch_timeout_probe(limit_ns, ctx->status, S(stream)) != 0)
    return cuda_fail("probe launch");
  return QI_OK;
}

}  // extern "C"
