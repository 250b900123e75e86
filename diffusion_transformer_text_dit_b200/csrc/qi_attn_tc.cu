// Block-causal flash attention on tcgen05 tensor cores (sm_100a), head_dim 128,
// bf16 in / bf16 out, fp32 softmax.
//
// Mask (RGBA-Image-2.1 Core AI port: "block-causal attention"; qwen-image-mnn:
// "block-causal mask"): the joint sequence is a list of contiguous groups
// [text | (reference) | target]; a token sees every token of its own group and
// of all earlier groups, so the keys of a query at global position t are
// exactly [0, end(group(t))) - a per-query key limit.  Key tiles at or past the
// largest limit of the CTA's queries are never loaded; tiles entirely below
// the smallest limit are not masked.  Queries may be a suffix of the sequence
// (q_offset > 0: the cached-prefix step processes only the target rows while
// keys/values cover the whole sequence).
//
// One CTA = one head x 256 queries, as two 128-row tiles A and B that share
// the key/value stream.  TMEM (512 columns): S_A | S_B | O_A | O_B, 128 fp32
// columns each.  Per key tile j of 128 keys:
//   S_X = Q_X K_j^T         tcgen05.mma kind::f16, A = Q (smem), B = K (smem), both K-major
//   softmax warps of X read S_X (one query row per thread), write P_X as bf16
//   into the first 64 columns of S_X
//   O_X += P_X V_j          tcgen05.mma with A = P from TMEM, B = V (smem, MN-major)
// Issue order (one thread): S_A0 S_B0 | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) ...
// so each tile's softmax overlaps the other tile's MMAs.  The softmax keeps a
// per-row reference maximum and rescales O (TMEM load / store) only when the
// running maximum exceeds it by more than 8 (base 2): P <= 256 in between,
// exact in value because the final normalisation divides by the same sum.
//
// Warps: 0-3 softmax of tile A (TMEM lanes 0-127), 4-7 softmax of tile B,
// 8 TMA producer, 9 TMEM allocator + MMA issuer.  K streams through a 3-stage
// ring (a stage is released once both S MMAs have read it), V through a
// 2-stage ring; every barrier wait is bounded (qi_common.cuh).
//
// Work units are (query tile pair, head); the grid is one CTA per unit,
// heaviest first.  A grid of U units on P SMs (one CTA per SM) leaves its
// last round partly idle when U mod P is small; the heaviest units of a few
// whole heads are then split over the key range: two CTAs take key tiles
// [0, n/2) and [n/2, n), each keeps its own reference maximum and row sum,
// writes its unnormalised O, maximum and sum to scratch, and the CTA that
// finishes second (an atomic counter per unit, no waiting) combines them:
// m = max(m0, m1), O = (O0 2^(m0-m) + O1 2^(m1-m)) / (l0 2^(m0-m) + l1 2^(m1-m)).
// The split is chosen from the shapes of the sequence, not of the launch, so
// a row is split the same way in every launch that computes it.
#include <algorithm>
#include <functional>
#include <mutex>
#include <vector>

#include "qi_common.cuh"
#include "qi_internal.h"

namespace qi {

constexpr int FA_ROWS = 128;                   // rows per Q tile, keys per K/V tile
constexpr int FA_THREADS = 320;
constexpr int FA_KST = 3;                      // K ring stages
constexpr int FA_VST = 2;                      // V ring stages
constexpr int FA_OUT_BOX = FA_ROWS * 128;      // bytes of one staged 64-column bf16 output box

// Tile geometry of the two element types.  A tile is 128 rows x 128 head
// columns: bf16 -> two 64-column (128-byte) swizzle regions of 16 KB; e4m3 ->
// one 128-column (128-byte) region of 16 KB.
template <bool FP8>
struct FaCfg {
  static constexpr int TILE = FP8 ? 128 * 128 : 128 * 128 * 2;
  static constexpr int REGION = 128 * 128;       // bytes of one 128-byte-wide swizzle region
  static constexpr int REGIONS = TILE / REGION;  // 1 (e4m3) or 2 (bf16)
  static constexpr int SMEM = 1024 + (2 + FA_KST + FA_VST) * TILE + 256;
  static_assert(4 * FA_OUT_BOX <= (2 + FA_KST) * TILE, "output staging overlaps the V ring");
};

// tcgen05.mma kind::f8f6f4 with A = B = e4m3 (format 0) and an fp32
// accumulator: D format 1 (bits 4-5), B major bit 16, N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int M, int N, bool b_mn_major) {
  return (1u << 4) | (b_mn_major ? (1u << 16) : 0u) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate));
}
// D (TMEM) += A (TMEM, e4m3, 4 keys per 32-bit column) x B (smem descriptor).
__device__ __forceinline__ void umma_e4m3_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}
// Four values rounded to e4m3 (nearest, ties to even, saturating at +-448),
// packed little-endian (a first).
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// MN-major operand with the 128-byte swizzle: 64 elements (128 B) contiguous
// along N, K rows 128 B apart inside an 8-row group, 8-row groups 1024 B
// apart (stride offset), 64-element column blocks lbo_bytes apart (leading
// offset).
__device__ __forceinline__ uint64_t umma_desc_mnmajor_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// D (TMEM) += A (TMEM, K-major) x B (smem descriptor), kind::f16.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One query row of S: 128 consecutive 32-bit TMEM columns of this thread's
// lane, loaded and waited for in one asm statement.
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ int fa_key_limit(const GroupTable& g, int t) {
  return g.end[group_of(g, t)];
}

// Per-unit scratch of the key-range split (floats per half).
constexpr int FA_PART_O = 2 * FA_ROWS * 128;   // 256 rows x 128 fp32
constexpr int FA_PART_ML = 2 * FA_ROWS * 2;    // 256 rows x (maximum, sum)

// Grid index -> (query tile pair, head, half, split unit).  Segments, in
// launch order: the longest-range tiles of the unsplit heads, the halves of
// the split heads' longest-range tiles, the remaining tiles of every head.
// Within a segment, head-major with the last tile first, so that CTAs
// dispatched together share a head's K/V in L2.  half = -1: not split.
struct FaUnit {
  int ct, h, half, su;
};
__device__ __forceinline__ FaUnit fa_unit(const AttnParams& p, int b) {
  FaUnit u;
  const int k = p.split_heads, nh = p.n_ctiles - p.ct_heavy;
  const int seg_a = nh * (p.heads - k), seg_b = 2 * nh * k;
  u.half = -1;
  u.su = -1;
  if (b < seg_a) {
    u.h = b / nh;
    u.ct = p.n_ctiles - 1 - b % nh;
  } else if (b < seg_a + seg_b) {
    const int v = b - seg_a;
    u.half = v & 1;
    u.su = v >> 1;
    u.h = p.heads - k + u.su / nh;
    u.ct = p.n_ctiles - 1 - u.su % nh;
  } else {
    const int v = b - seg_a - seg_b;
    u.h = v / p.ct_heavy;
    u.ct = p.ct_heavy - 1 - v % p.ct_heavy;
  }
  return u;
}

// o f + b g with both products rounded before the sum: symmetric in the two
// halves of a split unit.
__device__ __forceinline__ float fa_combine(uint32_t o, float f, float b, float g) {
  return __fadd_rn(__fmul_rn(__uint_as_float(o), f), __fmul_rn(b, g));
}

// Lane-wise minimum / maximum of two bf16 pairs.
__device__ __forceinline__ uint32_t bf16x2_min(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t bf16x2_max(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Named barrier 1 over the 8 softmax warps (threads 0-255): plain, and with
// an AND of a predicate across them.
__device__ __forceinline__ void fa_softmax_bar() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}
__device__ __forceinline__ bool fa_softmax_all(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, 256, p;\n\t"
      "selp.b32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred))
      : "memory");
  return r != 0;
}

template <bool FP8>
__global__ void __launch_bounds__(FA_THREADS, 1)
    fa_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
              const AttnParams p) {
  using Cfg = FaCfg<FP8>;
  constexpr int FA_TILE = Cfg::TILE;
  constexpr int FA_HALF = Cfg::REGION;
  int* status = p.status;
  extern __shared__ uint8_t fa_smem_raw[];
  const uint32_t raw_addr = smem_u32(fa_smem_raw);
  uint8_t* smem = fa_smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* sQ = smem;                              // [2][FA_TILE]: tile A, tile B
  uint8_t* sK = smem + 2 * FA_TILE;                // [FA_KST][FA_TILE]
  uint8_t* sV = smem + (2 + FA_KST) * FA_TILE;     // [FA_VST][FA_TILE]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (2 + FA_KST + FA_VST) * FA_TILE);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                     // [FA_KST]
  uint64_t* k_empty = k_full + FA_KST;             // [FA_KST]
  uint64_t* v_full = k_empty + FA_KST;             // [FA_VST]
  uint64_t* v_empty = v_full + FA_VST;             // [FA_VST]
  uint64_t* s_full = v_empty + FA_VST;             // [2] per Q tile
  uint64_t* p_full = s_full + 2;                   // [2] per Q tile
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  uint32_t* order_slot = tmem_slot + 1;   // split: the counter value this CTA saw
  // output staging for the TMA store, over Q and the first K stages (free
  // once every MMA has completed): [tile][64-column box][128 rows][128 B]
  uint8_t* fa_stage = smem;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const FaUnit unit = fa_unit(p, static_cast<int>(blockIdx.x));
  const int h = unit.h;
  const int q0 = unit.ct * 2 * FA_ROWS;
  const int q_last = min(q0 + 2 * FA_ROWS, p.Sq) - 1;
  const int kv_end = min(fa_key_limit(p.groups, p.q_offset + q_last), p.Sk);
  const int kv_min = min(fa_key_limit(p.groups, p.q_offset + q0), p.Sk);
  const int n_kv_all = (kv_end + FA_ROWS - 1) / FA_ROWS;
  // key tiles [kv_lo, kv_lo + n_kv) of this CTA; local tile index i drives
  // every ring stage and barrier phase, kv_lo + i the key coordinates
  const int kv_lo = unit.half == 1 ? n_kv_all / 2 : 0;
  const int n_kv = unit.half == 0 ? n_kv_all / 2 : n_kv_all - kv_lo;
  const int hc = h * 128;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < FA_KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < FA_VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 128);
    }
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmO);
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();      // the previous kernel's outputs are complete from here on
  pdl_trigger();

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, 2 * FA_TILE);
      for (int t = 0; t < 2; ++t)
        for (int half = 0; half < Cfg::REGIONS; ++half)
          tma_load_2d(&tmQ, q_full, sQ + t * FA_TILE + half * FA_HALF, hc + 64 * half,
                      q0 + t * FA_ROWS);
      // K(j) into stage j % FA_KST once S_B(j - FA_KST) has read it; V(j) into
      // stage j % FA_VST once PV_B(j - FA_VST) has.  K runs further ahead:
      // the next S MMA needs it well before the next PV needs V.
      bool ok = true;
      int jk = 0, jv = 0;   // tiles whose loads were issued
      for (int j = 0; j < n_kv; ++j) {
        const int ks = j % FA_KST, kr = j / FA_KST;
        if (!mbar_wait(&k_empty[ks], (kr & 1) ^ 1u, status)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[ks], FA_TILE);
        for (int half = 0; half < Cfg::REGIONS; ++half)
          tma_load_2d(&tmK, &k_full[ks], sK + ks * FA_TILE + half * FA_HALF, hc + 64 * half,
                      (kv_lo + j) * FA_ROWS);
        jk = j + 1;
        const int vs = j % FA_VST, vr = j / FA_VST;
        if (!mbar_wait(&v_empty[vs], (vr & 1) ^ 1u, status)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[vs], FA_TILE);
        for (int half = 0; half < Cfg::REGIONS; ++half)
          tma_load_2d(&tmV, &v_full[vs], sV + vs * FA_TILE + half * FA_HALF, hc + 64 * half,
                      (kv_lo + j) * FA_ROWS);
        jv = j + 1;
      }
      if (!ok) {
        // bounded drain of the loads already armed (Q, the last K and V tiles)
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(q_full, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
        }
        for (int jj = (jk > FA_KST ? jk - FA_KST : 0); jj < jk; ++jj) {
          const uint64_t t1 = globaltimer_ns();
          while (!mbar_try_wait(&k_full[jj % FA_KST], (jj / FA_KST) & 1) &&
                 globaltimer_ns() - t1 < QI_WAIT_NS) {
          }
        }
        for (int jj = (jv > FA_VST ? jv - FA_VST : 0); jj < jv; ++jj) {
          const uint64_t t1 = globaltimer_ns();
          while (!mbar_try_wait(&v_full[jj % FA_VST], (jj / FA_VST) & 1) &&
                 globaltimer_ns() - t1 < QI_WAIT_NS) {
          }
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = FP8 ? umma_idesc_e4m3(128, 128, false) : umma_idesc(false, 128, 128);
      constexpr uint32_t idesc_pv = FP8 ? umma_idesc_e4m3(128, 128, true)
                                        : (umma_idesc(false, 128, 128) | (1u << 16));   // B MN-major
      bool ok = mbar_wait(q_full, 0, status);
      auto issue_s = [&](int X, int jj) -> bool {
        const int st = jj % FA_KST;
        if (!mbar_wait(&k_full[st], (jj / FA_KST) & 1, status)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(sQ + X * FA_TILE), kb = smem_u32(sK + st * FA_TILE);
        if (FP8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 32 e4m3 values (32 bytes) of the head per instruction
            umma_e4m3(tmem_base + X * 128, umma_desc_kmajor_sw128(qa + kk * 32),
                      umma_desc_kmajor_sw128(kb + kk * 32), idesc_s, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * FA_HALF + (kk & 3) * 32;
            umma_f16(tmem_base + X * 128, umma_desc_kmajor_sw128(qa + off),
                     umma_desc_kmajor_sw128(kb + off), idesc_s, kk > 0);
          }
        }
        umma_commit(&s_full[X]);
        return true;
      };
      auto issue_pv = [&](int X, int jj) -> bool {
        const int st = jj % FA_VST;
        if (!mbar_wait(&v_full[st], (jj / FA_VST) & 1, status)) return false;
        if (!mbar_wait(&p_full[X], jj & 1, status)) return false;
        tc_fence_after();
        const uint32_t vb = smem_u32(sV + st * FA_TILE);
        if (FP8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 32 keys per instruction (8 columns of e4m3 P)
            umma_e4m3_ts(tmem_base + 256 + X * 128, tmem_base + X * 128 + kk * 8,
                         umma_desc_mnmajor_sw128(vb + kk * 32 * 128, FA_HALF), idesc_pv,
                         (jj > 0 || kk > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // 16 keys per instruction: two 8-row groups
            umma_f16_ts(tmem_base + 256 + X * 128, tmem_base + X * 128 + kk * 8,
                        umma_desc_mnmajor_sw128(vb + kk * 2048, FA_HALF), idesc_pv,
                        (jj > 0 || kk > 0) ? 1u : 0u);
        }
        return true;
      };
      if (ok && n_kv > 0) {
        ok = issue_s(0, 0) && issue_s(1, 0);
        if (ok) umma_commit(&k_empty[0]);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        ok = issue_pv(0, j);
        if (ok && j + 1 < n_kv) ok = issue_s(0, j + 1);
        if (ok) ok = issue_pv(1, j);
        if (ok) umma_commit(&v_empty[j % FA_VST]);
        if (ok && j + 1 < n_kv) {
          ok = issue_s(1, j + 1);
          if (ok) umma_commit(&k_empty[(j + 1) % FA_KST]);
        }
      }
      if (ok) {
        umma_commit(o_full);
      } else {
        umma_commit(drain);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < QI_WAIT_NS) {
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int X = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_bits = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem_base + lane_bits + X * 128;
    const uint32_t tO = tmem_base + lane_bits + 256 + X * 128;
    const int qrow = q0 + X * FA_ROWS + row;
    const int lim = qrow < p.Sq ? min(fa_key_limit(p.groups, p.q_offset + qrow), p.Sk) : p.Sk;
    const float sl2 = p.sm_scale * 1.4426950408889634f;
    float m_ref = -INFINITY;   // reference maximum, base-2 scaled
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait_warp(&s_full[X], j & 1, status)) { ok = false; break; }
      tc_fence_after();
      const int k0 = (kv_lo + j) * FA_ROWS;
      const bool masked = k0 + FA_ROWS > kv_min;
      uint32_t r[128];
      tmem_ld128(tS, r);                     // the whole S row, read once
      if (masked) {
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (k0 + i >= lim) r[i] = __float_as_uint(-INFINITY);
      }
      if constexpr (!FP8) {
        // bf16: the tile's row maximum first (base-2 scaled, in 8 independent
        // chains of three-input maxima: a single chain over 128 values would
        // put the max latency 128 times on the critical path), then the
        // reference decision, then P = 2^(s sl2 - m_ref) once (the
        // scale-subtract as paired fp32 FMAs, the row sum in 4 paired partial
        // sums).  The reference moves only if the tile's maximum exceeds it
        // by more than 8 (base 2), so P <= 256 (exact in value: the final
        // normalisation divides by the same sum).
        float m8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) m8[k] = fmaxf(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k)
            m8[k] = fmax3(m8[k], __uint_as_float(r[i + 2 * k]), __uint_as_float(r[i + 2 * k + 1]));
        const float mx2 = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
        if (j == 0) {
          m_ref = mx2 == -INFINITY ? 0.f : mx2;   // a row with no key in this tile: P = 0
        } else {
          // move the reference (and rescale O, warp-collectively) before any
          // P of this tile is written; O is complete up to tile j-1
          const bool grow = mx2 > m_ref + 8.0f;
          if (__any_sync(0xffffffffu, grow)) {
            float f = 1.0f;
            if (grow) {
              const float m_new = fmaxf(m_ref, mx2);
              f = exp2f(m_ref - m_new);
              l *= f;
              m_ref = m_new;
            }
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
              tmem_st32(tO + c * 32, o);
            }
            tmem_st_wait();
          }
        }
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
        uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float s0 = __uint_as_float(r[32 * c + 2 * i]), s1 = __uint_as_float(r[32 * c + 2 * i + 1]);
            const uint64_t x2 = f2_fma(f2_pack(s0, s1), sl2x2, negm2);
            float x0, x1;
            f2_unpack(x2, x0, x1);
            const float p0 = ex2_approx(x0);
            const float p1 = ex2_approx(x1);
            acc2[i & 3] = f2_add(acc2[i & 3], f2_pack(p0, p1));
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);   // P (bf16) over the first 64 columns of S
        }
        float a0, a1, b0, b1;
        f2_unpack(f2_add(acc2[0], acc2[1]), a0, a1);
        f2_unpack(f2_add(acc2[2], acc2[3]), b0, b1);
        l += (a0 + b0) + (a1 + b1);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[X]);
      } else {
        // e4m3: P with the current reference maximum, the tile's row maximum
        // taken on the side.  Only if that maximum exceeds the reference by
        // more than 8 (base 2) does the row move its reference; then O is
        // rescaled and P computed again from the S values still in registers
        // (rare after the first tiles), so P and the sum are exactly those of
        // taking the maximum first.  (Measured: for e4m3 P this order is
        // faster than the bf16 one above, and slower for bf16 P.)
        if (j == 0) {
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = fmaxf(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1]));
#pragma unroll
          for (int i = 16; i < 128; i += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              m8[k] = fmax3(m8[k], __uint_as_float(r[i + 2 * k]), __uint_as_float(r[i + 2 * k + 1]));
          m_ref = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7])) * sl2;
          if (m_ref == -INFINITY) m_ref = 0.f;   // a row with no key in this tile: P = 0
        }
        const uint64_t sl2x2 = f2_pack(sl2, sl2);
        float sum = 0.f;
#pragma unroll 1
        for (int attempt = 0; attempt < 2; ++attempt) {
          const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
          uint64_t acc2[4] = {0ull, 0ull, 0ull, 0ull};
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[8];   // 8 words of 4 keys
            float e0 = 0.f, e1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float s0 = __uint_as_float(r[32 * c + 2 * i]), s1 = __uint_as_float(r[32 * c + 2 * i + 1]);
              m4[i & 3] = fmax3(m4[i & 3], s0, s1);
              const uint64_t x2 = f2_fma(f2_pack(s0, s1), sl2x2, negm2);
              float x0, x1;
              f2_unpack(x2, x0, x1);
              const float p0 = ex2_approx(x0);
              const float p1 = ex2_approx(x1);
              acc2[i & 3] = f2_add(acc2[i & 3], f2_pack(p0, p1));
              if (i & 1) {
                pk[i >> 1] = pack_e4m3x4(e0, e1, p0, p1);   // keys 2i-2 .. 2i+1 of the chunk
              } else {
                e0 = p0;
                e1 = p1;
              }
            }
            tmem_st8(tS + c * 8, pk);   // P (e4m3) over the first 32 columns of S
          }
          {
            float a0, a1, b0, b1;
            f2_unpack(f2_add(acc2[0], acc2[1]), a0, a1);
            f2_unpack(f2_add(acc2[2], acc2[3]), b0, b1);
            sum = (a0 + b0) + (a1 + b1);
          }
          if (j == 0 || attempt == 1) break;
          const float mx2 = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
          const bool grow = mx2 > m_ref + 8.0f;
          // The O rescale and the P stores are warp-collective TMEM accesses,
          // so the decision is taken per warp: if any row of the warp moved its
          // reference, the whole warp rescales (factor 1 for the other rows)
          // and recomputes P (the same values for the other rows).  O is
          // complete up to tile j-1: the commit that released S_X(j) covers
          // every earlier MMA.
          if (!__any_sync(0xffffffffu, grow)) break;
          float f = 1.0f;
          if (grow) {
            const float m_new = fmaxf(m_ref, mx2);
            f = exp2f(m_ref - m_new);
            l *= f;
            m_ref = m_new;
          }
          tmem_st_wait();   // this attempt's P stores land before the next ones
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + c * 32, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st32(tO + c * 32, o);
          }
          tmem_st_wait();
        }
        l += sum;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[X]);
      }
    }
    ok = __all_sync(0xffffffffu, ok);
    // split unit: publish this half's partial, then count; the half that
    // counts second combines (every softmax warp reaches both barriers: the
    // o_full wait result is made uniform across them first)
    bool store = ok && n_kv > 0 && mbar_wait_warp(o_full, 0, status);
    float* other_o = nullptr;
    float m_oth = 0.f, l_oth = 0.f;
    if (unit.half >= 0) {
      uint32_t* counter = static_cast<uint32_t*>(p.split_scratch) + unit.su;
      const size_t n_units = static_cast<size_t>(p.n_ctiles - p.ct_heavy) * p.split_heads;
      float* ml = reinterpret_cast<float*>(static_cast<uint8_t*>(p.split_scratch) +
                                           ((n_units * 4 + 255) & ~static_cast<size_t>(255)));
      float* po = ml + n_units * 2 * FA_PART_ML;
      // partial O layout [32 column quads][256 rows] of float4: the 32 lanes
      // of a warp (32 consecutive rows) store and load 512 contiguous bytes
      const int prow = X * FA_ROWS + row;
      if (store) {
        tc_fence_after();
        float4* mine = reinterpret_cast<float4*>(
            po + (static_cast<size_t>(unit.su) * 2 + unit.half) * FA_PART_O) + prow;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            mine[(c * 8 + v) * 2 * FA_ROWS] =
                make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                            __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
        float* mml = ml + (static_cast<size_t>(unit.su) * 2 + unit.half) * FA_PART_ML + prow * 2;
        mml[0] = m_ref;
        mml[1] = l;
      }
      __threadfence();
      const bool all = fa_softmax_all(store);
      if (threadIdx.x == 0) *order_slot = all ? atomicAdd(counter, 1u) : 0u;
      fa_softmax_bar();
      store = all && *order_slot == 1u;
      if (store) {
        __threadfence();
        const size_t oth = static_cast<size_t>(unit.su) * 2 + (unit.half ^ 1);
        other_o = po + oth * FA_PART_O + prow * 4;
        m_oth = __ldcg(ml + oth * FA_PART_ML + prow * 2);
        l_oth = __ldcg(ml + oth * FA_PART_ML + prow * 2 + 1);
        if (threadIdx.x == 0) *counter = 0u;   // ready for the next launch
      }
    }
    if (store) {
      tc_fence_after();
      // this CTA's O is scaled by f_me, the other half's by f_oth, and the
      // sum of both normalises (an empty half, l = 0, has weight 0).  Products
      // and sums are rounded separately (no FMA contraction), so the result
      // does not depend on which half finished second.
      float f_me = 1.f, f_oth = 0.f, lsum = l;
      if (other_o) {
        const float m = fmaxf(l > 0.f ? m_ref : -INFINITY, l_oth > 0.f ? m_oth : -INFINITY);
        f_me = l > 0.f ? exp2f(m_ref - m) : 0.f;
        f_oth = l_oth > 0.f ? exp2f(m_oth - m) : 0.f;
        lsum = __fadd_rn(__fmul_rn(l, f_me), __fmul_rn(l_oth, f_oth));
      }
      const float inv = lsum > 0.f ? 1.0f / lsum : 0.f;
      const uint64_t inv2 = f2_pack(inv, inv);
      uint32_t lo2 = 0u, hi2 = 0u;   // range of the stored bf16 values of this row, as bf16 pairs
      // the other half's partial is loaded one 32-column chunk ahead
      const float4* src = reinterpret_cast<const float4*>(other_o);
      float4 ahead[8];
      if (other_o) {
#pragma unroll
        for (int v = 0; v < 8; ++v) ahead[v] = __ldcg(src + v * 2 * FA_ROWS);
      }
      // every lane of the warp takes part in the (warp-wide) TMEM loads
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tO + c * 32, r);
        if (other_o) {
          float4 cur[8];
#pragma unroll
          for (int v = 0; v < 8; ++v) cur[v] = ahead[v];
          if (c + 1 < 4) {
#pragma unroll
            for (int v = 0; v < 8; ++v) ahead[v] = __ldcg(src + ((c + 1) * 8 + v) * 2 * FA_ROWS);
          }
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 b = cur[v];
            r[4 * v] = __float_as_uint(fa_combine(r[4 * v], f_me, b.x, f_oth));
            r[4 * v + 1] = __float_as_uint(fa_combine(r[4 * v + 1], f_me, b.y, f_oth));
            r[4 * v + 2] = __float_as_uint(fa_combine(r[4 * v + 2], f_me, b.z, f_oth));
            r[4 * v + 3] = __float_as_uint(fa_combine(r[4 * v + 3], f_me, b.w, f_oth));
          }
        }
        // O / l in paired fp32 multiplies, rounded to bf16 pairs; the row's
        // range is taken over the stored bf16 pairs themselves
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a, b;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])), inv2),
                    a, b);
          pk[i] = pack_bf16x2(a, b);
          lo2 = bf16x2_min(lo2, pk[i]);
          hi2 = bf16x2_max(hi2, pk[i]);
        }
        // staged in the TMA store's layout: per tile and 64-column box, 128
        // rows of 128 bytes, 16-byte chunk j of row r at chunk j ^ (r mod 8)
        uint8_t* rowp = fa_stage + X * 2 * FA_OUT_BOX + (c >> 1) * FA_OUT_BOX + row * 128;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int j = (c & 1) * 4 + v;
          *reinterpret_cast<uint4*>(rowp + ((j ^ (row & 7)) << 4)) =
              make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      fence_proxy_async_smem();
      const float rlo = fminf(bf16_bits_to_float(static_cast<uint16_t>(lo2)),
                              bf16_bits_to_float(static_cast<uint16_t>(lo2 >> 16)));
      const float rhi = fmaxf(bf16_bits_to_float(static_cast<uint16_t>(hi2)),
                              bf16_bits_to_float(static_cast<uint16_t>(hi2 >> 16)));
      if (p.row_range && qrow < p.Sq) {
        // per-row range for the next quantizer (non-negative floats order like
        // their bit patterns; negative zero is normalised to +0)
        atomicMax(p.row_range + 2 * static_cast<size_t>(qrow), __float_as_uint(__fsub_rn(0.0f, rlo)));
        atomicMax(p.row_range + 2 * static_cast<size_t>(qrow) + 1, __float_as_uint(__fadd_rn(rhi, 0.0f)));
      }
    }
    // every softmax thread arrives here; the staged tiles go out by TMA only
    // if all of them were staged (rows past Sq are clipped by the store)
    if (fa_softmax_all(store) && threadIdx.x == 0) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (q0 + t * FA_ROWS >= p.Sq) break;
#pragma unroll
        for (int box = 0; box < 2; ++box)
          tma_store_2d(&tmO, fa_stage + (2 * t + box) * FA_OUT_BOX, hc + 64 * box, q0 + t * FA_ROWS);
      }
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- split plan

static int host_key_limit(const GroupTable& g, int t) {
  int k = 0;
  while (k < g.n - 1 && t >= g.end[k]) ++k;
  return g.end[k];
}

// Key tiles of query tile pair ct of a launch.
static int host_n_kv(const AttnParams& p, int ct) {
  const int q_last = std::min((ct + 1) * 2 * FA_ROWS, p.Sq) - 1;
  const int kv_end = std::min(host_key_limit(p.groups, p.q_offset + q_last), p.Sk);
  return (kv_end + FA_ROWS - 1) / FA_ROWS;
}

// Finish time of greedy dispatch, in grid order, of `n_full` units of cost
// c_full and then `n_half` of cost c_half onto `sms` SMs (one CTA each).
static long fa_makespan(int sms, int n_full, long c_full, int n_half, long c_half) {
  std::vector<long> t(static_cast<size_t>(sms), 0);   // a min-heap of SM free times
  auto push = [&](long cost) {
    std::pop_heap(t.begin(), t.end(), std::greater<long>());
    t.back() += cost;
    std::push_heap(t.begin(), t.end(), std::greater<long>());
  };
  std::make_heap(t.begin(), t.end(), std::greater<long>());
  for (int i = 0; i < n_full; ++i) push(c_full);
  for (int i = 0; i < n_half; ++i) push(c_half);
  return *std::max_element(t.begin(), t.end());
}

static size_t fa_split_scratch_bytes(size_t units) {
  return ((units * 4 + 255) & ~static_cast<size_t>(255)) +
         units * 2 * (FA_PART_ML + FA_PART_O) * sizeof(float);
}

// The split depends on the sequence (Sk, the group table), heads, the SM
// count and the scratch the caller guarantees, never on the launch's query
// rows.  It models the launch as the last group's query tiles of every head
// (the rows a cached-prefix launch computes; in an uncached launch they are
// the longest-range tiles too) and picks the number of whole heads whose
// tiles are split in two that minimises the modelled finish time: costs in
// key tiles plus two tiles of fixed work per CTA and one more per split half
// (the partial write and the combine).  The shorter tiles of earlier groups
// run after these and are left out of the model.
static void attention_split_plan_compute(const AttnParams& p, int* split_heads, size_t* bytes,
                                         size_t* counter_bytes) {
  *split_heads = 0;
  *bytes = 0;
  *counter_bytes = 0;
  const int n_kv = (p.Sk + FA_ROWS - 1) / FA_ROWS;
  if (p.num_sms < 2 || n_kv < 8 || p.heads < 1) return;
  const int start_last = p.groups.n >= 2 ? p.groups.end[p.groups.n - 2] : 0;
  const int tiles = (p.Sk - start_last + 2 * FA_ROWS - 1) / (2 * FA_ROWS);
  // capacity for tiles + 1 per head: an uncached launch whose last group does
  // not start on a tile boundary has one more longest-range tile
  int k_max = p.heads;
  while (k_max > 0 && fa_split_scratch_bytes(static_cast<size_t>(tiles + 1) * k_max) > p.split_bytes)
    --k_max;
  const long c_full = n_kv + 2, c_half = (n_kv + 1) / 2 + 3;
  const long base = fa_makespan(p.num_sms, tiles * p.heads, c_full, 0, c_half);
  long best = base;
  for (int k = 1; k <= k_max; ++k) {
    const long t = fa_makespan(p.num_sms, tiles * (p.heads - k), c_full, 2 * tiles * k, c_half);
    if (t < best) {
      best = t;
      *split_heads = k;
    }
  }
  if (best * 100 > base * 97) *split_heads = 0;   // less than 3% modelled gain: no split
  if (*split_heads > 0) {
    const size_t units = static_cast<size_t>(tiles + 1) * *split_heads;
    *bytes = fa_split_scratch_bytes(units);
    *counter_bytes = units * 4;
  }
}

// The plan is a pure function of a few integers; a step asks for the same
// one in every block, so recent plans are kept (the model simulation costs
// about a tenth of a millisecond of host time).
void attention_split_plan(const AttnParams& p, int* split_heads, size_t* bytes,
                          size_t* counter_bytes) {
  struct Entry {
    bool used;
    int sk, heads, sms, n;
    int end[16];
    size_t cap;
    int k;
    size_t bytes, counters;
  };
  static Entry memo[16];
  static int next = 0;
  static std::mutex mu;
  auto same = [&](const Entry& e) {
    if (!e.used || e.sk != p.Sk || e.heads != p.heads || e.sms != p.num_sms ||
        e.cap != p.split_bytes || e.n != p.groups.n)
      return false;
    for (int i = 0; i < p.groups.n; ++i)
      if (e.end[i] != p.groups.end[i]) return false;
    return true;
  };
  {
    std::lock_guard<std::mutex> g(mu);
    for (const Entry& e : memo)
      if (same(e)) {
        *split_heads = e.k;
        *bytes = e.bytes;
        *counter_bytes = e.counters;
        return;
      }
  }
  attention_split_plan_compute(p, split_heads, bytes, counter_bytes);
  std::lock_guard<std::mutex> g(mu);
  Entry& e = memo[next];
  next = (next + 1) % 16;
  e.used = true;
  e.sk = p.Sk;
  e.heads = p.heads;
  e.sms = p.num_sms;
  e.n = p.groups.n;
  for (int i = 0; i < 16; ++i) e.end[i] = i < p.groups.n ? p.groups.end[i] : 0;
  e.cap = p.split_bytes;
  e.k = *split_heads;
  e.bytes = *bytes;
  e.counters = *counter_bytes;
}

template <bool FP8>
static int launch_attention_t(const AttnParams& p_in, cudaStream_t st) {
  using Cfg = FaCfg<FP8>;
  static bool attr = false;   // per instantiation
  if (!attr) {
    if (cudaFuncSetAttribute(fa_kernel<FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM) != cudaSuccess) {
      launch_result();
      return -1;
    }
    attr = true;
  }
  AttnParams p = p_in;
  p.n_ctiles = (p.Sq + 2 * FA_ROWS - 1) / (2 * FA_ROWS);
  // tiles [ct_heavy, n_ctiles) reach the last key tile (the key range grows
  // with the query position)
  const int n_kv_max = (p.Sk + FA_ROWS - 1) / FA_ROWS;
  p.ct_heavy = p.n_ctiles;
  while (p.ct_heavy > 0 && host_n_kv(p, p.ct_heavy - 1) == n_kv_max) --p.ct_heavy;
  size_t need = 0, counters = 0;
  p.split_heads = 0;
  if (p.split_scratch) attention_split_plan(p, &p.split_heads, &need, &counters);
  // The plan bounds k by split_bytes with a tile more than any launch over
  // all of the last group can have; a launch over fewer rows (a block call
  // on part of the last group) may hold less scratch than that and then
  // does not split.
  if (p.split_heads > 0 &&
      fa_split_scratch_bytes(static_cast<size_t>(p.n_ctiles - p.ct_heavy) * p.split_heads) >
          std::min(p.split_bytes, p.split_have))
    p.split_heads = 0;
  const int W = p.heads * 128;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t esz = FP8 ? 1 : 2;
  const uint32_t box = FP8 ? 128 : 64;   // one 128-byte swizzle row per box
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_2d(&tq, p.q, dt, W, p.Sq, static_cast<uint64_t>(p.ldq) * esz, box, FA_ROWS) ||
      !make_tmap_2d(&tk, p.k, dt, W, p.Sk, static_cast<uint64_t>(p.ldkv) * esz, box, FA_ROWS) ||
      !make_tmap_2d(&tv, p.v, dt, W, p.Sk, static_cast<uint64_t>(p.ldkv) * esz, box, FA_ROWS) ||
      !make_tmap_2d(&to, p.o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, p.Sq,
                    static_cast<uint64_t>(p.ldo) * 2, 64, FA_ROWS))
    return -2;
  dim3 grid(static_cast<unsigned>(p.n_ctiles * p.heads +
                                  (p.n_ctiles - p.ct_heavy) * p.split_heads));
  launch_pdl(fa_kernel<FP8>, grid, dim3(FA_THREADS), Cfg::SMEM, st, 1, tq, tk, tv, to, p);
  return launch_result();
}

int launch_attention(const AttnParams& p, cudaStream_t st) {
  if (p.Sq == 0) return 0;
  return p.fp8 ? launch_attention_t<true>(p, st) : launch_attention_t<false>(p, st);
}

}  // namespace qi
