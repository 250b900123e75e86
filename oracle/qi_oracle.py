"""CPU oracle for the Qwen-Image-2.1 single-stream DiT step with W8A8 Linears.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's ``cpu_baseline`` / ``--impl reference`` legs may import this module.
The product path (the CUDA library and its binding) never calls it, and this
module imports nothing from the product package: both sides only share the
seeded input tensors drawn by ``synth``.

Plain, slow and written to be read against the pages.  Arithmetic is float64
except where the pages fix a precision:

  * activation / weight quantization: fp32 IEEE operations
    (FlagRelease "Qwen-Image-2.1-W8A8-arm-FlagOS", "Quantization and validation":
    symmetric per-output-channel INT8 weights with FP32 scales; dynamic
    asymmetric per-token INT8 activations with FP32 scales),
  * the W8A8 Linear: exact integer accumulation, then scaling, then a BF16
    output (same section: "INT32, followed by FP32 scaling and BF16 output"),
  * Q/K RMSNorm: the normalized activation is cast to the scale's dtype (bf16)
    before the scale multiplies ("Qwen Image 2.1 native qualification",
    "Numerical checks"),
  * the FlowMatch Euler update ``x += (sigma_next - sigma) * v`` in fp32
    ("RGBA-Image-2.1 - Core AI port of Qwen-Image-2.1", "Graph contracts",
    Sampler; fp32 inputs and outputs).

Every function names the passage it follows.  Where the pages leave a step
open, the reading taken is stated in the function and in the design notes.
Each function is pinned by ``tests/test_oracle_pins.py`` against facts the
pages or the mathematics fix; none is "parity unpinned" except where noted.

Library primitives used as single steps: ``numpy.matmul`` (float64; exact for
the integer GEMM because every partial sum stays below 2**53), ``numpy.exp``,
``numpy.tanh``, ``numpy.cos`` / ``numpy.sin``.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

F32 = np.float32
F64 = np.float64

# ----------------------------------------------------------------------------
# bfloat16 rounding
# ----------------------------------------------------------------------------


def bf16_round(x) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even; returned as float32.

    Input is first rounded to float32 (finite values only; NaN is not handled).
    bfloat16 keeps the top 16 bits of the float32 pattern.
    """
    a = np.ascontiguousarray(np.asarray(x, dtype=F32))
    bits = a.view(np.uint32).astype(np.uint64)
    keep_lsb = (bits >> np.uint64(16)) & np.uint64(1)
    r = ((bits + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(F32).reshape(a.shape)


# ----------------------------------------------------------------------------
# W8A8 quantization  (FlagOS card, "Quantization and validation")
# ----------------------------------------------------------------------------


def prepare_w8(w) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Symmetric INT8 per output channel, zero point 0, FP32 scales.

    Reading: per row n, s = max|W[n,:]| / 127 (fp32 division; s = 1 for an
    all-zero row), q = clamp(rint(W / s), -127, 127) with round-half-even.
    Returns (q int8 [N,K], s float32 [N], rowsum int64 [N] = sum_k q[n,k]).
    """
    w = np.asarray(w, dtype=F32)
    amax = np.max(np.abs(w), axis=1)
    s = (amax / F32(127)).astype(F32)
    s = np.where(amax == 0, F32(1), s).astype(F32)
    q = np.clip(np.rint(w / s[:, None]), -127, 127).astype(np.int8)
    rowsum = q.astype(np.int64).sum(axis=1)
    return q, s, rowsum


def quantize_act(u) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Dynamic asymmetric INT8 per token (row), FP32 scale.

    Reading (all fp32 IEEE operations, rint = round-half-even):
      lo = min(min_k u, 0), hi = max(max_k u, 0), s = (hi - lo) / 255
      zp = clamp(rint(-128 - lo / s), -128, 127)
      q  = clamp(rint(u / s) + zp, -128, 127)
    A row whose range is empty (all zeros) gets s = 1, zp = 0, q = 0.
    Dequantization is u ~= s * (q - zp).
    Returns (q int8 [M,K], s float32 [M], zp int32 [M]).
    """
    u = np.asarray(u, dtype=F32)
    lo = np.minimum(u.min(axis=1), F32(0)).astype(F32)
    hi = np.maximum(u.max(axis=1), F32(0)).astype(F32)
    s = ((hi - lo) / F32(255)).astype(F32)
    empty = s == 0
    s = np.where(empty, F32(1), s).astype(F32)
    zp = np.clip(np.rint(F32(-128) - lo / s), -128, 127)
    zp = np.where(empty, 0, zp).astype(np.int32)
    q = np.clip(np.rint(u / s[:, None]) + zp[:, None], -128, 127).astype(np.int8)
    return q, s, zp


def int_gemm(qa, qw) -> np.ndarray:
    """acc[m, n] = sum_k qa[m, k] * qw[n, k] exactly, as int64.

    float64 matmul is exact here: |qa*qw| <= 128*127 and K <= 2**17, so every
    partial sum is an integer below 2**53.
    """
    qa = np.asarray(qa)
    qw = np.asarray(qw)
    assert qa.shape[1] == qw.shape[1] and qa.shape[1] <= (1 << 17)
    acc = np.asarray(qa, F64) @ np.asarray(qw, F64).T
    return np.rint(acc).astype(np.int64)


def w8a8_linear(qa, sa, zpa, qw, sw, rowsum, bias=None) -> Tuple[np.ndarray, np.ndarray]:
    """INT32 accumulation, FP32 scaling, BF16 output.

    y[m,n] = bf16( (acc[m,n] - zp[m] * rowsum[n]) * s_a[m] * s_w[n] + bias[n] )
    The subtraction of zp * rowsum removes the activation zero point: with
    u ~= s_a (q_a - zp) and w ~= s_w q_w,  sum_k u w ~= s_a s_w (acc - zp rowsum).
    Returns (acc int64 [M,N], y as bf16 values in float32 [M,N]).
    """
    acc = int_gemm(qa, qw)
    corr = acc - np.asarray(zpa, np.int64)[:, None] * np.asarray(rowsum, np.int64)[None, :]
    y = corr.astype(F64) * np.asarray(sa, F64)[:, None] * np.asarray(sw, F64)[None, :]
    if bias is not None:
        y = y + np.asarray(bias, F64)[None, :]
    return acc, bf16_round(y)


def w8a8_apply(u, wq) -> np.ndarray:
    """Quantize activations ``u`` per token, then apply the prepared W8A8 Linear ``wq``."""
    qa, sa, zpa = quantize_act(u)
    return w8a8_linear(qa, sa, zpa, *wq)[1]


def bf16_linear(x, w, b=None) -> np.ndarray:
    """A Linear kept in BF16 (FlagOS card, "Quantization and validation": the
    Linears outside the W8A8 set and the activations stay BF16): the input is
    the bf16 activation, the weight is bf16, the products are summed exactly
    (float64 is exact for the short sums of bf16 x bf16 products used here to
    far below bf16 resolution) and the output is rounded to bf16 once.
    Returns bf16 values as float32."""
    y = np.asarray(bf16_round(x), F64) @ np.asarray(bf16_round(w), F64).T
    if b is not None:
        y = y + np.asarray(b, F64)[None, :]
    return bf16_round(y)


def linear_apply(u, lin) -> np.ndarray:
    """Apply one block Linear as prepared by ``prepare_block``: a W8A8 tuple
    (q, s, rowsum, bias) or a BF16 one ("bf16", w, bias)."""
    if isinstance(lin[0], str):
        return bf16_linear(u, lin[1], lin[2])
    return w8a8_apply(u, lin)


# ----------------------------------------------------------------------------
# Norms, modulation, activation
# ----------------------------------------------------------------------------


def layer_norm(x, eps) -> np.ndarray:
    """Non-affine LayerNorm over the last axis (reading: eps = 1e-6, no affine)."""
    x = np.asarray(x, F64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps)


def modulate(u, shift, scale) -> np.ndarray:
    """adaLN modulation u * (1 + scale) + shift (reading of the pages' modulation rows)."""
    return np.asarray(u, F64) * (1.0 + np.asarray(scale, F64)) + np.asarray(shift, F64)


def rms_norm_cast(x, w, eps) -> np.ndarray:
    """Q/K RMSNorm with the cast ordering of "Qwen Image 2.1 native qualification".

    Per vector of length d (fp32 IEEE operations):
      r = 1 / sqrt(mean(x^2) + eps),  n = x * r,
      out = bf16( bf16(n) * w )        # n is cast to bf16 BEFORE the bf16 scale w
    Returns bf16 values as float32.
    """
    x = np.asarray(x, F32)
    ms = (np.sum(x * x, axis=-1, keepdims=True, dtype=F32) / F32(x.shape[-1])).astype(F32)
    r = (F32(1) / np.sqrt((ms + F32(eps)).astype(F32))).astype(F32)
    n = bf16_round(x * r)
    return bf16_round(n * np.asarray(w, F32))


def gelu_tanh(x) -> np.ndarray:
    """GELU, tanh form: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = np.asarray(x, F64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


# ----------------------------------------------------------------------------
# 3-axis RoPE  (Core AI port, "Graph contracts", RoPE; qwen-image-mnn "What runs where")
# ----------------------------------------------------------------------------

ROPE_THETA = 10000.0
ROPE_AXIS_PAIRS = (8, 28, 28)   # rotation pairs for (frame, h, w): axis dims 16/56/56


def rope_positions(groups: Sequence[Tuple[str, int, Optional[Tuple[int, int]]]]) -> np.ndarray:
    """(frame, h, w) position of every token of the joint sequence.

    Text token i sits at (i, i, i).  An image token at row y, column x of an
    h x w grid sits at (L + k, y - (h - h//2), x - (w - w//2)), L = number of
    text tokens, k = index of the image group (reading: reference = 0,
    target = 1 in an edit sequence).  Image tokens are in raster order.
    """
    L = sum(n for kind, n, _ in groups if kind == "text")
    pos: List[Tuple[int, int, int]] = []
    ti = 0
    k = 0
    for kind, n, grid in groups:
        if kind == "text":
            for _ in range(n):
                pos.append((ti, ti, ti))
                ti += 1
        else:
            h, w = grid
            assert h * w == n
            for y in range(h):
                for x in range(w):
                    pos.append((L + k, y - (h - h // 2), x - (w - w // 2)))
            k += 1
    return np.asarray(pos, dtype=np.int64)


def rope_tables(positions) -> Tuple[np.ndarray, np.ndarray]:
    """cos/sin tables [S, 64] (fp32) for 64 rotation pairs of a 128-wide head.

    Reading: pairs 0..7 rotate with the frame axis, 8..35 with h, 36..63 with w;
    pair i of an axis with n pairs has frequency theta^(-i/n) (theta = 1e4),
    i.e. theta^(-2i/D) for axis dim D = 2n.
    """
    positions = np.asarray(positions, F64)
    angles = []
    for axis, n in enumerate(ROPE_AXIS_PAIRS):
        freq = ROPE_THETA ** (-np.arange(n, dtype=F64) / n)
        angles.append(positions[:, axis:axis + 1] * freq[None, :])
    ang = np.concatenate(angles, axis=1)
    return np.cos(ang).astype(F32), np.sin(ang).astype(F32)


def rope_apply(x, cos, sin) -> np.ndarray:
    """Rotate adjacent pairs (x[2j], x[2j+1]) by the angle of pair j; bf16 result.

    x: [S, heads, 128]; cos/sin: [S, 64].  fp32 operations, no fused
    multiply-add:  a' = a c - b s,  b' = a s + b c.
    """
    x = np.asarray(x, F32)
    a = x[..., 0::2]
    b = x[..., 1::2]
    c = np.asarray(cos, F32)[:, None, :]
    s = np.asarray(sin, F32)[:, None, :]
    out = np.empty_like(x)
    out[..., 0::2] = (a * c).astype(F32) - (b * s).astype(F32)
    out[..., 1::2] = (a * s).astype(F32) + (b * c).astype(F32)
    return bf16_round(out)


# ----------------------------------------------------------------------------
# Block-causal attention  (Core AI port intro: "block-causal attention";
# qwen-image-mnn: "block-causal mask")
# ----------------------------------------------------------------------------


def group_ids(group_ends: Sequence[int]) -> np.ndarray:
    """Group index of every token, from the cumulative group ends."""
    ids = np.zeros(group_ends[-1], dtype=np.int64)
    start = 0
    for g, end in enumerate(group_ends):
        ids[start:end] = g
        start = end
    return ids


def attention_block_causal(q, k, v, q_group, k_group, sm_scale) -> np.ndarray:
    """Masked softmax attention, brute force in float64.

    q: [Sq, heads, d], k/v: [Sk, heads, d]; q_group/k_group: group index of
    every query / key.  Query i may attend to key j iff group(j) <= group(i): a
    token sees its own group and every earlier group.
    Returns [Sq, heads, d] float64.
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    visible = np.asarray(k_group)[None, :] <= np.asarray(q_group)[:, None]
    out = np.empty(q.shape, dtype=F64)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * sm_scale
        s = np.where(visible, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out


def mxfp4_decode(packed, scales, k=None) -> np.ndarray:
    """MXFP4 checkpoint weights to fp32 ("Qwen_Image-2.1-MXFP4-Paiton-RDNA4",
    "What was quantized": E2M1 values packed low nibble first, one E8M0 scale
    per group of 32 input columns, rows zero-padded to a multiple of 32 columns
    and the padding removed on load).

    E2M1: code = sign << 3 | exponent << 1 | mantissa, exponent bias 1:
    exponent 0 -> mantissa * 0.5 (subnormal), else (1 + mantissa / 2) 2^(e-1).
    E8M0: 2^(e - 127), 255 = NaN.  w[r, c] = e2m1 * scale, in fp32.
    """
    packed = np.asarray(packed, np.uint8)
    scales = np.asarray(scales, np.uint8)
    n, half = packed.shape
    k_stored = 2 * half
    k = k_stored if k is None else k
    codes = np.empty((n, k_stored), np.int64)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    e = (codes >> 1) & 3
    m = codes & 1
    mag = np.where(e == 0, 0.5 * m, (1.0 + 0.5 * m) * np.exp2(np.maximum(e - 1, 0)))
    val = np.where(codes & 8, -mag, mag).astype(F32)
    sc = np.ldexp(np.float32(1.0), np.minimum(scales.astype(np.int64), 254) - 127).astype(F32)
    sc = np.where(scales == 255, np.float32(np.nan), sc).astype(F32)
    with np.errstate(over="ignore"):   # 6 x 2^127 overflows to inf in fp32, as it must
        w = (val * np.repeat(sc, 32, axis=1)).astype(F32)
    return w[:, :k]


def e4m3_round(x) -> np.ndarray:
    """Round to the nearest FP8 E4M3 value (ties to even), saturating at +-448.

    E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; normal values
    (1 + m/8) 2^(e-7) for e = 1..15 (all mantissas except e = 15, m = 7, the
    NaN code), subnormals (m/8) 2^-6.  So the spacing of the values in
    [2^e, 2^(e+1)) is 2^(e-3) for e >= -6, and 2^-9 below 2^-6.  (The
    reduced-precision attention of "Qwen_Image-2.1-MXFP4-Paiton-RDNA4",
    "Runtime precision and quality": int8/fp8 attention for later steps.)
    """
    x = np.asarray(x, F64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))          # a = m 2^ex, m in [0.5, 1)
    e = np.maximum(ex - 1, -6)                          # binade exponent, subnormals share -6
    quantum = np.ldexp(1.0, e - 3)
    r = np.rint(a / quantum) * quantum                  # a / quantum is exact: quantum is 2^k
    r = np.minimum(r, 448.0)
    return np.where(x < 0, -r, r)


def attention_block_causal_fp8(q, k, v, q_group, k_group, sm_scale, tile=128,
                               quantize=True, fp32_scores=True) -> np.ndarray:
    """Block-causal attention with e4m3 operands, following the method of the
    reduced-precision attention step by step (the reading of "int8/fp8
    attention" this build takes; the pages give no further detail):

      * q, k, v are rounded to e4m3;
      * keys are processed in tiles of ``tile`` keys from key 0; each row keeps
        a reference maximum m (base 2) set by the first tile and moved only
        when a tile's row maximum exceeds it by more than 8, rescaling the
        running sums by 2^(m_old - m_new);
      * per tile P = 2^(s log2(e) sm_scale - m), rounded to e4m3 before it
        multiplies V; the row sum takes the unrounded P;
      * O = (sum_tiles P_e4m3 V) / (sum_tiles P).

    With ``quantize=False, fp32_scores=False`` (no rounding anywhere) this is
    exactly the masked softmax attention above, which pins the tile
    bookkeeping.  By default S and the reference-maximum decisions are taken
    in fp32, like the tensor-core accumulation and the softmax they restate;
    everything else is float64.
    """
    rnd = e4m3_round if quantize else (lambda a: np.asarray(a, F64))
    q = rnd(q)
    k = rnd(k)
    v = rnd(v)
    qg = np.asarray(q_group)
    kg = np.asarray(k_group)
    Sq, heads, _ = q.shape
    Sk = k.shape[0]
    R = F32 if fp32_scores else F64
    sl2 = R(R(sm_scale) * R(1.4426950408889634))
    out = np.empty(q.shape, dtype=F64)
    for h in range(heads):
        for i in range(Sq):
            vis = kg <= qg[i]
            m = -np.inf
            l = 0.0
            o = np.zeros(q.shape[2], F64)
            for t0 in range(0, Sk, tile):
                t1 = min(t0 + tile, Sk)
                sv = vis[t0:t1]
                if not sv.any():
                    continue
                s = (k[t0:t1, h, :] @ q[i, h, :]).astype(R)        # scores of the tile
                mx2 = R(R(s[sv].max()) * sl2)
                if t0 == 0 or mx2 > R(m + R(8.0)):
                    m_new = max(m, float(mx2)) if t0 else float(mx2)
                    f = 2.0 ** (m - m_new) if t0 else 1.0
                    l *= f
                    o *= f
                    m = R(m_new)
                x = s.astype(F64) * float(sl2) - float(m)
                p = np.where(sv, np.exp2(x), 0.0)
                l += p.sum()
                o += rnd(p) @ v[t0:t1, h, :]
            out[i, h, :] = o / l
    return out


def attention_block_causal_fp8_plain(q, k, v, q_group, k_group, sm_scale) -> np.ndarray:
    """Block-causal attention with e4m3 operands, in the plainest reading of
    the pages' "int8/fp8 attention" ("Qwen_Image-2.1-MXFP4-Paiton-RDNA4",
    "Runtime precision and quality"), with no tiling:

      * q, k, v are rounded to e4m3;
      * per query row, s = (q . k) sm_scale over the visible keys, m = max s;
      * P = exp(s - m) (float64), rounded to e4m3 before it multiplies V;
      * O = (sum_j e4m3(P_j) v_j) / (sum_j P_j), the row sum over unrounded P.

    It differs from a tiled kernel only where the kernel takes scheduling
    decisions (which maximum each tile subtracts): those shift P by a power
    of two, which e4m3 rounds identically except below its smallest normal
    value 2^-6.
    """
    q = e4m3_round(q)
    k = e4m3_round(k)
    v = e4m3_round(v)
    visible = np.asarray(k_group)[None, :] <= np.asarray(q_group)[:, None]
    out = np.empty(q.shape, dtype=F64)
    for h in range(q.shape[1]):
        s = (q[:, h, :] @ k[:, h, :].T) * sm_scale
        s = np.where(visible, s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        out[:, h, :] = (e4m3_round(p) @ v[:, h, :]) / p.sum(axis=1, keepdims=True)
    return out


# ----------------------------------------------------------------------------
# One transformer block
# ----------------------------------------------------------------------------


PRECISION_W8A8 = {"qk": "w8", "v": "w8", "out": "w8", "up": "w8", "down": "w8"}


def prepare_block(wts: dict, precision: Optional[dict] = None) -> dict:
    """Prepare the Linears of a block from fp32 weights: W8A8 ones quantized
    (codes, scales, rowsums), BF16 ones rounded to bf16.

    precision maps "qk" (the q and k rows of the fused projection), "v", "out",
    "up", "down" to "w8", "bf16" or "mx"; default all W8A8.  "mx" Linears come
    as MXFP4 codes ``wts[name + "_mx"] = (packed, scales)`` and run as BF16
    Linears on their decoded weights ("Qwen_Image-2.1-MXFP4-Paiton-RDNA4":
    MXFP4 weights, the exact profile with BF16 activation arithmetic).  The pages' deployed
    layout (FlagOS card, "Quantization and validation", Scope) keeps only q, k
    and the MLP Linears of blocks 2-29 in W8A8.  W8A8 weights are quantized per
    output row, so splitting the q | k | v projection by rows leaves every
    code and scale unchanged.  "qkv" holds the projection's parts in column
    order: a list of (Linear, first column)."""
    prec = dict(PRECISION_W8A8)
    prec.update(precision or {})
    out = {}

    def prep(w, b, kind):
        b = np.asarray(b, F32)
        if kind == "mx":        # MXFP4 codes (packed, scales), decoded; exact in bf16
            return ("bf16", mxfp4_decode(*w), b)
        w = np.asarray(w, F32)
        if kind == "bf16":
            return ("bf16", bf16_round(w), b)
        q, s, rs = prepare_w8(w)
        return (q, s, rs, b)

    def weight(name, kind):
        return wts[name + "_mx"] if kind == "mx" else wts[name]

    b3 = np.asarray(wts["qkv_b"], F32)
    H = b3.shape[0] // 3
    if prec["qk"] == "mx" or prec["v"] == "mx":
        assert prec["qk"] == prec["v"] == "mx", "an MXFP4 q | k | v projection is MXFP4 throughout"
        out["qkv"] = [(prep(wts["qkv_mx"], b3, "mx"), 0)]
        w3 = None
    else:
        w3 = np.asarray(wts["qkv"], F32)
    if w3 is None:
        pass
    elif prec["qk"] == prec["v"]:
        out["qkv"] = [(prep(w3, b3, prec["qk"]), 0)]
    else:
        out["qkv"] = [(prep(w3[:2 * H], b3[:2 * H], prec["qk"]), 0),
                      (prep(w3[2 * H:], b3[2 * H:], prec["v"]), 2 * H)]
    for name in ("out", "up", "down"):
        out[name] = prep(weight(name, prec[name]), wts[name + "_b"], prec[name])
    out["norm_q"] = np.asarray(wts["norm_q"], F32)
    out["norm_k"] = np.asarray(wts["norm_k"], F32)
    return out


def dit_block(x, pw: dict, mod, row_set, q_group, k_group, cos, sin, heads, head_dim, eps,
              kv_prefix: Optional[Tuple[np.ndarray, np.ndarray]] = None,
              return_kv: bool = False, attn: str = "bf16"):
    """One single-stream block on the rows in ``x``.

    x: [T, H] residual stream of the rows processed (float64);
    mod: [R, 6, H] modulation rows (shift1, scale1, gate1, shift2, scale2, gate2);
    row_set: [T] which modulation row set each row uses;
    q_group / k_group: group of each processed row / of each key
    (k_group covers kv_prefix rows first, then the processed rows);
    cos/sin: [T, 64] RoPE tables of the processed rows;
    kv_prefix: cached (K, V) of earlier rows ([P, heads, d] bf16 values), used
    as the leading keys when only later rows are processed.

    Steps (reading of the pages' block; see the design notes):
      u1 = LN(x)(1 + scale1) + shift1 -> W8A8 QKV -> Q/K RMSNorm (cast first) -> RoPE
      o  = bf16(block-causal attention)
      x += gate1 * W8A8 out(o)
      u2 = LN(x)(1 + scale2) + shift2 -> W8A8 up -> bf16(GELU-tanh) -> W8A8 down
      x += gate2 * down
    Returns the new x (and the (K, V) of the processed rows if return_kv).
    """
    x = np.asarray(x, F64)
    T, H = x.shape
    m = np.asarray(mod, F64)[np.asarray(row_set)]          # [T, 6, H]
    shift1, scale1, gate1, shift2, scale2, gate2 = (m[:, i, :] for i in range(6))

    u1 = modulate(layer_norm(x, eps), shift1, scale1)
    parts = pw["qkv"] if isinstance(pw["qkv"], list) else [(pw["qkv"], 0)]
    qkv = np.concatenate([linear_apply(u1, lin) for lin, _ in parts], axis=1)   # bf16 [T, 3H]
    q = qkv[:, 0:H].reshape(T, heads, head_dim)
    k = qkv[:, H:2 * H].reshape(T, heads, head_dim)
    v = qkv[:, 2 * H:3 * H].reshape(T, heads, head_dim)
    q = rope_apply(rms_norm_cast(q, pw["norm_q"], eps), cos, sin)
    k = rope_apply(rms_norm_cast(k, pw["norm_k"], eps), cos, sin)

    if kv_prefix is not None:
        k_all = np.concatenate([kv_prefix[0], k], axis=0)
        v_all = np.concatenate([kv_prefix[1], v], axis=0)
    else:
        k_all, v_all = k, v
    if attn == "fp8":
        o = attention_block_causal_fp8(q, k_all, v_all, q_group, k_group, 1.0 / math.sqrt(head_dim))
    else:
        o = attention_block_causal(q, k_all, v_all, q_group, k_group, 1.0 / math.sqrt(head_dim))
    # The attention output and the GELU output are activation tensors of the
    # BF16 transformer (FlagOS card: the Linears outside the W8A8 set and the
    # activations stay BF16), so the per-token quantizer sees them as bf16
    # values: the code decision is taken on the same bf16 input precision as
    # the CUDA path.
    o = bf16_round(o.reshape(T, H))

    x = x + gate1 * linear_apply(o, pw["out"])
    u2 = modulate(layer_norm(x, eps), shift2, scale2)
    g = bf16_round(gelu_tanh(linear_apply(u2, pw["up"])))
    x = x + gate2 * linear_apply(g, pw["down"])
    if return_kv:
        return x, (k, v)
    return x


# ----------------------------------------------------------------------------
# Timestep embedding and adaLN rows
# ----------------------------------------------------------------------------


def timestep_embedding(t, dim=256) -> np.ndarray:
    """Sinusoidal embedding of 1000 t (reading: dim 256, cos half first).

    The pages fix only that the DiT's timestep input is sigma in fp32
    (Core AI port, "Graph contracts", Sampler); the embedding is the usual
    one: freq_i = exp(-ln(1e4) i / 128), emb = [cos(1000 t f), sin(1000 t f)].
    """
    half = dim // 2
    freqs = np.exp(-math.log(10000.0) * np.arange(half, dtype=F64) / half)
    arg = 1000.0 * float(t) * freqs
    return np.concatenate([np.cos(arg), np.sin(arg)])


def silu(x) -> np.ndarray:
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def linear(x, w, b) -> np.ndarray:
    """BF16-weight Linear evaluated in float64: x W^T + b."""
    return np.asarray(x, F64) @ np.asarray(w, F64).T + np.asarray(b, F64)


def time_embed(t, mw: dict) -> np.ndarray:
    """temb = Linear_2(SiLU(Linear_1(sinusoid(t))))  [H]."""
    e = timestep_embedding(t)
    return linear(silu(linear(e, mw["t1"], mw["t1_b"])), mw["t2"], mw["t2_b"])


def adaln_rows(temb, w_mod, b_mod) -> np.ndarray:
    """Modulation rows of one block: Linear_{H->6H}(SiLU(temb)) reshaped to [6, H]."""
    y = linear(silu(temb), w_mod, b_mod)
    return y.reshape(6, -1)


# ----------------------------------------------------------------------------
# Sampler  (Core AI port, "Graph contracts", Sampler)
# ----------------------------------------------------------------------------


def sigma_schedule(steps: int, image_tokens: int, base_len=256, max_len=8192,
                   base_shift=0.5, max_shift=0.9, terminal=0.02) -> np.ndarray:
    """Shifted FlowMatch sigmas [steps + 1] (fp32), ending in 0.

    mu is linear in the image-token count (base_shift at base_len tokens,
    max_shift at max_len); the base grid linspace(1, 1/steps, steps) is
    shifted exponentially, sigma' = e^mu / (e^mu + 1/sigma - 1); the tail is
    stretched so the last non-zero sigma equals ``terminal``; 0 is appended.
    The endpoints (256 / 8192 tokens, shifts 0.5 / 0.9) are a reading.
    """
    slope = (max_shift - base_shift) / (max_len - base_len)
    mu = image_tokens * slope + (base_shift - slope * base_len)
    base = np.linspace(1.0, 1.0 / steps, steps)
    shifted = math.exp(mu) / (math.exp(mu) + (1.0 / base - 1.0))
    one_minus = 1.0 - shifted
    stretch = one_minus[-1] / (1.0 - terminal)
    sig = 1.0 - one_minus / stretch
    return np.append(sig, 0.0).astype(F32)


def euler_update(x, v, sigma, sigma_next) -> np.ndarray:
    """x + (sigma_next - sigma) * v in fp32: one rounding per operation, no FMA."""
    x = np.asarray(x, F32)
    v = np.asarray(v, F32)
    dt = F32(sigma_next) - F32(sigma)
    return (x + (dt * v).astype(F32)).astype(F32)


def cfg_combine(v_cond, v_uncond, guidance) -> np.ndarray:
    """True classifier-free guidance of one step (qwen-image-mnn, "Install /
    run": a true CFG scale with a negative prompt): v_u + g (v_c - v_u) in
    fp32, one rounding per operation, no FMA.  The pages give the scale, not
    the formula; this is the plain reading, with no renormalization."""
    vc = np.asarray(v_cond, F32)
    vu = np.asarray(v_uncond, F32)
    d = (vc - vu).astype(F32)
    return (vu + (F32(guidance) * d).astype(F32)).astype(F32)


# ----------------------------------------------------------------------------
# Whole denoising step
# ----------------------------------------------------------------------------


def joint_inputs(latents, txt, ref_latents, mw: dict, groups, mode: str = "none"):
    """Rows of the joint sequence that enter the first block, and their indices.

    Core AI port, "Graph contracts": the DiT takes the text features and the
    latent tokens as separate inputs and runs one single-stream sequence
    [text | image].  Reading (see the design notes): text rows enter through
    the text in-projection (a BF16 Linear H -> H), reference-image rows of an
    edit sequence through the same image in-projection as the target latents
    (P -> H), in the order of the groups.  In "read" mode (cached prefix) only
    the target rows are formed.
    Returns (x [rows, H] float64, row indices into the sequence).
    """
    sizes = [n for _, n, _ in groups]
    S = sum(sizes)
    P_tok = S - sizes[-1]
    x_img = linear(np.asarray(latents, F64), mw["img_in"], mw["img_in_b"])
    if mode == "read":
        return x_img, np.arange(P_tok, S)
    parts = [linear(np.asarray(txt, F64), mw["txt_in"], mw["txt_in_b"])]
    if ref_latents is not None:
        parts.append(linear(np.asarray(ref_latents, F64), mw["img_in"], mw["img_in_b"]))
    parts.append(x_img)
    x = np.concatenate(parts, axis=0)
    assert x.shape[0] == S
    return x, np.arange(S)


def step_forward(latents, txt, ref_latents, mw: dict, blocks_pw: Sequence[dict],
                 blocks_mod_w: Sequence[Tuple], groups, heads, head_dim, eps, sigma, sigma_next,
                 kv_cache: Optional[Dict[int, Tuple[np.ndarray, np.ndarray]]] = None,
                 mode: str = "none", return_v: bool = False, attn: str = "bf16"):
    """One FlowMatch Euler step of the DiT.

    latents [N, P] fp32 (target tokens); txt [L, H] text features (bf16 values);
    ref_latents [R, P] fp32 reference-image tokens of an edit sequence, or None;
    mw: step-level BF16 Linears; blocks_pw: prepared W8A8 block weights;
    blocks_mod_w: (W_mod [6H, H], b_mod [6H]) per block;
    groups: [(kind, tokens, grid)] of the joint sequence, the target last.
    mode: "none"   - all tokens processed, nothing cached;
          "write"  - all tokens processed, the prefix (K, V) of every block
                     stored in kv_cache;
          "read"   - only the target rows processed, prefix keys from kv_cache.
    Reading: prefix groups use modulation rows of the clean timestep t = 0,
    the target uses the step's sigma; this is what makes the cached prefix
    K/V of the first step exact for later steps.
    """
    sizes = [n for _, n, _ in groups]
    ends = list(np.cumsum(sizes))
    S, P_tok = ends[-1], ends[-2] if len(ends) > 1 else 0
    gid = group_ids(ends)
    row_set_all = np.where(gid < len(groups) - 1, 0, 1)
    cos_all, sin_all = rope_tables(rope_positions(groups))

    temb_t = time_embed(sigma, mw)
    temb_0 = time_embed(0.0, mw)

    x, rows = joint_inputs(latents, txt, ref_latents, mw, groups, mode)

    for l, (pw, (wm, bm)) in enumerate(zip(blocks_pw, blocks_mod_w)):
        mod = np.stack([adaln_rows(temb_0, wm, bm), adaln_rows(temb_t, wm, bm)])
        kvp = kv_cache[l] if mode == "read" else None
        x, kv = dit_block(x, pw, mod, row_set_all[rows], gid[rows], gid, cos_all[rows],
                          sin_all[rows], heads, head_dim, eps, kv_prefix=kvp, return_kv=True,
                          attn=attn)
        if mode == "write":
            kv_cache[l] = (kv[0][:P_tok], kv[1][:P_tok])

    xt = x[-sizes[-1]:]
    # final adaLN: two rows (shift, scale) from the step's timestep embedding
    fm = linear(silu(temb_t), mw["final_mod"], mw["final_mod_b"]).reshape(2, -1)
    u = modulate(layer_norm(xt, eps), fm[0], fm[1])
    v = linear(u, mw["proj_out"], mw["proj_out_b"]).astype(F32)
    new_lat = euler_update(latents, v, sigma, sigma_next)
    if return_v:
        return new_lat, v
    return new_lat
