"""Pins for the CPU oracle: facts fixed by the pages or by mathematics.

Each test checks the oracle against something other than itself: values
derived by hand from a formula the pages state, closed forms, invariants,
library routines that the method reduces to in a special case, and brute
force on tiny inputs.  They are chosen so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import qi_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32 = np.float32
rng = np.random.default_rng(1234)


# --------------------------------------------------------------------- bf16


def test_bf16_round_matches_torch_cast():
    x = np.concatenate([rng.standard_normal(4096).astype(F32) * 100,
                        # exact ties between two bf16 neighbours (both parities)
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 ** -130], F32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(O.bf16_round(x), ref)


# ------------------------------------------------------------ weight quant


def test_prepare_w8_hand_example():
    # FlagOS card, "Quantization and validation": symmetric INT8 per output
    # channel, zero point 0, FP32 scale.  amax = 1.27 -> s = 1.27/127 ~ 0.01:
    # 0.5/s = 50, -1.27/s = -127, 0.0149/s = 1.49 -> 1, 0.0151/s -> 2.
    w = np.array([[0.5, -1.27, 0.0149, 0.0151, 0.0],
                  [0.0, 0.0, 0.0, 0.0, 0.0]], F32)
    q, s, rs = O.prepare_w8(w)
    assert q.dtype == np.int8
    assert q[0].tolist() == [50, -127, 1, 2, 0]
    assert s[0] == F32(1.27) / F32(127)
    assert rs[0] == 50 - 127 + 1 + 2
    assert q[1].tolist() == [0] * 5 and s[1] == 1.0 and rs[1] == 0


def test_prepare_w8_bounds():
    w = rng.standard_normal((64, 300)).astype(F32) * 0.02
    q, s, rs = O.prepare_w8(w)
    amax_idx = np.argmax(np.abs(w), axis=1)
    assert np.all(np.abs(q[np.arange(64), amax_idx]) == 127)
    assert np.all(np.sign(q[np.arange(64), amax_idx]) == np.sign(w[np.arange(64), amax_idx]))
    err = np.abs(w.astype(np.float64) - s[:, None].astype(np.float64) * q)
    assert np.all(err <= s[:, None] * (0.5 + 1e-6))
    assert np.array_equal(rs, q.astype(np.int64).sum(1))


# -------------------------------------------------------- activation quant


def test_quantize_act_hand_example():
    # FlagOS card: dynamic asymmetric INT8 per token/row.  Row [-1, 0, 0.5, 1.55]:
    # lo = -1, hi = 1.55, s = 2.55/255 ~ 0.01, zp = rint(-128 + 100) = -28,
    # q = rint(u/s) + zp = [-100, 0, 50, 155] - 28 = [-128, -28, 22, 127].
    u = np.array([[-1.0, 0.0, 0.5, 1.55]], F32)
    q, s, zp = O.quantize_act(u)
    assert q[0].tolist() == [-128, -28, 22, 127]
    assert zp[0] == -28
    assert s[0] == (F32(1.55) - F32(-1.0)) / F32(255)


def test_quantize_act_edge_rows():
    u = np.array([[0.0, 0.0, 0.0],          # empty range
                  [0.5, 1.0, 2.0],          # all positive: lo = 0 -> zp = -128
                  [-0.5, -1.0, -2.0]], F32)  # all negative: hi = 0 -> zp = 127
    q, s, zp = O.quantize_act(u)
    assert (s[0], zp[0]) == (1.0, 0) and q[0].tolist() == [0, 0, 0]
    assert zp[1] == -128 and q[1].tolist()[-1] == 127
    assert zp[2] == 127 and q[2].tolist()[-1] == -128


def test_quantize_act_invariants():
    u = (rng.standard_normal((50, 257)) * rng.uniform(0.01, 10, (50, 1))).astype(F32)
    u[:, 7] = 0.0
    q, s, zp = O.quantize_act(u)
    assert np.all(q[:, 7] == zp)                                # zero is exact
    rec = s[:, None].astype(np.float64) * (q.astype(np.float64) - zp[:, None])
    assert np.all(np.abs(rec - u) <= s[:, None] * 0.5 * (1 + 1e-5))
    assert np.all(q[np.arange(50), np.argmin(u, 1)] <= -127)     # row min -> bottom code
    assert np.all(q[np.arange(50), np.argmax(u, 1)] >= 126)      # row max -> top code
    q2, s2, zp2 = O.quantize_act(u * F32(4))                     # power-of-two scaling
    assert np.array_equal(q2, q) and np.array_equal(zp2, zp) and np.array_equal(s2, s * 4)


# -------------------------------------------------------------- int GEMM


def test_int_gemm_brute_force():
    qa = rng.integers(-128, 128, (3, 37)).astype(np.int8)
    qw = rng.integers(-127, 128, (4, 37)).astype(np.int8)
    acc = O.int_gemm(qa, qw)
    for m in range(3):
        for n in range(4):
            assert acc[m, n] == sum(int(qa[m, k]) * int(qw[n, k]) for k in range(37))


def test_int_gemm_special_cases():
    qa = rng.integers(-128, 128, (5, 64)).astype(np.int8)
    qa[2] = 0
    eye = (127 * np.eye(64)).astype(np.int8)
    acc = O.int_gemm(qa, eye)
    assert np.array_equal(acc, 127 * qa.astype(np.int64))
    assert np.all(acc[2] == 0)
    # extreme magnitude at the largest K the block uses (16384): -128 * -127 * K
    big_a = np.full((1, 16384), -128, np.int8)
    big_w = np.full((2, 16384), -127, np.int8)
    assert O.int_gemm(big_a, big_w)[0, 0] == 128 * 127 * 16384 < 2 ** 31


def test_w8a8_linear_approximates_float_linear():
    M, N, K = 6, 40, 512
    u = rng.standard_normal((M, K)).astype(F32) + F32(0.3)   # non-symmetric range -> zp != 0
    w = (rng.standard_normal((N, K)) * 0.02).astype(F32)
    b = O.bf16_round(rng.standard_normal(N) * 0.02)
    qa, sa, zpa = O.quantize_act(u)
    assert np.any(zpa != -0)
    qw, sw, rs = O.prepare_w8(w)
    acc, y = O.w8a8_linear(qa, sa, zpa, qw, sw, rs, b)
    exact = u.astype(np.float64) @ w.astype(np.float64).T + b
    # |u w - s_a(q_a - zp) s_w q_w| <= sum_k s_a/2 |w| + s_w/2 |u| + s_a s_w / 4
    bound = (sa[:, None] / 2 * np.abs(w).sum(1)[None, :]
             + sw[None, :] / 2 * np.abs(u).sum(1)[:, None]
             + K * sa[:, None] * sw[None, :] / 4)
    bound = bound + np.abs(exact) * 2 ** -8                    # one bf16 rounding
    assert np.all(np.abs(y - exact) <= bound)
    # the error is far below the bound's worst case; catch a missing zp term
    assert np.linalg.norm(y - exact) / np.linalg.norm(exact) < 0.05


# ----------------------------------------------------------------- norms


def test_layer_norm_vs_torch():
    x = rng.standard_normal((7, 256)) * 3 + 1
    ref = F.layer_norm(torch.from_numpy(x), (256,), eps=1e-6).numpy()
    assert np.allclose(O.layer_norm(x, 1e-6), ref, rtol=1e-12, atol=1e-12)


def test_modulate_closed_form():
    u = np.array([[1.0, -2.0]])
    assert np.allclose(O.modulate(u, np.array([0.5, 0.25]), np.array([1.0, -0.5])), [[2.5, -0.75]])


def test_rms_norm_cast_first_hand_example():
    # "Qwen Image 2.1 native qualification", Numerical checks: the normalized
    # activation is cast to the scale's dtype before the scale multiplies.
    # x = [1]*64 + [0.25]*64: mean(x^2) = (64 + 4)/128 = 0.53125,
    # n = x / sqrt(0.53125 + 1e-6): 1.3719873 -> bf16 1.375 and 0.3429968 -> bf16 0.34375.
    # w = 1.015625: cast-first 1.375*w = 1.3964844 -> bf16 1.3984375, 0.34375*w -> 0.34960938;
    # cast-last (n*w then bf16) would give 1.390625 and 0.34765625.
    x = np.array([[1.0] * 64 + [0.25] * 64], F32)
    w = np.full(128, 1.015625, F32)
    out = O.rms_norm_cast(x, w, 1e-6)
    assert out[0, 0] == F32(1.3984375) and out[0, -1] == F32(0.349609375)
    assert out[0, 0] != F32(1.390625) and out[0, -1] != F32(0.34765625)


def test_rms_norm_invariants():
    x = rng.standard_normal((20, 128)).astype(F32)
    w = np.ones(128, F32)
    a = O.rms_norm_cast(x, w, 0.0)
    assert np.array_equal(a, O.rms_norm_cast(x * F32(8), w, 0.0))   # scale invariance
    rms = np.sqrt((a.astype(np.float64) ** 2).mean(1))
    assert np.allclose(rms, 1.0, atol=5e-3)


def test_gelu_tanh_vs_torch():
    x = np.linspace(-8, 8, 2001)
    ref = F.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    assert np.allclose(O.gelu_tanh(x), ref, rtol=1e-13, atol=1e-15)


# ------------------------------------------------------------------ RoPE


def test_rope_positions_golden():
    ref = np.loadtxt(os.path.join(GOLDEN, "rope_positions_L3_2x3.txt"), dtype=np.int64)
    pos = O.rope_positions([("text", 3, None), ("image", 6, (2, 3))])
    assert np.array_equal(pos, ref)


def test_rope_positions_edit_frames_and_range():
    pos = O.rope_positions([("text", 4, None), ("image", 4, (2, 2)), ("image", 16, (4, 4))])
    assert np.all(pos[4:8, 0] == 4) and np.all(pos[8:, 0] == 5)
    # a 128x128 grid stays inside the tables' -1024..8191 range
    p = O.rope_positions([("text", 512, None), ("image", 128 * 128, (128, 128))])
    assert p.min() >= -1024 and p.max() <= 8191
    assert p[512:, 1].min() == -64 and p[512:, 1].max() == 63


def test_rope_positions_multi_reference_frames():
    # k-th image group at frame L + k: three references, then the target
    groups = [("text", 5, None), ("image", 4, (2, 2)), ("image", 9, (3, 3)),
              ("image", 6, (2, 3)), ("image", 16, (4, 4))]
    pos = O.rope_positions(groups)
    ends = np.cumsum([n for _, n, _ in groups])
    for k, (a, b) in enumerate(zip(ends[:-1], ends[1:])):
        assert np.all(pos[a:b, 0] == 5 + k)
    # each image group is centred on its own grid, whatever precedes it
    assert np.array_equal(pos[9:18, 1:], O.rope_positions([("image", 9, (3, 3))])[:, 1:])


def test_rope_tables_axis_layout():
    pos = np.array([[5, -3, 7]])
    c, s = O.rope_tables(pos)
    assert c.shape == (1, 64)
    # pair 0 / 8 / 36 are each axis' first pair, frequency 1
    assert np.isclose(c[0, 0], math.cos(5)) and np.isclose(s[0, 0], math.sin(5))
    assert np.isclose(c[0, 8], math.cos(-3)) and np.isclose(s[0, 8], math.sin(-3))
    assert np.isclose(c[0, 36], math.cos(7)) and np.isclose(s[0, 36], math.sin(7))
    # pair 1 of the frame axis: 10000^(-1/8);  pair 9 (h axis, i=1): 10000^(-1/28)
    assert np.isclose(c[0, 1], math.cos(5 * 10000 ** (-1 / 8)))
    assert np.isclose(s[0, 9], math.sin(-3 * 10000 ** (-1 / 28)))


def _rope_complex(x, pos):
    """Independent RoPE: complex multiplication of adjacent pairs (torch)."""
    c, s = O.rope_tables(pos)
    ang = torch.atan2(torch.from_numpy(s).double(), torch.from_numpy(c).double())
    z = torch.view_as_complex(torch.from_numpy(np.asarray(x, np.float64)).reshape(*x.shape[:-1], 64, 2).contiguous())
    return torch.view_as_real(z * torch.polar(torch.ones_like(ang), ang)[:, None, :]).reshape(x.shape).numpy()


def test_rope_apply_vs_complex_rotation():
    x = O.bf16_round(rng.standard_normal((9, 2, 128)))
    pos = O.rope_positions([("text", 3, None), ("image", 6, (2, 3))])
    c, s = O.rope_tables(pos)
    out = O.rope_apply(x, c, s)
    ref = _rope_complex(x, pos)
    assert np.allclose(out, ref, rtol=2 ** -8, atol=1e-6)


def test_rope_identity_and_relative_invariance():
    x = O.bf16_round(rng.standard_normal((4, 1, 128)))
    c, s = O.rope_tables(np.zeros((4, 3), np.int64))
    assert np.array_equal(O.rope_apply(x, c, s), x)
    q = rng.standard_normal((1, 1, 128))
    k = rng.standard_normal((1, 1, 128))
    pq, pk = np.array([[3, 5, -2]]), np.array([[1, -4, 6]])
    d0 = (_rope_complex(q, pq) * _rope_complex(k, pk)).sum()
    for axis in range(3):
        sh = np.zeros((1, 3), np.int64)
        sh[0, axis] = 17
        d1 = (_rope_complex(q, pq + sh) * _rope_complex(k, pk + sh)).sum()
        assert abs(d1 - d0) < 1e-6 * np.linalg.norm(q) * np.linalg.norm(k)   # fp32 tables
    # and the oracle's fp32/bf16 form keeps the same dot product to rounding
    a = O.rope_apply(O.bf16_round(q), *O.rope_tables(pq)) * O.rope_apply(O.bf16_round(k), *O.rope_tables(pk))
    sh = np.array([[0, 0, 17]])
    b = O.rope_apply(O.bf16_round(q), *O.rope_tables(pq + sh)) * O.rope_apply(O.bf16_round(k), *O.rope_tables(pk + sh))
    assert abs(a.sum() - b.sum()) < 0.05 * np.linalg.norm(q) * np.linalg.norm(k)


# ------------------------------------------------------------- attention


def _sdpa(q, k, v, causal=False, mask=None):
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64)).permute(1, 0, 2)
    o = F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=mask, is_causal=causal)
    return o.permute(1, 0, 2).numpy()


def test_attention_one_group_is_full_attention():
    q, k, v = (rng.standard_normal((11, 2, 16)) for _ in range(3))
    g = np.zeros(11, np.int64)
    out = O.attention_block_causal(q, k, v, g, g, 1 / 4)
    assert np.allclose(out, _sdpa(q, k, v), atol=1e-12)


def test_attention_singleton_groups_is_causal():
    q, k, v = (rng.standard_normal((9, 3, 8)) for _ in range(3))
    g = np.arange(9)
    out = O.attention_block_causal(q, k, v, g, g, 1 / math.sqrt(8))
    assert np.allclose(out, _sdpa(q, k, v, causal=True), atol=1e-12)


def test_attention_text_image_and_mask_invariance():
    ends = [5, 12, 20]
    g = O.group_ids(ends)
    q, k, v = (rng.standard_normal((20, 2, 8)) for _ in range(3))
    out = O.attention_block_causal(q, k, v, g, g, 0.3)
    # text rows see only text; last group sees everything
    sc = 0.3 * math.sqrt(8)
    assert np.allclose(out[:5], _sdpa(q[:5] * sc, k[:5], v[:5]), atol=1e-12)
    assert np.allclose(out[12:], _sdpa(q[12:] * sc, k, v), atol=1e-12)
    # perturbing later-group keys/values leaves earlier groups bit-identical
    k2, v2 = k.copy(), v.copy()
    k2[12:] += 5.0
    v2[12:] -= 3.0
    out2 = O.attention_block_causal(q, k2, v2, g, g, 0.3)
    assert np.array_equal(out2[:12], out[:12])
    assert not np.allclose(out2[12:], out[12:])


def test_attention_many_groups_reduce_to_full_attention_on_prefixes():
    # [text | ref1 | ref2 | ref3 | target]: the rows of group g attend exactly
    # like full (one-group) attention over the sequence cut at the end of g
    ends = [4, 9, 12, 18, 27]
    g = O.group_ids(ends)
    q, k, v = (rng.standard_normal((27, 2, 8)) for _ in range(3))
    out = O.attention_block_causal(q, k, v, g, g, 0.25)
    start = 0
    for e in ends:
        sub = O.attention_block_causal(q[:e], k[:e], v[:e], np.zeros(e, np.int64),
                                       np.zeros(e, np.int64), 0.25)
        assert np.allclose(out[start:e], sub[start:e], atol=1e-12)
        start = e
    sc = 0.25 * math.sqrt(8)
    assert np.allclose(out[9:12], _sdpa(q[9:12] * sc, k[:12], v[:12]), atol=1e-12)


def test_mxfp4_decode_format():
    # one row of 64 codes: the 16 E2M1 codes twice per 32-column group, scales 2^0 and 2^3
    codes = np.array(list(range(16)) * 4, np.uint8)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)[None, :]   # low nibble first
    scales = np.array([[127, 130]], np.uint8)
    w = O.mxfp4_decode(packed, scales)
    e2m1 = [0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    assert np.array_equal(w[0, :16], e2m1) and np.array_equal(w[0, 16:32], e2m1)
    assert np.array_equal(w[0, 32:48], np.array(e2m1) * 8)
    # padding columns are dropped; E8M0 extremes: 2^-127 (denormal) and NaN
    assert O.mxfp4_decode(packed, scales, k=40).shape == (1, 40)
    ext = O.mxfp4_decode(np.full((1, 16), 0x22, np.uint8), np.array([[0]], np.uint8))
    assert ext[0, 0] == np.float32(2.0 ** -127)          # code 2 = 1.0, E8M0 0 = 2^-127 (an fp32 denormal)
    assert np.all(np.isnan(O.mxfp4_decode(packed[:, :16], np.array([[255]], np.uint8))))


def _e4m3_decode(b):
    # straight from the format: 1 sign, 4 exponent (bias 7), 3 mantissa bits
    sgn = -1.0 if b & 0x80 else 1.0
    e, m = (b >> 3) & 15, b & 7
    if e == 15 and m == 7:
        return None                                   # NaN code
    return sgn * (m / 8.0 * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))


def test_e4m3_round_codes_ties_and_saturation():
    vals = sorted({v for v in (_e4m3_decode(b) for b in range(256)) if v is not None})
    assert len(vals) == 253 and max(vals) == 448.0 and min(vals) == -448.0
    a = np.array(vals)
    assert np.array_equal(O.e4m3_round(a), a)         # every value is its own rounding
    pos = np.array([v for v in vals if v >= 0])
    codes = {(_e4m3_decode(b)): b for b in range(128) if _e4m3_decode(b) is not None}
    mid = (pos[:-1] + pos[1:]) / 2                    # ties go to the even mantissa
    want = np.where([codes[lo] % 2 == 0 for lo in pos[:-1]], pos[:-1], pos[1:])
    assert np.array_equal(O.e4m3_round(mid), want)
    assert O.e4m3_round(np.array([0.3]))[0] == 0.3125  # quantum 2^-5 in [0.25, 0.5)
    assert np.array_equal(O.e4m3_round(np.array([460.0, 1e6, -500.0])), [448.0, 448.0, -448.0])
    assert np.array_equal(O.e4m3_round(np.array([2.0 ** -10, 1.5 * 2.0 ** -10, -2.0 ** -12])),
                          [0.0, 2.0 ** -9, 0.0])


def test_attention_fp8_unquantized_reduces_to_exact_attention():
    ends = [6, 13, 30]
    g = O.group_ids(ends)
    q, k, v = (rng.standard_normal((30, 2, 8)) for _ in range(3))
    # scores that grow along the keys force the reference-maximum rescales
    k[:, :, 0] += np.linspace(0, 60, 30)[:, None]
    q[:, :, 0] = np.abs(q[:, :, 0]) + 1.0
    ref = O.attention_block_causal(q, k, v, g, g, 0.4)
    for tile in (4, 7, 128):
        out = O.attention_block_causal_fp8(q, k, v, g, g, 0.4, tile=tile, quantize=False,
                                           fp32_scores=False)
        assert np.allclose(out, ref, rtol=1e-10, atol=1e-12)
        # fp32 scores: within fp32 rounding of the scores
        out32 = O.attention_block_causal_fp8(q, k, v, g, g, 0.4, tile=tile, quantize=False)
        assert np.linalg.norm(out32 - ref) / np.linalg.norm(ref) < 1e-5


def test_attention_fp8_error_is_e4m3_sized():
    ends = [16, 80]
    g = O.group_ids(ends)
    q, k, v = (rng.standard_normal((80, 2, 32)) for _ in range(3))
    ref = O.attention_block_causal(q, k, v, g, g, 1 / math.sqrt(32))
    out = O.attention_block_causal_fp8(q, k, v, g, g, 1 / math.sqrt(32), tile=16)
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert 1e-3 < err < 8e-2


def test_attention_fp8_plain_uniform_scores_closed_form():
    """q = 0: every visible score is 0, so P = exp(0) = 1 exactly (an e4m3
    value) and the output is the plain mean of the e4m3-rounded values of the
    visible keys; a numerator or denominator over the wrong key set, or P
    rounded in the row sum, would move it."""
    ends = [5, 12, 20]
    g = O.group_ids(ends)
    k = rng.standard_normal((20, 2, 16))
    v = rng.standard_normal((20, 2, 16)) * 3
    q = np.zeros((20, 2, 16))
    out = O.attention_block_causal_fp8_plain(q, k, v, g, g, 0.3)
    v8 = O.e4m3_round(v)
    for i in range(20):
        n_vis = ends[g[i]]
        assert np.allclose(out[i], v8[:n_vis].mean(axis=0), rtol=0, atol=1e-12)


def test_attention_fp8_plain_row_sum_uses_unrounded_p():
    """Constant V rows (an e4m3 value c): O = c * sum(e4m3(P)) / sum(P), which
    differs from c by at most one e4m3 half-step (2^-4 relative) and, with
    varied scores, is not exactly c -- the row sum takes the unrounded P."""
    g = O.group_ids([40])
    q = rng.standard_normal((40, 1, 16))
    k = rng.standard_normal((40, 1, 16))
    v = np.full((40, 1, 16), 0.75)          # e4m3-exact
    out = O.attention_block_causal_fp8_plain(q, k, v, g, g, 0.7)
    q8, k8 = O.e4m3_round(q), O.e4m3_round(k)
    for i in range(40):
        s = (k8[:, 0] @ q8[i, 0]) * 0.7
        p = np.exp(s - s.max())
        want = 0.75 * O.e4m3_round(p).sum() / p.sum()
        assert np.allclose(out[i, 0], want, rtol=1e-12)
    ratio = out[:, 0, 0] / 0.75
    assert np.all(np.abs(ratio - 1) <= 2.0 ** -4) and np.any(ratio != 1)


def test_attention_fp8_plain_error_is_e4m3_sized():
    ends = [16, 80]
    g = O.group_ids(ends)
    q, k, v = (rng.standard_normal((80, 2, 32)) for _ in range(3))
    ref = O.attention_block_causal(q, k, v, g, g, 1 / math.sqrt(32))
    out = O.attention_block_causal_fp8_plain(q, k, v, g, g, 1 / math.sqrt(32))
    err = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert 1e-3 < err < 8e-2


# ------------------------------------------------------------ timestep


def test_timestep_embedding_closed_form():
    e0 = O.timestep_embedding(0.0)
    assert np.array_equal(e0[:128], np.ones(128)) and np.array_equal(e0[128:], np.zeros(128))
    t = 0.37
    e = O.timestep_embedding(t)
    assert np.isclose(e[0], math.cos(1000 * t)) and np.isclose(e[128], math.sin(1000 * t))
    assert np.isclose(e[64], math.cos(1000 * t * 10000 ** -0.5))


# -------------------------------------------------------------- sampler


def test_sigma_schedule_page_facts():
    facts = json.load(open(os.path.join(GOLDEN, "sampler_facts.json")))
    n = facts["default_steps"]
    for tokens in (256, 1024, 4096, 16384):
        sig = O.sigma_schedule(n, tokens)
        assert sig.dtype == np.float32 and len(sig) == n + 1
        assert sig[0] == F32(facts["first_sigma"])
        assert abs(sig[-2] - facts["terminal_sigma"]) < 1e-7
        assert sig[-1] == facts["final_sigma"]
        assert np.all(np.diff(sig) < 0)


def test_sigma_schedule_hand_values():
    # 3 steps at 256 tokens: mu = 0.5, e^mu = 1.6487213; base = [1, 2/3, 1/3]
    # shifted = [1, 1.6487213/2.1487213, 1.6487213/3.6487213] = [1, 0.767303, 0.451863]
    # 1 - shifted = [0, 0.232697, 0.548137]; stretch = 0.548137/0.98 = 0.559323
    # sigma = [1, 1 - 0.232697/0.559323, 0.02, 0] = [1, 0.583964, 0.02, 0]
    sig = O.sigma_schedule(3, 256)
    assert np.allclose(sig, [1.0, 0.583964, 0.02, 0.0], atol=2e-6)
    # more image tokens -> larger mu -> larger mid sigmas
    assert O.sigma_schedule(3, 8192)[1] > sig[1]


def test_token_counts_golden():
    tc = json.load(open(os.path.join(GOLDEN, "token_counts.json")))
    from diffusion_transformer_text_dit_b200 import synth
    assert synth.STEP1024.target_tokens == tc["tokens"]["1024"]
    assert synth.BLOCK512.groups[-1].tokens == tc["tokens"]["512"]
    assert synth.GEN2048.target_tokens == tc["tokens"]["2048"]
    for size, n in tc["tokens"].items():
        assert (int(size) // tc["patch_px"]) ** 2 == n


def test_euler_fp32_rounding():
    x = rng.standard_normal(1000).astype(F32)
    v = rng.standard_normal(1000).astype(F32)
    out = O.euler_update(x, v, 0.7316, 0.6801)
    tx, tv = torch.from_numpy(x), torch.from_numpy(v)
    dt = torch.tensor(0.6801, dtype=torch.float32) - torch.tensor(0.7316, dtype=torch.float32)
    ref = (tx + (dt * tv)).numpy()
    assert np.array_equal(out, ref)
    # a constant velocity integrates exactly over a whole schedule: x_end ~ x0 - v
    sig = O.sigma_schedule(40, 4096)
    z = x.copy()
    for i in range(40):
        z = O.euler_update(z, v, sig[i], sig[i + 1])
    assert np.allclose(z, x - v, atol=1e-5)


def test_cfg_combine_special_cases():
    vc = rng.standard_normal(257).astype(np.float32)
    vu = rng.standard_normal(257).astype(np.float32)
    # scale 0 is the unconditional velocity, equal velocities are unchanged
    assert np.array_equal(O.cfg_combine(vc, vu, 0.0), vu)
    assert np.array_equal(O.cfg_combine(vu, vu, 7.5), vu)
    # scale 1 gives v_c exactly where v_c - v_u is exact (Sterbenz: v_u/2 <= v_c <= 2 v_u)
    a = np.float32(1.0) + rng.random(100).astype(np.float32)
    b = a * np.float32(1.5)
    assert np.array_equal(O.cfg_combine(b, a, 1.0), b)
    # hand values: 0.5 + 3 (1 - 0.5) = 2
    assert O.cfg_combine(np.float32([1.0]), np.float32([0.5]), 3.0)[0] == np.float32(2.0)
    # within a few fp32 ulps of the exact value
    g = 4.0
    exact = vu.astype(np.float64) + g * (vc.astype(np.float64) - vu.astype(np.float64))
    assert np.allclose(O.cfg_combine(vc, vu, g), exact, rtol=0, atol=4e-6 * (1 + np.abs(exact)).max())


def test_w8_call_count_golden():
    g = json.load(open(os.path.join(GOLDEN, "w8_call_count.json")))
    blocks = range(g["first_block"], g["last_block"] + 1)
    assert len(blocks) * g["modules_per_block"] == g["modules"]
    assert g["modules"] * g["steps"] == g["calls_per_request"]


# ---------------------------------------------------------------- block


def _tiny_weights(H, F_, d, seed):
    r = np.random.default_rng(seed)
    w = {}
    for name, (n, k) in {"qkv": (3 * H, H), "out": (H, H), "up": (F_, H), "down": (H, F_)}.items():
        w[name] = (r.standard_normal((n, k)) * 0.05).astype(F32)
        w[name + "_b"] = O.bf16_round(r.standard_normal(n) * 0.05)
    w["norm_q"] = O.bf16_round(1 + 0.1 * r.standard_normal(d))
    w["norm_k"] = O.bf16_round(1 + 0.1 * r.standard_normal(d))
    return w


def _torch_block(x, w, mod, row_set, groups_ids, pos, heads, d, eps):
    """Independent float64 formulation of the block without quantization:
    torch layer_norm, Linear, complex-number RoPE, SDPA with a boolean mask."""
    X = torch.from_numpy(x)
    m = torch.from_numpy(mod.astype(np.float64))[torch.from_numpy(row_set)]
    sh1, sc1, g1, sh2, sc2, g2 = m.unbind(1)
    lin = lambda a, n: a @ torch.from_numpy(w[n].astype(np.float64)).T + torch.from_numpy(w[n + "_b"].astype(np.float64))
    T, H = X.shape
    u1 = F.layer_norm(X, (H,), eps=eps) * (1 + sc1) + sh1
    qkv = lin(u1, "qkv")
    q, k, v = qkv.split(H, dim=1)

    def rms(a, wn):
        a = a.reshape(T, heads, d)
        return a * torch.rsqrt(a.pow(2).mean(-1, keepdim=True) + eps) * torch.from_numpy(w[wn].astype(np.float64))

    q = torch.from_numpy(_rope_complex(rms(q, "norm_q").numpy(), pos))
    k = torch.from_numpy(_rope_complex(rms(k, "norm_k").numpy(), pos))
    gid = torch.from_numpy(groups_ids)
    mask = gid[None, :] <= gid[:, None]
    o = F.scaled_dot_product_attention(q.permute(1, 0, 2), k.permute(1, 0, 2),
                                       v.reshape(T, heads, d).permute(1, 0, 2), attn_mask=mask)
    o = o.permute(1, 0, 2).reshape(T, H)
    X = X + g1 * lin(o, "out")
    u2 = F.layer_norm(X, (H,), eps=eps) * (1 + sc2) + sh2
    X = X + g2 * lin(F.gelu(lin(u2, "up"), approximate="tanh"), "down")
    return X.numpy()


@pytest.mark.parametrize("sizes", [[1], [4, 8], [3, 5, 6]])
def test_block_vs_unquantized_torch_formulation(sizes):
    H, F_, heads, d, eps = 256, 512, 2, 128, 1e-6
    w = _tiny_weights(H, F_, d, 7)
    pw = O.prepare_block(w)
    S = sum(sizes)
    ends = list(np.cumsum(sizes))
    gid = O.group_ids(ends)
    row_set = np.where(gid < len(sizes) - 1, 0, 1)
    groups = [("text", sizes[0], None)] + [("image", n, (1, n)) for n in sizes[1:]]
    pos = O.rope_positions(groups)
    c, s = O.rope_tables(pos)
    r = np.random.default_rng(3)
    x = r.standard_normal((S, H))
    mod = O.bf16_round(r.standard_normal((2, 6, H)) * 0.5)
    out = O.dit_block(x, pw, mod, row_set, gid, gid, c, s, heads, d, eps)
    ref = _torch_block(x, w, mod, row_set, gid, pos, heads, d, eps)
    delta_rel = np.linalg.norm((out - x) - (ref - x)) / np.linalg.norm(ref - x)
    assert delta_rel < 0.03, delta_rel
    # a swapped modulation row or a dropped gate changes the delta by O(1)
    mod_sw = mod.copy()
    mod_sw[:, [0, 3]] = mod[:, [3, 0]]
    bad = O.dit_block(x, pw, mod_sw, row_set, gid, gid, c, s, heads, d, eps)
    assert np.linalg.norm((bad - x) - (ref - x)) / np.linalg.norm(ref - x) > 0.1


def test_bf16_linear_exact_sum_brute_force():
    """BF16 Linear: bf16 input and weight, the exact sum of the products (here
    with Python fractions), the bias, one rounding to bf16."""
    from fractions import Fraction
    r = np.random.default_rng(21)
    x = r.standard_normal((3, 24)) * 3
    w = r.standard_normal((5, 24)) * 0.1
    b = O.bf16_round(r.standard_normal(5) * 0.1)
    y = O.bf16_linear(x, w, b)
    xb, wb = O.bf16_round(x), O.bf16_round(w)
    for i in range(3):
        for j in range(5):
            exact = sum(Fraction(float(xb[i, k])) * Fraction(float(wb[j, k])) for k in range(24))
            exact += Fraction(float(b[j]))
            assert y[i, j] == O.bf16_round(np.array([float(exact)]))[0]
    # identity weight, no bias: the bf16-rounded input itself
    assert np.array_equal(O.bf16_linear(x[:, :5], np.eye(5)), O.bf16_round(x[:, :5]))


def test_prepare_block_precision_split_and_bf16_block():
    """Mixed precision (the pages' layout): the q, k rows keep exactly the
    codes of the all-W8A8 projection (per-row quantization), the v rows and
    the BF16 Linears are bf16 weights; a block with every Linear in BF16 is
    much closer to the unquantized formulation than the W8A8 block, and the
    W8A8 q, k / BF16 v block sits in between."""
    H, F_, heads, d, eps = 256, 512, 2, 128, 1e-6
    w = _tiny_weights(H, F_, d, 7)
    full = O.prepare_block(w)
    mixed = O.prepare_block(w, {"v": "bf16", "out": "bf16"})
    (q8, s8, rs8, b8), c0 = full["qkv"][0]
    (qk, sk, rsk, bk), c1 = mixed["qkv"][0]
    assert c0 == c1 == 0 and np.array_equal(qk, q8[:2 * H]) and np.array_equal(sk, s8[:2 * H])
    (tag, wv, bv), cv = mixed["qkv"][1]
    assert tag == "bf16" and cv == 2 * H and np.array_equal(wv, O.bf16_round(w["qkv"][2 * H:]))
    assert mixed["out"][0] == "bf16" and not isinstance(mixed["up"][0], str)
    allbf = O.prepare_block(w, {k: "bf16" for k in O.PRECISION_W8A8})
    sizes = [4, 8]
    S = sum(sizes)
    gid = O.group_ids(list(np.cumsum(sizes)))
    row_set = np.where(gid < 1, 0, 1)
    groups = [("text", 4, None), ("image", 8, (1, 8))]
    pos = O.rope_positions(groups)
    c, sn = O.rope_tables(pos)
    r = np.random.default_rng(3)
    x = r.standard_normal((S, H))
    mod = O.bf16_round(r.standard_normal((2, 6, H)) * 0.5)
    ref = _torch_block(x, w, mod, row_set, gid, pos, heads, d, eps)
    err = {}
    for name, pw in (("w8", full), ("mixed", mixed), ("bf16", allbf)):
        out = O.dit_block(x, pw, mod, row_set, gid, gid, c, sn, heads, d, eps)
        err[name] = np.linalg.norm((out - x) - (ref - x)) / np.linalg.norm(ref - x)
    assert err["bf16"] < 0.01 and err["bf16"] < err["mixed"] < err["w8"] < 0.03, err


def test_block_zero_gates_is_identity():
    H, F_, heads, d = 256, 512, 2, 128
    pw = O.prepare_block(_tiny_weights(H, F_, d, 9))
    x = rng.standard_normal((6, H))
    mod = O.bf16_round(rng.standard_normal((2, 6, H)))
    mod[:, 2] = 0
    mod[:, 5] = 0
    gid = O.group_ids([2, 6])
    c, s = O.rope_tables(np.zeros((6, 3), np.int64))
    out = O.dit_block(x, pw, mod, np.array([0, 0, 1, 1, 1, 1]), gid, gid, c, s, heads, d, 1e-6)
    assert np.array_equal(out, x)


# ------------------------------------------------------------------ step


def _tiny_model(H, P, seed):
    r = np.random.default_rng(seed)
    b = lambda n: O.bf16_round(r.standard_normal(n) * 0.02)
    wt = lambda n, k: O.bf16_round(r.standard_normal((n, k)) * 0.05)
    return {"t1": wt(H, 256), "t1_b": b(H), "t2": wt(H, H), "t2_b": b(H),
            "img_in": wt(H, P), "img_in_b": b(H), "txt_in": wt(H, H), "txt_in_b": b(H),
            "final_mod": wt(2 * H, H), "final_mod_b": b(2 * H),
            "proj_out": wt(P, H), "proj_out_b": b(P)}


def test_adaln_rows_chunk_order():
    """Zero weights and a bias equal to the chunk index: the six rows come out
    as (shift1, scale1, gate1, shift2, scale2, gate2) = 0, 1, ..., 5 in that
    order; an interleaved reshape would mix them."""
    H = 8
    b = np.repeat(np.arange(6.0), H)
    rows = O.adaln_rows(rng.standard_normal(H), np.zeros((6 * H, H)), b)
    assert rows.shape == (6, H)
    for i in range(6):
        assert np.array_equal(rows[i], np.full(H, float(i)))


def test_adaln_rows_linear_part_closed_form():
    """Chunk i of W_mod = (i + 1) I: row i = (i + 1) SiLU(temb), SiLU written
    out with math.exp element by element."""
    H = 6
    t = rng.standard_normal(H) * 2
    w = np.concatenate([(i + 1) * np.eye(H) for i in range(6)])
    rows = O.adaln_rows(t, w, np.zeros(6 * H))
    silu = np.array([x / (1.0 + math.exp(-x)) for x in t])
    for i in range(6):
        assert np.allclose(rows[i], (i + 1) * silu, rtol=1e-14, atol=0)


def test_joint_inputs_routing():
    """Text rows go through the text in-projection, reference and target
    latent rows through the image in-projection, in the groups' order; in
    the cached mode only the target rows are formed (torch float64 Linears)."""
    H, P = 256, 64
    mw = _tiny_model(H, P, 12)
    groups = [("text", 3, None), ("image", 4, (2, 2)), ("image", 6, (2, 3))]
    r = np.random.default_rng(13)
    lat = r.standard_normal((6, P)).astype(F32)
    ref = r.standard_normal((4, P)).astype(F32)
    txt = O.bf16_round(r.standard_normal((3, H)))
    T = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    want_t = F.linear(T(txt), T(mw["txt_in"]), T(mw["txt_in_b"])).numpy()
    want_r = F.linear(T(ref), T(mw["img_in"]), T(mw["img_in_b"])).numpy()
    want_l = F.linear(T(lat), T(mw["img_in"]), T(mw["img_in_b"])).numpy()
    x, rows = O.joint_inputs(lat, txt, ref, mw, groups, "none")
    assert np.array_equal(rows, np.arange(13))
    assert np.allclose(x[:3], want_t, rtol=1e-12, atol=1e-12)
    assert np.allclose(x[3:7], want_r, rtol=1e-12, atol=1e-12)
    assert np.allclose(x[7:], want_l, rtol=1e-12, atol=1e-12)
    # the two in-projections differ, so a swapped route fails the checks above
    assert not np.allclose(F.linear(T(ref), T(mw["txt_in"][:, :P]), T(mw["txt_in_b"])).numpy(), want_r)
    xr, rows_r = O.joint_inputs(lat, None, None, mw, groups, "read")
    assert np.array_equal(rows_r, np.arange(7, 13)) and np.allclose(xr, want_l, rtol=1e-12, atol=1e-12)


def test_step_text_reaches_v_only_through_blocks():
    """With identity blocks (zero gates) v does not depend on the text rows;
    with one real block it does (the target attends to the text group)."""
    H, P, heads, d, eps = 256, 64, 2, 128, 1e-6
    mw = _tiny_model(H, P, 14)
    groups = [("text", 4, None), ("image", 6, (2, 3))]
    r = np.random.default_rng(15)
    lat = r.standard_normal((6, P)).astype(F32)
    txt_a = O.bf16_round(r.standard_normal((4, H)))
    txt_b = O.bf16_round(r.standard_normal((4, H)))
    pw = [O.prepare_block(_tiny_weights(H, 512, d, 3))]
    zero_mod = (np.zeros((6 * H, H)), np.zeros(6 * H))
    live_mod = (O.bf16_round(r.standard_normal((6 * H, H)) * 0.02), O.bf16_round(r.standard_normal(6 * H) * 0.3))
    run = lambda txt, mod: O.step_forward(lat, txt, None, mw, pw, [mod], groups, heads, d, eps,
                                          0.8, 0.75, return_v=True)[1]
    assert np.array_equal(run(txt_a, zero_mod), run(txt_b, zero_mod))
    assert not np.allclose(run(txt_a, live_mod), run(txt_b, live_mod))


def test_step_with_identity_blocks_closed_form():
    H, P, heads, d, eps = 256, 64, 2, 128, 1e-6
    mw = _tiny_model(H, P, 5)
    groups = [("text", 4, None), ("image", 6, (2, 3))]
    r = np.random.default_rng(8)
    lat = r.standard_normal((6, P)).astype(F32)
    txt = O.bf16_round(r.standard_normal((4, H)))
    pw = [O.prepare_block(_tiny_weights(H, 512, d, 1))]
    zero_mod = (np.zeros((6 * H, H)), np.zeros(6 * H))            # gates = 0: identity block
    sig, sig2 = 0.8, 0.75
    new, v = O.step_forward(lat, txt, None, mw, pw, [zero_mod], groups, heads, d, eps,
                            sig, sig2, return_v=True)
    # closed form with torch: v = proj(LN(img_in(lat))(1 + scale) + shift)
    T = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    e = T(O.timestep_embedding(sig))
    temb = F.linear(F.silu(F.linear(e, T(mw["t1"]), T(mw["t1_b"]))), T(mw["t2"]), T(mw["t2_b"]))
    shift, scale = F.linear(F.silu(temb), T(mw["final_mod"]), T(mw["final_mod_b"])).chunk(2)
    xi = F.linear(T(lat), T(mw["img_in"]), T(mw["img_in_b"]))
    ref_v = F.linear(F.layer_norm(xi, (H,), eps=eps) * (1 + scale) + shift, T(mw["proj_out"]), T(mw["proj_out_b"]))
    assert np.allclose(v, ref_v.numpy(), rtol=1e-5, atol=1e-5)
    assert np.allclose(new, lat + (F32(sig2) - F32(sig)) * v, atol=1e-6)


def test_step_cached_equals_uncached():
    H, P, heads, d, eps = 256, 64, 2, 128, 1e-6
    mw = _tiny_model(H, P, 6)
    groups = [("text", 4, None), ("image", 4, (2, 2)), ("image", 6, (2, 3))]
    r = np.random.default_rng(9)
    lat = r.standard_normal((6, P)).astype(F32)
    ref = r.standard_normal((4, P)).astype(F32)
    txt = O.bf16_round(r.standard_normal((4, H)))
    nb = 2
    pw = [O.prepare_block(_tiny_weights(H, 512, d, 10 + i)) for i in range(nb)]
    mods = [(O.bf16_round(r.standard_normal((6 * H, H)) * 0.02), O.bf16_round(r.standard_normal(6 * H) * 0.1))
            for _ in range(nb)]
    cache = {}
    a1 = O.step_forward(lat, txt, ref, mw, pw, mods, groups, heads, d, eps, 1.0, 0.9, kv_cache=cache, mode="write")
    a2 = O.step_forward(a1, txt, ref, mw, pw, mods, groups, heads, d, eps, 0.9, 0.8)
    b2 = O.step_forward(a1, None, None, mw, pw, mods, groups, heads, d, eps, 0.9, 0.8, kv_cache=cache, mode="read")
    assert len(cache) == nb and cache[0][0].shape == (8, heads, d)
    assert np.allclose(a2, b2, rtol=0, atol=1e-6)
