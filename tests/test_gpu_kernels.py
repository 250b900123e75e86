"""Per-kernel parity of the CUDA path against the CPU oracle, through the C ABI.

Integer and byte results (weight codes, activation codes/scales/zero points,
int32 accumulators, the Q/K norm ordering on exactly summable inputs, the
Euler update) must match bit for bit.  Floating-point results are compared
within a tolerance derived from the arithmetic (stated per test).
"""
import math

import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, rel_l2

pytestmark = pytest.mark.gpu
BF16_ULP = 2.0 ** -7   # relative spacing of bf16 at the top of a binade


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _bf16(shape, seed, scale=1.0):
    return (torch.randn(*shape, generator=_gen(seed)) * scale).to(torch.bfloat16)


# ------------------------------------------------------------------ weight prep

@pytest.mark.parametrize("n,k", [(48, 256), (768, 256), (4096, 4096), (64, 16384)])
def test_prepare_w8_bit_exact(ctx, n, k):
    w = synth.linear_weight(3, ("prep", n, k), n, k)
    w[1] = 0.0
    q, s, rs = qi.qi_prepare_w8(ctx, cuda(w))
    oq, os_, ors = O.prepare_w8(w.numpy())
    assert np.array_equal(q.cpu().numpy(), oq)
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(rs.cpu().numpy(), ors)


# ------------------------------------------------------------------ activation quant

@pytest.mark.parametrize("M,K", [(1, 256), (80, 256), (5, 1032), (77, 4096), (1280, 4096), (33, 16384)])
def test_quantize_plain_bit_exact(ctx, M, K):
    x = _bf16((M, K), M * 7 + K, 1.0) * torch.logspace(-3, 2, M).reshape(M, 1).to(torch.bfloat16)
    x = x.to(torch.bfloat16)
    if M > 3:
        x[0] = 0
        x[1] = x[1].abs()
        x[2] = -x[2].abs()
        x[3] = 0.5
    q, s, zp = qi.qi_quantize_act(ctx, cuda(x))
    oq, os_, ozp = O.quantize_act(bf16_np(x))
    assert np.array_equal(s.cpu().numpy(), os_)
    assert np.array_equal(zp.cpu().numpy(), ozp)
    assert np.array_equal(q.cpu().numpy(), oq)


@pytest.mark.parametrize("K", [4096, 1000, 16384])   # 16384 fp32: the largest staged row (64 KB)
def test_quantize_fp32_input_bit_exact(ctx, K):
    x = torch.randn(300, K, generator=_gen(5)) * 3 + 0.7
    q, s, zp = qi.qi_quantize_act(ctx, cuda(x))
    oq, os_, ozp = O.quantize_act(x.numpy())
    assert np.array_equal(s.cpu().numpy(), os_) and np.array_equal(zp.cpu().numpy(), ozp)
    assert np.array_equal(q.cpu().numpy(), oq)


def test_empty_inputs_are_noops(ctx):
    """Zero rows: quantization and attention return OK and write nothing (a
    zero-element tensor hands the library a NULL pointer, which is allowed
    for a call on zero rows)."""
    x = cuda(_bf16((4, 256), 3, 1.0))
    q = torch.full((4, 256), 7, dtype=torch.int8, device="cuda")
    s = torch.full((4,), 2.0, device="cuda")
    zp = torch.full((4,), 5, dtype=torch.int32, device="cuda")
    qi.qi_quantize_act(ctx, x[:0], out=(q[:0], s[:0], zp[:0]))
    y = torch.full((4, 64), 3.0, dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((64, 256), dtype=torch.int8, device="cuda")
    w = qi.w8_struct(wq, torch.ones(64, device="cuda"), torch.zeros(64, dtype=torch.int32, device="cuda"))
    qi.qi_w8a8_linear(ctx, q[:0], s[:0], zp[:0], w, y=y[:0])
    H, S = 256, 40
    qkv = cuda(_bf16((3, S, H), 4, 1.0))
    o = torch.full((S, H), 1.5, dtype=torch.bfloat16, device="cuda")
    g = qi.groups_struct([8, S], [0, 1])
    qi.qi_attn_block_causal(ctx, qkv[0][:0], qkv[1], qkv[2], g, q_offset=S, o=o[:0])
    torch.cuda.synchronize()
    ctx.check()
    assert bool((q == 7).all()) and bool((s == 2.0).all()) and bool((zp == 5).all())
    assert bool((o == 1.5).all()) and bool((y == 3.0).all())


def test_empty_inputs_still_validate_their_other_arguments(ctx):
    """A zero-row call is rejected for the same bad weight, dtype, shape,
    epilogue or group table as a call with rows: only its row pointers may be
    NULL."""
    L = qi.lib()
    h = ctx.handle
    st = qi.stream_ptr()
    # quantizer: bad dtype, bad K
    assert L.qi_quantize_act(h, None, 7, 0, 256, 256, None, None, 0, None, 0, 1e-6, None, None,
                             None, st) == qi.QI_ERR_INVALID_ARG
    assert L.qi_quantize_act(h, None, qi.QI_BF16, 0, 100, 100, None, None, 0, None, 0, 1e-6,
                             None, None, None, st) == qi.QI_ERR_UNSUPPORTED_SHAPE
    # W8A8 Linear: NULL weight codes, bad K, bad epilogue kind
    bad_w = qi.qi_w8()
    assert L.qi_w8a8_linear(h, None, None, None, 0, qi.C.byref(bad_w), None, None, 0, None,
                            st) == qi.QI_ERR_INVALID_ARG
    q = torch.zeros((64, 100), dtype=torch.int8, device="cuda")
    s = torch.ones(64, device="cuda")
    rs = torch.zeros(64, dtype=torch.int32, device="cuda")
    w = qi.w8_struct(q, s, rs)
    assert L.qi_w8a8_linear(h, None, None, None, 0, qi.C.byref(w), None, None, 64, None,
                            st) == qi.QI_ERR_UNSUPPORTED_SHAPE
    q2 = torch.zeros((64, 128), dtype=torch.int8, device="cuda")
    w2 = qi.w8_struct(q2, s, rs)
    ep = qi.qi_epilogue()
    ep.kind = 9
    assert L.qi_w8a8_linear(h, None, None, None, 0, qi.C.byref(w2), qi.C.byref(ep), None, 64,
                            None, st) == qi.QI_ERR_INVALID_ARG
    # ... while the same zero-row call with good arguments is a no-op
    assert L.qi_w8a8_linear(h, None, None, None, 0, qi.C.byref(w2), None, None, 64, None,
                            st) == qi.QI_OK
    # BF16 Linear: k not a multiple of 64
    wb = torch.zeros((64, 96), dtype=torch.bfloat16, device="cuda")
    assert L.qi_bf16_linear(h, None, 0, 96, qi.C.byref(qi.bf16_struct(wb)), None, 64,
                            st) == qi.QI_ERR_UNSUPPORTED_SHAPE
    # attention: head_dim 64, and a group table that does not end at Sk
    g = qi.groups_struct([8, 40], [0, 1])
    assert L.qi_attn_block_causal(h, None, 256, 0, 40, None, None, 256, 40, 2, 64,
                                  qi.C.byref(g), 0.1, None, 256, st) == qi.QI_ERR_UNSUPPORTED_SHAPE
    g_bad = qi.groups_struct([8, 30], [0, 1])
    assert L.qi_attn_block_causal(h, None, 256, 0, 40, None, None, 256, 40, 2, 128,
                                  qi.C.byref(g_bad), 0.1, None, 256, st) == qi.QI_ERR_INVALID_ARG
    ctx.check()


@pytest.mark.parametrize("H,L,N", [(256, 16, 64), (4096, 256, 1024)])
def test_quantize_ln_modulate(ctx, H, L, N):
    cfg = synth.TINY.replace(hidden=H)
    x = synth.hidden_states(cfg, L + N)
    mod = synth.mod_table(cfg)
    g = qi.groups_struct([L, L + N], [0, 1])
    mod_g = cuda(mod)   # [2, 6, H]: row set r's shift at r*6H, scale at r*6H + H
    q, s, zp = qi.qi_quantize_act(ctx, cuda(x), shift=mod_g[0, 0], scale=mod_g[0, 1],
                                  mod_ld=6 * H, groups=g, row0=0, eps=1e-6)
    m = bf16_np(mod)
    rs = np.array([0] * L + [1] * N)
    u = O.modulate(O.layer_norm(x.numpy(), 1e-6), m[rs, 0], m[rs, 1])
    oq, os_, ozp = O.quantize_act(u)
    q, s, zp = q.cpu().numpy(), s.cpu().numpy(), zp.cpu().numpy()
    # LayerNorm in fp32 vs float64: scales agree to fp32 rounding, codes to +-1
    assert np.all(np.abs(s - os_) <= 1e-5 * os_)
    assert np.mean(zp == ozp) > 0.95 and np.all(np.abs(zp - ozp) <= 1)
    deq = s[:, None] * (q.astype(np.float64) - zp[:, None])
    odeq = os_[:, None] * (oq.astype(np.float64) - ozp[:, None])
    assert np.all(np.abs(deq - odeq) <= 1.01 * np.maximum(s, os_)[:, None])
    same = zp == ozp
    assert np.mean(q[same] == oq[same]) > 0.999


# ------------------------------------------------------------------ W8A8 GEMM

def _w8_pair(ctx, n, k, seed):
    w = synth.linear_weight(seed, ("gemm", n, k), n, k)
    b = synth.bias(seed, ("gemm", n), n)
    q, s, rs = qi.qi_prepare_w8(ctx, cuda(w))
    ow = O.prepare_w8(w.numpy())
    return qi.w8_struct(q, s, rs, cuda(b)), (q, s, rs, cuda(b)), ow, bf16_np(b)


def _acts(M, K, seed):
    x = torch.randn(M, K, generator=_gen(seed)) + 0.25
    return x, O.quantize_act(x.numpy())


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (80, 768, 256), (200, 1024, 4096),
                                   (1280, 4096, 4096), (300, 4096, 16384), (130, 64 * 3, 128)])
def test_w8a8_accumulators_bit_exact_and_output(ctx, M, N, K):
    ws, keep, (oq, os_, ors), ob = _w8_pair(ctx, N, K, 11)
    x, (qa, sa, zpa) = _acts(M, K, M + N)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qi.qi_w8a8_linear(ctx, cuda(torch.from_numpy(qa)), cuda(torch.from_numpy(sa)),
                      cuda(torch.from_numpy(zpa)), ws, y=y, acc_debug=acc)
    oacc, oy = O.w8a8_linear(qa, sa, zpa, oq, os_, ors, ob)
    assert np.array_equal(acc.cpu().numpy().astype(np.int64), oacc)
    gy = bf16_np(y)
    # one fp32 evaluation of (acc - zp rowsum) s_a s_w + b vs float64, each rounded to bf16
    assert np.all(np.abs(gy - oy) <= BF16_ULP * np.abs(oy) + 2.0 ** -20 * np.abs(oy).max())


def test_w8a8_full_size_sampled_rows(ctx):
    # QKV projection of the 1024x1024 step: M = 4608, N = 3*4096, K = 4096
    M, N, K = 4608, 12288, 4096
    ws, keep, (oq, os_, ors), ob = _w8_pair(ctx, N, K, 12)
    qa = torch.randint(-128, 128, (M, K), generator=_gen(1), dtype=torch.int8)
    sa = torch.rand(M, generator=_gen(2)) * 0.05 + 1e-3
    zpa = torch.randint(-128, 128, (M,), generator=_gen(3), dtype=torch.int32)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qi.qi_w8a8_linear(ctx, cuda(qa), cuda(sa), cuda(zpa), ws, y=y, acc_debug=acc)
    rows = np.concatenate([np.random.default_rng(0).choice(M, 24, replace=False), [0, M - 1]])
    oacc, oy = O.w8a8_linear(qa.numpy()[rows], sa.numpy()[rows], zpa.numpy()[rows], oq, os_, ors, ob)
    assert np.array_equal(acc.cpu().numpy()[rows].astype(np.int64), oacc)
    gy = bf16_np(y)[rows]
    assert np.all(np.abs(gy - oy) <= BF16_ULP * np.abs(oy) + 2.0 ** -20 * np.abs(oy).max())


def test_w8a8_gelu_epilogue(ctx):
    M, N, K = 96, 1024, 256
    ws, keep, (oq, os_, ors), ob = _w8_pair(ctx, N, K, 13)
    x, (qa, sa, zpa) = _acts(M, K, 5)
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ep = qi.qi_epilogue()
    ep.kind = qi.QI_EPI_GELU_TANH
    qi.qi_w8a8_linear(ctx, cuda(torch.from_numpy(qa)), cuda(torch.from_numpy(sa)),
                      cuda(torch.from_numpy(zpa)), ws, epilogue=ep, y=y)
    _, oy = O.w8a8_linear(qa, sa, zpa, oq, os_, ors, ob)
    og = O.bf16_round(O.gelu_tanh(oy))
    # the Linear output may differ by 1 bf16 ulp; GELU' <= 1.13 and one more rounding
    assert np.all(np.abs(bf16_np(y) - og) <= 3 * BF16_ULP * np.abs(og) + 1e-6)


def test_w8a8_gated_residual_epilogue(ctx):
    H, L, N, K = 256, 16, 64, 256
    M = L + N
    ws, keep, (oq, os_, ors), ob = _w8_pair(ctx, H, K, 14)
    x, (qa, sa, zpa) = _acts(M, K, 6)
    res = torch.randn(M, H, generator=_gen(7))
    mod = synth.mod_table(synth.TINY)
    g = qi.groups_struct([L, M], [0, 1])
    r_gpu = cuda(res)
    ep = qi.qi_epilogue()
    ep.kind = qi.QI_EPI_GATED_RESIDUAL
    ep.residual = r_gpu.data_ptr()
    ep.ld_residual = H
    gate = cuda(mod[:, 2].contiguous())
    ep.gate = gate.data_ptr()
    ep.gate_ld = H
    ep.groups = torch_groups = None
    import ctypes as C
    ep.groups = C.pointer(g)
    ep.row0 = 0
    qi.qi_w8a8_linear(ctx, cuda(torch.from_numpy(qa)), cuda(torch.from_numpy(sa)),
                      cuda(torch.from_numpy(zpa)), ws, epilogue=ep)
    _, oy = O.w8a8_linear(qa, sa, zpa, oq, os_, ors, ob)
    gate_np = bf16_np(mod[:, 2])[np.array([0] * L + [1] * N)]
    ref = res.numpy().astype(np.float64) + gate_np * oy
    got = r_gpu.cpu().numpy()
    assert np.all(np.abs(got - ref) <= BF16_ULP * np.abs(gate_np * oy) + 1e-6 * np.abs(ref) + 1e-7)


# ------------------------------------------------------------------ BF16 GEMM

@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (80, 4096, 64), (4096, 64, 4096), (300, 4096, 4096)])
def test_bf16_linear(ctx, M, N, K):
    a = _bf16((M, K), 21 + M)
    w = _bf16((N, K), 22 + N, 0.05)
    b = _bf16((N,), 23, 0.05)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    qi.qi_bf16_linear(ctx, cuda(a), qi.bf16_struct(cuda(w), cuda(b)), y)
    A, W, B = bf16_np(a).astype(np.float64), bf16_np(w).astype(np.float64), bf16_np(b)
    ref = A @ W.T + B
    bound = 1e-5 * (np.abs(A) @ np.abs(W).T) + 1e-6
    assert np.all(np.abs(y.cpu().numpy() - ref) <= bound)


# ------------------------------------------------------------------ Q/K norm + RoPE

def _norm_rope_case(T, heads, seed, exact):
    H = heads * 128
    if exact:
        # values k/8, |k| <= 8: squares and their sums are exact in fp32 in any order
        qkv = (torch.randint(-8, 9, (T, 3 * H), generator=_gen(seed)).float() / 8).to(torch.bfloat16)
    else:
        qkv = _bf16((T, 3 * H), seed, 2.0)
    wq = synth.norm_weight(1, "q", 128)
    wk = synth.norm_weight(1, "k", 128)
    groups = [("text", 3, None), ("image", T - 3, (1, T - 3))]
    cos, sin = O.rope_tables(O.rope_positions(groups))
    return qkv, wq, wk, torch.from_numpy(cos), torch.from_numpy(sin)


@pytest.mark.parametrize("exact", [True, False])
def test_qk_norm_rope(ctx, exact):
    T, heads = 67, 4
    H = heads * 128
    qkv, wq, wk, cos, sin = _norm_rope_case(T, heads, 31, exact)
    q = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    k = torch.empty_like(q)
    v = torch.empty_like(q)
    qi.qi_qk_norm_rope(ctx, cuda(qkv), heads, cuda(wq), cuda(wk), cuda(cos), cuda(sin), 1e-6, q, k, v)
    x = bf16_np(qkv)
    oq = O.rope_apply(O.rms_norm_cast(x[:, :H].reshape(T, heads, 128), bf16_np(wq), 1e-6), cos.numpy(), sin.numpy())
    ok = O.rope_apply(O.rms_norm_cast(x[:, H:2 * H].reshape(T, heads, 128), bf16_np(wk), 1e-6), cos.numpy(), sin.numpy())
    gq, gk = bf16_np(q).reshape(T, heads, 128), bf16_np(k).reshape(T, heads, 128)
    assert np.array_equal(bf16_np(v), x[:, 2 * H:])
    if exact:
        assert np.array_equal(gq, oq) and np.array_equal(gk, ok)
    else:
        # sums of squares in another order: at most one bf16 step apart, rarely
        for g, o in ((gq, oq), (gk, ok)):
            assert np.all(np.abs(g - o) <= 2 * BF16_ULP * np.abs(o) + 1e-6)
            assert np.mean(g == o) > 0.98


def test_qk_norm_cast_ordering_example(ctx):
    # "Qwen Image 2.1 native qualification": cast to bf16 before the scale.
    qkv = torch.zeros((1, 3 * 128), dtype=torch.bfloat16)
    qkv[0, :64] = 1.0
    qkv[0, 64:128] = 0.25
    w = torch.full((128,), 1.015625, dtype=torch.bfloat16)
    cos = torch.ones((1, 64))
    sin = torch.zeros((1, 64))
    q = torch.empty((1, 128), dtype=torch.bfloat16, device="cuda")
    k, v = torch.empty_like(q), torch.empty_like(q)
    qi.qi_qk_norm_rope(ctx, cuda(qkv), 1, cuda(w), cuda(w), cuda(cos), cuda(sin), 1e-6, q, k, v)
    g = bf16_np(q)[0]
    assert g[0] == np.float32(1.3984375) and g[127] == np.float32(0.349609375)


# ------------------------------------------------------------------ attention

def _attn_case(sizes, heads, seed):
    S = sum(sizes)
    q = _bf16((S, heads * 128), seed, 1.0)
    k = _bf16((S, heads * 128), seed + 1, 1.0)
    v = _bf16((S, heads * 128), seed + 2, 1.0)
    ends = [int(e) for e in np.cumsum(sizes)]
    return q, k, v, ends


def _oracle_attn(q, k, v, ends, heads, q_rows=None):
    S = k.shape[0]
    gid = O.group_ids(ends)
    qn = bf16_np(q).reshape(-1, heads, 128)
    rows = np.arange(S) if q_rows is None else q_rows
    return O.attention_block_causal(qn[rows], bf16_np(k).reshape(S, heads, 128),
                                    bf16_np(v).reshape(S, heads, 128), gid[rows], gid,
                                    1 / math.sqrt(128)).reshape(len(rows), heads * 128)


@pytest.mark.parametrize("sizes,heads", [([16, 64], 2), ([5, 70, 3], 2), ([200], 1),
                                         ([1] * 16, 1), ([256, 1024], 32), ([100, 30, 130], 3)])
def test_attention_vs_oracle(ctx, sizes, heads):
    q, k, v, ends = _attn_case(sizes, heads, 41 + len(sizes))
    g = qi.groups_struct(ends, [0] * len(ends))
    o = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k), cuda(v), g)
    ref = _oracle_attn(q, k, v, ends, heads)
    got = bf16_np(o)
    # P is rounded to bf16 before P V and O to bf16: ~2^-8 relative per term
    assert rel_l2(got, ref) < 4e-3
    assert np.abs(got - ref).max() < 2e-2


def test_attention_cached_rows_bit_identical_and_mask_invariance(ctx):
    sizes = [256, 1024, 4096 // 4]
    heads = 4
    q, k, v, ends = _attn_case(sizes, heads, 77)
    g = qi.groups_struct(ends, [0, 0, 1])
    full = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k), cuda(v), g)
    P = ends[-2]
    part = qi.qi_attn_block_causal(ctx, cuda(q[P:].contiguous()), cuda(k), cuda(v), g, q_offset=P)
    assert torch.equal(full[P:], part)
    # later groups never influence earlier ones
    k2, v2 = k.clone(), v.clone()
    k2[ends[0]:] = 3.0
    v2[ends[0]:] = -2.0
    o2 = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k2), cuda(v2), g)
    assert torch.equal(o2[:ends[0]], full[:ends[0]])
    ref = _oracle_attn(q, k, v, ends, heads, q_rows=np.arange(P, ends[-1], 7))
    assert rel_l2(bf16_np(full)[P::7], ref) < 4e-3


def _num_sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def test_attention_key_split_vs_oracle_and_cached_rows(ctx):
    """Every head's longest-range query tiles split over the key range and
    combined (4 heads x 17 tiles leave most SMs idle).  The first tile holds
    rows of all three groups; those of the first two see no key of the upper
    half (a zero-weight half in the combine).  Sampled rows against the
    oracle; the cached-prefix call (the prefix not a multiple of the tile)
    computes the target rows bit for bit as the uncached call does."""
    sizes, heads = [100, 30, 4000], 4
    q, k, v, ends = _attn_case(sizes, heads, 123)
    S = ends[-1]
    g = qi.groups_struct(ends, [0, 0, 1])
    ks, need = qi.qi_attn_split_plan(S, heads, g, _num_sms())
    assert ks == heads
    qi.qi_ctx_reserve_attention(ctx, need)
    full = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k), cuda(v), g)
    ctx.check()
    P = ends[-2]
    part = qi.qi_attn_block_causal(ctx, cuda(q[P:].contiguous()), cuda(k), cuda(v), g, q_offset=P)
    ctx.check()
    assert torch.equal(full[P:], part)
    rows = np.concatenate([np.arange(256), np.arange(256, S, 13)])
    ref = _oracle_attn(q, k, v, ends, heads, q_rows=rows)
    got = bf16_np(full)[rows]
    assert rel_l2(got, ref) < 4e-3
    assert np.abs(got - ref).max() < 2e-2


def test_attention_key_split_full_size_1024px(ctx):
    """The 1024x1024 step's attention ([512 | 4096] tokens, 32 heads): the
    split takes some heads; sampled rows of every head against the oracle,
    and rows of split and unsplit heads alike within the same tolerance."""
    sizes, heads = [512, 4096], 32
    q, k, v, ends = _attn_case(sizes, heads, 5)
    g = qi.groups_struct(ends, [0, 1])
    ks, need = qi.qi_attn_split_plan(ends[-1], heads, g, _num_sms())
    assert 0 < ks < heads
    qi.qi_ctx_reserve_attention(ctx, need)
    o = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k), cuda(v), g)
    ctx.check()
    rows = np.arange(3, ends[-1], 29)
    ref = _oracle_attn(q, k, v, ends, heads, q_rows=rows).reshape(len(rows), heads, 128)
    got = bf16_np(o)[rows].reshape(len(rows), heads, 128)
    for hs in (slice(0, heads - ks), slice(heads - ks, heads)):
        assert rel_l2(got[:, hs], ref[:, hs]) < 4e-3
        assert np.abs(got[:, hs] - ref[:, hs]).max() < 2e-2


# ------------------------------------------------------------------ Euler, conditioning, probe

def test_euler_bit_exact(ctx):
    x = torch.randn(4096 * 64, generator=_gen(9))
    v = torch.randn(4096 * 64, generator=_gen(10))
    sig = O.sigma_schedule(40, 4096)
    xg = cuda(x)
    for i in (0, 17, 38, 39):
        qi.qi_euler_update(ctx, xg, cuda(v), float(sig[i]), float(sig[i + 1]))
        x = torch.from_numpy(O.euler_update(x.numpy(), v.numpy(), sig[i], sig[i + 1]))
    assert torch.equal(xg.cpu(), x)


def test_time_conditioning(ctx):
    cfg = synth.TINY.replace(blocks=3)
    H = cfg.hidden
    glob = synth.model_weights(cfg)
    blocks = [synth.block_weights(cfg, l) for l in range(cfg.blocks)]
    dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    model = qi.Model(ctx, dims, [qi.BlockWeights(ctx, b) for b in blocks], glob)
    ws = torch.empty(qi.qi_step_workspace_bytes(dims, 8), dtype=torch.uint8, device="cuda")
    bm = torch.empty((cfg.blocks, 2, 6 * H), dtype=torch.bfloat16, device="cuda")
    fm = torch.empty((2, 2 * H), dtype=torch.bfloat16, device="cuda")
    sigma = 0.73
    qi.qi_time_conditioning(ctx, model, sigma, bm, fm, ws)
    mw = {k: bf16_np(t) for k, t in glob.items()}
    for r, t in enumerate((0.0, sigma)):
        temb = O.time_embed(t, mw)
        for l, b in enumerate(blocks):
            ref = O.adaln_rows(temb, bf16_np(b["mod"]), bf16_np(b["mod_b"])).reshape(-1)
            assert rel_l2(bf16_np(bm[l, r]), ref) < 5e-3
        if r == 1:
            ref = O.linear(O.silu(temb), mw["final_mod"], mw["final_mod_b"])
            assert rel_l2(bf16_np(fm[1]), ref) < 5e-3


def test_timeout_probe_reports_and_context_survives(ctx):
    qi.qi_debug_timeout_probe(ctx, 20_000_000)   # 20 ms
    with pytest.raises(qi.QiError) as e:
        ctx.check()
    assert e.value.code == qi.QI_ERR_TIMEOUT
    ctx.check()   # cleared; the context is still usable
    x = torch.randn(4, 256, device="cuda")
    qi.qi_quantize_act(ctx, x)
    ctx.check()


def test_attention_growing_scores_rescale_path(ctx):
    # later keys are scaled up so each key tile's row maximum exceeds the
    # previous one by a wide margin: the running-maximum rescale of O is taken,
    # in some lanes of a warp and not in others
    sizes = [128, 640]
    heads = 2
    q, k, v, ends = _attn_case(sizes, heads, 91)
    S = sum(sizes)
    ramp = torch.linspace(0.5, 6.0, S).reshape(S, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    g = qi.groups_struct(ends, [0, 1])
    o = qi.qi_attn_block_causal(ctx, cuda(q), cuda(k), cuda(v), g)
    ctx.check()
    ref = _oracle_attn(q, k, v, ends, heads)
    assert rel_l2(bf16_np(o), ref) < 4e-3


@pytest.mark.parametrize("M,heads", [(80, 2), (300, 4), (4608, 32)])
def test_qkv_fused_epilogue_matches_two_step_path(ctx, M, heads):
    # The fused QKV epilogue (W8A8 GEMM + Q/K RMSNorm + RoPE) against the
    # two-step path (W8A8 GEMM storing bf16, then qi_qk_norm_rope).  v must be
    # identical; q and k may differ only where the sum of squares, accumulated
    # in another order, moves the normalisation by one ulp.
    H = heads * 128
    ws, keep, _, _ = _w8_pair(ctx, 3 * H, H, 17)
    x, (qa, sa, zpa) = _acts(M, H, 23)
    qa_g, sa_g, zp_g = (cuda(torch.from_numpy(a)) for a in (qa, sa, zpa))
    wq = cuda(synth.norm_weight(2, "q", 128))
    wk = cuda(synth.norm_weight(2, "k", 128))
    groups = [("text", 16, None), ("image", M - 16, (1, M - 16))]
    cos, sin = (cuda(t) for t in qi.qi_rope_tables(groups))
    y = torch.empty((M, 3 * H), dtype=torch.bfloat16, device="cuda")
    qi.qi_w8a8_linear(ctx, qa_g, sa_g, zp_g, ws, y=y)
    q2, k2, v2 = (torch.empty((M, H), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    qi.qi_qk_norm_rope(ctx, y, heads, wq, wk, cos, sin, 1e-6, q2, k2, v2)
    q1, k1, v1 = (torch.empty((M, H), dtype=torch.bfloat16, device="cuda") for _ in range(3))
    ep = qi.qi_epilogue()
    ep.kind = qi.QI_EPI_QKV_NORM_ROPE
    ep.hidden, ep.eps, ep.ld_out = H, 1e-6, H
    ep.norm_q, ep.norm_k = wq.data_ptr(), wk.data_ptr()
    ep.rope_cos, ep.rope_sin = cos.data_ptr(), sin.data_ptr()
    ep.q_out, ep.k_out, ep.v_out = q1.data_ptr(), k1.data_ptr(), v1.data_ptr()
    qi.qi_w8a8_linear(ctx, qa_g, sa_g, zp_g, ws, epilogue=ep)
    ctx.check()
    assert torch.equal(v1, v2)
    for a, b in ((q1, q2), (k1, k2)):
        a, b = bf16_np(a), bf16_np(b)
        # a rotated pair whose inputs differ by at most one bf16 step each can
        # differ by up to ~2 steps of the pair's norm (which the rotation keeps),
        # even where the rotated value itself is near zero
        pair_norm = np.sqrt((b.reshape(M, -1, 2) ** 2).sum(-1, keepdims=True))
        bound = 4 * BF16_ULP * np.broadcast_to(pair_norm, (M, H // 2, 2)).reshape(M, H) + 1e-6
        assert np.all(np.abs(a - b) <= bound)
        assert np.mean(a == b) > 0.99
