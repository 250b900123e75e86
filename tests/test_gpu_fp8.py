"""fp8 (e4m3) attention: the cast, the attention kernel against the oracle's
step-by-step emulation of the same method, cached rows, and denoising steps
with fp8 attention against the oracle's fp8 step (cached == uncached)."""
import math

import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, rel_l2

pytestmark = pytest.mark.gpu


def _gen(seed):
    return torch.Generator().manual_seed(seed)


def _decode_e4m3(b: np.ndarray) -> np.ndarray:
    """e4m3 bytes -> values, from the format (1 sign, 4 exponent bits with bias 7, 3 mantissa bits)."""
    b = b.astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e, m = (b >> 3) & 15, b & 7
    return s * np.where(e == 0, m / 8.0 * 2.0 ** -6, (1 + m / 8.0) * np.exp2(e - 7.0))


def test_e4m3_cast_bit_exact(ctx):
    n = 4096 * 16
    g = _gen(3)
    x = torch.randn(n, generator=g) * torch.exp2(torch.randint(-14, 10, (n,), generator=g).float())
    x[:6] = torch.tensor([1000.0, -600.0, 0.0, 2.0 ** -12, 448.0, 464.0])
    x = x.to(torch.bfloat16)
    got = _decode_e4m3(qi.qi_to_e4m3(ctx, cuda(x)).cpu().numpy())
    assert np.array_equal(got, O.e4m3_round(bf16_np(x)))


def _case(sizes, heads, seed):
    S = sum(sizes)
    mk = lambda s: (torch.randn((S, heads * 128), generator=_gen(s))).to(torch.bfloat16)
    return mk(seed), mk(seed + 1), mk(seed + 2), [int(e) for e in np.cumsum(sizes)]


def _run_fp8(ctx, q, k, v, ends, q_offset=0):
    g = qi.groups_struct(ends, [0] * len(ends))
    q8, k8, v8 = (qi.qi_to_e4m3(ctx, cuda(t)) for t in (q, k, v))
    return qi.qi_attn_block_causal_fp8(ctx, q8, k8, v8, g, q_offset=q_offset)


def _oracle(q, k, v, ends, heads, fp8=True, rows=None):
    S = k.shape[0]
    gid = O.group_ids(ends)
    rows = np.arange(S) if rows is None else rows
    qn = bf16_np(q).reshape(-1, heads, 128)[rows]
    kn, vn = (bf16_np(t).reshape(S, heads, 128) for t in (k, v))
    f = {True: O.attention_block_causal_fp8, False: O.attention_block_causal,
         "plain": O.attention_block_causal_fp8_plain}[fp8]
    return f(qn, kn, vn, gid[rows], gid, 1 / math.sqrt(128)).reshape(len(rows), heads * 128)


# RMS relative error of one e4m3 rounding of a value whose mantissa is spread
# uniformly: half a step of 2^-3 relative, i.e. 2^-4 at most, 2^-4 / sqrt(3) RMS
E4M3_RMS = 2.0 ** -4 / math.sqrt(3.0)


@pytest.mark.parametrize("sizes,heads", [([16, 64], 2), ([5, 70, 3], 2), ([200], 1),
                                         ([100, 30, 130], 3), ([256, 640], 2)])
def test_attention_fp8_vs_oracle(ctx, sizes, heads):
    q, k, v, ends = _case(sizes, heads, 61 + len(sizes))
    got = bf16_np(_run_fp8(ctx, q, k, v, ends))
    # the same method in the oracle: differences come from the fp32 score
    # accumulation order, ex2.approx and the final bf16 rounding only
    assert rel_l2(got, _oracle(q, k, v, ends, heads)) < 5e-3
    # and the method itself sits an e4m3-sized step from exact attention
    e_exact = rel_l2(got, _oracle(q, k, v, ends, heads, fp8=False))
    assert e_exact < 8e-2
    # the plain reading (exact row maximum, no tiles): the kernel subtracts a
    # per-tile reference maximum instead, which rescales P before its e4m3
    # rounding, so the two differ by at most the noise of one e4m3 rounding,
    # and the kernel is closer to it than to exact attention
    e_plain = rel_l2(got, _oracle(q, k, v, ends, heads, fp8="plain"))
    assert e_plain < E4M3_RMS and e_plain < e_exact


def test_attention_fp8_cached_rows_bit_identical(ctx):
    sizes, heads = [256, 512, 384], 2
    q, k, v, ends = _case(sizes, heads, 90)
    full = _run_fp8(ctx, q, k, v, ends)
    P = ends[-2]
    part = _run_fp8(ctx, q[P:].contiguous(), k, v, ends, q_offset=P)
    assert torch.equal(full[P:], part)


def test_attention_fp8_key_split(ctx):
    """The key-range split on e4m3 operands (every head split, as in the bf16
    case): target rows of the cached call equal the uncached call's; the
    split halves keep their own reference maxima, so sampled rows are held to
    the plain reading's e4m3 bound, and closer to it than to exact attention."""
    sizes, heads = [100, 30, 4000], 4
    q, k, v, ends = _case(sizes, heads, 17)
    g = qi.groups_struct(ends, [0] * len(ends))
    n_sms = torch.cuda.get_device_properties(0).multi_processor_count
    ks, need = qi.qi_attn_split_plan(ends[-1], heads, g, n_sms)
    assert ks == heads
    qi.qi_ctx_reserve_attention(ctx, need)
    full = _run_fp8(ctx, q, k, v, ends)
    P = ends[-2]
    part = _run_fp8(ctx, q[P:].contiguous(), k, v, ends, q_offset=P)
    ctx.check()
    assert torch.equal(full[P:], part)
    rows = np.concatenate([np.arange(256), np.arange(256, ends[-1], 31)])
    got = bf16_np(full)[rows]
    e_plain = rel_l2(got, _oracle(q, k, v, ends, heads, fp8="plain", rows=rows))
    e_exact = rel_l2(got, _oracle(q, k, v, ends, heads, fp8=False, rows=rows))
    assert e_plain < E4M3_RMS and e_plain < e_exact and e_exact < 8e-2


class _StepFp8:
    def __init__(self, ctx, blocks=2):
        from tests.test_gpu_step import Setup
        cfg = synth.TINY.replace(name="fp8_step", blocks=blocks, patch=64,
                                 groups=(synth.Group("text", 12), synth.Group("image", 16, (4, 4)),
                                         synth.Group("image", 144, (12, 12))))
        self.s = Setup(ctx, cfg)


def test_step_fp8_attention_vs_oracle(ctx):
    st = _StepFp8(ctx)
    s = st.s
    sig = O.sigma_schedule(40, s.cfg.target_tokens)
    a, b = float(sig[10]), float(sig[11])
    ctx.set_attention_fp8(True)
    try:
        lat, v = s.gpu_step(ctx, s.lat, a, b)
    finally:
        ctx.set_attention_fp8(False)
    cfg = s.cfg
    mw = {k_: bf16_np(t) for k_, t in s.glob.items()}
    pws = [O.prepare_block({k_: v_.float().numpy() for k_, v_ in blk.items()}) for blk in s.blocks]
    mods = [(bf16_np(blk["mod"]), bf16_np(blk["mod_b"])) for blk in s.blocks]
    _, ov = O.step_forward(s.lat.numpy(), bf16_np(s.txt), s.ref.numpy(), mw, pws, mods, s.gd,
                           cfg.heads, cfg.head_dim, cfg.eps, a, b, return_v=True, attn="fp8")
    assert np.all(np.isfinite(v.numpy()))
    assert rel_l2(v.numpy(), ov) < 3e-2
    assert np.array_equal(lat.numpy(), O.euler_update(s.lat.numpy(), v.numpy(), a, b))
    # fp8 attention changes the result, by an amount of the order of its rounding
    _, v16 = s.gpu_step(ctx, s.lat, a, b)
    assert 0 < rel_l2(v.numpy(), v16.numpy()) < 0.1


def test_step_fp8_cached_equals_uncached(ctx):
    st = _StepFp8(ctx, blocks=3)
    s = st.s
    sig = O.sigma_schedule(40, s.cfg.target_tokens)
    ctx.set_attention_fp8(True)
    try:
        a1, _ = s.gpu_step(ctx, s.lat, float(sig[0]), float(sig[1]), qi.QI_KV_WRITE_PREFIX)
        u2, _ = s.gpu_step(ctx, a1, float(sig[1]), float(sig[2]), qi.QI_KV_NONE)
        c2, _ = s.gpu_step(ctx, a1, float(sig[1]), float(sig[2]), qi.QI_KV_READ_PREFIX)
    finally:
        ctx.set_attention_fp8(False)
    assert torch.equal(u2, c2)


def test_schedule_bf16_prefix_then_fp8_steps_vs_oracle(ctx):
    # the pages' schedule: the prefix pass (and the first steps) at full
    # precision, a later step with fp8 attention reading the cached prefix K/V
    st = _StepFp8(ctx, blocks=2)
    s = st.s
    cfg = s.cfg
    sig = O.sigma_schedule(40, cfg.target_tokens)
    lat1, _ = s.gpu_step(ctx, s.lat, float(sig[0]), float(sig[1]), qi.QI_KV_WRITE_PREFIX)
    ctx.set_attention_fp8(True)
    try:
        _, v = s.gpu_step(ctx, lat1, float(sig[7]), float(sig[8]), qi.QI_KV_READ_PREFIX)
    finally:
        ctx.set_attention_fp8(False)
    mw = {k_: bf16_np(t) for k_, t in s.glob.items()}
    pws = [O.prepare_block({k_: v_.float().numpy() for k_, v_ in blk.items()}) for blk in s.blocks]
    mods = [(bf16_np(blk["mod"]), bf16_np(blk["mod_b"])) for blk in s.blocks]
    cache = {}
    O.step_forward(s.lat.numpy(), bf16_np(s.txt), s.ref.numpy(), mw, pws, mods, s.gd, cfg.heads,
                   cfg.head_dim, cfg.eps, float(sig[0]), float(sig[1]), kv_cache=cache,
                   mode="write")
    _, ov = O.step_forward(lat1.numpy(), None, None, mw, pws, mods, s.gd, cfg.heads, cfg.head_dim,
                           cfg.eps, float(sig[7]), float(sig[8]), kv_cache=cache, mode="read",
                           return_v=True, attn="fp8")
    assert rel_l2(v.numpy(), ov) < 3e-2


# ------------------------------------------------------------------ MXFP4 checkpoint weights

def test_mxfp4_decode_bit_exact_and_w8_prepare(ctx):
    g = _gen(11)
    n, k_stored, k = 96, 4096 + 32, 4096 + 16          # padded rows, padding removed on decode
    packed = torch.randint(0, 256, (n, k_stored // 2), generator=g, dtype=torch.uint8)
    scales = torch.randint(110, 135, (n, k_stored // 32), generator=g, dtype=torch.uint8)
    scales[0, :4] = torch.tensor([0, 1, 254, 255], dtype=torch.uint8)   # denormal, extremes, NaN
    w = qi.qi_mxfp4_decode(ctx, cuda(packed), cuda(scales), k=k).cpu().numpy()
    ref = O.mxfp4_decode(packed.numpy(), scales.numpy(), k=k)
    assert np.array_equal(w, ref, equal_nan=True)
    # the decoded (finite) weights go through the W8A8 weight preparation unchanged
    wd = torch.from_numpy(ref[1:]).contiguous()
    q, s, rs = qi.qi_prepare_w8(ctx, cuda(wd))
    oq, os_, ors = O.prepare_w8(ref[1:])
    assert np.array_equal(q.cpu().numpy(), oq) and np.array_equal(s.cpu().numpy(), os_)
