"""Parity at the 2048x2048 workload's shapes (512 text + 16384 image tokens,
S = 16896): the whole 40-step denoise is far beyond the CPU oracle, so each
operation is checked on its own at full size, the oracle computing sampled
rows one by one from the same seeded inputs."""
import math

import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, rel_l2

pytestmark = pytest.mark.gpu
CFG = synth.GEN2048
S = CFG.tokens
ROWS = np.array([0, 1, 511, 512, 513, 4095, 9000, 12345, S - 129, S - 2, S - 1])


def _gen(seed):
    return torch.Generator().manual_seed(seed)


@pytest.mark.parametrize("N,K", [(4096, 4096), (4096, 16384)])
def test_w8a8_2048_shapes_sampled_rows(ctx, N, K):
    w = synth.linear_weight(5, ("g2048", N, K), N, K)
    b = synth.bias(5, ("g2048", N), N)
    q, s, rs = qi.qi_prepare_w8(ctx, cuda(w))
    oq, os_, ors = O.prepare_w8(w.numpy())
    qa = torch.randint(-128, 128, (S, K), generator=_gen(1), dtype=torch.int8)
    sa = torch.rand(S, generator=_gen(2)) * 0.05 + 1e-3
    zp = torch.randint(-128, 128, (S,), generator=_gen(3), dtype=torch.int32)
    acc = torch.empty((S, N), dtype=torch.int32, device="cuda")
    y = torch.empty((S, N), dtype=torch.bfloat16, device="cuda")
    qi.qi_w8a8_linear(ctx, cuda(qa), cuda(sa), cuda(zp), qi.w8_struct(q, s, rs, cuda(b)), y=y,
                      acc_debug=acc)
    ctx.check()
    oacc, oy = O.w8a8_linear(qa.numpy()[ROWS], sa.numpy()[ROWS], zp.numpy()[ROWS], oq, os_, ors,
                             bf16_np(b))
    assert np.array_equal(acc.cpu().numpy()[ROWS].astype(np.int64), oacc)
    gy = bf16_np(y)[ROWS]
    assert np.all(np.abs(gy - oy) <= 2.0 ** -7 * np.abs(oy) + 2.0 ** -20 * np.abs(oy).max())


def test_attention_2048_shapes_sampled_rows_and_cached_rows(ctx):
    heads = CFG.heads
    ends = [int(e) for e in np.cumsum(CFG.group_sizes())]
    q = torch.randn(S, heads * 128, generator=_gen(11)).to(torch.bfloat16)
    k = torch.randn(S, heads * 128, generator=_gen(12)).to(torch.bfloat16)
    v = torch.randn(S, heads * 128, generator=_gen(13)).to(torch.bfloat16)
    g = qi.groups_struct(ends, [0, 1])
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o = qi.qi_attn_block_causal(ctx, qg, kg, vg, g)
    P = ends[0]
    part = qi.qi_attn_block_causal(ctx, qg[P:].contiguous(), kg, vg, g, q_offset=P)
    ctx.check()
    assert torch.equal(o[P:], part)
    gid = O.group_ids(ends)
    qn = bf16_np(q).reshape(S, heads, 128)
    ref = O.attention_block_causal(qn[ROWS], bf16_np(k).reshape(S, heads, 128),
                                   bf16_np(v).reshape(S, heads, 128), gid[ROWS], gid,
                                   1 / math.sqrt(128)).reshape(len(ROWS), -1)
    got = bf16_np(o)[ROWS]
    assert rel_l2(got, ref) < 4e-3
    assert np.abs(got - ref).max() < 2e-2


def test_quantize_2048_rows_bit_exact(ctx):
    x = (torch.randn(S, 4096, generator=_gen(21)) * 2).to(torch.bfloat16)
    q, s, zp = qi.qi_quantize_act(ctx, cuda(x))
    oq, os_, ozp = O.quantize_act(bf16_np(x[ROWS]))
    assert np.array_equal(q.cpu().numpy()[ROWS], oq)
    assert np.array_equal(s.cpu().numpy()[ROWS], os_)
    assert np.array_equal(zp.cpu().numpy()[ROWS], ozp)
