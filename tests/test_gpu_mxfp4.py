"""MXFP4 weights at run time (EliovpAI "Qwen_Image-2.1-MXFP4-Paiton-RDNA4",
"What was quantized": E2M1 codes two per byte, low nibble first, one E8M0 scale
per 32 input columns; "Runtime precision and quality": the exact profile keeps
BF16 activation arithmetic).

The GEMM decodes the codes to bf16 in shared memory, tile by tile, and never
holds a decoded copy in HBM.  Every decoded value is exact in bf16, so the
oracle reference is its MXFP4 decode followed by its BF16 Linear (bf16 inputs,
exact sum, one bf16 rounding); the GPU sums in fp32, so an output may land one
bf16 step away from the oracle's rounding (tolerance: one bf16 ulp relative,
2^-7, plus a tiny absolute term).
"""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, oracle_weights, rel_l2

pytestmark = pytest.mark.gpu


def _case(M, N, K, seed):
    packed, scales = synth.mxfp4_weight(seed, ("linear", N, K), N, K)
    g = torch.Generator().manual_seed(seed)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = synth.bias(seed, ("mxb", N), N)
    return a, packed, scales, b


def _oracle(a, packed, scales, b):
    w = O.mxfp4_decode(packed.numpy(), scales.numpy())
    return O.bf16_linear(bf16_np(a), w, bf16_np(b))


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (77, 512, 512), (300, 768, 4096),
                                   (1280, 4096, 16384), (1000, 16384, 4096)])
def test_mxfp4_linear_vs_oracle(ctx, M, N, K):
    a, packed, scales, b = _case(M, N, K, M + N + K)
    w = qi.mx_struct(cuda(packed), cuda(scales), cuda(b))
    y = qi.qi_mxfp4_linear(ctx, cuda(a), w)
    ctx.check()
    got = bf16_np(y)
    ref = _oracle(a, packed, scales, b)
    assert np.all(np.isfinite(got))
    tol = 2.0 ** -7 * np.abs(ref) + 1e-6 * np.abs(ref).max()
    assert np.all(np.abs(got - ref) <= tol), np.abs(got - ref).max()
    assert rel_l2(got, ref) < 2e-3


def test_mxfp4_linear_extreme_scales(ctx):
    """Scale bytes outside the table decoder's range take the general decode:
    E8M0 0 and 1 (subnormal-sized weights), 255 (NaN marker); every other
    output stays finite and matches."""
    M, N, K = 64, 256, 256
    a, packed, scales, b = _case(M, N, K, 5)
    scales = scales.clone()
    scales[3, 1] = 0
    scales[4, :] = 1
    scales[7, 2] = 255
    w = qi.mx_struct(cuda(packed), cuda(scales), cuda(b))
    got = bf16_np(qi.qi_mxfp4_linear(ctx, cuda(a), w))
    ctx.check()
    ref = _oracle(a, packed, scales, b)
    assert np.array_equal(np.isnan(got), np.isnan(ref)) and np.isnan(got[:, 7]).all()
    fin = np.isfinite(ref)
    tol = 2.0 ** -7 * np.abs(ref[fin]) + 1e-6 * np.abs(ref[fin]).max()
    assert np.all(np.abs(got[fin] - ref[fin]) <= tol)


def test_mxfp4_linear_rejects_bad_shapes(ctx):
    a, packed, scales, b = _case(8, 256, 256, 1)
    y = torch.empty((8, 256), dtype=torch.bfloat16, device="cuda")
    for field, bad in (("n", 128), ("k", 128)):   # n % 256 != 0, k % 256 != 0
        w = qi.mx_struct(cuda(packed), cuda(scales), cuda(b))
        setattr(w, field, bad)
        with pytest.raises(qi.QiError) as e:
            qi.qi_mxfp4_linear(ctx, cuda(a)[:, :w.k].contiguous(), w, y=y)
        assert e.value.code == qi.QI_ERR_UNSUPPORTED_SHAPE


def test_mxfp4_expand_bf16_bit_exact(ctx):
    """The bf16 expansion equals the oracle's decode value for value, at the
    extreme scales too (E8M0 0 and 1: subnormal-sized weights; 255: NaN)."""
    N, K = 512, 1024
    packed, scales = synth.mxfp4_weight(3, ("expand", N, K), N, K)
    scales = scales.clone()
    scales[0, :4] = torch.tensor([0, 1, 254, 255], dtype=torch.uint8)
    scales[9, :] = 0
    got = bf16_np(qi.qi_mxfp4_expand_bf16(ctx, cuda(packed), cuda(scales)))
    ctx.check()
    ref = O.mxfp4_decode(packed.numpy(), scales.numpy())
    assert np.array_equal(got, ref.astype(np.float32), equal_nan=True)
    assert np.isnan(got[0, 96:128]).all() and not np.isnan(got[1:]).any()


@pytest.mark.parametrize("N,K", [(1, 32), (100, 96), (257, 4096)])
def test_mxfp4_expand_bf16_ragged_shapes(ctx, N, K):
    """Any row count and any multiple of 32 columns (one scale group), the
    grid's last partial block of words included."""
    packed, scales = synth.mxfp4_weight(N + K, ("ragged", N, K), N, K)
    got = bf16_np(qi.qi_mxfp4_expand_bf16(ctx, cuda(packed), cuda(scales)))
    ctx.check()
    assert np.array_equal(got, O.mxfp4_decode(packed.numpy(), scales.numpy()).astype(np.float32))


def _block(ctx, cfg, mx_expand=None):
    H, S = cfg.hidden, cfg.tokens
    wts = synth.block_weights(cfg, 0)
    prec = synth.linear_precision(cfg, 0)
    bw = qi.BlockWeights(ctx, wts, precision=prec, mx_expand=mx_expand)
    ends = list(np.cumsum(cfg.group_sizes()))
    gd = [(gr.kind, gr.tokens, gr.grid) for gr in cfg.groups]
    g = qi.groups_struct(ends, cfg.group_row_sets())
    cos, sin = qi.qi_rope_tables(gd)
    dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, 1)
    x = synth.hidden_states(cfg, S)
    mod = synth.mod_table(cfg)
    kl = torch.zeros((S, H), dtype=torch.bfloat16, device="cuda")
    vl = torch.zeros_like(kl)
    ws = torch.empty(qi.qi_block_workspace_bytes(dims, S), dtype=torch.uint8, device="cuda")
    xg = cuda(x)
    qi.qi_dit_block_forward(ctx, dims, bw.struct, xg, 0, cuda(mod), g, cuda(cos), cuda(sin), kl, vl,
                            qi.QI_KV_NONE, ws)
    ctx.check()
    gid = O.group_ids(ends)
    rs = np.where(gid < len(ends) - 1, 0, 1)
    ocos, osin = O.rope_tables(O.rope_positions(gd))
    ref = O.dit_block(x.numpy(), O.prepare_block(oracle_weights(wts), prec), bf16_np(mod), rs, gid,
                      gid, ocos, osin, cfg.heads, cfg.head_dim, cfg.eps)
    return x.numpy(), xg.cpu().numpy(), ref


@pytest.mark.parametrize("cfg", [synth.TINY.replace(precision="mxfp4"),
                                 synth.BLOCK512.replace(precision="mxfp4")],
                         ids=["tiny", "block_512px"])
def test_block_mxfp4_vs_oracle(ctx, cfg):
    x, out, ref = _block(ctx, cfg)
    assert np.all(np.isfinite(out))
    assert rel_l2(out, ref) < 1e-2
    assert rel_l2(out - x, ref - x) < 1e-2


@pytest.mark.parametrize("cfg", [synth.TINY.replace(precision="mxfp4"),
                                 synth.BLOCK512.replace(precision="mxfp4")],
                         ids=["tiny", "block_512px"])
def test_block_mxfp4_expanded_equals_tile_decode(ctx, cfg):
    """Expanding each MXFP4 Linear to bf16 before a BF16 GEMM gives the block
    output of the GEMM that decodes in shared memory, bit for bit (the same
    exact bf16 weights meet the same MMA sequence), with the scratch split in
    two alternating halves or used whole."""
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, 1)
    _, tile, _ = _block(ctx, cfg)
    # two halves (each expansion overlapping the kernel before it), and one
    for buffers in (2, 1):
        _, expd, ref = _block(ctx, cfg, mx_expand=qi.mx_expand_scratch(dims, buffers=buffers))
        assert np.array_equal(tile, expd), buffers
        assert rel_l2(expd, ref) < 1e-2
