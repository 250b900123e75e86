"""Block-level parity: qi_dit_block_forward against the oracle's block, and the
cached-prefix invariant (target rows computed with prefix K/V read from the
cache equal the uncached computation bit for bit)."""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, oracle_weights, rel_l2

pytestmark = pytest.mark.gpu


def oracle_block_weights(wts, precision=None):
    return O.prepare_block(oracle_weights(wts), precision)


def run_block(ctx, cfg, wts, x, mod, sizes, kv=None, row0=0, mode=qi.QI_KV_NONE, bw=None):
    H = cfg.hidden
    ends = list(np.cumsum(sizes))
    S = ends[-1]
    g = qi.groups_struct(ends, [0] * (len(sizes) - 1) + [1])
    gd = [(gr.kind, gr.tokens, gr.grid) for gr in cfg.groups] if cfg.groups and sum(
        gg.tokens for gg in cfg.groups) == S else [("text", sizes[0], None)] + [
        ("image", n, (1, n)) for n in sizes[1:]]
    cos, sin = qi.qi_rope_tables(gd)
    dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, 1)
    bw = bw or qi.BlockWeights(ctx, wts)
    if kv is None:
        kv = (torch.zeros((S, H), dtype=torch.bfloat16, device="cuda"),
              torch.zeros((S, H), dtype=torch.bfloat16, device="cuda"))
    T = S - row0
    ws = torch.empty(qi.qi_block_workspace_bytes(dims, T), dtype=torch.uint8, device="cuda")
    xg = cuda(x)
    qi.qi_dit_block_forward(ctx, dims, bw.struct, xg, row0, cuda(mod), g,
                            cuda(cos[row0:].contiguous()), cuda(sin[row0:].contiguous()),
                            kv[0], kv[1], mode, ws)
    ctx.check()
    return xg, kv, bw, gd


def oracle_block(cfg, wts, x, mod, sizes, gd, precision=None):
    ends = list(np.cumsum(sizes))
    gid = O.group_ids(ends)
    rs = np.where(gid < len(sizes) - 1, 0, 1)
    cos, sin = O.rope_tables(O.rope_positions(gd))
    return O.dit_block(x.numpy(), oracle_block_weights(wts, precision), bf16_np(mod), rs, gid, gid,
                       cos, sin, cfg.heads, cfg.head_dim, cfg.eps)


# Per-Linear precision layouts (FlagRelease W8A8 card, "Quantization and
# validation", Scope: only q, k and the MLP Linears of blocks 2-29 are W8A8;
# the rest stays BF16).  Together they take every branch of the block: the
# q | k | v projection all W8A8, W8A8 q, k with BF16 v, all BF16; the output
# projection and each MLP Linear in either precision.
PRECISIONS = {
    "pages_mid": {"v": "bf16", "out": "bf16"},
    "all_bf16": {"qk": "bf16", "v": "bf16", "out": "bf16", "up": "bf16", "down": "bf16"},
    "bf16_mlp": {"up": "bf16", "down": "bf16"},
    "bf16_down": {"down": "bf16"},
}


@pytest.mark.parametrize("cfg", [synth.TINY, synth.BLOCK512], ids=["tiny", "block_512px"])
@pytest.mark.parametrize("prec", list(PRECISIONS), ids=list(PRECISIONS))
def test_block_mixed_precision_vs_oracle(ctx, cfg, prec):
    precision = PRECISIONS[prec]
    wts = synth.block_weights(cfg, 0)
    sizes = cfg.group_sizes()
    x = synth.hidden_states(cfg, cfg.tokens)
    mod = synth.mod_table(cfg)
    bw = qi.BlockWeights(ctx, wts, precision=precision)
    xg, _, _, gd = run_block(ctx, cfg, wts, x, mod, sizes, bw=bw)
    ref = oracle_block(cfg, wts, x, mod, sizes, gd, precision)
    out = xg.cpu().numpy()
    assert np.all(np.isfinite(out))
    assert rel_l2(out, ref) < 1e-2
    assert rel_l2(out - x.numpy(), ref - x.numpy()) < 1e-2


def test_block_mixed_precision_cached_prefix_bit_identical(ctx):
    cfg = synth.TINY
    sizes = [128, 64, 192]
    wts = synth.block_weights(cfg, 1)
    S = sum(sizes)
    x = synth.hidden_states(cfg, S, tag="xc")
    mod = synth.mod_table(cfg, tag="modc")
    bw = qi.BlockWeights(ctx, wts, precision=PRECISIONS["pages_mid"])
    full, kv, bw, _ = run_block(ctx, cfg, wts, x, mod, sizes, mode=qi.QI_KV_WRITE_PREFIX, bw=bw)
    P = S - sizes[-1]
    part, _, _, _ = run_block(ctx, cfg, wts, x[P:].contiguous(), mod, sizes, kv=kv, row0=P,
                              mode=qi.QI_KV_READ_PREFIX, bw=bw)
    assert torch.equal(full[P:], part)


@pytest.mark.parametrize("cfg", [synth.TINY, synth.TINY.replace(
    name="tiny_ragged", groups=(synth.Group("text", 21), synth.Group("image", 35, (5, 7))))],
    ids=["tiny", "ragged"])
def test_block_tiny_vs_oracle(ctx, cfg):
    wts = synth.block_weights(cfg, 0)
    sizes = cfg.group_sizes()
    x = synth.hidden_states(cfg, cfg.tokens)
    mod = synth.mod_table(cfg)
    xg, _, _, gd = run_block(ctx, cfg, wts, x, mod, sizes)
    ref = oracle_block(cfg, wts, x, mod, sizes, gd)
    out = xg.cpu().numpy()
    assert np.all(np.isfinite(out))
    assert rel_l2(out, ref) < 1e-2
    assert rel_l2(out - x.numpy(), ref - x.numpy()) < 1e-2   # the block's own contribution


def test_block_512px_vs_oracle(ctx):
    cfg = synth.BLOCK512
    wts = synth.block_weights(cfg, 0)
    sizes = cfg.group_sizes()
    x = synth.hidden_states(cfg, cfg.tokens)
    mod = synth.mod_table(cfg)
    xg, _, _, gd = run_block(ctx, cfg, wts, x, mod, sizes)
    ref = oracle_block(cfg, wts, x, mod, sizes, gd)
    out = xg.cpu().numpy()
    assert rel_l2(out, ref) < 1e-2
    assert rel_l2(out - x.numpy(), ref - x.numpy()) < 1e-2


@pytest.mark.parametrize("sizes", [[128, 64, 192], [16, 64], [21, 35, 30]])
def test_block_cached_prefix_bit_identical(ctx, sizes):
    cfg = synth.TINY
    wts = synth.block_weights(cfg, 1)
    S = sum(sizes)
    x = synth.hidden_states(cfg, S, tag="xc")
    mod = synth.mod_table(cfg, tag="modc")
    full, kv, bw, _ = run_block(ctx, cfg, wts, x, mod, sizes, mode=qi.QI_KV_WRITE_PREFIX)
    P = S - sizes[-1]
    part, _, _, _ = run_block(ctx, cfg, wts, x[P:].contiguous(), mod, sizes, kv=kv, row0=P,
                              mode=qi.QI_KV_READ_PREFIX, bw=bw)
    assert torch.equal(full[P:], part)


def test_block_1024px_partial_cached_rows(ctx):
    """Full-width block ([512 | 4096] tokens), cached calls on the last 64 and
    the last 16 rows of the target group.  The attention splits the longest
    query tiles of some heads over the key range; with 64 rows the block's
    scratch holds the split's partials and the rows equal the uncached pass
    bit for bit; with 16 rows it does not, so that call runs unsplit (no
    write past its workspace) and differs only by rounding."""
    cfg = synth.STEP1024.replace(blocks=1)
    sizes = cfg.group_sizes()
    S = sum(sizes)
    ends = [int(e) for e in np.cumsum(sizes)]
    assert qi.qi_attn_split_plan(S, cfg.heads, qi.groups_struct(ends, [0, 1]),
                                 torch.cuda.get_device_properties(0).multi_processor_count)[0] > 0
    wts = synth.block_weights(cfg, 0)
    x = synth.hidden_states(cfg, S, tag="xp")
    mod = synth.mod_table(cfg, tag="modp")
    full, kv, bw, _ = run_block(ctx, cfg, wts, x, mod, sizes, mode=qi.QI_KV_WRITE_PREFIX)
    for T, exact in ((64, True), (16, False)):
        P = S - T
        kv_copy = (kv[0].clone(), kv[1].clone())
        part, _, _, _ = run_block(ctx, cfg, wts, x[P:].contiguous(), mod, sizes, kv=kv_copy, row0=P,
                                  mode=qi.QI_KV_READ_PREFIX, bw=bw)
        if exact:
            assert torch.equal(full[P:], part)
        else:
            got, want, x0 = part.cpu().numpy(), full[P:].cpu().numpy(), x[P:].numpy()
            assert np.all(np.isfinite(got))
            assert rel_l2(got - x0, want - x0) < 2e-2


def test_block_rejects_bad_arguments(ctx):
    cfg = synth.TINY
    wts = synth.block_weights(cfg, 0)
    with pytest.raises(qi.QiError) as e:
        run_block(ctx, cfg, wts, synth.hidden_states(cfg, 80), synth.mod_table(cfg), [16, 64],
                  row0=16, mode=qi.QI_KV_NONE)
    assert e.value.code == qi.QI_ERR_INVALID_ARG
