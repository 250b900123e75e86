"""Full-width parity of the two 1024x1024 workloads against the oracle.

The full 32-block step (hidden 4096, 32 heads, MLP 16384, [512 text | 4096
image] tokens, uncached) and the image-conditioned edit ([256 text | 1024
reference | 4096 target]: a first step that writes the text + reference K/V,
then a second step that reads them and processes the target rows only) are
compared with velocities the float64 oracle computed on the same seeded
inputs (tests/golden/make_step_goldens.py; the oracle needs 10-30 minutes per
step, so its outputs are stored).  The Euler update must be bit-exact given
the GPU's own v (RGBA-Image-2.1 Core AI port, "Graph contracts", Sampler),
and the cached second step must equal the uncached one bit for bit ("Qwen
Image 2.1 native qualification", "Numerical checks": cached vs uncached
second steps).

Tolerances.  The BF16 path (every block Linear in BF16) and the MXFP4 path (every block
Linear in MXFP4, bf16 activations) must be within rel-L2 2e-2 of the oracle
after the 32-block stack.  The W8A8 stack re-quantizes
every activation per token in every block, so a rounding-sized difference
anywhere flips int8 codes and the flips compound over 32 blocks: the oracle
itself moves v by ``s`` (tests/golden/step_1024px_sensitivity.json, the oracle
run again on latents moved by one fp32 ulp each) when its input changes by
one ulp.  Two correct implementations that round differently are each such a
perturbation of the exact quantized step, so they may differ by about
sqrt(2) s; the W8A8 stack is held to max(2e-2, 2 s).  Every block on its own
is held to 1e-2 at full width (the teacher-forced test below).
"""
import json
import os

import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import cuda, oracle_weights, rel_l2
from tests.golden.make_step_goldens import input_hashes

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, f"{name}.json")) as f:
        meta = json.load(f)
    return meta, [np.load(os.path.join(GOLDEN, st["v"])) for st in meta["steps"]]


@pytest.fixture(scope="module")
def model(ctx):
    """The 32-block model of both workloads (same weight seed and shapes),
    drawn on the host one block at a time exactly as the oracle run drew it."""
    cfg = synth.STEP1024
    assert synth.EDIT1024.weight_seed == cfg.weight_seed and synth.EDIT1024.hidden == cfg.hidden
    blocks = []
    for l in range(cfg.blocks):
        wts = synth.block_weights(cfg, l)
        blocks.append(qi.BlockWeights(ctx, wts))
        del wts
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    m = qi.Model(ctx, dims, blocks, synth.model_weights(cfg))
    yield m
    del m, blocks
    torch.cuda.empty_cache()


class Run:
    def __init__(self, ctx, model, cfg):
        self.ctx, self.model, self.cfg = ctx, model, cfg
        S, H = cfg.tokens, cfg.hidden
        gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
        self.groups = qi.groups_struct(list(np.cumsum(cfg.group_sizes())), cfg.group_row_sets())
        cos, sin = qi.qi_rope_tables(gd)
        self.cos, self.sin = cuda(cos), cuda(sin)
        self.ws = torch.empty(qi.qi_step_workspace_bytes(model.dims, S), dtype=torch.uint8,
                              device="cuda")
        self.kv = torch.zeros((cfg.blocks, 2, S, H), dtype=torch.bfloat16, device="cuda")
        self.txt = cuda(synth.text_features(cfg))
        ref = synth.ref_latents(cfg)
        self.ref = cuda(ref) if ref is not None else None

    def step(self, lat, sigma, sigma_next, mode):
        latg = cuda(torch.from_numpy(np.ascontiguousarray(lat)))
        v = torch.empty_like(latg)
        cached = mode == qi.QI_KV_READ_PREFIX
        qi.qi_denoise_step(self.ctx, self.model, latg, None if cached else self.txt,
                           self.cfg.text_tokens, None if cached else self.ref, self.groups,
                           self.cos, self.sin, sigma, sigma_next, mode,
                           None if mode == qi.QI_KV_NONE else self.kv, v, self.ws)
        self.ctx.check()
        return latg.cpu().numpy(), v.cpu().numpy()


def _check_inputs(cfg, meta):
    assert meta["inputs"] == input_hashes(cfg), "the seeded inputs changed since the oracle ran"


def w8a8_stack_tolerance(step: str = "step_1024px") -> float:
    """max(2e-2, 2 x the oracle's one-ulp sensitivity of v after the 32 blocks
    of `step`, a stack with W8A8 Linears)."""
    with open(os.path.join(GOLDEN, f"{step}_sensitivity.json")) as f:
        s = json.load(f)["steps"][0][f"v_rel_l2_vs_{step}"]
    return max(2e-2, 2.0 * s)


def test_step_1024px_vs_oracle(ctx, model):
    cfg = synth.STEP1024
    meta, (ov,) = _golden("step_1024px")
    _check_inputs(cfg, meta)
    st = meta["steps"][0]
    lat0 = synth.latents(cfg).numpy()
    lat1, v = Run(ctx, model, cfg).step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
    assert np.all(np.isfinite(v))
    err, tol = rel_l2(v, ov), w8a8_stack_tolerance()
    print(f"step_1024px: v rel-L2 {err:.4e} (tolerance {tol:.4e})")
    assert err <= tol, f"v rel-L2 {err:.3e} after 32 W8A8 blocks (tolerance {tol:.3e})"
    assert np.array_equal(lat1, O.euler_update(lat0, v, st["sigma"], st["sigma_next"]))


def test_step_1024px_bf16_path_vs_oracle(ctx):
    """The same step with every block Linear in BF16: within rel-L2 2e-2 of
    the oracle's BF16 step after the 32-block stack."""
    cfg = synth.STEP1024_BF16
    meta, (ov,) = _golden("step_1024px_bf16")
    _check_inputs(cfg, meta)
    st = meta["steps"][0]
    blocks = [qi.BlockWeights(ctx, synth.block_weights(cfg, l),
                              precision=synth.linear_precision(cfg, l)) for l in range(cfg.blocks)]
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    m = qi.Model(ctx, dims, blocks, synth.model_weights(cfg))
    lat0 = synth.latents(cfg).numpy()
    lat1, v = Run(ctx, m, cfg).step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
    del m, blocks
    torch.cuda.empty_cache()
    assert np.all(np.isfinite(v))
    err = rel_l2(v, ov)
    print(f"step_1024px_bf16: v rel-L2 {err:.4e} (tolerance 2e-2)")
    assert err <= 2e-2, f"v rel-L2 {err:.3e} after 32 BF16 blocks"
    assert np.array_equal(lat1, O.euler_update(lat0, v, st["sigma"], st["sigma_next"]))


def test_step_1024px_pagesmask_vs_oracle(ctx):
    """The step with the pages' layout (W8A8 q, k and MLP Linears in blocks
    2-29, every other Linear BF16): within the W8A8-stack tolerance of its
    own one-ulp sensitivity."""
    cfg = synth.STEP1024_PAGES
    meta, (ov,) = _golden("step_1024px_pagesmask")
    _check_inputs(cfg, meta)
    st = meta["steps"][0]
    blocks = [qi.BlockWeights(ctx, synth.block_weights(cfg, l),
                              precision=synth.linear_precision(cfg, l)) for l in range(cfg.blocks)]
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    m = qi.Model(ctx, dims, blocks, synth.model_weights(cfg))
    lat0 = synth.latents(cfg).numpy()
    lat1, v = Run(ctx, m, cfg).step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
    del m, blocks
    torch.cuda.empty_cache()
    assert np.all(np.isfinite(v))
    err, tol = rel_l2(v, ov), w8a8_stack_tolerance("step_1024px_pagesmask")
    print(f"step_1024px_pagesmask: v rel-L2 {err:.4e} (tolerance {tol:.4e})")
    assert err <= tol
    assert np.array_equal(lat1, O.euler_update(lat0, v, st["sigma"], st["sigma_next"]))


def test_step_1024px_blocks_teacher_forced(ctx, model):
    """Blocks of the full-width step against the oracle's block on the GPU's
    own input to that block (the residual stream tapped before and after
    every block): the first, a middle and the last block each within rel-L2
    1e-2 of the oracle, on the whole block output and on the block's own
    contribution (the delta), as for the single 512px block."""
    cfg = synth.STEP1024
    S, H = cfg.tokens, cfg.hidden
    meta, _ = _golden("step_1024px")
    st = meta["steps"][0]
    r = Run(ctx, model, cfg)
    x_layers = torch.empty((cfg.blocks + 1, S, H), dtype=torch.float32, device="cuda")
    ctx.set_block_taps({"x_layers": x_layers})
    try:
        r.step(synth.latents(cfg).numpy(), st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
    finally:
        ctx.set_block_taps(None)
    mw = oracle_weights(synth.model_weights(cfg))
    temb_0, temb_t = O.time_embed(0.0, mw), O.time_embed(st["sigma"], mw)
    gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
    ends = list(np.cumsum(cfg.group_sizes()))
    gid = O.group_ids(ends)
    rs = np.where(gid < len(ends) - 1, 0, 1)
    cos, sin = O.rope_tables(O.rope_positions(gd))
    for l in (0, cfg.blocks // 2, cfg.blocks - 1):
        wts = oracle_weights(synth.block_weights(cfg, l))
        mod = np.stack([O.adaln_rows(temb_0, wts["mod"], wts["mod_b"]),
                        O.adaln_rows(temb_t, wts["mod"], wts["mod_b"])])
        x_in = x_layers[l].cpu().numpy()
        got = x_layers[l + 1].cpu().numpy()
        ref = O.dit_block(x_in, O.prepare_block(wts), mod, rs, gid, gid, cos, sin, cfg.heads,
                          cfg.head_dim, cfg.eps)
        e_out, e_delta = rel_l2(got, ref), rel_l2(got - x_in, ref - x_in)
        print(f"block {l}: output rel-L2 {e_out:.4e}, delta rel-L2 {e_delta:.4e}")
        assert e_out <= 1e-2 and e_delta <= 1e-2, (l, e_out, e_delta)


def test_edit_1024px_write_then_cached_step_vs_oracle(ctx, model):
    cfg = synth.EDIT1024
    meta, (ov1, ov2) = _golden("edit_1024px")
    _check_inputs(cfg, meta)
    s1, s2 = meta["steps"]
    r = Run(ctx, model, cfg)
    lat0 = synth.latents(cfg).numpy()
    # first step: every token processed, the text + reference K/V kept
    lat1, v1 = r.step(lat0, s1["sigma"], s1["sigma_next"], qi.QI_KV_WRITE_PREFIX)
    tol = w8a8_stack_tolerance()
    err1 = rel_l2(v1, ov1)
    print(f"edit_1024px step 1: v rel-L2 {err1:.4e} (tolerance {tol:.4e})")
    assert np.all(np.isfinite(v1)) and err1 <= tol, f"step 1 v rel-L2 {err1:.3e} (tol {tol:.3e})"
    assert np.array_equal(lat1, O.euler_update(lat0, v1, s1["sigma"], s1["sigma_next"]))
    # second step from the oracle's step-1 latents: the target rows only,
    # attending over the cached prefix K/V of the first step
    olat1 = O.euler_update(lat0, ov1, s1["sigma"], s1["sigma_next"])
    c2, v2 = r.step(olat1, s2["sigma"], s2["sigma_next"], qi.QI_KV_READ_PREFIX)
    err2 = rel_l2(v2, ov2)
    print(f"edit_1024px cached step 2: v rel-L2 {err2:.4e} (tolerance {tol:.4e})")
    assert np.all(np.isfinite(v2)) and err2 <= tol, f"cached step 2 v rel-L2 {err2:.3e} (tol {tol:.3e})"
    assert np.array_equal(c2, O.euler_update(olat1, v2, s2["sigma"], s2["sigma_next"]))
    # and the uncached second step gives the same latents bit for bit
    u2, _ = r.step(olat1, s2["sigma"], s2["sigma_next"], qi.QI_KV_NONE)
    assert np.array_equal(u2, c2)


def test_step_1024px_mxfp4_vs_oracle_and_decode_paths(ctx):
    """The full-width 32-block step with MXFP4 weights (every block Linear;
    bf16 activations, no re-quantization): within rel-L2 2e-2 of the
    oracle's step on the decoded weights, like the BF16 path.  Expanding each
    Linear to bf16 in two alternating scratch halves (every expansion
    overlapping the kernel before it) gives the velocity of decoding inside
    the GEMMs bit for bit, so no expansion overwrites weights a GEMM is still
    reading."""
    cfg = synth.STEP1024_MXFP4
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    scratch = qi.mx_expand_scratch(dims)
    blocks = [qi.BlockWeights(ctx, synth.block_weights(cfg, l), precision=synth.linear_precision(cfg, l),
                              mx_expand=scratch) for l in range(cfg.blocks)]
    glob = synth.model_weights(cfg)
    expanded = qi.Model(ctx, dims, blocks, glob)
    for b in blocks:
        b.struct.mx_expand, b.struct.mx_expand_bytes = None, 0
    tiled = qi.Model(ctx, dims, blocks, glob)
    meta, (ov,) = _golden("step_1024px_mxfp4")
    _check_inputs(cfg, meta)
    st = meta["steps"][0]
    lat0 = synth.latents(cfg).numpy()
    runs = [Run(ctx, m, cfg).step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
            for m in (expanded, tiled, expanded)]
    del expanded, tiled, blocks, scratch
    torch.cuda.empty_cache()
    (lat1, v), vs = runs[0], [r[1] for r in runs]
    assert np.all(np.isfinite(v))
    assert np.array_equal(vs[0], vs[1]) and np.array_equal(vs[0], vs[2])
    err = rel_l2(v, ov)
    print(f"step_1024px_mxfp4: v rel-L2 {err:.4e} (tolerance 2e-2)")
    assert err <= 2e-2, f"v rel-L2 {err:.3e} after 32 MXFP4 blocks"
    assert np.array_equal(lat1, O.euler_update(lat0, v, st["sigma"], st["sigma_next"]))


def test_edit_3ref_1024px_vs_oracle_and_cache(ctx, model):
    """The multi-reference edit at full width ([256 text | 1024 | 1024 | 576
    references | 4096 target], each reference its own group of the
    block-causal mask): one uncached step within the W8A8-stack tolerance of
    the oracle; writing the four prefix groups' K/V gives the same velocity
    bit for bit, and a second step that reads them equals the uncached second
    step bit for bit."""
    cfg = synth.EDIT3REF1024
    assert cfg.weight_seed == synth.STEP1024.weight_seed and cfg.hidden == synth.STEP1024.hidden
    meta, (ov,) = _golden("edit_3ref_1024px")
    _check_inputs(cfg, meta)
    st = meta["steps"][0]
    r = Run(ctx, model, cfg)
    lat0 = synth.latents(cfg).numpy()
    lat1, v = r.step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_NONE)
    assert np.all(np.isfinite(v))
    err, tol = rel_l2(v, ov), w8a8_stack_tolerance()
    print(f"edit_3ref_1024px: v rel-L2 {err:.4e} (tolerance {tol:.4e})")
    assert err <= tol, f"v rel-L2 {err:.3e} (tolerance {tol:.3e})"
    assert np.array_equal(lat1, O.euler_update(lat0, v, st["sigma"], st["sigma_next"]))
    w1, vw = r.step(lat0, st["sigma"], st["sigma_next"], qi.QI_KV_WRITE_PREFIX)
    assert np.array_equal(vw, v) and np.array_equal(w1, lat1)
    sig = O.sigma_schedule(40, cfg.target_tokens)
    c2, _ = r.step(lat1, float(sig[1]), float(sig[2]), qi.QI_KV_READ_PREFIX)
    u2, _ = r.step(lat1, float(sig[1]), float(sig[2]), qi.QI_KV_NONE)
    assert np.array_equal(c2, u2)


def test_cfg_1024px_vs_oracle(ctx, model):
    """True CFG at full width: the prompt's sequence is the 1024x1024 step
    ([512 text | 4096]), the negative prompt's [256 text | 4096], guidance 4,
    both in one batched step.  The batch's guided velocity equals the
    guidance of the two single-sequence velocities bit for bit, and each of
    those is within the W8A8-stack tolerance of the oracle's."""
    cfg = synth.CFG1024
    cond, ucfg = synth.STEP1024, cfg.uncond()
    assert cfg.replace(name=cond.name, uncond_text=0) == cond
    meta_c, (ovc,) = _golden("step_1024px")
    meta_u, (ovu,) = _golden("cfg_1024px_uncond")
    _check_inputs(cond, meta_c)
    _check_inputs(ucfg, meta_u)
    st = meta_u["steps"][0]
    assert (st["sigma"], st["sigma_next"]) == (meta_c["steps"][0]["sigma"], meta_c["steps"][0]["sigma_next"])
    a, b = st["sigma"], st["sigma_next"]
    rc, ru = Run(ctx, model, cond), Run(ctx, model, ucfg)
    lat0 = synth.latents(cfg).numpy()
    _, vc = rc.step(lat0, a, b, qi.QI_KV_NONE)
    _, vu = ru.step(lat0, a, b, qi.QI_KV_NONE)
    ws = torch.empty(qi.qi_step_cfg_workspace_bytes(model.dims, cond.tokens, ucfg.tokens,
                                                    cfg.target_tokens), dtype=torch.uint8, device="cuda")
    sc = qi.seq_struct(rc.txt, cond.text_tokens, None, rc.groups, rc.cos, rc.sin)
    su = qi.seq_struct(ru.txt, ucfg.text_tokens, None, ru.groups, ru.cos, ru.sin)
    latg = cuda(torch.from_numpy(lat0.copy()))
    vg = torch.empty_like(latg)
    qi.qi_denoise_step_cfg(ctx, model, latg, sc, su, cfg.guidance, a, b, qi.QI_KV_NONE, vg, ws)
    ctx.check()
    v, lat1 = vg.cpu().numpy(), latg.cpu().numpy()
    del ws, rc, ru
    torch.cuda.empty_cache()
    assert np.all(np.isfinite(v))
    assert np.array_equal(v, O.cfg_combine(vc, vu, cfg.guidance))
    assert np.array_equal(lat1, O.euler_update(lat0, v, a, b))
    tol = w8a8_stack_tolerance()
    ec, eu = rel_l2(vc, ovc), rel_l2(vu, ovu)
    eg = rel_l2(v, O.cfg_combine(ovc, ovu, cfg.guidance))
    print(f"cfg_1024px: prompt v rel-L2 {ec:.4e}, negative prompt v rel-L2 {eu:.4e} "
          f"(tolerance {tol:.4e}); guided v rel-L2 {eg:.4e}")
    assert ec <= tol and eu <= tol, (ec, eu, tol)
