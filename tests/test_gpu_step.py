"""Step-level parity: qi_denoise_step against the oracle's step (velocity and
updated latents), the 32-block stack, cached == uncached steps for text-only
and edit sequences, and A-B-A determinism at the 1024x1024 workload."""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, oracle_weights, rel_l2

pytestmark = pytest.mark.gpu

# Ten reference images of mixed grids: the most the pages' edit flow takes
# (each reference its own group of the block-causal mask).
REF10 = tuple(synth.Group("image", h * w, (h, w))
              for h, w in ((4, 4), (3, 3), (2, 2), (4, 4), (2, 3), (3, 3), (3, 4), (2, 2), (4, 4), (2, 4)))


class Setup:
    def __init__(self, ctx, cfg):
        self.cfg = cfg
        H = cfg.hidden
        self.glob = synth.model_weights(cfg)
        self.blocks = [synth.block_weights(cfg, l) for l in range(cfg.blocks)]
        self.dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
        self.model = qi.Model(ctx, self.dims,
                              [qi.BlockWeights(ctx, b, precision=synth.linear_precision(cfg, l))
                               for l, b in enumerate(self.blocks)], self.glob)
        self.gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
        self.ends = list(np.cumsum(cfg.group_sizes()))
        self.groups = qi.groups_struct(self.ends, cfg.group_row_sets())
        cos, sin = qi.qi_rope_tables(self.gd)
        self.cos, self.sin = cuda(cos), cuda(sin)
        S = cfg.tokens
        self.ws = torch.empty(qi.qi_step_workspace_bytes(self.dims, S), dtype=torch.uint8,
                              device="cuda")
        self.kv = torch.zeros((cfg.blocks, 2, S, H), dtype=torch.bfloat16, device="cuda")
        self.txt = synth.text_features(cfg)
        self.ref = synth.ref_latents(cfg)
        self.lat = synth.latents(cfg)

    def gpu_step(self, ctx, lat, sigma, sigma_next, mode=qi.QI_KV_NONE):
        latg = cuda(lat)
        v = torch.empty_like(latg)
        cfg = self.cfg
        qi.qi_denoise_step(ctx, self.model, latg,
                           cuda(self.txt) if mode != qi.QI_KV_READ_PREFIX else None,
                           cfg.text_tokens,
                           cuda(self.ref) if (self.ref is not None and mode != qi.QI_KV_READ_PREFIX) else None,
                           self.groups, self.cos, self.sin, sigma, sigma_next, mode,
                           self.kv if mode != qi.QI_KV_NONE else None, v, self.ws)
        ctx.check()
        return latg.cpu(), v.cpu()

    def oracle_step(self, lat, sigma, sigma_next):
        cfg = self.cfg
        mw = {k: bf16_np(t) for k, t in self.glob.items()}
        pws = [O.prepare_block(oracle_weights(b), synth.linear_precision(cfg, l))
               for l, b in enumerate(self.blocks)]
        mods = [(bf16_np(b["mod"]), bf16_np(b["mod_b"])) for b in self.blocks]
        return O.step_forward(lat.numpy(), bf16_np(self.txt),
                              None if self.ref is None else self.ref.numpy(), mw, pws, mods,
                              self.gd, cfg.heads, cfg.head_dim, cfg.eps, sigma, sigma_next,
                              return_v=True)


@pytest.mark.parametrize("cfg", [
    synth.TINY.replace(name="tiny_step_2blk", blocks=2),
    synth.TINY.replace(name="tiny_step_32blk", blocks=32),
    synth.TINY.replace(name="tiny_edit", blocks=2, patch=64,
                       groups=(synth.Group("text", 12), synth.Group("image", 16, (4, 4)),
                               synth.Group("image", 64, (8, 8)))),
    synth.TINY.replace(name="tiny_edit_3ref", blocks=2, patch=64,
                       groups=(synth.Group("text", 12), synth.Group("image", 16, (4, 4)),
                               synth.Group("image", 36, (6, 6)), synth.Group("image", 9, (3, 3)),
                               synth.Group("image", 64, (8, 8)))),
    synth.TINY.replace(name="tiny_edit_10ref", blocks=2, patch=64,
                       groups=(synth.Group("text", 12),) + REF10 + (synth.Group("image", 64, (8, 8)),)),
    synth.TINY.replace(name="tiny_edit_14ref", blocks=2, patch=64,
                       groups=(synth.Group("text", 12),) + REF10 + REF10[:4] + (synth.Group("image", 64, (8, 8)),)),
    synth.TINY.replace(name="tiny_pages", blocks=6, precision="pages"),
    synth.TINY.replace(name="tiny_mxfp4", blocks=3, patch=64, precision="mxfp4")],
    ids=["2blk", "32blk", "edit", "edit_3ref", "edit_10ref", "edit_14ref_max_groups", "pages_mask_6blk",
         "mxfp4_3blk"])
def test_step_vs_oracle(ctx, cfg):
    s = Setup(ctx, cfg)
    sig = O.sigma_schedule(40, cfg.target_tokens)
    lat1, v = s.gpu_step(ctx, s.lat, float(sig[3]), float(sig[4]))
    olat, ov = s.oracle_step(s.lat, float(sig[3]), float(sig[4]))
    assert np.all(np.isfinite(v.numpy()))
    assert rel_l2(v.numpy(), ov) < 2e-2
    # the Euler update is bit-exact given the velocity
    assert np.array_equal(lat1.numpy(), O.euler_update(s.lat.numpy(), v.numpy(), sig[3], sig[4]))


@pytest.mark.parametrize("edit,precision", [(0, "w8a8"), (1, "w8a8"), (3, "w8a8"), (10, "w8a8"),
                                            (1, "pages"), (1, "mxfp4")],
                         ids=["text_image", "text_ref_image", "text_3ref_image", "text_10ref_image",
                              "pages_mask", "mxfp4"])
def test_step_cached_equals_uncached(ctx, edit, precision):
    refs = ([synth.Group("image", 64, (8, 8)), synth.Group("image", 100, (10, 10)),
             synth.Group("image", 48, (6, 8))][:edit] if edit <= 3 else list(REF10[:edit]))
    groups = ((synth.Group("text", 128 if edit else 100),) + tuple(refs) +
              (synth.Group("image", 256, (16, 16)),))
    cfg = synth.TINY.replace(name="cache", blocks=3 if precision == "w8a8" else 5, patch=64,
                             groups=groups, precision=precision)
    s = Setup(ctx, cfg)
    sig = O.sigma_schedule(40, cfg.target_tokens)
    a1, _ = s.gpu_step(ctx, s.lat, float(sig[0]), float(sig[1]), qi.QI_KV_WRITE_PREFIX)
    u2, _ = s.gpu_step(ctx, a1, float(sig[1]), float(sig[2]), qi.QI_KV_NONE)
    c2, _ = s.gpu_step(ctx, a1, float(sig[1]), float(sig[2]), qi.QI_KV_READ_PREFIX)
    assert torch.equal(u2, c2)


def test_step_1024px_deterministic_aba(ctx):
    cfg = synth.STEP1024
    s = Setup(ctx, cfg)
    sig = O.sigma_schedule(40, cfg.target_tokens)
    a, va = s.gpu_step(ctx, s.lat, float(sig[0]), float(sig[1]))
    other = synth.latents(cfg.replace(latent_seed=77))
    b, vb = s.gpu_step(ctx, other, float(sig[0]), float(sig[1]))
    a2, va2 = s.gpu_step(ctx, s.lat, float(sig[0]), float(sig[1]))
    assert torch.equal(a, a2) and torch.equal(va, va2)
    assert not torch.equal(va, vb)
    assert torch.isfinite(va).all()


# ------------------------------------------------------------------ true CFG

class CfgSetup:
    """A conditional and an unconditional (negative prompt) sequence over the
    same target; the negative prompt is shorter."""

    def __init__(self, ctx, blocks=2, refs=0, text_c=12, text_u=7):
        ref_groups = (tuple(synth.Group("image", n, g) for n, g in
                            ((16, (4, 4)), (36, (6, 6)))[:refs]) if refs <= 2 else REF10[:refs])
        tgt = synth.Group("image", 64, (8, 8))
        self.cfg_c = synth.TINY.replace(name="cfg_c", blocks=blocks, patch=64,
                                        groups=(synth.Group("text", text_c),) + ref_groups + (tgt,))
        self.cfg_u = self.cfg_c.replace(name="cfg_u", groups=(synth.Group("text", text_u),) + ref_groups + (tgt,))
        self.c = Setup(ctx, self.cfg_c)
        self.u = Setup(ctx, self.cfg_u)
        self.u.model = self.c.model   # one model: same weights for both passes
        # the negative prompt's text rows: another draw of the same distribution
        self.u.txt = synth.text_features(self.cfg_u.replace(input_seed=9))
        self.u.ref = self.c.ref
        S_c, S_u, N = self.cfg_c.tokens, self.cfg_u.tokens, self.cfg_c.target_tokens
        self.ws = torch.empty(qi.qi_step_cfg_workspace_bytes(self.c.dims, S_c, S_u, N),
                              dtype=torch.uint8, device="cuda")

    def seq(self, s, mode):
        return qi.seq_struct(cuda(s.txt) if mode != qi.QI_KV_READ_PREFIX else None,
                             s.cfg.text_tokens,
                             cuda(s.ref) if (s.ref is not None and mode != qi.QI_KV_READ_PREFIX) else None,
                             s.groups, s.cos, s.sin, s.kv if mode != qi.QI_KV_NONE else None)

    def step(self, ctx, lat, g, sigma, sigma_next, mode=qi.QI_KV_NONE):
        sc, su = self.seq(self.c, mode), self.seq(self.u, mode)
        latg = cuda(lat)
        v = torch.empty_like(latg)
        qi.qi_denoise_step_cfg(ctx, self.c.model, latg, sc, su, g, sigma, sigma_next, mode, v,
                               self.ws)
        ctx.check()
        return latg.cpu(), v.cpu()


@pytest.mark.parametrize("refs", [0, 2, 10], ids=["text_image", "text_2ref_image", "text_10ref_image"])
def test_cfg_batch_equals_two_single_steps(ctx, refs):
    s = CfgSetup(ctx, refs=refs)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    a, b = float(sig[5]), float(sig[6])
    lat, v = s.step(ctx, s.c.lat, 4.0, a, b)
    _, vc = s.c.gpu_step(ctx, s.c.lat, a, b)
    _, vu = s.u.gpu_step(ctx, s.c.lat, a, b)
    # each sequence of the batch computes exactly its single-sequence velocity
    assert np.array_equal(v.numpy(), O.cfg_combine(vc.numpy(), vu.numpy(), 4.0))
    assert np.array_equal(lat.numpy(), O.euler_update(s.c.lat.numpy(), v.numpy(), a, b))
    assert not np.array_equal(vc.numpy(), vu.numpy())


def test_cfg_step_vs_oracle(ctx):
    s = CfgSetup(ctx, refs=1)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    a, b = float(sig[2]), float(sig[3])
    _, v = s.step(ctx, s.c.lat, 3.0, a, b)
    _, ovc = s.c.oracle_step(s.c.lat, a, b)
    _, ovu = s.u.oracle_step(s.c.lat, a, b)
    ov = O.cfg_combine(ovc, ovu, 3.0)
    assert np.all(np.isfinite(v.numpy()))
    assert rel_l2(v.numpy(), ov) < 2e-2


def test_cfg_10ref_step_vs_oracle(ctx):
    """True CFG over ten references (24 groups in the two sequences): the
    batch's row table merges neighbouring groups of the same row set, so it
    runs, and its guided velocity matches the oracle's."""
    s = CfgSetup(ctx, refs=10)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    a, b = float(sig[2]), float(sig[3])
    _, v = s.step(ctx, s.c.lat, 3.0, a, b)
    _, ovc = s.c.oracle_step(s.c.lat, a, b)
    _, ovu = s.u.oracle_step(s.c.lat, a, b)
    ov = O.cfg_combine(ovc, ovu, 3.0)
    assert np.all(np.isfinite(v.numpy()))
    assert rel_l2(v.numpy(), ov) < 2e-2


@pytest.mark.parametrize("refs", [1, 10], ids=["1ref", "10ref"])
def test_cfg_cached_equals_uncached(ctx, refs):
    s = CfgSetup(ctx, blocks=3, refs=refs)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    a1, _ = s.step(ctx, s.c.lat, 2.5, float(sig[0]), float(sig[1]), qi.QI_KV_WRITE_PREFIX)
    u2, _ = s.step(ctx, a1, 2.5, float(sig[1]), float(sig[2]), qi.QI_KV_NONE)
    c2, _ = s.step(ctx, a1, 2.5, float(sig[1]), float(sig[2]), qi.QI_KV_READ_PREFIX)
    assert torch.equal(u2, c2)


@pytest.mark.parametrize("refs", [0, 2], ids=["text_image", "text_2ref_image"])
def test_cfg_fp8_batch_equals_two_single_fp8_steps(ctx, refs):
    """fp8 attention in a true-CFG batch: the QKV epilogue writes each
    sequence's e4m3 K/V rows at that sequence's own place, so each velocity of
    the batch is exactly its single-sequence fp8 velocity."""
    s = CfgSetup(ctx, refs=refs)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    a, b = float(sig[5]), float(sig[6])
    ctx.set_attention_fp8(True)
    try:
        _, v = s.step(ctx, s.c.lat, 4.0, a, b)
        _, vc = s.c.gpu_step(ctx, s.c.lat, a, b)
        _, vu = s.u.gpu_step(ctx, s.c.lat, a, b)
    finally:
        ctx.set_attention_fp8(False)
    assert np.array_equal(v.numpy(), O.cfg_combine(vc.numpy(), vu.numpy(), 4.0))
    assert not np.array_equal(vc.numpy(), vu.numpy())


def test_cfg_fp8_cached_equals_uncached(ctx):
    """Cached fp8 steps cast only the cached prefix K/V rows of each sequence
    to e4m3; the uncached step gets all of them from the QKV epilogue."""
    s = CfgSetup(ctx, blocks=3, refs=1)
    sig = O.sigma_schedule(40, s.cfg_c.target_tokens)
    ctx.set_attention_fp8(True)
    try:
        a1, _ = s.step(ctx, s.c.lat, 2.5, float(sig[0]), float(sig[1]), qi.QI_KV_WRITE_PREFIX)
        u2, _ = s.step(ctx, a1, 2.5, float(sig[1]), float(sig[2]), qi.QI_KV_NONE)
        c2, _ = s.step(ctx, a1, 2.5, float(sig[1]), float(sig[2]), qi.QI_KV_READ_PREFIX)
    finally:
        ctx.set_attention_fp8(False)
    assert torch.equal(u2, c2)


def test_cfg_rejects_mismatched_targets(ctx):
    s = CfgSetup(ctx)
    other = synth.TINY.replace(name="cfg_bad", blocks=2, patch=64,
                               groups=(synth.Group("text", 7), synth.Group("image", 16, (4, 4))))
    bad = Setup(ctx, other)
    latg = cuda(s.c.lat)
    before = latg.clone()
    with pytest.raises(qi.QiError) as e:
        qi.qi_denoise_step_cfg(ctx, s.c.model, latg, s.seq(s.c, qi.QI_KV_NONE),
                               s.seq(bad, qi.QI_KV_NONE), 2.0, 1.0, 0.9, qi.QI_KV_NONE, None, s.ws)
    assert e.value.code == qi.QI_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(latg, before)


def test_cfg_rejects_row_sets_other_than_prefix_and_target(ctx):
    """The step fixes the row sets (0 for text and references, 1 for the
    target), so each sequence is two runs of the batch's row table whatever
    its number of references; other row sets are rejected before any launch,
    latents untouched."""
    s = CfgSetup(ctx, refs=10)
    alt = lambda st: qi.groups_struct(st.ends, [g % 2 for g in range(len(st.ends))])
    sc, su = s.seq(s.c, qi.QI_KV_NONE), s.seq(s.u, qi.QI_KV_NONE)
    gc, gu = alt(s.c), alt(s.u)
    sc.groups, su.groups = qi.C.pointer(gc), qi.C.pointer(gu)
    latg = cuda(s.c.lat)
    before = latg.clone()
    with pytest.raises(qi.QiError) as e:
        qi.qi_denoise_step_cfg(ctx, s.c.model, latg, sc, su, 2.0, 1.0, 0.9, qi.QI_KV_NONE, None, s.ws)
    assert e.value.code == qi.QI_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert torch.equal(latg, before)
