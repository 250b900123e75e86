"""Step-level parity: qi_denoise_step against the oracle's step (velocity and
updated latents), the 32-block stack, cached == uncached steps for text-only
and edit sequences, and A-B-A determinism at the 1024x1024 workload."""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda, rel_l2

pytestmark = pytest.mark.gpu


class Setup:
    def __init__(self, ctx, cfg):
        self.cfg = cfg
        H = cfg.hidden
        self.glob = synth.model_weights(cfg)
        self.blocks = [synth.block_weights(cfg, l) for l in range(cfg.blocks)]
        self.dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
        self.model = qi.Model(ctx, self.dims, [qi.BlockWeights(ctx, b) for b in self.blocks],
                              self.glob)
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
        pws = [O.prepare_block({k: v.float().numpy() for k, v in b.items()}) for b in self.blocks]
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
                               synth.Group("image", 64, (8, 8))))],
    ids=["2blk", "32blk", "edit", "edit_3ref"])
def test_step_vs_oracle(ctx, cfg):
    s = Setup(ctx, cfg)
    sig = O.sigma_schedule(40, cfg.target_tokens)
    lat1, v = s.gpu_step(ctx, s.lat, float(sig[3]), float(sig[4]))
    olat, ov = s.oracle_step(s.lat, float(sig[3]), float(sig[4]))
    assert np.all(np.isfinite(v.numpy()))
    assert rel_l2(v.numpy(), ov) < 2e-2
    # the Euler update is bit-exact given the velocity
    assert np.array_equal(lat1.numpy(), O.euler_update(s.lat.numpy(), v.numpy(), sig[3], sig[4]))


@pytest.mark.parametrize("edit", [0, 1, 3], ids=["text_image", "text_ref_image", "text_3ref_image"])
def test_step_cached_equals_uncached(ctx, edit):
    refs = [synth.Group("image", 64, (8, 8)), synth.Group("image", 100, (10, 10)),
            synth.Group("image", 48, (6, 8))][:edit]
    groups = ((synth.Group("text", 128 if edit else 100),) + tuple(refs) +
              (synth.Group("image", 256, (16, 16)),))
    cfg = synth.TINY.replace(name="cache", blocks=3, patch=64, groups=groups)
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
