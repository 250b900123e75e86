"""Seeded synthetic workloads for the Qwen-Image-2.1 single-stream DiT step.

This module holds shapes, seeds and value distributions only; it performs none
of the method's arithmetic.  Both the CUDA path (through the tests and the
benchmark) and the CPU oracle receive the tensors drawn here, so the two sides
see bit-identical inputs.

Draws use torch's CPU generator (``torch.Generator``, one per named tensor,
seeded from the workload seed and the tensor's name), the same kind of draw the
RGBA-Image-2.1 Core AI port describes for its initial noise ("Use it":
``torch.randn`` on a CPU generator seeded with ``--seed``).  Weights are random-init: no trained checkpoint is
involved anywhere.

Value distributions (fixed for every workload):
  * Linear weights N(0, 0.02) in fp32 (quantized later for W8A8 Linears, cast
    to bf16 for BF16 Linears), biases N(0, 0.02) as bf16,
  * Q/K RMSNorm weights 1 + N(0, 0.1) as bf16,
  * latents N(0, 1) fp32, text features N(0, 1) bf16,
  * block-level modulation tables N(0, 0.5) bf16 (block tests only; the full
    step derives them from the timestep embedding).
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "Group", "DitConfig", "TINY", "BLOCK512", "STEP1024", "EDIT1024", "EDIT3REF1024", "CFG1024",
    "GEN2048", "GEN2048_SCHED", "STEP1024_PAGES", "STEP1024_MXFP4", "STEP1024_BF16", "linear_precision",
    "mxfp4_weight",
    "CONFIGS", "gen", "linear_weight", "bias", "norm_weight", "latents",
    "text_features", "ref_latents", "hidden_states", "mod_table", "block_weights", "model_weights",
]


@dataclasses.dataclass(frozen=True)
class Group:
    """One contiguous token group of the joint sequence."""
    kind: str                                  # "text" or "image"
    tokens: int
    grid: Optional[Tuple[int, int]] = None     # (h, w) for image groups


@dataclasses.dataclass(frozen=True)
class DitConfig:
    name: str
    hidden: int
    heads: int
    head_dim: int
    mlp: int
    blocks: int
    patch: int
    groups: Tuple[Group, ...]                  # last group = target latent tokens
    eps: float = 1e-6
    weight_seed: int = 0
    input_seed: int = 1
    latent_seed: int = 1
    steps: int = 1
    t: Optional[float] = None                  # fixed timestep for block-only workloads
    uncond_text: int = 0                       # true CFG: negative-prompt tokens (0 = no guidance)
    fp8_from_step: int = 0                     # precision schedule: fp8 attention from this step (1-based; 0 = never)
    guidance: float = 4.0                      # true CFG scale
    precision: str = "w8a8"                    # "w8a8" | "pages" (W8A8/BF16 layout) | "mxfp4" | "bf16"

    @property
    def tokens(self) -> int:
        return sum(g.tokens for g in self.groups)

    @property
    def prefix_tokens(self) -> int:
        return sum(g.tokens for g in self.groups[:-1])

    @property
    def target_tokens(self) -> int:
        return self.groups[-1].tokens

    @property
    def text_tokens(self) -> int:
        return sum(g.tokens for g in self.groups if g.kind == "text")

    def group_sizes(self) -> Tuple[int, ...]:
        return tuple(g.tokens for g in self.groups)

    def group_row_sets(self) -> Tuple[int, ...]:
        """Modulation row set per group: 0 for conditioning prefix groups, 1 for the target."""
        return tuple(0 if i < len(self.groups) - 1 else 1 for i in range(len(self.groups)))

    def uncond(self) -> "DitConfig":
        """The unconditional (negative prompt) sequence of a true-CFG workload:
        the text group holds uncond_text tokens, the rest is unchanged."""
        assert self.uncond_text > 0 and self.groups[0].kind == "text"
        return dataclasses.replace(self, name=self.name + "_uncond", input_seed=self.input_seed + 1000,
                                   groups=(Group("text", self.uncond_text),) + self.groups[1:],
                                   uncond_text=0)

    def replace(self, **kw) -> "DitConfig":
        return dataclasses.replace(self, **kw)


_TEXT = "text"
_IMAGE = "image"

# 16 text + 64 image tokens (8x8 grid of 2x2-patched 64-channel latents), one block.
TINY = DitConfig("tiny_h256_1block", 256, 2, 128, 1024, 1, 256,
                 (Group(_TEXT, 16), Group(_IMAGE, 64, (8, 8))),
                 weight_seed=0, input_seed=0, latent_seed=0, t=0.5)
# One full-width block at 512x512: 256 text + 1024 image tokens.
BLOCK512 = DitConfig("block_512px", 4096, 32, 128, 16384, 1, 64,
                     (Group(_TEXT, 256), Group(_IMAGE, 1024, (32, 32))), t=0.5)
# Full 32-block step at 1024x1024: 512 text + 4096 image tokens.
STEP1024 = DitConfig("step_1024px", 4096, 32, 128, 16384, 32, 64,
                     (Group(_TEXT, 512), Group(_IMAGE, 4096, (64, 64))))
# Edit step: 256 text + 1024 reference + 4096 target tokens.
EDIT1024 = DitConfig("edit_1024px", 4096, 32, 128, 16384, 32, 64,
                     (Group(_TEXT, 256), Group(_IMAGE, 1024, (32, 32)),
                      Group(_IMAGE, 4096, (64, 64))))
# True-CFG step at 1024x1024: the 512-token prompt and a 256-token negative
# prompt over the same 4096 target tokens, run as one batch.
CFG1024 = DitConfig("cfg_1024px", 4096, 32, 128, 16384, 32, 64,
                    (Group(_TEXT, 512), Group(_IMAGE, 4096, (64, 64))), uncond_text=256)
# Multi-reference edit step: 256 text + three references (32x32, 32x32, 24x24)
# + 4096 target tokens; each reference is its own group of the block-causal mask.
EDIT3REF1024 = DitConfig("edit_3ref_1024px", 4096, 32, 128, 16384, 32, 64,
                         (Group(_TEXT, 256), Group(_IMAGE, 1024, (32, 32)),
                          Group(_IMAGE, 1024, (32, 32)), Group(_IMAGE, 576, (24, 24)),
                          Group(_IMAGE, 4096, (64, 64))))
# 40-step denoise at 2048x2048: 512 text + 16384 image tokens.
GEN2048 = DitConfig("denoise40_2048px", 4096, 32, 128, 16384, 32, 64,
                    (Group(_TEXT, 512), Group(_IMAGE, 16384, (128, 128))),
                    steps=40, latent_seed=42)

# The same denoise with the pages' precision schedule: the prefix pass and
# steps 1-7 with bf16 attention, steps 8-40 with fp8 (e4m3) attention.
GEN2048_SCHED = GEN2048.replace(name="denoise40_2048px_sched", fp8_from_step=8)

# The same step with the pages' mixed-precision layout (FlagRelease W8A8 card,
# "Quantization and validation", Scope): W8A8 for the attention q, k and the
# two MLP Linears of blocks 2-29 (112 modules), BF16 for v, the output
# projection and every Linear of blocks 0, 1, 30 and 31.
STEP1024_PAGES = STEP1024.replace(name="step_1024px_pagesmask", precision="pages")

CONFIGS = {c.name: c for c in (TINY, BLOCK512, STEP1024, EDIT1024, EDIT3REF1024, CFG1024, GEN2048,
                               GEN2048_SCHED, STEP1024_PAGES)}


# The same step with every block Linear stored as MXFP4 and run on bf16
# activations (EliovpAI "Qwen_Image-2.1-MXFP4-Paiton-RDNA4": MXFP4 weights;
# the exact profile keeps BF16 activation arithmetic).  The block Linears are
# a synthetic MXFP4 checkpoint (random codes and scales), see mxfp4_weight.
STEP1024_MXFP4 = STEP1024.replace(name="step_1024px_mxfp4", precision="mxfp4")
CONFIGS[STEP1024_MXFP4.name] = STEP1024_MXFP4
# The same step on the BF16 path: every block Linear in BF16 (same weight draws).
STEP1024_BF16 = STEP1024.replace(name="step_1024px_bf16", precision="bf16")
CONFIGS[STEP1024_BF16.name] = STEP1024_BF16


def linear_precision(cfg: DitConfig, layer: int) -> dict:
    """Which Linears of block ``layer`` are W8A8 ("w8") and which BF16
    ("bf16"): keys "qk" (the q and k rows of the fused projection), "v",
    "out", "up", "down".  The pages' layout keeps the first two and the last
    two blocks entirely in BF16 (blocks 2-29 of 32 carry the W8A8 Linears)."""
    if cfg.precision == "w8a8":
        return {"qk": "w8", "v": "w8", "out": "w8", "up": "w8", "down": "w8"}
    if cfg.precision == "mxfp4":
        return {"qk": "mx", "v": "mx", "out": "mx", "up": "mx", "down": "mx"}
    if cfg.precision == "bf16":
        return {"qk": "bf16", "v": "bf16", "out": "bf16", "up": "bf16", "down": "bf16"}
    assert cfg.precision == "pages"
    if 2 <= layer < cfg.blocks - 2:
        return {"qk": "w8", "v": "bf16", "out": "bf16", "up": "w8", "down": "w8"}
    return {"qk": "bf16", "v": "bf16", "out": "bf16", "up": "bf16", "down": "bf16"}


def gen(seed: int, *tags) -> torch.Generator:
    """A CPU generator whose seed is a stable function of ``seed`` and ``tags``."""
    key = repr((seed,) + tuple(tags)).encode()
    return torch.Generator().manual_seed((seed * 0x9E3779B1 + zlib.crc32(key)) % (2 ** 63))


def _normal(shape, std, g, device="cpu") -> torch.Tensor:
    """N(0, std^2) draws.  On the CPU (every parity test) the draw comes from
    the CPU generator ``g``.  For a CUDA device the tensor is drawn on that
    device from a CUDA generator seeded identically: the values then differ
    from the CPU draw (another counter stream) but are just as reproducible;
    that path only serves workloads too large to draw on the host (the full
    32-block model of the benchmark), which no oracle comparison uses."""
    dev = torch.device(device)
    if dev.type == "cpu":
        t = torch.randn(*shape, generator=g, dtype=torch.float32)
    else:
        gd = torch.Generator(device=dev).manual_seed(g.initial_seed())
        t = torch.randn(*shape, generator=gd, dtype=torch.float32, device=dev)
    t.mul_(std)
    return t


def linear_weight(seed, tag, n, k, device="cpu") -> torch.Tensor:
    """fp32 [n, k] ~ N(0, 0.02)."""
    return _normal((n, k), 0.02, gen(seed, "w", tag), device)


def bias(seed, tag, n, device="cpu") -> torch.Tensor:
    """bf16 [n] ~ N(0, 0.02)."""
    return _normal((n,), 0.02, gen(seed, "b", tag), device).to(torch.bfloat16)


def norm_weight(seed, tag, d, device="cpu") -> torch.Tensor:
    """bf16 [d] ~ 1 + N(0, 0.1)."""
    return (1.0 + _normal((d,), 0.1, gen(seed, "n", tag), device)).to(torch.bfloat16)


def latents(cfg: DitConfig, device="cpu") -> torch.Tensor:
    """fp32 [target_tokens, patch] ~ N(0, 1)."""
    return _normal((cfg.target_tokens, cfg.patch), 1.0, gen(cfg.latent_seed, "latents"), device)


def ref_latents(cfg: DitConfig, device="cpu"):
    """fp32 [reference_tokens, patch] ~ N(0, 1) for edit sequences, else None."""
    ref = [g for g in cfg.groups[:-1] if g.kind == "image"]
    if not ref:
        return None
    n = sum(g.tokens for g in ref)
    return _normal((n, cfg.patch), 1.0, gen(cfg.latent_seed, "ref_latents"), device)


def text_features(cfg: DitConfig, device="cpu") -> torch.Tensor:
    """bf16 [text_tokens, hidden] ~ N(0, 1): the encoder's last hidden state stand-in."""
    return _normal((cfg.text_tokens, cfg.hidden), 1.0,
                   gen(cfg.input_seed, "txt"), device).to(torch.bfloat16)


def hidden_states(cfg: DitConfig, tokens: int, device="cpu", tag="x") -> torch.Tensor:
    """fp32 [tokens, hidden] ~ N(0, 1): a block-level residual-stream input."""
    return _normal((tokens, cfg.hidden), 1.0, gen(cfg.input_seed, tag), device)


def mod_table(cfg: DitConfig, rows: int = 2, device="cpu", tag="mod") -> torch.Tensor:
    """bf16 [rows, 6, hidden] ~ N(0, 0.5): block-level modulation rows."""
    return _normal((rows, 6, cfg.hidden), 0.5, gen(cfg.input_seed, tag), device).to(torch.bfloat16)


def mxfp4_weight(seed, tag, n, k, device="cpu"):
    """A synthetic MXFP4 checkpoint tensor [n, k]: E2M1 codes, two per byte
    (low nibble first), uniform over the 16 codes -> packed uint8 [n, k/2];
    one E8M0 scale byte per 32 columns, uniform in 118..121 (2^-9 .. 2^-6)
    -> uint8 [n, k/32].  Random bytes only: no value is computed."""
    g = gen(seed, "mx", tag)
    packed = torch.randint(0, 256, (n, k // 2), generator=g, dtype=torch.uint8)
    scales = torch.randint(118, 122, (n, k // 32), generator=g, dtype=torch.uint8)
    return packed.to(device), scales.to(device)


def block_weights(cfg: DitConfig, layer: int, device="cpu") -> dict:
    """Random-init weights of one block.

    W8A8 Linears come as fp32 (``qkv`` [3H, H], ``out`` [H, H], ``up`` [F, H],
    ``down`` [H, F]); each side quantizes them itself.  ``mod`` is the block's
    adaLN Linear [6H, H] as bf16.
    """
    s, H, F, d = cfg.weight_seed, cfg.hidden, cfg.mlp, cfg.head_dim
    L = ("blk", layer)
    if cfg.precision == "mxfp4":
        # the four Linears as MXFP4 codes (``<name>_mx`` = (packed, scales))
        out = {name + "_mx": mxfp4_weight(s, L + (name,), n, k, device)
               for name, n, k in (("qkv", 3 * H, H), ("out", H, H), ("up", F, H), ("down", H, F))}
        out.update({
            "qkv_b": bias(s, L + ("qkv",), 3 * H, device), "out_b": bias(s, L + ("out",), H, device),
            "up_b": bias(s, L + ("up",), F, device), "down_b": bias(s, L + ("down",), H, device),
            "norm_q": norm_weight(s, L + ("nq",), d, device),
            "norm_k": norm_weight(s, L + ("nk",), d, device),
            "mod": linear_weight(s, L + ("mod",), 6 * H, H, device).to(torch.bfloat16),
            "mod_b": bias(s, L + ("mod",), 6 * H, device),
        })
        return out
    return {
        "qkv": linear_weight(s, L + ("qkv",), 3 * H, H, device),
        "qkv_b": bias(s, L + ("qkv",), 3 * H, device),
        "out": linear_weight(s, L + ("out",), H, H, device),
        "out_b": bias(s, L + ("out",), H, device),
        "up": linear_weight(s, L + ("up",), F, H, device),
        "up_b": bias(s, L + ("up",), F, device),
        "down": linear_weight(s, L + ("down",), H, F, device),
        "down_b": bias(s, L + ("down",), H, device),
        "norm_q": norm_weight(s, L + ("nq",), d, device),
        "norm_k": norm_weight(s, L + ("nk",), d, device),
        "mod": linear_weight(s, L + ("mod",), 6 * H, H, device).to(torch.bfloat16),
        "mod_b": bias(s, L + ("mod",), 6 * H, device),
    }


def model_weights(cfg: DitConfig, device="cpu") -> dict:
    """Random-init weights of the step-level BF16 Linears (no blocks)."""
    s, H, P = cfg.weight_seed, cfg.hidden, cfg.patch

    def lin(tag, n, k):
        return linear_weight(s, ("g", tag), n, k, device).to(torch.bfloat16)

    return {
        "t1": lin("t1", H, 256), "t1_b": bias(s, ("g", "t1"), H, device),
        "t2": lin("t2", H, H), "t2_b": bias(s, ("g", "t2"), H, device),
        "img_in": lin("img_in", H, P), "img_in_b": bias(s, ("g", "img_in"), H, device),
        "txt_in": lin("txt_in", H, H), "txt_in_b": bias(s, ("g", "txt_in"), H, device),
        "final_mod": lin("final_mod", 2 * H, H),
        "final_mod_b": bias(s, ("g", "final_mod"), 2 * H, device),
        "proj_out": lin("proj_out", P, H), "proj_out_b": bias(s, ("g", "proj_out"), P, device),
    }


def group_layout(sizes: Sequence[int]):
    """Cumulative group ends for a list of group sizes (pure bookkeeping)."""
    ends, acc = [], 0
    for n in sizes:
        acc += int(n)
        ends.append(acc)
    return ends
