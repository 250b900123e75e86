"""Write the oracle's velocities for the full-width 1024x1024 workloads.

The GPU parity tests of the full 32-block step (512 text + 4096 image tokens)
and of the 1024x1024 edit step ([256 text | 1024 reference | 4096 target],
first step writing the prefix K/V, second step reading it) compare the CUDA
path's velocity with the values this script stores.  It imports only the
oracle and the seeded input generators, draws every block's weights on the
CPU exactly as the tests do (one block at a time, so host memory stays
bounded), and runs ``oracle.qi_oracle.step_forward``.

    python tests/golden/make_step_goldens.py step_1024px
    python tests/golden/make_step_goldens.py edit_1024px
    python tests/golden/make_step_goldens.py step_1024px_bf16
    python tests/golden/make_step_goldens.py step_1024px_mxfp4
    python tests/golden/make_step_goldens.py step_1024px_pagesmask
    python tests/golden/make_step_goldens.py step_1024px_sensitivity
    python tests/golden/make_step_goldens.py step_1024px_pagesmask_sensitivity
    python tests/golden/make_step_goldens.py cfg_1024px_uncond
    python tests/golden/make_step_goldens.py edit_3ref_1024px

``cfg_1024px_uncond`` is the unconditional (negative prompt) sequence of the
true-CFG workload, [256 text | 4096 image]: its conditional sequence is the
1024x1024 step itself (same seeds), so the two stored velocities give the
guided one.  ``edit_3ref_1024px`` is one uncached step of the multi-reference
edit, [256 text | 1024 | 1024 | 576 references | 4096 target].

``step_1024px_bf16`` is the same step with every block Linear in BF16 (the
BF16 path), ``step_1024px_mxfp4`` with every block Linear in MXFP4 (decoded
weights, bf16 activations), ``step_1024px_pagesmask`` with the pages' W8A8 /
BF16 layout; ``<step>_sensitivity`` runs that step once more on the
latents moved by one fp32 ulp each and records how far that moves v: the
spread that two correct implementations of the same quantized stack, which
round differently, can show after 32 blocks.

Writes ``<workload>_v*.npy`` (fp32 [4096, 64] velocities) and
``<workload>.json`` (seeds, sigmas, input hashes, output hashes, oracle
wall time) beside this file.  A 1024x1024 step takes the float64 oracle
roughly 10-30 minutes on 8 cores.
"""
from __future__ import annotations

import hashlib
import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from diffusion_transformer_text_dit_b200 import synth  # noqa: E402
from oracle import qi_oracle as O  # noqa: E402


def sha(*arrays) -> str:
    """sha256 (first 16 hex digits) over the raw bytes of the given tensors/arrays."""
    h = hashlib.sha256()
    for a in arrays:
        a = a.detach().contiguous().view(-1).view(dtype=__import__("torch").uint8).numpy() \
            if hasattr(a, "detach") else np.ascontiguousarray(a).view(np.uint8)
        h.update(a.tobytes())
    return h.hexdigest()[:16]


def input_hashes(cfg) -> dict:
    """Hashes of the inputs both sides draw: latents, text, references, the
    step-level weights and the first and last block's weights."""
    out = {"latents": sha(synth.latents(cfg)), "txt": sha(synth.text_features(cfg))}
    ref = synth.ref_latents(cfg)
    if ref is not None:
        out["ref_latents"] = sha(ref)
    g = synth.model_weights(cfg)
    out["model_weights"] = sha(*[g[k] for k in sorted(g)])
    for l in (0, cfg.blocks - 1):
        b = synth.block_weights(cfg, l)
        parts = []
        for k in sorted(b):   # MXFP4 weights are (packed, scales) pairs
            parts.extend(b[k] if isinstance(b[k], tuple) else [b[k]])
        out[f"block{l}"] = sha(*parts)
    return out


class LazyBlocks:
    """The block weights of a workload, drawn one block at a time.

    ``step_forward`` zips its per-block prepared weights with the per-block
    adaLN weights; ``prepared()`` draws block l and leaves its adaLN weights
    in a slot that ``modulation()`` hands out next, so zip(prepared(),
    modulation()) sees the pairs of one draw."""

    def __init__(self, cfg):
        self.cfg = cfg
        self.slot = None

    def prepared(self):
        for l in range(self.cfg.blocks):
            wts = synth.block_weights(self.cfg, l)
            self.slot = (wts["mod"].float().numpy(), wts["mod_b"].float().numpy())
            pw = O.prepare_block({k: tuple(t.numpy() for t in v) if isinstance(v, tuple)
                                  else v.float().numpy() for k, v in wts.items()},
                                 synth.linear_precision(self.cfg, l))
            del wts
            t = time.time() - self.t0
            print(f"  block {l + 1}/{self.cfg.blocks} drawn at {t:.0f} s", flush=True)
            yield pw

    def modulation(self):
        for _ in range(self.cfg.blocks):
            yield self.slot


def run_step(cfg, lat, sigma, sigma_next, mode, kv_cache):
    glob = synth.model_weights(cfg)
    mw = {k: v.float().numpy() for k, v in glob.items()}
    txt = synth.text_features(cfg).float().numpy()
    ref = synth.ref_latents(cfg)
    gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
    lb = LazyBlocks(cfg)
    lb.t0 = time.time()
    new_lat, v = O.step_forward(lat, txt, None if ref is None else ref.numpy(), mw, lb.prepared(),
                                lb.modulation(), gd, cfg.heads, cfg.head_dim, cfg.eps, sigma,
                                sigma_next, kv_cache=kv_cache, mode=mode, return_v=True)
    return new_lat, np.asarray(v, np.float32), time.time() - lb.t0


def main(name: str):
    base = name[:-len("_sensitivity")] if name.endswith("_sensitivity") else name
    cfg = synth.CFG1024.uncond() if base == "cfg_1024px_uncond" else synth.CONFIGS[base]
    sig = O.sigma_schedule(40, cfg.target_tokens)
    lat0 = synth.latents(cfg).numpy()
    meta = {"workload": name, "tokens": cfg.tokens, "groups": list(cfg.group_sizes()),
            "blocks": cfg.blocks, "weight_seed": cfg.weight_seed, "input_seed": cfg.input_seed,
            "latent_seed": cfg.latent_seed, "sigmas": [float(sig[0]), float(sig[1]), float(sig[2])],
            "inputs": input_hashes(cfg), "oracle": "oracle.qi_oracle.step_forward (float64 numpy)",
            "cores": os.cpu_count()}
    if name in ("step_1024px", "step_1024px_bf16", "step_1024px_mxfp4", "step_1024px_pagesmask",
                "cfg_1024px_uncond", "edit_3ref_1024px"):
        # one uncached step sigma_0 -> sigma_1
        _, v, secs = run_step(cfg, lat0, float(sig[0]), float(sig[1]), "none", None)
        np.save(os.path.join(HERE, f"{name}_v.npy"), v)
        meta["precision"] = cfg.precision
        meta["steps"] = [{"mode": "none", "sigma": float(sig[0]), "sigma_next": float(sig[1]),
                          "v": f"{name}_v.npy", "v_sha": sha(v), "oracle_seconds": secs}]
    elif name.endswith("_sensitivity"):
        # the step on latents moved by one ulp (toward +inf), against the
        # stored velocity of the unmoved latents
        v_base = np.load(os.path.join(HERE, f"{base}_v.npy"))
        lat_up = np.nextafter(lat0, np.float32(np.inf)).astype(np.float32)
        _, v, secs = run_step(cfg, lat_up, float(sig[0]), float(sig[1]), "none", None)
        d = float(np.linalg.norm(v.astype(np.float64) - v_base) / np.linalg.norm(v_base))
        meta["steps"] = [{"mode": "none", "sigma": float(sig[0]), "sigma_next": float(sig[1]),
                          "latents": "nextafter(latents, +inf): every latent moved by one fp32 ulp",
                          f"v_rel_l2_vs_{base}": d, "v_sha": sha(v), "oracle_seconds": secs}]
    elif name == "edit_1024px":
        # step 1 writes the text + reference K/V; step 2 reads them and
        # processes the target rows only, from the oracle's step-1 latents
        cache = {}
        lat1, v1, s1 = run_step(cfg, lat0, float(sig[0]), float(sig[1]), "write", cache)
        np.save(os.path.join(HERE, f"{name}_v1.npy"), v1)
        _, v2, s2 = run_step(cfg, lat1, float(sig[1]), float(sig[2]), "read", cache)
        np.save(os.path.join(HERE, f"{name}_v2.npy"), v2)
        meta["steps"] = [
            {"mode": "write", "sigma": float(sig[0]), "sigma_next": float(sig[1]),
             "v": f"{name}_v1.npy", "v_sha": sha(v1), "oracle_seconds": s1},
            {"mode": "read", "sigma": float(sig[1]), "sigma_next": float(sig[2]),
             "latents": "euler_update(latents, v1, sigma_0, sigma_1)",
             "v": f"{name}_v2.npy", "v_sha": sha(v2), "oracle_seconds": s2}]
    else:
        raise SystemExit(f"unknown workload {name}")
    with open(os.path.join(HERE, f"{name}.json"), "w") as f:
        json.dump(meta, f, indent=1)
    print(json.dumps(meta, indent=1))


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else "step_1024px")
