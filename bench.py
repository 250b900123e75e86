#!/usr/bin/env python
"""Benchmark: DiT denoising steps/s at 1024x1024 (512 text + 4096 image tokens).

One step = one full pass of the hot path: time conditioning and adaLN rows,
text/image in-projections, 32 single-stream W8A8 blocks (block-causal
attention, 3-axis RoPE, Q/K RMSNorm), final layer and the FlowMatch Euler
update, all in libqi's sm_100a kernels, with random-init weights and seeded
synthetic inputs resident in HBM.  Prints one JSON line (rank 0).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun as independent replicas (one step per GPU per
iteration; the step does not shard).  The reference arm times the CPU oracle
on the host cores (rank 0 only), a bounded sample per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_transformer_text_dit_b200 import synth  # noqa: E402

METRIC = "DiT steps/s at 1024² (4096 img+512 txt tok); W8A8 GEMM & attn % of peak"
CFG = synth.STEP1024


# ------------------------------------------------------------------ workload arithmetic

def algorithmic_work(cfg: synth.DitConfig, cached: bool = False):
    """Per-step algorithmic work: int8 ops of the W8A8 Linears and bf16 FLOPs of
    the visible (unmasked) query-key pairs.  A cached step processes only the
    target rows, which still attend over every key.  A true-CFG step does the
    work of both of its sequences."""
    if cfg.uncond_text:
        a = algorithmic_work(dataclasses.replace(cfg, uncond_text=0), cached)
        b = algorithmic_work(cfg.uncond(), cached)
        return {k: a[k] + b[k] for k in a}
    H, F, d, h = cfg.hidden, cfg.mlp, cfg.head_dim, cfg.heads
    rows = cfg.target_tokens if cached else cfg.tokens
    per_block_ops = 2 * rows * (3 * H * H + H * H + F * H + H * F)
    ends = np.cumsum(cfg.group_sizes())
    starts = np.concatenate([[0], ends[:-1]])
    if cached:
        pairs = int(cfg.target_tokens * ends[-1])
    else:
        pairs = int(sum((e - s) * e for s, e in zip(starts, ends)))   # query x visible keys
    attn_flops = 4 * d * h * pairs
    return {
        "gemm_i8_ops_per_step": cfg.blocks * per_block_ops,
        "attn_flops_per_step": cfg.blocks * attn_flops,
        "attn_pairs_per_head": pairs,
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling every 200 ms during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = set(gpus)
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                if int(f[0]) not in self.gpus:
                    continue
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ model setup

def build_model(ctx, qi, cfg, device):
    blocks = []
    for l in range(cfg.blocks):
        wts = synth.block_weights(cfg, l, device=device)
        blocks.append(qi.BlockWeights(ctx, wts, device=device))
        del wts
    glob = synth.model_weights(cfg, device=device)
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    return qi.Model(ctx, dims, blocks, glob, device=device), dims


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sust": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "src": "fallback"}


def kernel_traffic(cls: str):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary,
    if it was captured from the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(cls)
    if not d:
        return None
    src = os.path.join(ROOT, d["source"])
    if not os.path.exists(src):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest()[:16] != d["source_sha256_16"]:
        return None
    return d["bytes_per_launch_full"]


# ------------------------------------------------------------------ CPU oracle sample

class OracleSample:
    """The CPU oracle on whole blocks of the 1024^2 step (S = 4608), prepared once."""

    def __init__(self):
        from oracle import qi_oracle as O
        self.O = O
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            self.cores = os.cpu_count()
        cfg = CFG
        wts = synth.block_weights(cfg, 0)
        self.pw = O.prepare_block({k: v.float().numpy() for k, v in wts.items()})
        del wts
        self.x = synth.hidden_states(cfg, cfg.tokens).numpy().astype(np.float64)
        self.mod = synth.mod_table(cfg).float().numpy()
        gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
        ends = list(np.cumsum(cfg.group_sizes()))
        self.gid = O.group_ids(ends)
        self.rs = np.where(self.gid < len(ends) - 1, 0, 1)
        self.cos, self.sin = O.rope_tables(O.rope_positions(gd))

    def time_block(self) -> float:
        cfg = CFG
        t0 = time.perf_counter()
        self.O.dit_block(self.x, self.pw, self.mod, self.rs, self.gid, self.gid, self.cos,
                         self.sin, cfg.heads, cfg.head_dim, cfg.eps)
        return time.perf_counter() - t0


def run_reference(args, rank):
    if rank != 0:
        return
    sample = OracleSample()
    per = []
    for i in range(args.warmup + args.steps):
        t = sample.time_block()
        if i >= args.warmup:
            per.append(t)
    step_s = float(np.mean(per)) * CFG.blocks
    value = 1.0 / step_s
    desc = (f"1 of {CFG.blocks} blocks of the 1024^2 step (S={CFG.tokens}) per step, float64 "
            f"numpy oracle, extrapolated x{CFG.blocks}; step-level ops (<1% of the work) omitted")
    out = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": CFG.name, "tokens": CFG.tokens, "blocks": CFG.blocks,
                   "global_batch": 1, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": sample.cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ ranks

class Ranks:
    """Barrier and max-over-ranks for the timing of independent replicas.  The
    step has no cross-device exchange: these are the only collectives."""

    def __init__(self, world: int, backend: str = "nccl", device=None):
        self.world = world
        self.dist = None
        self.device = device
        if world > 1:
            import torch.distributed as dist
            kw = {"device_id": device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.dist is None:
            return v
        dev = self.device if self.device is not None else "cpu"
        t = torch.tensor([v], device=dev, dtype=torch.float64)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def aggregate_throughput(world: int, steps: int, max_ms: float) -> float:
    """Whole-job steps/s: every replica runs `steps` steps; the slowest sets the time."""
    return world * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ GPU arm

WORKLOADS = {c.name: c for c in (synth.STEP1024, synth.EDIT1024, synth.EDIT3REF1024, synth.CFG1024,
                                  synth.GEN2048, synth.GEN2048_SCHED)}


def run_ours(args, rank, world, local_rank):
    from diffusion_transformer_text_dit_b200 import build_lib, qi
    build_lib.build()
    torch.cuda.set_device(local_rank)
    ranks = Ranks(world, "nccl", torch.device("cuda", local_rank))

    ctx = qi.Context(local_rank)
    cfg = WORKLOADS[args.workload]
    denoise = cfg.steps > 1            # the 40-step 2048^2 workload
    model, dims = build_model(ctx, qi, cfg, "cuda")
    S, H = cfg.tokens, cfg.hidden
    gd = [(g.kind, g.tokens, g.grid) for g in cfg.groups]
    ends = list(np.cumsum(cfg.group_sizes()))
    groups = qi.groups_struct(ends, cfg.group_row_sets())
    cos, sin = qi.qi_rope_tables(gd)
    cos, sin = cos.cuda(), sin.cuda()
    sig = qi.qi_sigma_schedule(40, cfg.target_tokens).tolist()
    ws = torch.empty(qi.qi_step_workspace_bytes(dims, S), dtype=torch.uint8, device="cuda")
    kv = torch.empty((cfg.blocks, 2, S, H), dtype=torch.bfloat16, device="cuda")
    txt = synth.text_features(cfg, device="cuda")
    ref = synth.ref_latents(cfg, device="cuda")
    lat0 = synth.latents(cfg, device="cuda")
    lat = lat0.clone()
    stream = torch.cuda.current_stream()
    if cfg.uncond_text:
        # true CFG: the negative prompt's sequence, run in one batch with the prompt's
        ucfg = cfg.uncond()
        S_u = ucfg.tokens
        gd_u = [(g.kind, g.tokens, g.grid) for g in ucfg.groups]
        groups_u = qi.groups_struct(list(np.cumsum(ucfg.group_sizes())), ucfg.group_row_sets())
        cos_u, sin_u = (t.cuda() for t in qi.qi_rope_tables(gd_u))
        kv_u = torch.empty((cfg.blocks, 2, S_u, H), dtype=torch.bfloat16, device="cuda")
        txt_u = synth.text_features(ucfg, device="cuda")
        ws = torch.empty(qi.qi_step_cfg_workspace_bytes(dims, S, S_u, cfg.target_tokens),
                         dtype=torch.uint8, device="cuda")

    def step(i, latents, text, mode=qi.QI_KV_NONE):
        j = i % 40
        cached = mode == qi.QI_KV_READ_PREFIX
        if cfg.uncond_text:
            sc = qi.seq_struct(None if cached else text, cfg.text_tokens, None if cached else ref,
                               groups, cos, sin, None if mode == qi.QI_KV_NONE else kv)
            su = qi.seq_struct(None if cached else txt_u, ucfg.text_tokens, None if cached else ref,
                               groups_u, cos_u, sin_u, None if mode == qi.QI_KV_NONE else kv_u)
            qi.qi_denoise_step_cfg(ctx, model, latents, sc, su, cfg.guidance, sig[j], sig[j + 1],
                                   mode, None, ws)
            return
        qi.qi_denoise_step(ctx, model, latents, None if cached else text, cfg.text_tokens,
                           None if cached else ref, groups, cos, sin, sig[j], sig[j + 1], mode,
                           None if mode == qi.QI_KV_NONE else kv, None, ws)

    def denoise_40(latents, text):
        # FlowMatch Euler over the 40-step schedule; the prefix K/V of the
        # first step are reused by the 39 later steps.  With a precision
        # schedule, attention switches to fp8 from step fp8_from_step on (the
        # prefix pass stays at full precision).
        step(0, latents, text, qi.QI_KV_WRITE_PREFIX)
        for i in range(1, 40):
            if cfg.fp8_from_step and i + 1 == cfg.fp8_from_step:
                ctx.set_attention_fp8(True)
            step(i, latents, text, qi.QI_KV_READ_PREFIX)
        ctx.set_attention_fp8(False)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)

    def timed(fn):
        ranks.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
        return ranks.max(e0.elapsed_time(e1))

    for i in range(args.warmup):
        step(i, lat, txt)
    ctx.check()

    # ---------------- device-resident timed region (profiled per kernel class)
    clocks = ClockSampler([local_rank]) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    ctx.profile(True)
    if denoise:
        n_steps = 40
        ms_max = timed(lambda: denoise_40(lat, txt))
    else:
        n_steps = args.steps
        ms_max = timed(lambda: [step(i, lat, txt) for i in range(n_steps)])
    prof = ctx.profile_read()
    ctx.profile(False)
    clk = clocks.stop() if clocks else None
    ctx.check()
    ms_per_step = ms_max / n_steps
    value = aggregate_throughput(world, n_steps, ms_max)

    # ---------------- cached-prefix steps (the pages' later denoising steps)
    extra = {}
    if not denoise:
        step(0, lat, txt, qi.QI_KV_WRITE_PREFIX)
        cms = timed(lambda: [step(i + 1, lat, txt, qi.QI_KV_READ_PREFIX) for i in range(args.steps)])
        extra["cached_step"] = {"value": aggregate_throughput(world, args.steps, cms),
                                "unit": "steps/s", "ms_per_step": cms / args.steps,
                                "note": "target rows only; prefix K/V read from the cache"}
    else:
        extra["seconds_per_40_steps"] = ms_max / 1e3

    # ---------------- end to end through the public call with host buffers
    h_lat = lat0.cpu().pin_memory()
    h_txt = txt.cpu().pin_memory()
    h_out = torch.empty_like(h_lat).pin_memory()
    d_lat = torch.empty_like(lat0)
    d_txt = torch.empty_like(txt)
    if denoise:
        # inputs copied in before the first step, the result copied out after the last
        def e2e_run():
            d_lat.copy_(h_lat, non_blocking=True)
            d_txt.copy_(h_txt, non_blocking=True)
            denoise_40(d_lat, d_txt)
            h_out.copy_(d_lat, non_blocking=True)
        h2d = (h_lat.numel() * 4 + h_txt.numel() * 2) / 40
        d2h = h_out.numel() * 4 / 40
        e2e_ms = timed(e2e_run)
        e2e = aggregate_throughput(world, 40, e2e_ms)
    else:
        def e2e_run():
            for i in range(args.steps):
                d_lat.copy_(h_lat, non_blocking=True)
                d_txt.copy_(h_txt, non_blocking=True)
                step(i, d_lat, d_txt)
                h_out.copy_(d_lat, non_blocking=True)
        h2d = h_lat.numel() * 4 + h_txt.numel() * 2
        d2h = h_out.numel() * 4
        e2e_run()
        e2e_ms = timed(e2e_run)
        e2e = aggregate_throughput(world, args.steps, e2e_ms)
    ctx.check()

    if rank != 0:
        ranks.close()
        return

    # ---------------- roofline of the dominant kernel class
    if denoise:
        w_full, w_cached = algorithmic_work(cfg, False), algorithmic_work(cfg, True)
        work = {k: (w_full[k] + 39 * w_cached[k]) / 40 for k in ("gemm_i8_ops_per_step", "attn_flops_per_step")}
    else:
        work = algorithmic_work(cfg)
    pk = peaks()
    tot = {k: v[2] for k, v in prof.items()}
    dom = max(tot, key=tot.get)
    kernels = {k: {"launches_per_step": prof[k][0] / n_steps,
                   "ms_per_step": tot[k] / n_steps,
                   "share": tot[k] / max(sum(tot.values()), 1e-9)} for k in tot if prof[k][0]}
    if dom == "attention":
        achieved = work["attn_flops_per_step"] * n_steps / (tot[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "unit": "TFLOP/s", "peak": pk["bf16_sust"],
                "peak_note": f"bf16 dense, sustained, {pk['src']}"}
    elif dom == "gemm_i8":
        achieved = work["gemm_i8_ops_per_step"] * n_steps / (tot[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "unit": "TOP/s", "peak": 2 * pk["bf16_sust"],
                "peak_note": f"int8 dense = bf16 sustained {pk['src']} x nominal int8/bf16 ratio 2"}
    else:
        achieved = None
        roof = {"bound": "hbm", "unit": "GB/s", "peak": pk["hbm"], "peak_note": pk["src"]}
    tr = kernel_traffic(dom) if not denoise and cfg is synth.STEP1024 else None
    roof.update({"kernel": dom, "achieved": achieved,
                 "frac": (achieved / roof["peak"]) if achieved else None,
                 "traffic": tr, "ms_per_step": tot[dom] / n_steps,
                 "launches_per_step": prof[dom][0] / n_steps})
    other = {}
    if prof["gemm_i8"][0]:
        a = work["gemm_i8_ops_per_step"] * n_steps / (tot["gemm_i8"] / 1e3) / 1e12
        other["gemm_i8"] = {"achieved_tops": a, "peak_tops": 2 * pk["bf16_sust"],
                            "frac": a / (2 * pk["bf16_sust"])}
    if prof["attention"][0]:
        a = work["attn_flops_per_step"] * n_steps / (tot["attention"] / 1e3) / 1e12
        other["attention"] = {"achieved_tflops": a, "peak_tflops": pk["bf16_sust"],
                              "frac": a / pk["bf16_sust"]}

    cpu = None
    if world == 1 and not args.no_cpu_baseline and cfg is synth.STEP1024:
        osamp = OracleSample()
        tb = osamp.time_block()
        v = 1.0 / (tb * cfg.blocks)
        cpu = {"value": v, "unit": "steps/s", "cores": osamp.cores, "kind": "oracle",
               "sample": (f"1 of {cfg.blocks} blocks of the 1024^2 step (S={cfg.tokens}), "
                          f"float64 numpy oracle, {tb:.1f} s, extrapolated x{cfg.blocks}")}

    desc = (f"{cfg.name}: {cfg.blocks} blocks, hidden {H}, {cfg.heads}x128 heads, MLP {cfg.mlp}, "
            f"groups {'|'.join(str(n) for n in cfg.group_sizes())} tokens, "
            + (f"true CFG with a {cfg.uncond_text}-token negative prompt in the same batch "
               f"(scale {cfg.guidance}), " if cfg.uncond_text else "")
            + ("40-step FlowMatch Euler denoise, prefix K/V cached from step 2"
               if denoise else "uncached step")
            + ", all attn/MLP Linears W8A8 (int8 GEMMs), "
            + (f"bf16 attention in steps 1-{cfg.fp8_from_step - 1} and fp8 (e4m3) attention from "
               f"step {cfg.fp8_from_step}" if cfg.fp8_from_step else "bf16 attention"))
    out = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": n_steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": desc, "tokens": S, "blocks": cfg.blocks, "global_batch": world,
                   "l2": "inputs larger than L2: ~12.8 GB of weights streamed per step",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "tensor_core_fracs": other,
        "kernels": kernels,
        "extra": extra,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": int(sum(v[0] for v in prof.values())),
        "clocks": clk,
    }
    print(json.dumps(out), flush=True)
    ranks.close()


def run_ncu_case(args):
    """A few launches of one kernel at the 1024^2 step's shapes, for ncu captures:
    gemms:     the block's four W8A8 GEMMs (QKV, out, up, down) in block order;
    gemm_down: W8A8 down projection, M = 4608, N = 4096, K = 16384 (operands
               142 MB > L2);
    attention: block-causal attention over [512 | 4096] tokens, 32 heads."""
    from diffusion_transformer_text_dit_b200 import build_lib, qi
    build_lib.build()
    ctx = qi.Context(0)
    cfg = CFG
    S, H, F = cfg.tokens, cfg.hidden, cfg.mlp
    g = torch.Generator(device="cuda").manual_seed(5)
    if args.ncu_case == "gemms":
        # the four W8A8 GEMMs of a block at the 1024^2 shapes, in block order:
        # QKV (fused norm/RoPE epilogue), out, up (+GELU), down (+gated residual)
        def w8(n, k, seed):
            w = torch.randn(n, k, device="cuda", generator=g) * 0.02
            q, s_, rs = qi.qi_prepare_w8(ctx, w)
            return q, s_, rs, torch.zeros(n, device="cuda", dtype=torch.bfloat16)
        Wqkv, Wout, Wup, Wdown = w8(3 * H, H, 1), w8(H, H, 2), w8(F, H, 3), w8(H, F, 4)
        qa = torch.randint(-128, 128, (S, F), device="cuda", generator=g, dtype=torch.int8)
        sa = torch.rand(S, device="cuda", generator=g) * 0.01 + 1e-3
        zp = torch.randint(-128, 128, (S,), device="cuda", generator=g, dtype=torch.int32)
        qa_h = qa[:, :H].contiguous()
        y = torch.empty((S, F), device="cuda", dtype=torch.bfloat16)
        x = torch.zeros((S, H), device="cuda", dtype=torch.float32)
        gate = torch.ones((2, H), device="cuda", dtype=torch.bfloat16)
        qo, ko, vo = (torch.empty((S, H), device="cuda", dtype=torch.bfloat16) for _ in range(3))
        nq = torch.ones(128, device="cuda", dtype=torch.bfloat16)
        cos_t = torch.ones((S, 64), device="cuda")
        sin_t = torch.zeros((S, 64), device="cuda")
        groups = qi.groups_struct(list(np.cumsum(cfg.group_sizes())), cfg.group_row_sets())
        import ctypes
        ep_qkv = qi.qi_epilogue()
        ep_qkv.kind = qi.QI_EPI_QKV_NORM_ROPE
        ep_qkv.hidden, ep_qkv.eps, ep_qkv.ld_out = H, 1e-6, H
        ep_qkv.norm_q = ep_qkv.norm_k = nq.data_ptr()
        ep_qkv.rope_cos, ep_qkv.rope_sin = cos_t.data_ptr(), sin_t.data_ptr()
        ep_qkv.q_out, ep_qkv.k_out, ep_qkv.v_out = qo.data_ptr(), ko.data_ptr(), vo.data_ptr()
        ep_gelu = qi.qi_epilogue()
        ep_gelu.kind = qi.QI_EPI_GELU_TANH
        ep_res = qi.qi_epilogue()
        ep_res.kind = qi.QI_EPI_GATED_RESIDUAL
        ep_res.residual, ep_res.ld_residual = x.data_ptr(), H
        ep_res.gate, ep_res.gate_ld = gate.data_ptr(), H
        ep_res.groups = ctypes.pointer(groups)
        yh = y[:, :H].contiguous()
        for _ in range(args.warmup + args.steps):
            qi.qi_w8a8_linear(ctx, qa_h, sa, zp, qi.w8_struct(*Wqkv), epilogue=ep_qkv)
            qi.qi_w8a8_linear(ctx, qa_h, sa, zp, qi.w8_struct(*Wout), y=yh)
            qi.qi_w8a8_linear(ctx, qa_h, sa, zp, qi.w8_struct(*Wup), epilogue=ep_gelu, y=y)
            qi.qi_w8a8_linear(ctx, qa, sa, zp, qi.w8_struct(*Wdown), epilogue=ep_res)
    elif args.ncu_case == "gemm_down":
        qa = torch.randint(-128, 128, (S, F), device="cuda", generator=g, dtype=torch.int8)
        sa = torch.rand(S, device="cuda", generator=g) * 0.01 + 1e-3
        zp = torch.randint(-128, 128, (S,), device="cuda", generator=g, dtype=torch.int32)
        w = torch.randn(H, F, device="cuda", generator=g) * 0.02
        q, s, rs = qi.qi_prepare_w8(ctx, w)
        del w
        b = torch.zeros(H, device="cuda", dtype=torch.bfloat16)
        ws = qi.w8_struct(q, s, rs, b)
        y = torch.empty((S, H), device="cuda", dtype=torch.bfloat16)
        for _ in range(args.warmup + args.steps):
            qi.qi_w8a8_linear(ctx, qa, sa, zp, ws, y=y)
    elif args.ncu_case == "attention":
        q = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        k = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        v = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        groups = qi.groups_struct(list(np.cumsum(cfg.group_sizes())), cfg.group_row_sets())
        o = torch.empty_like(q)
        for _ in range(args.warmup + args.steps):
            qi.qi_attn_block_causal(ctx, q, k, v, groups, o=o)
    torch.cuda.synchronize()
    ctx.check()
    print(json.dumps({"ncu_case": args.ncu_case, "launches": args.warmup + args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default=synth.STEP1024.name,
                    help="step_1024px (default): one uncached 1024^2 step per iteration, plus "
                         "a cached-prefix measurement; edit_1024px: the edit sequence; "
                         "edit_3ref_1024px: an edit with three reference images; "
                         "cfg_1024px: true classifier-free guidance (prompt + negative prompt "
                         "as one batch); "
                         "denoise40_2048px: the full 40-step 2048^2 denoise; "
                         "denoise40_2048px_sched: the same with the pages' precision schedule "
                         "(fp8 attention from step 8)")
    ap.add_argument("--ncu-case", choices=("gemms", "gemm_down", "attention"), default=None,
                    help="launch one kernel a few times (for ncu captures) and exit")
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args)
        return
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
