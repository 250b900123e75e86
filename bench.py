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
        out = {k: a[k] + b[k] for k in a}
        out["gemv_bytes_per_step"] = a["gemv_bytes_per_step"]   # one time conditioning
        return out
    H, F, d, h = cfg.hidden, cfg.mlp, cfg.head_dim, cfg.heads
    rows = cfg.target_tokens if cached else cfg.tokens
    # 2 x rows x (weights) of each block Linear, split by its precision
    sizes = {"qk": 2 * H * H, "v": H * H, "out": H * H, "up": F * H, "down": H * F}
    i8_ops = bf16_block = mx_weights = 0
    for l in range(cfg.blocks):
        for name, kind in synth.linear_precision(cfg, l).items():
            if kind == "w8":
                i8_ops += 2 * rows * sizes[name]
            else:   # BF16 weights, or MXFP4 weights decoded to bf16 in the GEMM
                bf16_block += 2 * rows * sizes[name]
            if kind == "mx":
                mx_weights += sizes[name]
    ends = np.cumsum(cfg.group_sizes())
    starts = np.concatenate([[0], ends[:-1]])
    if cached:
        pairs = int(cfg.target_tokens * ends[-1])
    else:
        pairs = int(sum((e - s) * e for s, e in zip(starts, ends)))   # query x visible keys
    attn_flops = 4 * d * h * pairs
    # HBM bytes of the four activation quantizers per row: LN1 reads the fp32
    # residual (4H) and writes int8 codes (H); the attention-output quantizer
    # reads bf16 (2H) and writes H; LN2 reads the residual and the output
    # projection (4H + 2H) and writes the codes (H) (the down projection's
    # epilogue adds the output projection's gated term to the stream itself);
    # the GELU-output quantizer reads 2F and writes F.  Plus 8 bytes (scale,
    # zero point) per row and quantizer, and the final LayerNorm (4H in, 2H out
    # per target row).
    quant = cfg.target_tokens * 6 * H
    for l in range(cfg.blocks):
        pr = synth.linear_precision(cfg, l)
        w8 = {k: v == "w8" for k, v in pr.items()}
        b = 4 * H                                             # LN1 reads the fp32 residual
        b += (H + 8) if w8["qk"] else 0                       # ... writes codes for W8A8 q, k
        b += 2 * H if not (w8["qk"] and w8["v"]) else 0       # ... and bf16 u for a BF16 part
        b += (3 * H + 8) if w8["out"] else 0                  # attention-output quantizer
        b += 6 * H + ((H + 8) if w8["up"] else 2 * H)         # LN2 with the residual add
        b += (3 * F + 8) if w8["down"] else 0                 # GELU-output quantizer
        quant += rows * b
    # GEMV weight bytes: the adaLN rows of every block (6H x H bf16), the final
    # adaLN (2H x H) and the timestep MLP (H x 256 + H x H)
    gemv = 2 * (cfg.blocks * 6 * H * H + 2 * H * H + H * 256 + H * H)
    # bf16 Linears: text and reference in-projections (uncached), image
    # in-projection and proj_out of the target rows
    P, N = cfg.patch, cfg.target_tokens
    bf16 = 2 * N * P * H * 2
    if not cached:
        bf16 += 2 * cfg.text_tokens * H * H + 2 * (cfg.prefix_tokens - cfg.text_tokens) * P * H
    bf16 += bf16_block
    return {
        "gemm_i8_ops_per_step": i8_ops,
        "attn_flops_per_step": cfg.blocks * attn_flops,
        "attn_pairs_per_head": pairs,
        "quant_bytes_per_step": quant,
        "gemv_bytes_per_step": gemv,
        "bf16_linear_flops_per_step": bf16,
        # expanding MXFP4 Linears to bf16: codes (0.5 B) + scales (1/32 B) in,
        # bf16 (2 B) out per weight
        "mx_expand_bytes_per_step": mx_weights * (0.5 + 1 / 32 + 2),
    }


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling every 100 ms; the summary keeps the samples whose
    timestamps fall inside the timed region (window() marks it)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = set(gpus)
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def window(self, t0, t1):
        """Wall-clock bounds (time.time()) of the timed region."""
        self.t0, self.t1 = t0, t1

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
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
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                if int(f[1]) not in self.gpus:
                    continue
                rows.append((ts, float(f[2]), float(f[3]),
                             {n for n, v in zip(names, f[6:10]) if v.lower().startswith("active")}))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.05 <= r[0] <= self.t1 + 0.05]
        use = inside if inside else rows
        sm = [r[1] for r in use]
        reasons = set().union(*[r[3] for r in use]) if use else set()
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(r[2] for r in use) if use else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "in_timed_region": bool(inside)}


# ------------------------------------------------------------------ model setup

def build_model(ctx, qi, cfg, device, mx_expand=True):
    """The model on the device.  MXFP4 Linears expand into one shared bf16
    scratch before their GEMMs unless mx_expand is False (then the GEMM
    decodes the codes tile by tile in shared memory)."""
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, cfg.blocks)
    scratch = qi.mx_expand_scratch(dims, device) if cfg.precision == "mxfp4" and mx_expand else None
    blocks = []
    for l in range(cfg.blocks):
        wts = synth.block_weights(cfg, l, device=device)
        blocks.append(qi.BlockWeights(ctx, wts, device=device,
                                      precision=synth.linear_precision(cfg, l), mx_expand=scratch))
        del wts
    glob = synth.model_weights(cfg, device=device)
    return qi.Model(ctx, dims, blocks, glob, device=device), dims


PEAKS_INT8 = os.path.join(ROOT, "profiles", "peaks_int8.json")


def peaks():
    """Roofline denominators.  HBM and dense bf16: the machine's measured copy and
    cuBLAS figures (MEASURED_PEAKS.json), else the recorded fallback.  Dense
    int8: cuBLASLt's int8 GEMM (torch._int_mm at 8192^3) measured by
    `bench.py --measure-peaks` into profiles/peaks_int8.json, burst and
    sustained (4 s), else 2 x bf16 (the nominal ratio)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        pk = {"hbm": d["hbm_gbs"], "bf16": d["bf16_tflops"],
              "bf16_sust": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    else:
        pk = {"hbm": 6650.0, "bf16": 1590.0, "bf16_sust": 1400.0, "src": "fallback"}
    if os.path.exists(PEAKS_INT8):
        dd = json.load(open(PEAKS_INT8))
        d = dd["int8_cublaslt"]
        pk.update({"int8": d["burst_tops"], "int8_sust": d["sustained_tops"],
                   "int8_src": "measured cuBLASLt int8 GEMM 8192^3 (profiles/peaks_int8.json)"})
        # the tensor pipe's own rate per MHz (back-to-back tcgen05.mma probe),
        # to put a kernel against the pipe at the clock its run actually held
        for kind in ("int8", "bf16"):
            pr = dd.get(f"{kind}_probe")
            if pr and pr["clocks"].get("sm_mhz"):
                pk[f"{kind}_pipe_per_mhz"] = pr["sustained_tops"] / pr["clocks"]["sm_mhz"]
    else:
        pk.update({"int8": 2 * pk["bf16"], "int8_sust": 2 * pk["bf16_sust"],
                   "int8_src": f"2 x bf16 {pk['src']} (nominal int8/bf16 ratio)"})
    return pk


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
    """The CPU oracle as it stands, on a bounded sample of the 1024^2 step
    (S = 4608): one block on its last `rows` rows (target tokens), which
    attend over all S keys; the K/V of the earlier rows are computed once at
    set-up by the same oracle block (untimed).  The block's cost is linear in
    its rows (the Linears per row, the attention per query row), so a sample
    extrapolates to the step by (S / rows) x blocks.  Target rows attend over
    all 4608 keys against 4153 on average over the sequence, so the
    extrapolation overstates the step's attention part by about 10%."""

    def __init__(self, rows: int = CFG.tokens // 4):
        from oracle import qi_oracle as O
        self.O = O
        try:
            from threadpoolctl import threadpool_info
            self.cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        except Exception:
            self.cores = os.cpu_count()
        cfg = CFG
        self.rows = rows
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
        self.split = cfg.tokens - rows
        sp = self.split
        _, self.kv = O.dit_block(self.x[:sp], self.pw, self.mod, self.rs[:sp], self.gid[:sp],
                                 self.gid[:sp], self.cos[:sp], self.sin[:sp], cfg.heads,
                                 cfg.head_dim, cfg.eps, return_kv=True)

    def time_sample(self) -> float:
        cfg, sp = CFG, self.split
        t0 = time.perf_counter()
        self.O.dit_block(self.x[sp:], self.pw, self.mod, self.rs[sp:], self.gid[sp:], self.gid,
                         self.cos[sp:], self.sin[sp:], cfg.heads, cfg.head_dim, cfg.eps,
                         kv_prefix=self.kv)
        return time.perf_counter() - t0

    def step_seconds(self, sample_s: float) -> float:
        return sample_s * (CFG.tokens / self.rows) * CFG.blocks

    def describe(self, sample_s: float) -> str:
        return (f"oracle block (float64 numpy) on the last {self.rows} of {CFG.tokens} rows of the "
                f"1024^2 step (target rows, attending over all keys; the earlier rows' K/V from an "
                f"untimed set-up run of the same block), {sample_s:.1f} s, extrapolated "
                f"x{CFG.tokens / self.rows:g} rows x{CFG.blocks} blocks; step-level ops "
                f"(<1% of the work) omitted")


def run_reference(args, rank):
    if rank != 0:
        return
    # each step times one sample (~5 s on 16 cores), so W + K steps end
    # within a few minutes
    sample = OracleSample(rows=CFG.tokens // 8)
    per = []
    for i in range(args.warmup + args.steps):
        t = sample.time_sample()
        if i >= args.warmup:
            per.append(t)
    mean_s = float(np.mean(per))
    step_s = sample.step_seconds(mean_s)
    value = 1.0 / step_s
    desc = sample.describe(mean_s) + " (mean of the timed steps)"
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
                                  synth.GEN2048, synth.GEN2048_SCHED, synth.STEP1024_PAGES,
                                  synth.STEP1024_MXFP4)}


def weight_bytes_per_step(cfg) -> float:
    """HBM bytes of weights one step streams: the block Linears at their
    storage width (int8 1 B, bf16 2 B, MXFP4 4.25 bits) and the bf16 adaLN rows."""
    H, F = cfg.hidden, cfg.mlp
    sizes = {"qk": 2 * H * H, "v": H * H, "out": H * H, "up": F * H, "down": H * F}
    width = {"w8": 1.0, "bf16": 2.0, "mx": 4.25 / 8}
    lin = sum(sizes[n] * width[k] for l in range(cfg.blocks)
              for n, k in synth.linear_precision(cfg, l).items())
    return lin + cfg.blocks * 6 * H * H * 2


def run_ours(args, rank, world, local_rank):
    from diffusion_transformer_text_dit_b200 import build_lib, qi
    build_lib.build()
    torch.cuda.set_device(local_rank)
    ranks = Ranks(world, "nccl", torch.device("cuda", local_rank))

    ctx = qi.Context(local_rank)
    cfg = WORKLOADS[args.workload]
    denoise = cfg.steps > 1            # the 40-step 2048^2 workload
    model, dims = build_model(ctx, qi, cfg, "cuda", mx_expand=not args.mx_tile_decode)
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

    def run_timed():
        if denoise:
            return 40, timed(lambda: denoise_40(lat, txt))
        return args.steps, timed(lambda: [step(i, lat, txt) for i in range(args.steps)])

    # ---------------- device-resident timed region: the headline, with no
    # per-launch instrumentation (launches are only counted)
    clocks = ClockSampler([local_rank]) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    ctx.profile(False)
    t_start = time.time()
    n_steps, ms_max = run_timed()
    if clocks:
        clocks.window(t_start, time.time())
    counts = ctx.profile_read()
    clk = clocks.stop() if clocks else None
    ctx.check()
    ms_per_step = ms_max / n_steps
    value = aggregate_throughput(world, n_steps, ms_max)

    # ---------------- end to end through the public call with host buffers,
    # right after the headline so that both meet the GPU in the same state
    # (a 1 kW part settles to lower clocks under the power cap as a run goes on)
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
        # every step's inputs come in from pinned host memory and its latents
        # go back out; the copies run on a second stream into two alternating
        # device buffers, so step i+1's inputs land while step i computes
        copy_st = torch.cuda.Stream()
        d_lats, d_txts = [d_lat, torch.empty_like(lat0)], [d_txt, torch.empty_like(txt)]
        h_outs = [h_out, torch.empty_like(h_lat).pin_memory()]
        landed = [torch.cuda.Event() for _ in range(2)]
        stepped = [torch.cuda.Event() for _ in range(2)]
        freed = [torch.cuda.Event() for _ in range(2)]

        def e2e_run():
            copy_st.wait_stream(stream)
            for i in range(args.steps):
                b = i % 2
                with torch.cuda.stream(copy_st):
                    if i >= 2:
                        copy_st.wait_event(freed[b])       # step i-2 and its read-back are done
                    d_lats[b].copy_(h_lat, non_blocking=True)
                    d_txts[b].copy_(h_txt, non_blocking=True)
                    landed[b].record(copy_st)
                stream.wait_event(landed[b])
                step(i, d_lats[b], d_txts[b])
                stepped[b].record(stream)
                with torch.cuda.stream(copy_st):
                    copy_st.wait_event(stepped[b])
                    h_outs[b].copy_(d_lats[b], non_blocking=True)
                    freed[b].record(copy_st)
            stream.wait_stream(copy_st)                   # the last read-back ends the region
        h2d = h_lat.numel() * 4 + h_txt.numel() * 2
        d2h = h_out.numel() * 4
        e2e_run()
        e2e_ms = timed(e2e_run)
        e2e = aggregate_throughput(world, args.steps, e2e_ms)
    ctx.check()

    # ---------------- the same steps again with every launch bracketed by CUDA
    # events on its stream: per-kernel-class device time for the rooflines
    ctx.profile(True)
    _, ms_prof = run_timed()
    prof = ctx.profile_read()
    ctx.profile(False)
    ctx.check()

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

    if rank != 0:
        ranks.close()
        return

    # ---------------- rooflines: the dominant kernel class, the tensor-core
    # classes, and the whole step (sum of every class's roofline time)
    if denoise:
        w_full, w_cached = algorithmic_work(cfg, False), algorithmic_work(cfg, True)
        work = {k: (w_full[k] + 39 * w_cached[k]) / 40 for k in w_full}
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
        roof = {"bound": "tensor", "unit": "TOP/s", "peak": pk["int8_sust"],
                "peak_note": f"int8 dense, sustained: {pk['int8_src']}"}
    elif dom == "gemm_bf16":
        # BF16 Linears (and MXFP4 weights decoded to bf16 inside the GEMM)
        achieved = work["bf16_linear_flops_per_step"] * n_steps / (tot[dom] / 1e3) / 1e12
        roof = {"bound": "tensor", "unit": "TFLOP/s", "peak": pk["bf16_sust"],
                "peak_note": f"bf16 dense, sustained, {pk['src']}"}
    else:
        achieved = None
        roof = {"bound": "hbm", "unit": "GB/s", "peak": pk["hbm"], "peak_note": pk["src"]}
    tr = kernel_traffic(dom) if not denoise and cfg is synth.STEP1024 else None
    roof.update({"kernel": dom, "achieved": achieved,
                 "frac": (achieved / roof["peak"]) if achieved else None,
                 "traffic": tr, "ms_per_step": tot[dom] / n_steps,
                 "launches_per_step": prof[dom][0] / n_steps,
                 "timing": "CUDA events around each launch on its stream, in a second run of "
                           "the same steps (the headline run is not instrumented)"})
    other = {}
    if prof["gemm_i8"][0]:
        a = work["gemm_i8_ops_per_step"] * n_steps / (tot["gemm_i8"] / 1e3) / 1e12
        other["gemm_i8"] = {"achieved_tops": a, "peak_tops": pk["int8_sust"],
                            "frac": a / pk["int8_sust"], "frac_of_burst": a / pk["int8"],
                            "peak_note": pk["int8_src"]}
    if prof["attention"][0]:
        a = work["attn_flops_per_step"] * n_steps / (tot["attention"] / 1e3) / 1e12
        other["attention"] = {"achieved_tflops": a, "peak_tflops": pk["bf16_sust"],
                              "frac": a / pk["bf16_sust"], "frac_of_burst": a / pk["bf16"],
                              "peak_note": f"bf16 dense {pk['src']}"}
    if prof["gemm_bf16"][0] and work["bf16_linear_flops_per_step"] and \
            tot["gemm_bf16"] > 0.05 * sum(tot.values()):   # block Linears in BF16 / MXFP4
        a = work["bf16_linear_flops_per_step"] * n_steps / (tot["gemm_bf16"] / 1e3) / 1e12
        other["gemm_bf16"] = {"achieved_tflops": a, "peak_tflops": pk["bf16_sust"],
                              "frac": a / pk["bf16_sust"], "frac_of_burst": a / pk["bf16"],
                              "peak_note": f"bf16 dense {pk['src']}"}
    mhz = (clk or {}).get("sm_mhz")
    for cls, kind, key in (("gemm_i8", "int8", "achieved_tops"), ("attention", "bf16", "achieved_tflops"),
                           ("gemm_bf16", "bf16", "achieved_tflops")):
        if cls in other and mhz and pk.get(f"{kind}_pipe_per_mhz"):
            pipe = pk[f"{kind}_pipe_per_mhz"] * mhz
            other[cls]["tensor_pipe_at_bench_clock"] = pipe
            other[cls]["frac_of_tensor_pipe_at_bench_clock"] = other[cls][key] / pipe
    # whole step: each class's algorithmic work at its own roofline, summed,
    # against the measured (uninstrumented) step time
    ideal = {
        "gemm_i8": work["gemm_i8_ops_per_step"] / (pk["int8_sust"] * 1e12) * 1e3,
        "attention": work["attn_flops_per_step"] / (pk["bf16_sust"] * 1e12) * 1e3,
        "quant": work["quant_bytes_per_step"] / (pk["hbm"] * 1e9) * 1e3,
        "gemv": work["gemv_bytes_per_step"] / (pk["hbm"] * 1e9) * 1e3,
        "gemm_bf16": work["bf16_linear_flops_per_step"] / (pk["bf16_sust"] * 1e12) * 1e3,
    }
    if cfg.precision == "mxfp4" and not args.mx_tile_decode:
        ideal["other"] = work["mx_expand_bytes_per_step"] / (pk["hbm"] * 1e9) * 1e3
    step_roof = {"ideal_ms": sum(ideal.values()), "measured_ms": ms_per_step,
                 "frac": sum(ideal.values()) / ms_per_step,
                 "ideal_ms_by_class": ideal,
                 "note": "sum over kernel classes of algorithmic work / peak (int8 and bf16 "
                         "sustained tensor peaks, HBM copy bandwidth) over the measured step"}

    cpu = None
    if world == 1 and not args.no_cpu_baseline and cfg is synth.STEP1024:
        osamp = OracleSample(rows=CFG.tokens // 4)
        ts = float(np.mean([osamp.time_sample() for _ in range(3)]))
        v = 1.0 / osamp.step_seconds(ts)
        cpu = {"value": v, "unit": "steps/s", "cores": osamp.cores, "kind": "oracle",
               "sample": osamp.describe(ts) + " (mean of 3 samples)"}

    desc = (f"{cfg.name}: {cfg.blocks} blocks, hidden {H}, {cfg.heads}x128 heads, MLP {cfg.mlp}, "
            f"groups {'|'.join(str(n) for n in cfg.group_sizes())} tokens, "
            + (f"true CFG with a {cfg.uncond_text}-token negative prompt in the same batch "
               f"(scale {cfg.guidance}), " if cfg.uncond_text else "")
            + ("40-step FlowMatch Euler denoise, prefix K/V cached from step 2"
               if denoise else "uncached step")
            + {"w8a8": ", all attn/MLP Linears W8A8 (int8 GEMMs), ",
               "pages": ", the pages' precision layout (W8A8 q, k, MLP up/down in blocks 2-29 on "
                        "int8 GEMMs; v, out projection and all Linears of blocks 0, 1, 30, 31 in "
                        "BF16 on bf16 GEMMs), ",
               "mxfp4": (", all attn/MLP Linears with MXFP4 weights (synthetic checkpoint) "
                         + ("decoded to bf16 inside bf16 GEMMs" if args.mx_tile_decode else
                            "expanded to bf16 (one Linear at a time, into a shared scratch) "
                            "before bf16 GEMMs")
                         + ", bf16 activations, ")}[cfg.precision]
            + (f"bf16 attention in steps 1-{cfg.fp8_from_step - 1} and fp8 (e4m3) attention from "
               f"step {cfg.fp8_from_step}" if cfg.fp8_from_step else "bf16 attention"))
    out = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": n_steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if cfg.precision in ("mxfp4", "bf16") else "int8",
        "data": "synthetic",
        "config": {"workload": desc, "tokens": S, "blocks": cfg.blocks, "global_batch": world,
                   "l2": f"inputs larger than L2: ~{weight_bytes_per_step(cfg) / 1e9:.1f} GB of "
                         f"weights streamed per step",
                   "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "tensor_core_fracs": other,
        "step_roofline": step_roof,
        "kernels": kernels,
        "extra": extra,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h,
                "note": ("qi_denoise_step from pinned host buffers: inputs copied in before "
                         "step 1, latents read back after step 40" if denoise else
                         "qi_denoise_step from pinned host buffers: every step copies its inputs "
                         "in and reads its latents back, on a second stream into two "
                         "alternating device buffers (the next step's inputs land while this "
                         "one computes)")},
        "gpu_launches": int(sum(v[0] for v in counts.values())),
        "clocks": clk,
    }
    print(json.dumps(out), flush=True)
    ranks.close()


def run_ncu_case(args):
    """A few launches of one kernel at the 1024^2 step's shapes, for ncu captures:
    gemms:     the block's four W8A8 GEMMs (QKV, out, up, down) in block order;
    gemm_down: W8A8 down projection, M = 4608, N = 4096, K = 16384 (operands
               142 MB > L2);
    attention: block-causal attention over [512 | 4096] tokens, 32 heads;
    block:     one whole block at S = 4608 (4 quantizer launches, 4 GEMMs, attention);
    gemv:      the time conditioning of an 8-block model (3 GEMV launches);
    mx_expand: MXFP4 -> bf16 expansion of a 16384 x 4096 weight."""
    import ctypes as C
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
    elif args.ncu_case == "block":
        # one whole block at the 1024^2 shapes (S = 4608): every quantizer form
        # (LayerNorm with and without the residual add, range-fed on the
        # attention and GELU outputs), the four GEMMs and the attention
        wts = synth.block_weights(cfg, 0, device="cuda")
        bw = qi.BlockWeights(ctx, wts)
        del wts
        dims = qi.dims_struct(H, cfg.heads, F, cfg.patch, 1)
        groups = qi.groups_struct(list(np.cumsum(cfg.group_sizes())), cfg.group_row_sets())
        cos, sin = (t.cuda() for t in qi.qi_rope_tables([(gr.kind, gr.tokens, gr.grid) for gr in cfg.groups]))
        x0 = synth.hidden_states(cfg, S, device="cuda")
        mod = synth.mod_table(cfg, device="cuda")
        kl = torch.empty((S, H), dtype=torch.bfloat16, device="cuda")
        vl = torch.empty_like(kl)
        ws = torch.empty(qi.qi_block_workspace_bytes(dims, S), dtype=torch.uint8, device="cuda")
        x = x0.clone()
        for _ in range(args.warmup + args.steps):
            x.copy_(x0)
            qi.qi_dit_block_forward(ctx, dims, bw.struct, x, 0, mod, groups, cos, sin, kl, vl,
                                    qi.QI_KV_NONE, ws)
    elif args.ncu_case == "gemv":
        # the time conditioning of an 8-block model (1.6 GB of adaLN weights;
        # a 32-block step reads 4x as many): one GEMV launch covers every
        # block's adaLN rows and the final adaLN
        nb = 8
        wts = synth.block_weights(cfg, 0, device="cuda")
        bw = qi.BlockWeights(ctx, wts)
        del wts
        mods = [synth.linear_weight(cfg.weight_seed, ("ncu_mod", l), 6 * H, H, "cuda").to(torch.bfloat16)
                for l in range(nb)]
        structs = []
        for l in range(nb):
            st_ = qi.qi_block_weights.from_buffer_copy(bw.struct)
            st_.mod = qi.bf16_struct(mods[l])
            structs.append(st_)
        dims = qi.dims_struct(H, cfg.heads, F, cfg.patch, nb)
        model = qi.Model.__new__(qi.Model)
        model.dims = dims
        model.g = {k: v.to(torch.bfloat16).contiguous() for k, v in synth.model_weights(cfg, device="cuda").items()}
        arr = (qi.qi_block_weights * nb)(*structs)
        m = qi.qi_model()
        m.dims = dims
        m.blocks = C.cast(arr, C.POINTER(qi.qi_block_weights))
        for name in ("t1", "t2", "img_in", "txt_in", "final_mod", "proj_out"):
            setattr(m, name, qi.bf16_struct(model.g[name], model.g[name + "_b"]))
        model.struct = m
        model._arr = arr
        ws = torch.empty(qi.qi_step_workspace_bytes(dims, 8), dtype=torch.uint8, device="cuda")
        bm = torch.empty((nb, 2, 6 * H), dtype=torch.bfloat16, device="cuda")
        fm = torch.empty((2, 2 * H), dtype=torch.bfloat16, device="cuda")
        for i in range(args.warmup + args.steps):
            qi.qi_time_conditioning(ctx, model, 0.5 + 0.01 * i, bm, fm, ws)
    elif args.ncu_case == "mx_expand":
        # MXFP4 -> bf16 expansion of the MLP up projection's weights
        pk = torch.randint(0, 256, (F, H // 2), dtype=torch.uint8, device="cuda", generator=g)
        sc = torch.randint(118, 122, (F, H // 32), dtype=torch.uint8, device="cuda", generator=g)
        w = torch.empty((F, H), dtype=torch.bfloat16, device="cuda")
        for _ in range(args.warmup + args.steps):
            qi.qi_mxfp4_expand_bf16(ctx, pk, sc, out=w)
    elif args.ncu_case == "attention":
        q = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        k = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        v = (torch.randn(S, H, device="cuda", generator=g)).to(torch.bfloat16)
        groups = qi.groups_struct(list(np.cumsum(cfg.group_sizes())), cfg.group_row_sets())
        o = torch.empty_like(q)
        # the key-range split as in the step (whose blocks use their workspace)
        _, need = qi.qi_attn_split_plan(S, cfg.heads, groups,
                                        torch.cuda.get_device_properties(0).multi_processor_count)
        if need:
            qi.qi_ctx_reserve_attention(ctx, need)
        for _ in range(args.warmup + args.steps):
            qi.qi_attn_block_causal(ctx, q, k, v, groups, o=o)
    torch.cuda.synchronize()
    ctx.check()
    print(json.dumps({"ncu_case": args.ncu_case, "launches": args.warmup + args.steps}))


def measure_peaks(args):
    """Dense tensor peaks on this GPU, each as a burst (20 launches after 3
    warm-up) and sustained (back-to-back launches for 4 s, SM clock sampled):
      int8_cublaslt  cuBLASLt int8 GEMM, torch._int_mm [8192 x 8192] x [8192 x 8192]
      bf16_cublas    cuBLAS bf16 GEMM, torch.matmul at 8192^3
      int8_probe / bf16_probe  libqi's tensor-pipe probe: back-to-back
                     tcgen05.mma on shared-memory operands on every SM (the
                     pipe's own rate at the clock it runs at)
    Writes profiles/peaks_int8.json (read by the roofline) and prints it."""
    from diffusion_transformer_text_dit_b200 import build_lib, qi
    build_lib.build()
    torch.cuda.set_device(0)
    ctx = qi.Context(0)
    st = torch.cuda.current_stream()
    n = 8192
    g = torch.Generator(device="cuda").manual_seed(0)
    a8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device="cuda", generator=g)
    b8 = torch.randint(-128, 128, (n, n), dtype=torch.int8, device="cuda", generator=g).t()
    ab = torch.randn(n, n, device="cuda", generator=g).to(torch.bfloat16)
    bb = torch.randn(n, n, device="cuda", generator=g).to(torch.bfloat16).t()
    probe_ops = {True: None, False: None}

    def probe(i8):
        probe_ops[i8] = qi.qi_debug_mma_probe(ctx, i8, 20000)

    cases = {"int8_cublaslt": (lambda: torch._int_mm(a8, b8), 2 * n ** 3),
             "bf16_cublas": (lambda: torch.matmul(ab, bb), 2 * n ** 3),
             "int8_probe": (lambda: probe(True), None),
             "bf16_probe": (lambda: probe(False), None)}
    out = {"gpu": torch.cuda.get_device_name(0),
           "date": datetime.datetime.now(datetime.timezone.utc).isoformat(timespec="seconds"),
           "command": "python bench.py --measure-peaks"}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for name, (fn, ops) in cases.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0.record(st)
        for _ in range(20):
            fn()
        e1.record(st)
        torch.cuda.synchronize()
        ops = ops if ops is not None else probe_ops[name.startswith("int8")]
        burst = ops * 20 / (e0.elapsed_time(e1) / 1e3) / 1e12
        clocks = ClockSampler([0])
        clocks.start()
        time.sleep(0.3)
        e0.record(st)
        t_start = time.time()
        t_end = t_start + 4.0
        launches = 0
        while time.time() < t_end:
            for _ in range(8):
                fn()
            launches += 8
            torch.cuda.synchronize()
        e1.record(st)
        torch.cuda.synchronize()
        clocks.window(t_start, time.time())
        clk = clocks.stop()
        sust = ops * launches / (e0.elapsed_time(e1) / 1e3) / 1e12
        out[name] = {"burst_tops": burst, "sustained_tops": sust, "sustained_seconds":
                     e0.elapsed_time(e1) / 1e3, "ops_per_launch": ops, "clocks": clk}
    ctx.check()
    with open(PEAKS_INT8, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=tuple(WORKLOADS), default=synth.STEP1024.name,
                    help="step_1024px (default): one uncached 1024^2 step per iteration, plus "
                         "a cached-prefix measurement; step_1024px_pagesmask: the same step with "
                         "the pages' W8A8/BF16 layout; edit_1024px: the edit sequence; "
                         "edit_3ref_1024px: an edit with three reference images; "
                         "cfg_1024px: true classifier-free guidance (prompt + negative prompt "
                         "as one batch); "
                         "denoise40_2048px: the full 40-step 2048^2 denoise; "
                         "denoise40_2048px_sched: the same with the pages' precision schedule "
                         "(fp8 attention from step 8); step_1024px_mxfp4: the 1024^2 step with "
                         "MXFP4 weights and bf16 activations")
    ap.add_argument("--mx-tile-decode", action="store_true",
                    help="step_1024px_mxfp4: decode the MXFP4 codes inside the GEMM (tile by "
                         "tile in shared memory) instead of expanding each Linear to bf16 first")
    ap.add_argument("--ncu-case", choices=("gemms", "gemm_down", "attention", "block", "gemv",
                                           "mx_expand"),
                    default=None,
                    help="launch one kernel a few times (for ncu captures) and exit")
    ap.add_argument("--measure-peaks", action="store_true",
                    help="measure dense int8 / bf16 tensor peaks (cuBLASLt, cuBLAS and libqi's "
                         "tcgen05 probe) into profiles/peaks_int8.json and exit")
    args = ap.parse_args()
    if args.measure_peaks:
        measure_peaks(args)
        return
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
