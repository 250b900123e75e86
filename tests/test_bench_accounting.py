"""The bench's algorithmic work per step (the numerators of every roofline
fraction it reports), checked on the CPU against the workloads' shapes: the
block Linears' operations split by precision, the visible query-key pairs of
the block-causal mask, and the MXFP4 expansion bytes."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from diffusion_transformer_text_dit_b200 import synth  # noqa: E402

H, F, HEADS, D = 4096, 16384, 32, 128


def test_step_1024px_work():
    w = bench.algorithmic_work(synth.STEP1024)
    S = 512 + 4096
    # q | k | v (3H x H), out (H x H), up (F x H), down (H x F), 32 blocks
    assert w["gemm_i8_ops_per_step"] == 2 * S * (3 * H * H + H * H + F * H + H * F) * 32
    assert abs(w["gemm_i8_ops_per_step"] / 1e12 - 59.4) < 0.05
    # text rows see the text; image rows see everything
    pairs = 512 * 512 + 4096 * S
    assert w["attn_pairs_per_head"] == pairs == 19_136_512
    assert w["attn_flops_per_step"] == 4 * D * HEADS * pairs * 32
    assert w["mx_expand_bytes_per_step"] == 0


def test_cached_step_processes_target_rows_only():
    w = bench.algorithmic_work(synth.STEP1024, cached=True)
    assert w["gemm_i8_ops_per_step"] == 2 * 4096 * (4 * H * H + 2 * F * H) * 32
    assert w["attn_pairs_per_head"] == 4096 * 4608


def test_pagesmask_splits_the_linears_by_precision():
    cfg = synth.STEP1024_PAGES
    w = bench.algorithmic_work(cfg)
    S = 4608
    # W8A8: q, k (2H x H) and both MLP Linears in blocks 2..29; BF16: the rest
    i8 = 2 * S * (2 * H * H + 2 * F * H) * 28
    bf16_block = 2 * S * (4 * H * H + 2 * F * H) * 32 - i8
    assert w["gemm_i8_ops_per_step"] == i8
    # plus the step-level BF16 Linears: img_in and proj_out (4096 target rows,
    # patch dim 64) and txt_in (512 text rows, H x H)
    step_level = 2 * 4096 * 64 * H * 2 + 2 * 512 * H * H
    assert w["bf16_linear_flops_per_step"] == bf16_block + step_level


def test_mxfp4_expansion_bytes():
    w = bench.algorithmic_work(synth.STEP1024_MXFP4)
    assert w["gemm_i8_ops_per_step"] == 0
    weights = (4 * H * H + 2 * F * H) * 32
    assert w["mx_expand_bytes_per_step"] == weights * (0.5 + 1 / 32 + 2)
    assert abs(w["mx_expand_bytes_per_step"] / 1e9 - 16.3) < 0.05


def test_cfg_counts_both_sequences_and_one_time_conditioning():
    cfg = synth.CFG1024
    w = bench.algorithmic_work(cfg)
    a = bench.algorithmic_work(cfg.replace(uncond_text=0))
    b = bench.algorithmic_work(cfg.uncond())
    assert w["gemm_i8_ops_per_step"] == a["gemm_i8_ops_per_step"] + b["gemm_i8_ops_per_step"]
    assert w["gemv_bytes_per_step"] == a["gemv_bytes_per_step"]


class _Done:
    """Stands in for the finished nvidia-smi process and its reader thread."""

    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0

    def join(self, timeout=None):
        pass


def test_clock_summary_keeps_the_timed_region():
    """Only samples stamped inside the timed region count: the idle clock
    before it and a throttle reason after it are left out."""
    import datetime
    cs = bench.ClockSampler([0])
    cs.proc, cs.t = _Done(), _Done()
    t0 = datetime.datetime(2026, 1, 1, 12, 0, 0).timestamp()

    def line(dt, mhz, gpu=0, power_cap="Not Active", thermal="Not Active"):
        ts = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return f"{ts}, {gpu}, {mhz}, 1965, 900.0, 0x4, Not Active, Not Active, {thermal}, {power_cap}"

    cs.lines = [line(-0.3, 1965), line(0.1, 1650, power_cap="Active"), line(0.2, 1640),
                line(0.3, 1700, gpu=1, thermal="Active"), line(0.4, 1660), line(0.9, 1965, thermal="Active")]
    cs.window(t0, t0 + 0.5)
    out = cs.stop()
    assert out["samples"] == 3 and out["in_timed_region"]
    assert out["sm_mhz"] == 1650 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_a_window_uses_every_sample():
    cs = bench.ClockSampler([0])
    cs.proc, cs.t = _Done(), _Done()
    cs.lines = ["2026/01/01 12:00:00.100, 0, 1800, 1965, 700.0, 0x0, Not Active, Not Active, "
                "Not Active, Not Active", "garbage"]
    out = cs.stop()
    assert out["samples"] == 1 and not out["in_timed_region"] and out["reasons"] == []


def test_quantizer_bytes_of_the_1024px_step():
    """Per row and block: LN1 4H + H + 8, attention-output quantizer
    3H + 8, LN2 6H + H + 8 (residual and output projection in, codes out),
    GELU-output quantizer 3F + 8; plus the final LayerNorm 6H per target row."""
    w = bench.algorithmic_work(synth.STEP1024)
    S = 4608
    per_row = (5 * H + 8) + (3 * H + 8) + (7 * H + 8) + (3 * F + 8)
    assert w["quant_bytes_per_step"] == S * per_row * 32 + 4096 * 6 * H
