"""The C-ABI library loads and exports every symbol include/qi.h declares; the
host-only helpers (RoPE tables, sigma schedule, workspace sizes) agree with the
oracle.  No GPU is touched."""
import os
import re

import numpy as np
import pytest

from diffusion_transformer_text_dit_b200 import build_lib, qi
from oracle import qi_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_lib.build()
    return qi.lib()


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "qi.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^int\s+(qi_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_five_hot_path_calls():
    syms = declared_symbols()
    for name in ("qi_quantize_act", "qi_w8a8_linear", "qi_attn_block_causal",
                 "qi_dit_block_forward", "qi_denoise_step"):
        assert name in syms


def test_library_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert len(syms) >= 15
    for name in syms:
        assert hasattr(L, name), name
    assert set(syms) == set(qi.EXPORTED)


def test_rope_tables_match_oracle(L):
    for groups in ([("text", 16, None), ("image", 64, (8, 8))],
                   [("text", 5, None), ("image", 6, (2, 3)), ("image", 12, (3, 4))],
                   [("text", 512, None), ("image", 4096, (64, 64))]):
        c, s = qi.qi_rope_tables(groups)
        oc, os_ = O.rope_tables(O.rope_positions(groups))
        # both evaluate cos/sin in double and round once to fp32
        assert np.abs(c.numpy() - oc).max() <= 1.2e-7
        assert np.abs(s.numpy() - os_).max() <= 1.2e-7


def test_sigma_schedule_matches_oracle(L):
    for steps, tokens in ((40, 4096), (40, 16384), (3, 256), (8, 1024)):
        a = qi.qi_sigma_schedule(steps, tokens).numpy()
        b = O.sigma_schedule(steps, tokens)
        assert np.abs(a - b).max() <= 1e-6
        assert a[-1] == 0 and a[0] == 1


def test_workspace_sizes(L):
    d = qi.dims_struct(4096, 32, 16384, 64, 32)
    b = qi.qi_block_workspace_bytes(d, 4608)
    # int8 [T,F] + q,o [T,H] + g [T,F] (bf16)
    T, H, F = 4608, 4096, 16384
    assert b >= T * F + 2 * T * (2 * H + F)
    s = qi.qi_step_workspace_bytes(d, 4608)
    assert s > b + 32 * 2 * T * H * 2


def test_invalid_arguments_rejected_without_a_device(L):
    import ctypes as C
    bad = qi.dims_struct(4096, 32, 16384, 64, 32)
    bad.head_dim = 64
    n = C.c_size_t()
    assert L.qi_block_workspace_bytes(C.byref(bad), 10, C.byref(n)) == qi.QI_ERR_UNSUPPORTED_SHAPE
    assert "head_dim" in qi.last_error()
    assert L.qi_rope_tables(0, None, None, None, None, None, None) == qi.QI_ERR_INVALID_ARG
    assert L.qi_ctx_reserve_attention(None, 1 << 20) == qi.QI_ERR_INVALID_ARG


def test_attention_split_plan(L):
    """The attention's key-range split (host-side plan): taken where the last
    round of CTAs would be mostly idle, bounded by the scratch, absent for
    short key ranges and for grids whose last round is nearly full."""
    g = lambda ends: qi.groups_struct(ends, [0] * len(ends))
    k, nbytes = qi.qi_attn_split_plan(4608, 32, g([512, 4608]), 148)   # 1024x1024 step
    assert 0 < k < 32 and nbytes > 0
    # the scratch holds 17 tiles per split head: partial O, max and sum of two halves
    assert nbytes >= 17 * k * 2 * 256 * (128 + 2) * 4
    assert qi.qi_attn_split_plan(4608, 32, g([512, 4608]), 148, scratch_bytes=0) == (0, 0)
    # one byte short: at most k - 1 heads fit, and then the last round still
    # holds unsplit tiles, so no split is taken at all
    assert qi.qi_attn_split_plan(4608, 32, g([512, 4608]), 148, scratch_bytes=nbytes - 1)[0] < k
    assert qi.qi_attn_split_plan(16896, 32, g([512, 16896]), 148)[0] == 0   # 13.8 rounds
    assert qi.qi_attn_split_plan(896, 32, g([128, 896]), 148)[0] == 0       # 7 key tiles
    assert qi.qi_attn_split_plan(4130, 4, g([100, 130, 4130]), 148)[0] == 4
    # the plan depends on the last group only through its length: the edit
    # ([256 | 1024 | 4096]) splits as the step does
    assert qi.qi_attn_split_plan(5376, 32, g([256, 1280, 5376]), 148)[0] == k
    with pytest.raises(qi.QiError):
        qi.qi_attn_split_plan(4608, 32, g([512, 4000]), 148)   # groups do not end at Sk
