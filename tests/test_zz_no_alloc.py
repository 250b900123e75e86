"""The allocation-free block entry point, for callers that cannot allocate
device memory (a program handed only input/output buffers by its host
framework, or one held to a fixed device-memory budget).

qi_dit_block_forward_noalloc runs the same block as qi_dit_block_forward but
takes its scratch from a fixed array inside the library instead of a
caller-owned workspace.  Its results must agree with the workspace call within
the block tolerance the other tests use (rel-L2 1e-2; the two run the same
kernels, so they are in fact identical), on two calls in a row, the second on
different inputs after the first left its data in the shared array.  This file
is collected last so that, if it fails, every other test has already run.
"""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from tests._util import cuda, rel_l2

pytestmark = pytest.mark.gpu


def _block_inputs(cfg, tag):
    H, S = cfg.hidden, cfg.tokens
    x = synth.hidden_states(cfg, S, tag="x" + tag)
    mod = synth.mod_table(cfg, tag="mod" + tag)
    return x, mod


def test_noalloc_block_matches_workspace_call_twice(ctx):
    cfg = synth.TINY
    H, S = cfg.hidden, cfg.tokens
    bw = qi.BlockWeights(ctx, synth.block_weights(cfg, 0))
    dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, 1)
    ends = list(np.cumsum(cfg.group_sizes()))
    g = qi.groups_struct(ends, cfg.group_row_sets())
    cos, sin = qi.qi_rope_tables([(gr.kind, gr.tokens, gr.grid) for gr in cfg.groups])
    cos, sin = cuda(cos), cuda(sin)
    ws = torch.empty(qi.qi_block_workspace_bytes(dims, S), dtype=torch.uint8, device="cuda")
    for call, tag in enumerate(("a", "b")):
        x, mod = _block_inputs(cfg, tag)
        modg = cuda(mod)
        ref_x = cuda(x)
        kr = torch.zeros((S, H), dtype=torch.bfloat16, device="cuda")
        vr = torch.zeros_like(kr)
        qi.qi_dit_block_forward(ctx, dims, bw.struct, ref_x, 0, modg, g, cos, sin, kr, vr,
                                qi.QI_KV_NONE, ws)
        got_x = cuda(x)
        kn = torch.zeros_like(kr)
        vn = torch.zeros_like(kr)
        qi.qi_dit_block_forward_noalloc(ctx, dims, bw.struct, got_x, 0, modg, g, cos, sin, kn, vn,
                                        qi.QI_KV_NONE)
        ctx.check()
        a, b = got_x.cpu().numpy(), ref_x.cpu().numpy()
        assert np.all(np.isfinite(a)), f"call {call}"
        assert rel_l2(a, b) <= 1e-2, f"call {call}"
        assert rel_l2(a - x.numpy(), b - x.numpy()) <= 1e-2, f"call {call}"
        assert torch.equal(got_x, ref_x) and torch.equal(kn, kr) and torch.equal(vn, vr)


def test_noalloc_rejects_rows_beyond_the_fixed_scratch(ctx):
    cfg = synth.BLOCK512   # hidden 4096, mlp 16384: 255 rows fit in the 16 MiB scratch
    dims = qi.dims_struct(cfg.hidden, cfg.heads, cfg.mlp, cfg.patch, 1)
    bw = qi.qi_block_weights()   # never reached: the size check comes first
    T = 256
    g = qi.groups_struct([T], [1])
    dummy = torch.zeros(16, device="cuda")
    with pytest.raises(qi.QiError) as e:
        qi.lib()
        qi.check(qi.lib().qi_dit_block_forward_noalloc(
            ctx.handle, qi.C.byref(dims), qi.C.byref(bw), dummy.data_ptr(), T, 0,
            dummy.data_ptr(), qi.C.byref(g), dummy.data_ptr(), dummy.data_ptr(),
            dummy.data_ptr(), dummy.data_ptr(), qi.QI_KV_NONE, qi.stream_ptr()))
    assert e.value.code == qi.QI_ERR_WORKSPACE
    assert "fixed" in str(e.value)
