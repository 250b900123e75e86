"""The activation quantizers that a block actually runs, checked bit for bit at
their own inputs.

FlagRelease "Qwen-Image-2.1-W8A8-arm-FlagOS", "Quantization and validation":
dynamic asymmetric INT8 activations per token with FP32 scales.  A block runs
four of them: two fused with the LayerNorm + adaLN modulate (fp32 input u), and
two on bf16 tensors whose row ranges were published by the producing kernel
(the attention epilogue and the GELU epilogue).  The block's taps
(qi_ctx_set_block_taps) expose each quantizer's exact input and its codes,
scales and zero points; the oracle's quantize_act of that same input must give
the same three arrays, and each published range must equal the range of the
stored bf16 row.  The LayerNorm values themselves are checked against the
float64 LayerNorm within fp32 rounding.

Also: rounding ties of u / s, and values a hair off a tie (the case where the
kernel's reciprocal-multiply shortcut hands over to the IEEE quotient).
"""
import numpy as np
import pytest
import torch

from diffusion_transformer_text_dit_b200 import qi, synth
from oracle import qi_oracle as O
from tests._util import bf16_np, cuda

pytestmark = pytest.mark.gpu

F32 = np.float32


def _range_bits(a: np.ndarray) -> np.ndarray:
    """[rows, 2] uint32: float bits of (0 - min(min, 0), max(max, 0) + 0)."""
    lo = np.minimum(a.min(axis=1), F32(0)).astype(F32)
    hi = np.maximum(a.max(axis=1), F32(0)).astype(F32)
    out = np.stack([(F32(0) - lo).astype(F32), (hi + F32(0)).astype(F32)], axis=1)
    return out.view(np.uint32)


def _assert_codes_equal(name, u, q, s, zp):
    oq, os_, ozp = O.quantize_act(u)
    assert np.array_equal(s, os_), f"{name}: scales differ in {np.sum(s != os_)} rows"
    assert np.array_equal(zp, ozp), f"{name}: zero points differ in {np.sum(zp != ozp)} rows"
    bad = q != oq
    assert not bad.any(), f"{name}: {bad.sum()} codes differ (first row {np.argwhere(bad)[0][0]})"


BLOCK1024 = synth.STEP1024.replace(name="block_1024px", blocks=1, t=0.5)


@pytest.mark.parametrize("cfg", [synth.TINY, synth.BLOCK512, BLOCK1024],
                         ids=["tiny", "block_512px", "block_1024px"])
def test_block_quantizers_bit_exact_at_their_inputs(ctx, cfg):
    H, F, S = cfg.hidden, cfg.mlp, cfg.tokens
    wts = synth.block_weights(cfg, 0)
    bw = qi.BlockWeights(ctx, wts)
    del wts
    dims = qi.dims_struct(H, cfg.heads, cfg.mlp, cfg.patch, 1)
    ends = list(np.cumsum(cfg.group_sizes()))
    g = qi.groups_struct(ends, cfg.group_row_sets())
    cos, sin = qi.qi_rope_tables([(gr.kind, gr.tokens, gr.grid) for gr in cfg.groups])
    x = synth.hidden_states(cfg, S)
    mod = synth.mod_table(cfg)
    dev = "cuda"
    f32 = lambda *sh: torch.empty(sh, dtype=torch.float32, device=dev)
    i8 = lambda *sh: torch.empty(sh, dtype=torch.int8, device=dev)
    i32 = lambda *sh: torch.empty(sh, dtype=torch.int32, device=dev)
    taps = {"u1": f32(S, H), "q1": i8(S, H), "s1": f32(S), "zp1": i32(S),
            "o": torch.empty((S, H), dtype=torch.bfloat16, device=dev), "o_range": i32(S, 2),
            "qo": i8(S, H), "so": f32(S), "zpo": i32(S),
            "x_mid": f32(S, H), "u2": f32(S, H), "q2": i8(S, H), "s2": f32(S), "zp2": i32(S),
            "g": torch.empty((S, F), dtype=torch.bfloat16, device=dev), "g_range": i32(S, 2),
            "qg": i8(S, F), "sg": f32(S), "zpg": i32(S)}
    xg = cuda(x)
    kl = torch.zeros((S, H), dtype=torch.bfloat16, device=dev)
    vl = torch.zeros_like(kl)
    ws = torch.empty(qi.qi_block_workspace_bytes(dims, S), dtype=torch.uint8, device=dev)
    ctx.set_block_taps(taps)
    try:
        qi.qi_dit_block_forward(ctx, dims, bw.struct, xg, 0, cuda(mod), g, cuda(cos), cuda(sin),
                                kl, vl, qi.QI_KV_NONE, ws)
        ctx.check()
    finally:
        ctx.set_block_taps(None)
    t = {k: v.cpu() for k, v in taps.items()}
    npy = lambda k: t[k].numpy()

    # the four quantizers, each at its own input
    _assert_codes_equal("LN1 quantizer", npy("u1"), npy("q1"), npy("s1"), npy("zp1"))
    _assert_codes_equal("attention-output quantizer", bf16_np(t["o"]), npy("qo"), npy("so"),
                        npy("zpo"))
    _assert_codes_equal("LN2 quantizer", npy("u2"), npy("q2"), npy("s2"), npy("zp2"))
    _assert_codes_equal("GELU-output quantizer", bf16_np(t["g"]), npy("qg"), npy("sg"), npy("zpg"))

    # the ranges the producers published are exactly the stored rows' ranges
    assert np.array_equal(npy("o_range").view(np.uint32), _range_bits(bf16_np(t["o"])))
    assert np.array_equal(npy("g_range").view(np.uint32), _range_bits(bf16_np(t["g"])))

    # the LayerNorm + modulate values against the float64 LayerNorm (fp32
    # arithmetic: sums over H values, a reciprocal square root, one FMA)
    m = bf16_np(mod)
    gid = O.group_ids(ends)
    rs = np.where(gid < len(ends) - 1, 0, 1)
    u1 = O.modulate(O.layer_norm(x.numpy(), cfg.eps), m[rs, 0], m[rs, 1])
    assert np.all(np.abs(npy("u1") - u1) <= 2e-5 * np.maximum(1.0, np.abs(u1)))
    u2 = O.modulate(O.layer_norm(npy("x_mid"), cfg.eps), m[rs, 3], m[rs, 4])
    assert np.all(np.abs(npy("u2") - u2) <= 2e-5 * np.maximum(1.0, np.abs(u2)))
    # and the taps are the block's own: the residual stream moved
    assert not np.array_equal(npy("x_mid"), x.numpy())


def _tie_rows(dtype):
    """Rows with an exactly known scale whose elements sit on rounding ties of
    u / s, or within a few ulps of one."""
    rows = []
    # power-of-two scale: lo = -8, hi = 127/16 -> s = 1/16, zp = 0; u = (k + 1/2)/16
    # for |k + 1/2| < 127 (both signs stay inside [lo, hi])
    k = np.arange(-127, 127)
    ties = ((k + 0.5) / 16).astype(F32)
    rows.append(np.concatenate([[-8.0, 127 / 16], ties, -ties[::-1]]).astype(F32))
    if dtype == "f32":
        # scales that are not powers of two: find u with fl(u / s) == k + 1/2
        # exactly, and the fp32 neighbours of such u (fraction a hair off 1/2)
        for lo, hi in ((-0.7, 1.3), (-3.1, 0.2), (-1e-3, 2e-3), (0.0, 5.5)):
            lo, hi = F32(lo), F32(hi)
            s = F32((hi - lo) / F32(255))
            cand = ((np.arange(-128, 128) + 0.5) * np.float64(s)).astype(F32)
            on_tie = cand[(cand / s).astype(F32) == (np.arange(-128, 128) + 0.5)]
            near = np.concatenate([np.nextafter(on_tie, F32(np.inf)), np.nextafter(on_tie, F32(-np.inf)),
                                   np.nextafter(np.nextafter(on_tie, F32(np.inf)), F32(np.inf))])
            vals = np.concatenate([on_tie, near])
            vals = vals[(vals >= lo) & (vals <= hi)]
            rows.append(np.concatenate([[lo, hi], vals]).astype(F32))
    K = max(len(r) for r in rows)
    K = (K + 7) // 8 * 8
    out = np.zeros((len(rows), K), F32)
    for i, r in enumerate(rows):
        out[i, :len(r)] = r
        out[i, len(r):] = r[0]      # pad with the row's minimum: the range is unchanged
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantizer_rounding_ties(ctx, dtype):
    u = _tie_rows(dtype)
    x = torch.from_numpy(u)
    if dtype == "bf16":
        x = x.to(torch.bfloat16)
        assert np.array_equal(bf16_np(x), u)     # every tie value is a bf16 value
    q, s, zp = qi.qi_quantize_act(ctx, cuda(x))
    oq, os_, ozp = O.quantize_act(u)
    assert np.array_equal(s.cpu().numpy(), os_) and np.array_equal(zp.cpu().numpy(), ozp)
    assert np.array_equal(q.cpu().numpy(), oq)
    # the power-of-two row: ties go to the even code
    assert s.cpu().numpy()[0] == F32(1 / 16) and zp.cpu().numpy()[0] == 0
    codes = q.cpu().numpy()[0, 2:2 + 2 * 254].astype(np.int64)
    assert np.all(codes % 2 == 0)
