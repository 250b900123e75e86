"""Thin ctypes binding of libqi (include/qi.h).

Argument marshalling only: every step of the DiT path runs in the CUDA
library.  Tensors are torch CUDA tensors (PyTorch provides device memory and
streams); the binding passes their data pointers and sizes.  Loading fails
loudly if the library is missing -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import List, Optional, Sequence

import torch

from . import build_lib

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqi.so")

QI_OK = 0
QI_ERR_INVALID_ARG = 1
QI_ERR_UNSUPPORTED_SHAPE = 2
QI_ERR_ALIGNMENT = 3
QI_ERR_CUDA = 4
QI_ERR_TIMEOUT = 5
QI_ERR_WORKSPACE = 6

QI_F32, QI_BF16 = 0, 1
QI_EPI_STORE, QI_EPI_GELU_TANH, QI_EPI_GATED_RESIDUAL, QI_EPI_QKV_NORM_ROPE = 0, 1, 2, 3
QI_KV_NONE, QI_KV_WRITE_PREFIX, QI_KV_READ_PREFIX = 0, 1, 2
QI_MAX_GROUPS = 16


class QiError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libqi error {code}: {msg}")
        self.code = code


# ------------------------------------------------------------------ structs

class qi_groups(C.Structure):
    _fields_ = [("n", C.c_int32), ("end", C.c_int32 * QI_MAX_GROUPS),
                ("row_set", C.c_int32 * QI_MAX_GROUPS)]


class qi_w8(C.Structure):
    _fields_ = [("q", C.c_void_p), ("s", C.c_void_p), ("rowsum", C.c_void_p),
                ("bias", C.c_void_p), ("n", C.c_int32), ("k", C.c_int32)]


class qi_linear_bf16(C.Structure):
    _fields_ = [("w", C.c_void_p), ("bias", C.c_void_p), ("n", C.c_int32), ("k", C.c_int32)]


class qi_epilogue(C.Structure):
    _fields_ = [("kind", C.c_int32), ("residual", C.c_void_p), ("ld_residual", C.c_int32),
                ("gate", C.c_void_p), ("gate_ld", C.c_int32), ("groups", C.POINTER(qi_groups)),
                ("row0", C.c_int32), ("hidden", C.c_int32), ("eps", C.c_float),
                ("norm_q", C.c_void_p), ("norm_k", C.c_void_p), ("rope_cos", C.c_void_p),
                ("rope_sin", C.c_void_p), ("q_out", C.c_void_p), ("k_out", C.c_void_p),
                ("v_out", C.c_void_p), ("ld_out", C.c_int32)]


class qi_dims(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("heads", C.c_int32), ("head_dim", C.c_int32),
                ("mlp", C.c_int32), ("patch", C.c_int32), ("blocks", C.c_int32),
                ("eps", C.c_float)]


class qi_mxfp4(C.Structure):
    _fields_ = [("packed", C.c_void_p), ("scales", C.c_void_p), ("bias", C.c_void_p),
                ("n", C.c_int32), ("k", C.c_int32)]


class qi_block_weights(C.Structure):
    _fields_ = [("qkv", qi_w8), ("out", qi_w8), ("up", qi_w8), ("down", qi_w8),
                ("norm_q", C.c_void_p), ("norm_k", C.c_void_p), ("mod", qi_linear_bf16),
                ("qkv_bf16", qi_linear_bf16), ("out_bf16", qi_linear_bf16),
                ("up_bf16", qi_linear_bf16), ("down_bf16", qi_linear_bf16),
                ("qkv_mx", qi_mxfp4), ("out_mx", qi_mxfp4), ("up_mx", qi_mxfp4),
                ("down_mx", qi_mxfp4), ("mx_expand", C.c_void_p), ("mx_expand_bytes", C.c_size_t)]


class qi_model(C.Structure):
    _fields_ = [("dims", qi_dims), ("blocks", C.POINTER(qi_block_weights)),
                ("t1", qi_linear_bf16), ("t2", qi_linear_bf16), ("img_in", qi_linear_bf16),
                ("txt_in", qi_linear_bf16), ("final_mod", qi_linear_bf16),
                ("proj_out", qi_linear_bf16)]


class qi_seq(C.Structure):
    _fields_ = [("txt", C.c_void_p), ("text_tokens", C.c_int32), ("ref_latents", C.c_void_p),
                ("groups", C.POINTER(qi_groups)), ("rope_cos", C.c_void_p),
                ("rope_sin", C.c_void_p), ("kv_cache", C.c_void_p)]


TAP_FIELDS = ("u1", "q1", "s1", "zp1", "o", "o_range", "qo", "so", "zpo", "x_mid", "u2", "q2",
              "s2", "zp2", "g", "g_range", "qg", "sg", "zpg", "x_layers")


class qi_block_taps(C.Structure):
    _fields_ = [(name, C.c_void_p) for name in TAP_FIELDS]


# ------------------------------------------------------------------ loading

_lib = None

_SIGS = {
    "qi_ctx_create": [C.c_int, C.POINTER(C.c_void_p)],
    "qi_ctx_destroy": [C.c_void_p],
    "qi_ctx_check": [C.c_void_p, C.c_void_p],
    "qi_last_error": [C.c_char_p, C.c_size_t],
    "qi_prepare_w8": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                      C.c_void_p, C.c_void_p],
    "qi_quantize_act": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p,
                        C.c_void_p, C.c_int, C.POINTER(qi_groups), C.c_int, C.c_float,
                        C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p],
    "qi_w8a8_linear": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                       C.POINTER(qi_w8), C.POINTER(qi_epilogue), C.c_void_p, C.c_int,
                       C.c_void_p, C.c_void_p],
    "qi_bf16_linear": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.POINTER(qi_linear_bf16),
                       C.c_void_p, C.c_int, C.c_void_p],
    "qi_mxfp4_linear": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.POINTER(qi_mxfp4),
                        C.c_void_p, C.c_int, C.c_void_p],
    "qi_qk_norm_rope": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                        C.c_void_p, C.c_void_p, C.c_void_p, C.c_float, C.c_void_p, C.c_void_p,
                        C.c_void_p, C.c_int, C.c_void_p],
    "qi_attn_block_causal": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                             C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int,
                             C.POINTER(qi_groups), C.c_float, C.c_void_p, C.c_int, C.c_void_p],
    "qi_attn_block_causal_fp8": [C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                 C.c_void_p, C.c_int, C.c_int, C.c_int, C.c_int,
                                 C.POINTER(qi_groups), C.c_float, C.c_void_p, C.c_int, C.c_void_p],
    "qi_to_e4m3": [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p, C.c_void_p],
    "qi_attn_split_plan": [C.c_int, C.c_int, C.POINTER(qi_groups), C.c_int, C.c_size_t,
                           C.POINTER(C.c_int), C.POINTER(C.c_size_t)],
    "qi_ctx_reserve_attention": [C.c_void_p, C.c_size_t],
    "qi_ctx_set_attention_fp8": [C.c_void_p, C.c_int],
    "qi_ctx_set_block_taps": [C.c_void_p, C.POINTER(qi_block_taps)],
    "qi_mxfp4_expand_bf16": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                             C.c_void_p],
    "qi_mxfp4_decode": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int, C.c_int, C.c_int,
                        C.c_void_p, C.c_void_p],
    "qi_block_workspace_bytes": [C.POINTER(qi_dims), C.c_int, C.POINTER(C.c_size_t)],
    "qi_dit_block_forward": [C.c_void_p, C.POINTER(qi_dims), C.POINTER(qi_block_weights),
                             C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.POINTER(qi_groups),
                             C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                             C.c_void_p, C.c_size_t, C.c_void_p],
    "qi_dit_block_forward_noalloc": [C.c_void_p, C.POINTER(qi_dims), C.POINTER(qi_block_weights),
                                     C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                                     C.POINTER(qi_groups), C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_int, C.c_void_p],
    "qi_time_conditioning": [C.c_void_p, C.POINTER(qi_model), C.c_float, C.c_void_p, C.c_void_p,
                             C.c_void_p, C.c_size_t, C.c_void_p],
    "qi_step_workspace_bytes": [C.POINTER(qi_dims), C.c_int, C.POINTER(C.c_size_t)],
    "qi_denoise_step": [C.c_void_p, C.POINTER(qi_model), C.c_void_p, C.c_void_p, C.c_int,
                        C.c_void_p, C.POINTER(qi_groups), C.c_void_p, C.c_void_p, C.c_float,
                        C.c_float, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                        C.c_void_p],
    "qi_step_cfg_workspace_bytes": [C.POINTER(qi_dims), C.c_int, C.c_int, C.c_int,
                                    C.POINTER(C.c_size_t)],
    "qi_denoise_step_cfg": [C.c_void_p, C.POINTER(qi_model), C.c_void_p, C.POINTER(qi_seq),
                            C.POINTER(qi_seq), C.c_float, C.c_float, C.c_float, C.c_int,
                            C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p],
    "qi_euler_update": [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_float, C.c_float,
                        C.c_void_p],
    "qi_rope_tables": [C.c_int, C.POINTER(C.c_int32), C.POINTER(C.c_int32),
                       C.POINTER(C.c_int32), C.POINTER(C.c_int32), C.c_void_p, C.c_void_p],
    "qi_sigma_schedule": [C.c_int, C.c_int, C.c_void_p],
    "qi_debug_timeout_probe": [C.c_void_p, C.c_uint64, C.c_void_p],
    "qi_debug_mma_probe": [C.c_void_p, C.c_int, C.c_int, C.c_void_p],
    "qi_ctx_profile": [C.c_void_p, C.c_int],
    "qi_ctx_profile_read": [C.c_void_p, C.c_int, C.POINTER(C.c_longlong), C.POINTER(C.c_int),
                            C.POINTER(C.c_double)],
}

KERNEL_CLASSES = ("gemm_i8", "gemm_bf16", "attention", "quant", "qk_norm_rope", "gemv", "other")

EXPORTED = tuple(_SIGS)


def lib(build: bool = False):
    """Load libqi.so (building it first if asked).  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if build:
        build_lib.build()
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m diffusion_transformer_text_dit_b200.build_lib`")
    L = C.CDLL(LIB_PATH)
    for name, args in _SIGS.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = C.c_int
    _lib = L
    return L


def last_error() -> str:
    buf = C.create_string_buffer(1024)
    lib().qi_last_error(buf, 1024)
    return buf.value.decode(errors="replace")


def check(code: int):
    if code != QI_OK:
        raise QiError(code, last_error())


def ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libqi takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libqi takes contiguous tensors")
    return t.data_ptr()


def stream_ptr(stream: Optional[torch.cuda.Stream] = None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def groups_struct(ends: Sequence[int], row_sets: Sequence[int]) -> qi_groups:
    g = qi_groups()
    g.n = len(ends)
    for i, (e, r) in enumerate(zip(ends, row_sets)):
        g.end[i] = int(e)
        g.row_set[i] = int(r)
    return g


# ------------------------------------------------------------------ context

class Context:
    """Owns a qi_ctx (one device status word) for the current CUDA device."""

    def __init__(self, device: Optional[int] = None):
        if not torch.cuda.is_available():
            raise RuntimeError("libqi needs a CUDA device (sm_100a); none is available")
        self.device = torch.cuda.current_device() if device is None else device
        h = C.c_void_p()
        check(lib().qi_ctx_create(self.device, C.byref(h)))
        self.handle = h

    def check(self, stream=None):
        check(lib().qi_ctx_check(self.handle, stream_ptr(stream)))

    def set_attention_fp8(self, enable: bool):
        """e4m3 attention in the steps run on this context (qi_ctx_set_attention_fp8)."""
        check(lib().qi_ctx_set_attention_fp8(self.handle, 1 if enable else 0))

    def set_block_taps(self, taps: Optional[dict]):
        """Copy each block quantizer's input and output into the given device
        tensors (qi_ctx_set_block_taps; keys from TAP_FIELDS), or stop (None)."""
        if taps is None:
            check(lib().qi_ctx_set_block_taps(self.handle, None))
            self._taps = None
            return
        st = qi_block_taps()
        for name in TAP_FIELDS:
            setattr(st, name, ptr(taps.get(name)))
        check(lib().qi_ctx_set_block_taps(self.handle, C.byref(st)))
        self._taps = taps   # keep the buffers alive while the library holds their pointers

    def profile(self, enable: bool):
        """Reset launch counters; time every launch with CUDA events if enable."""
        check(lib().qi_ctx_profile(self.handle, 1 if enable else 0))

    def profile_read(self) -> dict:
        """{class: (launches, timed launches, total ms)} since the last profile() call."""
        out = {}
        for i, name in enumerate(KERNEL_CLASSES):
            n, t, ms = C.c_longlong(), C.c_int(), C.c_double()
            check(lib().qi_ctx_profile_read(self.handle, i, C.byref(n), C.byref(t), C.byref(ms)))
            out[name] = (n.value, t.value, ms.value)
        return out

    def close(self):
        if self.handle:
            lib().qi_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ entry points

def qi_prepare_w8(ctx: Context, w: torch.Tensor, stream=None):
    """fp32 [n, k] -> (q int8 [n, k], s fp32 [n], rowsum int32 [n])."""
    n, k = w.shape
    q = torch.empty((n, k), dtype=torch.int8, device=w.device)
    s = torch.empty(n, dtype=torch.float32, device=w.device)
    rs = torch.empty(n, dtype=torch.int32, device=w.device)
    check(lib().qi_prepare_w8(ctx.handle, ptr(w), n, k, ptr(q), ptr(s), ptr(rs),
                              stream_ptr(stream)))
    return q, s, rs


def qi_quantize_act(ctx: Context, x: torch.Tensor, shift=None, scale=None, mod_ld: int = 0,
                    groups: Optional[qi_groups] = None, row0: int = 0, eps: float = 1e-6,
                    out=None, stream=None):
    """Per-token int8 quantization of x [M, K] (fp32 or bf16), optionally LN + modulate."""
    M, K = x.shape
    dt = QI_BF16 if x.dtype == torch.bfloat16 else QI_F32
    if out is None:
        out = (torch.empty((M, K), dtype=torch.int8, device=x.device),
               torch.empty(M, dtype=torch.float32, device=x.device),
               torch.empty(M, dtype=torch.int32, device=x.device))
    q, s, zp = out
    check(lib().qi_quantize_act(ctx.handle, ptr(x), dt, M, K, K, ptr(shift), ptr(scale), mod_ld,
                                C.byref(groups) if groups is not None else None, row0, eps,
                                ptr(q), ptr(s), ptr(zp), stream_ptr(stream)))
    return q, s, zp


# The weight structs hold raw device pointers, so each keeps references to the
# tensors it points to: a tensor freed while the struct lives would let the
# caching allocator hand its memory to a later tensor before a call reads it.

def w8_struct(q, s, rowsum, bias=None) -> qi_w8:
    w = qi_w8()
    w.q, w.s, w.rowsum, w.bias = ptr(q), ptr(s), ptr(rowsum), ptr(bias)
    w.n, w.k = q.shape
    w._keep = (q, s, rowsum, bias)
    return w


def bf16_struct(w, bias=None) -> qi_linear_bf16:
    s = qi_linear_bf16()
    s.w, s.bias = ptr(w), ptr(bias)
    s.n, s.k = w.shape
    s._keep = (w, bias)
    return s


def qi_w8a8_linear(ctx: Context, qa, s_a, zp_a, w: qi_w8, epilogue: Optional[qi_epilogue] = None,
                   y: Optional[torch.Tensor] = None, acc_debug: Optional[torch.Tensor] = None,
                   stream=None):
    M = qa.shape[0]
    ldy = y.shape[1] if y is not None else 0
    check(lib().qi_w8a8_linear(ctx.handle, ptr(qa), ptr(s_a), ptr(zp_a), M, C.byref(w),
                               C.byref(epilogue) if epilogue is not None else None, ptr(y), ldy,
                               ptr(acc_debug), stream_ptr(stream)))
    return y


def qi_bf16_linear(ctx: Context, a: torch.Tensor, w: qi_linear_bf16, y: torch.Tensor, stream=None):
    M = a.shape[0]
    check(lib().qi_bf16_linear(ctx.handle, ptr(a), M, a.shape[1], C.byref(w), ptr(y),
                               y.shape[1], stream_ptr(stream)))
    return y


def mx_struct(packed, scales, bias=None) -> qi_mxfp4:
    """An MXFP4 Linear: packed [n, k/2] uint8 codes, scales [n, k/32] uint8 E8M0."""
    m = qi_mxfp4()
    m.packed, m.scales, m.bias = ptr(packed), ptr(scales), ptr(bias)
    m.n = packed.shape[0]
    m.k = 2 * packed.shape[1]
    m._keep = (packed, scales, bias)
    return m


def qi_mxfp4_linear(ctx: Context, a: torch.Tensor, w: qi_mxfp4, y: Optional[torch.Tensor] = None,
                    stream=None):
    """bf16 y [M, n] = a [M, k] (bf16) x decode(w)^T + bias, MXFP4 decoded inside the GEMM."""
    M = a.shape[0]
    if y is None:
        y = torch.empty((M, w.n), dtype=torch.bfloat16, device=a.device)
    check(lib().qi_mxfp4_linear(ctx.handle, ptr(a), M, a.shape[1], C.byref(w), ptr(y), y.shape[1],
                                stream_ptr(stream)))
    return y


def qi_qk_norm_rope(ctx: Context, qkv, heads, wq, wk, cos, sin, eps, q_out, k_out, v_out,
                    stream=None):
    T = qkv.shape[0]
    check(lib().qi_qk_norm_rope(ctx.handle, ptr(qkv), T, heads, 128, ptr(wq), ptr(wk), ptr(cos),
                                ptr(sin), eps, ptr(q_out), ptr(k_out), ptr(v_out),
                                q_out.shape[1], stream_ptr(stream)))


def qi_attn_block_causal(ctx: Context, q, k, v, groups: qi_groups, q_offset: int = 0,
                         heads: Optional[int] = None, sm_scale: Optional[float] = None,
                         o: Optional[torch.Tensor] = None, stream=None):
    Sq, W = q.shape
    Sk = k.shape[0]
    heads = heads if heads is not None else W // 128
    sm_scale = sm_scale if sm_scale is not None else 128 ** -0.5
    if o is None:
        o = torch.empty((Sq, W), dtype=torch.bfloat16, device=q.device)
    check(lib().qi_attn_block_causal(ctx.handle, ptr(q), q.shape[1], Sq, q_offset, ptr(k), ptr(v),
                                     k.shape[1], Sk, heads, 128, C.byref(groups), sm_scale,
                                     ptr(o), o.shape[1], stream_ptr(stream)))
    return o


def qi_attn_block_causal_fp8(ctx: Context, q8, k8, v8, groups: qi_groups, q_offset: int = 0,
                             heads: Optional[int] = None, sm_scale: Optional[float] = None,
                             o: Optional[torch.Tensor] = None, stream=None):
    """Block-causal attention on e4m3 operands (uint8 tensors of e4m3 bytes)."""
    Sq, W = q8.shape
    Sk = k8.shape[0]
    heads = heads if heads is not None else W // 128
    sm_scale = sm_scale if sm_scale is not None else 128 ** -0.5
    if o is None:
        o = torch.empty((Sq, W), dtype=torch.bfloat16, device=q8.device)
    check(lib().qi_attn_block_causal_fp8(ctx.handle, ptr(q8), q8.shape[1], Sq, q_offset, ptr(k8),
                                         ptr(v8), k8.shape[1], Sk, heads, 128, C.byref(groups),
                                         sm_scale, ptr(o), o.shape[1], stream_ptr(stream)))
    return o


def qi_attn_split_plan(Sk: int, heads: int, groups: qi_groups, num_sms: int,
                       scratch_bytes: Optional[int] = None):
    """(split_heads, scratch bytes) of the attention's key-range split (host only)."""
    k, nb = C.c_int(0), C.c_size_t(0)
    sb = (1 << 64) - 1 if scratch_bytes is None else scratch_bytes
    check(lib().qi_attn_split_plan(Sk, heads, C.byref(groups), num_sms, sb, C.byref(k),
                                   C.byref(nb)))
    return k.value, nb.value


def qi_ctx_reserve_attention(ctx: Context, bytes_: int) -> None:
    """Reserve the context's scratch for the standalone attention calls' key-range split."""
    check(lib().qi_ctx_reserve_attention(ctx.handle, bytes_))


def qi_to_e4m3(ctx: Context, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """e4m3 bytes (uint8) of a bf16 tensor."""
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    check(lib().qi_to_e4m3(ctx.handle, ptr(x), x.numel(), ptr(out), stream_ptr(stream)))
    return out


def qi_mxfp4_expand_bf16(ctx: Context, packed, scales, out=None, stream=None):
    """bf16 weights [n, k] from MXFP4 codes (packed [n, k/2] uint8, scales [n, k/32])."""
    n, half = packed.shape
    k = 2 * half
    if out is None:
        out = torch.empty((n, k), dtype=torch.bfloat16, device=packed.device)
    check(lib().qi_mxfp4_expand_bf16(ctx.handle, ptr(packed), ptr(scales), n, k, ptr(out),
                                     stream_ptr(stream)))
    return out


def mx_expand_scratch(dims: "qi_dims", device="cuda", buffers: int = 2) -> torch.Tensor:
    """Scratch for expanding MXFP4 block Linears to bf16: room for `buffers`
    of the largest (max(3 hidden, mlp) x hidden); two let each expansion
    overlap the kernel before it.  One tensor may serve every block."""
    H, F = dims.hidden, dims.mlp
    return torch.empty(buffers * max(3 * H, F) * H, dtype=torch.bfloat16, device=device)


def qi_mxfp4_decode(ctx: Context, packed, scales, k: Optional[int] = None, out=None, stream=None):
    """fp32 weights [n, k] from MXFP4 codes (packed [n, k_stored/2] uint8) and E8M0 scales."""
    n, half = packed.shape
    k_stored = 2 * half
    k = k_stored if k is None else k
    if out is None:
        out = torch.empty((n, k), dtype=torch.float32, device=packed.device)
    check(lib().qi_mxfp4_decode(ctx.handle, ptr(packed), ptr(scales), n, k_stored, k, ptr(out),
                                stream_ptr(stream)))
    return out


def dims_struct(hidden, heads, mlp, patch, blocks, eps=1e-6) -> qi_dims:
    d = qi_dims()
    d.hidden, d.heads, d.head_dim, d.mlp, d.patch, d.blocks, d.eps = (
        hidden, heads, 128, mlp, patch, blocks, eps)
    return d


def qi_block_workspace_bytes(dims: qi_dims, T: int) -> int:
    n = C.c_size_t()
    check(lib().qi_block_workspace_bytes(C.byref(dims), T, C.byref(n)))
    return n.value


def qi_step_workspace_bytes(dims: qi_dims, S: int) -> int:
    n = C.c_size_t()
    check(lib().qi_step_workspace_bytes(C.byref(dims), S, C.byref(n)))
    return n.value


def qi_dit_block_forward(ctx: Context, dims: qi_dims, bw: qi_block_weights, x, row0, mod,
                         groups: qi_groups, cos, sin, k_layer, v_layer, kv_mode, workspace,
                         stream=None):
    T = x.shape[0]
    check(lib().qi_dit_block_forward(ctx.handle, C.byref(dims), C.byref(bw), ptr(x), T, row0,
                                     ptr(mod), C.byref(groups), ptr(cos), ptr(sin), ptr(k_layer),
                                     ptr(v_layer), kv_mode, ptr(workspace), workspace.numel(),
                                     stream_ptr(stream)))


def qi_dit_block_forward_noalloc(ctx: Context, dims: qi_dims, bw: qi_block_weights, x, row0, mod,
                                 groups: qi_groups, cos, sin, k_layer, v_layer, kv_mode,
                                 stream=None):
    """qi_dit_block_forward without a workspace: the library's fixed scratch is used."""
    T = x.shape[0]
    check(lib().qi_dit_block_forward_noalloc(ctx.handle, C.byref(dims), C.byref(bw), ptr(x), T,
                                             row0, ptr(mod), C.byref(groups), ptr(cos), ptr(sin),
                                             ptr(k_layer), ptr(v_layer), kv_mode,
                                             stream_ptr(stream)))


def qi_time_conditioning(ctx: Context, model: "Model", sigma: float, block_mod, final_mod,
                         workspace, stream=None):
    check(lib().qi_time_conditioning(ctx.handle, C.byref(model.struct), sigma, ptr(block_mod),
                                     ptr(final_mod), ptr(workspace), workspace.numel(),
                                     stream_ptr(stream)))


def qi_denoise_step(ctx: Context, model: "Model", latents, txt, text_tokens, ref_latents,
                    groups: qi_groups, cos, sin, sigma, sigma_next, kv_mode, kv_cache, v_out,
                    workspace, stream=None):
    check(lib().qi_denoise_step(ctx.handle, C.byref(model.struct), ptr(latents), ptr(txt),
                                text_tokens, ptr(ref_latents), C.byref(groups), ptr(cos),
                                ptr(sin), sigma, sigma_next, kv_mode, ptr(kv_cache), ptr(v_out),
                                ptr(workspace), workspace.numel(), stream_ptr(stream)))


def seq_struct(txt, text_tokens, ref_latents, groups: qi_groups, cos, sin, kv_cache=None):
    """A qi_seq for qi_denoise_step_cfg.  The struct holds raw device pointers,
    so it keeps references to every tensor (and the groups) it points to: a
    tensor freed while the struct lives would let the caching allocator hand
    its memory to a later tensor before the step reads it."""
    s = qi_seq()
    s.txt, s.text_tokens, s.ref_latents = ptr(txt), text_tokens, ptr(ref_latents)
    s.groups = C.pointer(groups)
    s.rope_cos, s.rope_sin, s.kv_cache = ptr(cos), ptr(sin), ptr(kv_cache)
    s._keep = (txt, ref_latents, groups, cos, sin, kv_cache)
    return s


def qi_step_cfg_workspace_bytes(dims: qi_dims, S_cond: int, S_uncond: int, target_tokens: int) -> int:
    n = C.c_size_t()
    check(lib().qi_step_cfg_workspace_bytes(C.byref(dims), S_cond, S_uncond, target_tokens,
                                            C.byref(n)))
    return n.value


def qi_denoise_step_cfg(ctx: Context, model: "Model", latents, cond: qi_seq, uncond: qi_seq,
                        guidance, sigma, sigma_next, kv_mode, v_out, workspace, stream=None):
    check(lib().qi_denoise_step_cfg(ctx.handle, C.byref(model.struct), ptr(latents),
                                    C.byref(cond), C.byref(uncond), guidance, sigma, sigma_next,
                                    kv_mode, ptr(v_out), ptr(workspace), workspace.numel(),
                                    stream_ptr(stream)))


def qi_euler_update(ctx: Context, x, v, sigma, sigma_next, stream=None):
    check(lib().qi_euler_update(ctx.handle, ptr(x), ptr(v), x.numel(), sigma, sigma_next,
                                stream_ptr(stream)))


def qi_rope_tables(groups_desc):
    """groups_desc: [(kind, tokens, grid)] -> host float32 tensors cos, sin [S, 64]."""
    n = len(groups_desc)
    kinds = (C.c_int32 * n)(*[0 if k == "text" else 1 for k, _, _ in groups_desc])
    toks = (C.c_int32 * n)(*[t for _, t, _ in groups_desc])
    gh = (C.c_int32 * n)(*[(g[0] if g else 0) for _, _, g in groups_desc])
    gw = (C.c_int32 * n)(*[(g[1] if g else 0) for _, _, g in groups_desc])
    S = sum(t for _, t, _ in groups_desc)
    cos = torch.empty((S, 64), dtype=torch.float32)
    sin = torch.empty((S, 64), dtype=torch.float32)
    check(lib().qi_rope_tables(n, kinds, toks, gh, gw, cos.data_ptr(), sin.data_ptr()))
    return cos, sin


def qi_sigma_schedule(steps: int, image_tokens: int):
    out = torch.empty(steps + 1, dtype=torch.float32)
    check(lib().qi_sigma_schedule(steps, image_tokens, out.data_ptr()))
    return out


def qi_debug_mma_probe(ctx: Context, int8: bool, iters: int, stream=None):
    """Back-to-back tcgen05.mma on every SM; returns the ops of the launch."""
    check(lib().qi_debug_mma_probe(ctx.handle, 1 if int8 else 0, iters, stream_ptr(stream)))
    sms = torch.cuda.get_device_properties(ctx.device).multi_processor_count
    return sms * iters * 4 * 2 * 128 * 256 * (32 if int8 else 16)


def qi_debug_timeout_probe(ctx: Context, limit_ns: int, stream=None):
    check(lib().qi_debug_timeout_probe(ctx.handle, limit_ns, stream_ptr(stream)))


# ------------------------------------------------------------------ model holders

class BlockWeights:
    """Device copies of one block's weights.  W8A8 Linears are quantized on the
    GPU by qi_prepare_w8; BF16 ones are cast to bf16; MXFP4 ones keep their
    codes and scales.  ``precision`` maps "qk", "v", "out", "up", "down" to
    "w8", "bf16" or "mx" (default: all W8A8); q and k share one setting (they
    are one GEMM).  ``mx_expand`` (mx_expand_scratch) lets the block expand
    each MXFP4 Linear to bf16 right before its GEMM instead of decoding tile
    by tile inside it."""

    def __init__(self, ctx: Context, wts: dict, device="cuda", precision: Optional[dict] = None,
                 mx_expand: Optional[torch.Tensor] = None):
        self.t = {}
        prec = {"qk": "w8", "v": "w8", "out": "w8", "up": "w8", "down": "w8"}
        prec.update(precision or {})
        st = qi_block_weights()

        def w8(w, b):
            w32 = w.to(device=device, dtype=torch.float32).contiguous()
            q, s, rs = qi_prepare_w8(ctx, w32)
            del w32
            b = b.to(device=device, dtype=torch.bfloat16).contiguous()
            return (q, s, rs, b), w8_struct(q, s, rs, b)

        def bf(w, b):
            wb = w.to(device=device, dtype=torch.bfloat16).contiguous()
            b = b.to(device=device, dtype=torch.bfloat16).contiguous()
            return (wb, b), bf16_struct(wb, b)

        def mx(codes, b):
            pk = codes[0].to(device=device, dtype=torch.uint8).contiguous()
            sc = codes[1].to(device=device, dtype=torch.uint8).contiguous()
            b = b.to(device=device, dtype=torch.bfloat16).contiguous()
            return (pk, sc, b), mx_struct(pk, sc, b)

        W, B = wts["qkv"] if "qkv" in wts else None, wts["qkv_b"]
        H = B.shape[0] // 3
        if prec["qk"] == "mx" or prec["v"] == "mx":
            if not (prec["qk"] == prec["v"] == "mx"):
                raise ValueError("an MXFP4 q | k | v projection is MXFP4 throughout")
            self.t["qkv_mx"], st.qkv_mx = mx(wts["qkv_mx"], B)
        elif prec["qk"] == "w8" and prec["v"] == "w8":
            self.t["qkv"], st.qkv = w8(W, B)
        elif prec["qk"] == "w8":
            self.t["qkv"], st.qkv = w8(W[:2 * H], B[:2 * H])
            self.t["qkv_bf16"], st.qkv_bf16 = bf(W[2 * H:], B[2 * H:])
        elif prec["v"] == "bf16":
            self.t["qkv_bf16"], st.qkv_bf16 = bf(W, B)
        else:
            raise ValueError("q, k in BF16 with v in W8A8 is not a supported layout")
        for name in ("out", "up", "down"):
            if prec[name] == "w8":
                self.t[name], s8 = w8(wts[name], wts[name + "_b"])
                setattr(st, name, s8)
            elif prec[name] == "mx":
                self.t[name + "_mx"], sm = mx(wts[name + "_mx"], wts[name + "_b"])
                setattr(st, name + "_mx", sm)
            else:
                self.t[name + "_bf16"], sb = bf(wts[name], wts[name + "_b"])
                setattr(st, name + "_bf16", sb)
        self.t["norm_q"] = wts["norm_q"].to(device=device, dtype=torch.bfloat16).contiguous()
        self.t["norm_k"] = wts["norm_k"].to(device=device, dtype=torch.bfloat16).contiguous()
        st.norm_q = ptr(self.t["norm_q"])
        st.norm_k = ptr(self.t["norm_k"])
        if "mod" in wts:
            self.t["mod"] = wts["mod"].to(device=device, dtype=torch.bfloat16).contiguous()
            self.t["mod_b"] = wts["mod_b"].to(device=device, dtype=torch.bfloat16).contiguous()
            st.mod = bf16_struct(self.t["mod"], self.t["mod_b"])
        if mx_expand is not None:   # shared scratch: the caller keeps it alive
            st.mx_expand = ptr(mx_expand)
            st.mx_expand_bytes = mx_expand.numel() * mx_expand.element_size()
            self.t["mx_expand"] = mx_expand
        self.struct = st


class Model:
    """Device weights of a whole DiT: blocks plus the step-level BF16 Linears."""

    def __init__(self, ctx: Context, dims: qi_dims, blocks: List[BlockWeights], glob: dict,
                 device="cuda"):
        self.dims = dims
        self.blocks = blocks
        self.g = {k: v.to(device=device, dtype=torch.bfloat16).contiguous() for k, v in glob.items()}
        arr = (qi_block_weights * len(blocks))(*[b.struct for b in blocks])
        self._arr = arr
        m = qi_model()
        m.dims = dims
        m.blocks = C.cast(arr, C.POINTER(qi_block_weights))
        for name in ("t1", "t2", "img_in", "txt_in", "final_mod", "proj_out"):
            setattr(m, name, bf16_struct(self.g[name], self.g[name + "_b"]))
        self.struct = m
