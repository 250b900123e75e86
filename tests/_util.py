"""Small helpers shared by the tests (no method arithmetic)."""
import numpy as np
import torch


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> float32 numpy array of the same values."""
    return t.detach().to("cpu", torch.float32).numpy()


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def cuda(t: torch.Tensor, dtype=None) -> torch.Tensor:
    return t.to(device="cuda", dtype=dtype or t.dtype).contiguous()


def oracle_weights(wts: dict) -> dict:
    """A block's drawn weights as the oracle takes them: float tensors as fp32
    numpy arrays, MXFP4 code pairs (packed, scales) as uint8 numpy arrays."""
    out = {}
    for k, v in wts.items():
        if isinstance(v, tuple):
            out[k] = tuple(t.detach().cpu().numpy() for t in v)
        else:
            out[k] = v.detach().to("cpu", torch.float32).numpy()
    return out
