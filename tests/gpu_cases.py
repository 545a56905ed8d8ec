"""Shared helpers for the GPU parity tests: draw inputs on the device, copy
them to host numpy arrays for the oracle, and compare."""
import numpy as np
import torch

ATTN_REL_L2 = 1e-3   # fp32 attention outputs vs the fp64 oracle
ATTN_MAX_ABS = 5e-3


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32_bits(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def assert_attn_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = gpu - ref
    rel = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    mx = np.abs(err).max() if err.size else 0.0
    assert rel <= ATTN_REL_L2 and mx <= ATTN_MAX_ABS, f"{what}: rel-L2 {rel:.3e}, max-abs {mx:.3e}"
    return rel, mx
