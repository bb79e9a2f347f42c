"""Shared test helpers: comparisons and host/device marshalling (no method arithmetic)."""
import numpy as np


def cos_sim(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))


def rel_l2(a, b) -> float:
    """||a - b|| / ||b||  (b is the reference)."""
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(np.linalg.norm(a - b) / (np.linalg.norm(b) + 1e-300))


def dev(x, dtype=None):
    """numpy -> CUDA tensor; uint16 (bf16 bits) travels as int16 with the same bits."""
    import torch
    x = np.ascontiguousarray(x)
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda()
    return torch.from_numpy(x if dtype is None else x.astype(dtype)).cuda()


def host(t) -> np.ndarray:
    import torch
    a = t.detach().cpu()
    if a.dtype in (torch.int16, torch.bfloat16):
        return a.view(torch.int16).numpy().view(np.uint16)
    return a.numpy()


def bf16_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
