"""Comparison helpers shared by the GPU parity tests."""
import numpy as np
import torch


def np64(t):
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().double().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().double().numpy()
    return np.asarray(t, dtype=np.float64)


def rel_l2(a, ref):
    a, ref = np64(a), np64(ref)
    return float(np.linalg.norm(a - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(a, ref):
    return float(np.max(np.abs(np64(a) - np64(ref)))) if np64(a).size else 0.0


def host_weights(w):
    """bf16 device/host weights -> dict of fp64 numpy arrays (values exactly the bf16 ones)."""
    return {k: np64(v) for k, v in w.items()}


def ulp_diff_f32(a, b):
    """Element-wise distance in units in the last place between two fp32 arrays."""
    ai = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    bi = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    ai = np.where(ai < 0, -(ai & 0x7FFFFFFF), ai)
    bi = np.where(bi < 0, -(bi & 0x7FFFFFFF), bi)
    return np.abs(ai - bi)
