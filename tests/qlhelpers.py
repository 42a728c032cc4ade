"""Helpers shared by the GPU parity tests: host arrays -> device tensors, and the error measure."""
import numpy as np
import torch

BENQ_TOL = 2e-3      # max over batch rows of max|y - y_ref| / max|y_ref|
MDBF_TOL = 5e-3


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bits16(a: np.ndarray) -> torch.Tensor:
    """uint16 bit patterns as a CUDA int16 tensor."""
    return dev(np.ascontiguousarray(a).view(np.int16))


def bf16(a: np.ndarray) -> torch.Tensor:
    return bits16(a).view(torch.bfloat16)


def f16(a: np.ndarray) -> torch.Tensor:
    return bits16(a).view(torch.float16)


def max_rel(y, y_ref) -> float:
    """Per batch row max|y - y_ref| / max|y_ref|, maximised over rows."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    num = np.abs(y - y_ref).max(axis=-1)
    den = np.abs(y_ref).max(axis=-1)
    return float((num / np.maximum(den, 1e-300)).max())


def f32_to_bf16_rne(y: np.ndarray) -> np.ndarray:
    u = np.ascontiguousarray(y, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def mdbf_dev_paths(paths):
    return [dict(S_A=dev(p.S_A), S_B=dev(p.S_B), A_amp=f16(p.A_amp), B_amp=f16(p.B_amp),
                 Q_U=f16(p.Q_U), Q_V=f16(p.Q_V)) for p in paths]
