"""Host <-> device helpers for the GPU parity tests (no method arithmetic)."""

import numpy as np
import torch


def to_dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(a).cuda()
    return t if dtype is None else t.view(dtype)


def bf16_to_np_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    bits = bf16_to_np_bits(t).astype(np.uint32) << np.uint32(16)
    return bits.view(np.float32).astype(np.float64)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy()


def same_bits_f32(a: np.ndarray, b: np.ndarray) -> bool:
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))
