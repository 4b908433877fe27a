"""Shared test plumbing: the ``gpu`` marker, conversions between torch tensors
and the numpy arrays the CPU oracle takes, and comparison helpers."""
from __future__ import annotations

import numpy as np
import pytest
import torch


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    if torch.cuda.is_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def to_np(t: torch.Tensor) -> np.ndarray:
    """CPU tensor -> numpy array in the oracle's convention (bf16 as uint16
    bits, E4M3 as uint8 bits).
    The tensor is made contiguous first; a strided view keeps its values, not
    its layout."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float32, torch.float16):
        return t.numpy()
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    raise TypeError(f"unsupported dtype {t.dtype}")


def buffer_np(t: torch.Tensor) -> tuple[np.ndarray, int]:
    """A 2-D strided CPU view -> (flat numpy array starting at its first
    element, row stride in elements), so the oracle reads the same layout."""
    assert t.dim() == 2 and t.stride(1) == 1
    stride = t.stride(0)
    T, H = t.shape
    n = (T - 1) * stride + H if T > 0 else 0
    flat = torch.as_strided(t, (n,), (1,)) if n > 0 else t.reshape(-1)[:0]
    return to_np(flat.clone()), stride


def bf16_bits_to_ordered(bits: np.ndarray) -> np.ndarray:
    """Map bfloat16 bit patterns onto integers whose difference is the number
    of representable values between them (negative values mirrored), so the
    distance is valid across zero and across binades; +0 and -0 coincide."""
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    return np.abs(bf16_bits_to_ordered(a_bits) - bf16_bits_to_ordered(b_bits))


def ordered_bits(bits: np.ndarray, nbits: int) -> np.ndarray:
    """Sign-magnitude bit patterns of an `nbits`-wide float format -> integers
    whose difference counts representable values between two numbers (+0 and
    -0 coincide)."""
    b = bits.astype(np.int64)
    sign = 1 << (nbits - 1)
    mag = b & (sign - 1)
    return np.where(b & sign, -mag, mag)


def ulp_distance(a: np.ndarray, b: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Distance in units of the last place between two arrays of the same
    narrow float type, given as the oracle's numpy arrays."""
    if dtype == torch.bfloat16:
        return np.abs(ordered_bits(a, 16) - ordered_bits(b, 16))
    if dtype == torch.float16:
        return np.abs(ordered_bits(a.view(np.uint16), 16) - ordered_bits(b.view(np.uint16), 16))
    if dtype == torch.float8_e4m3fn:
        return np.abs(ordered_bits(a, 8) - ordered_bits(b, 8))
    raise TypeError(f"no ulp distance for {dtype}")
