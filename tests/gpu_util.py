"""Helpers shared by the GPU tests: move bf16 bit arrays to the device and back."""

import numpy as np
import torch


def to_dev(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> CUDA bf16 tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_host_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def glu_dst_rows(F: int) -> np.ndarray:
    """Row of the folded GLU weight that holds source column c of W [d, 2F] (block interleave of 16)."""
    c = np.arange(2 * F)
    up = c >= F
    j = np.where(up, c - F, c)
    return (j // 16) * 32 + np.where(up, 16, 0) + (j % 16)


def oracle_layout(wstar_dn_bits: np.ndarray, glu: bool) -> np.ndarray:
    """Place the oracle's W* [d, N] in the library's K-major [N, d] layout (a pure permutation)."""
    N = wstar_dn_bits.shape[1]
    out = np.empty((N, wstar_dn_bits.shape[0]), dtype=np.uint16)
    rows = glu_dst_rows(N // 2) if glu else np.arange(N)
    out[rows] = wstar_dn_bits.T
    return out
