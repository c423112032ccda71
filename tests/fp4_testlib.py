"""Helpers shared by the GPU parity tests (layout bookkeeping only).

Nothing here computes the quantization method: these functions move bytes
between the logical scale layout the oracle produces and the tensor-core
scale layout declared in include/fp4.h, and upload oracle results as device
operands.
"""
from __future__ import annotations

import numpy as np
import torch


def mma_sf_offsets(R: int, S: int) -> np.ndarray:
    """Byte offset of logical scale (r, s) in the tensor-core layout:
    512-byte atoms of 128 rows x 4 blocks, atoms row-block major, inside an
    atom row r%32 owns 16 bytes (rows r, r+32, r+64, r+96; 4 blocks each)."""
    S4 = (S + 3) // 4 * 4
    r = np.arange(R, dtype=np.int64)[:, None]
    s = np.arange(S, dtype=np.int64)[None, :]
    return ((r // 128) * (S4 // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4


def mma_sf_bytes(R: int, S: int) -> int:
    return ((R + 127) // 128 * 128) * ((S + 3) // 4 * 4)


def to_mma_layout(per_row_scales: np.ndarray) -> np.ndarray:
    R, S = per_row_scales.shape
    out = np.zeros(mma_sf_bytes(R, S), np.uint8)
    out[mma_sf_offsets(R, S).reshape(-1)] = per_row_scales.reshape(-1)
    return out


def from_mma_layout(buf: np.ndarray, R: int, S: int) -> np.ndarray:
    return buf[mma_sf_offsets(R, S)]


def expand_2d(tile_scales: np.ndarray, rows: int) -> np.ndarray:
    """16x16 tile scales [rows/16, S] -> one scale per row [rows, S]."""
    return np.repeat(tile_scales, 16, axis=0)[:rows]


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    lo = packed & 0xF
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[0], -1)


def upload_qtensor(F, q: dict, rows: int, cols: int, fmt: int, block: int, device="cuda"):
    """An oracle quantization result as a device QTensor (GEMM input)."""
    t = F.QTensor.empty(rows, cols, fmt, block, device)
    t.codes.copy_(torch.from_numpy(q["codes"].reshape(-1)))
    sc = q["scales"]
    t.scales.copy_(torch.from_numpy(sc.reshape(-1)))
    per_row = expand_2d(sc, rows) if block == F.BLOCK_2D else sc
    t.scales_mma.copy_(torch.from_numpy(to_mma_layout(per_row)))
    t.s_dec.fill_(float(q["s_dec"]))
    t.amax.fill_(float(q.get("amax", 0.0)))
    return t


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (nb if nb > 0 else 1.0))
