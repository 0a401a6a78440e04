"""Packed INT4 container and dequantization.  Oracle (test infrastructure only).

The pages fix only that both methods emit "the same INT4 plus group scales"
("GPTQ versus AWQ objectives", section "What interviewers probe next") and that
act-order needs a group index per column (same section).  The byte layout is
this library's own: code c of memory column k is stored as u = c + 2^(bits-1)
in nibble k % 8 (bits 4(k%8) .. 4(k%8)+3) of uint32 word k // 8 of its row;
scales are FP16 (round to nearest even) of the scale the quantizer used.
With a zero-point per group (asymmetric groups) the stored code is
u = c + zero instead, and the zero-points are one byte each, [out, ngroups].
"""
from __future__ import annotations

import numpy as np


def pack_ref(codes_mem: np.ndarray, bits: int) -> np.ndarray:
    """[out, in] signed codes in memory order -> uint32 [out, in / 8]."""
    c = np.asarray(codes_mem, dtype=np.int64)
    out, inp = c.shape
    assert inp % 8 == 0
    u = (c + (1 << (bits - 1))).astype(np.uint64)
    assert u.min() >= 0 and u.max() < 16
    words = np.zeros((out, inp // 8), dtype=np.uint64)
    for k in range(8):
        words |= u[:, k::8] << np.uint64(4 * k)
    return words.astype(np.uint32)


def unpack_ref(qweight: np.ndarray, bits: int) -> np.ndarray:
    q = np.asarray(qweight, dtype=np.uint32).astype(np.int64)
    out, nw = q.shape
    codes = np.zeros((out, nw * 8), dtype=np.int64)
    for k in range(8):
        codes[:, k::8] = ((q >> (4 * k)) & 0xF) - (1 << (bits - 1))
    return codes


def to_memory_order(codes_q: np.ndarray, perm: np.ndarray) -> np.ndarray:
    out = np.empty_like(codes_q)
    out[:, perm] = codes_q
    return out


def g_idx_ref(perm: np.ndarray, g: int) -> np.ndarray:
    """Group of each memory-order column: position of the column in the
    quantization order, divided by g."""
    inv = np.empty_like(np.asarray(perm))
    inv[perm] = np.arange(len(perm))
    return inv // g


def dequant_ref(codes_q: np.ndarray, scales: np.ndarray, perm: np.ndarray, g: int,
                fp16: bool = True) -> np.ndarray:
    """What in memory order: code * scale of its group; ``fp16`` rounds the
    scales to half precision first (what a user of the packed format sees)."""
    sc = np.asarray(scales, dtype=np.float64)
    if fp16:
        sc = sc.astype(np.float16).astype(np.float64)
    cols = np.arange(codes_q.shape[1]) // g
    What_q = codes_q.astype(np.float64) * sc[:, cols]
    return to_memory_order(What_q, np.asarray(perm))


def pack_asym_ref(codes_mem: np.ndarray, zeros: np.ndarray, g_idx: np.ndarray,
                  bits: int) -> np.ndarray:
    """Asymmetric groups: stored code u = code + zero of the column's group
    (0 <= u <= 2^bits - 1), packed like pack_ref's words."""
    c = np.asarray(codes_mem, dtype=np.int64)
    z = np.asarray(zeros, dtype=np.int64)[:, np.asarray(g_idx)]
    u = c + z
    assert u.min() >= 0 and u.max() <= 2 ** bits - 1
    return pack_ref(u - 2 ** (bits - 1), bits)
