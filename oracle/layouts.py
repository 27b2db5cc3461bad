"""Byte layouts in HBM of the SharQ operands, written as plain CPU permutations.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

These are the layouts in which the preparation kernel writes its outputs and the GEMM
reads them. They are fixed by the consumer, the sm_100a block-scaled (sparse) MMA, as
described in the public PTX ISA (tcgen05 "Matrix fragments", scale-factor and
sparse-metadata layouts in tensor memory), not by the SharQ pages, which give none:

* FP4 codes: two per byte along K, the even K index in the low nibble; rows K-major.
* Block scales: one byte per (row, block). Rows are grouped by 128 and scale columns by
  4; each 128x4 tile is a 512-byte chunk in which (row r, column c) sits at
  (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4. Chunks run along the scale columns
  first, then along the 128-row groups. Rows are padded to 128 and columns to 4 with 0.
  This is the order in which a 32-lane x 128-bit copy, replicated over the four lane
  quarters, leaves every row's scales in its own tensor-memory lane.
* pair48 metadata: one nibble per group of 8 logical K, i0 | i1 << 2. For every 256
  logical K (32 nibbles = 16 bytes per row) the rows are stored one after another
  (row r at byte 16 r, the lower group in the low nibble), rows padded to a multiple of
  128 with the valid pattern 0x4 (pairs 0 and 1); the 256-K slices follow each other.
  A 128-row x 16-byte slice is what one 128-lane x 128-bit copy places in tensor
  memory, one row per lane.
* elem24 metadata (no hardware consumer on sm_100a for FP4): row-major nibbles, K/8
  bytes per row.
"""
from __future__ import annotations

import numpy as np


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[..., 2n] 4-bit codes -> [..., n] bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8) & 0xF
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def round_up(a: int, b: int) -> int:
    return (a + b - 1) // b * b


def scale_offset(r: np.ndarray, c: np.ndarray, n_cols: int) -> np.ndarray:
    """Byte offset of scale (row r, column c) in the 128x4-tiled layout."""
    cp = round_up(n_cols, 4)
    chunk = (r // 128) * (cp // 4) + (c // 4)
    return chunk * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (c % 4)


def scale_layout_size(n_rows: int, n_cols: int) -> int:
    return round_up(n_rows, 128) * round_up(n_cols, 4)


def to_scale_layout(s: np.ndarray) -> np.ndarray:
    """[R, C] scale codes -> flat bytes in the tiled layout (padding = 0)."""
    R, C = s.shape
    out = np.zeros(scale_layout_size(R, C), np.uint8)
    r, c = np.meshgrid(np.arange(R), np.arange(C), indexing="ij")
    out[scale_offset(r, c, C)] = s
    return out


def from_scale_layout(buf: np.ndarray, R: int, C: int) -> np.ndarray:
    r, c = np.meshgrid(np.arange(R), np.arange(C), indexing="ij")
    return np.asarray(buf)[scale_offset(r, c, C)]


META_PAD_NIBBLE = 0x4


def meta48_size(M: int, K: int) -> int:
    return round_up(M, 128) * K // 16


def to_meta48_layout(nib: np.ndarray) -> np.ndarray:
    """[M, K/8] nibbles -> flat bytes: slices of 256 K, each [M_pad rows x 16 bytes]."""
    M, G = nib.shape
    K = G * 8
    Mp = round_up(M, 128)
    full = np.full((Mp, G), META_PAD_NIBBLE, np.uint8)
    full[:M] = nib
    per_row = pack_nibbles(full)  # [Mp, K/16] bytes, group 2i low nibble
    slices = per_row.reshape(Mp, K // 256, 16).transpose(1, 0, 2)  # [K/256, Mp, 16]
    return np.ascontiguousarray(slices).reshape(-1)


def from_meta48_layout(buf: np.ndarray, M: int, K: int) -> np.ndarray:
    Mp = round_up(M, 128)
    s = np.asarray(buf, np.uint8).reshape(K // 256, Mp, 16).transpose(1, 0, 2).reshape(Mp, K // 16)
    return unpack_nibbles(s)[:M]


def to_meta24_layout(nib: np.ndarray) -> np.ndarray:
    return pack_nibbles(nib).reshape(-1)
