"""Readers that turn the library's hardware layouts back into the oracle's canonical arrays.

Test infrastructure, written from the layout contract in include/sharq.h (not from
the CUDA sources): E2M1 pairs with the lower K index in the low nibble, 128x4 scale
atoms, metadata slabs of 128 bits per row.
"""
from __future__ import annotations

import numpy as np
import torch


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def unpack_e2m1(buf: np.ndarray, rows: int, n_codes: int) -> np.ndarray:
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)[: rows * n_codes // 2].reshape(rows, n_codes // 2)
    out = np.empty((rows, n_codes), dtype=np.uint8)
    out[:, 0::2] = b & 0xF
    out[:, 1::2] = b >> 4
    return out


def atom_index(rows: int, spr: int) -> np.ndarray:
    """Byte offset of every (row, scale) in a 128x4-atom scale tensor: [rows, spr]."""
    r = np.arange(rows)[:, None]
    s = np.arange(spr)[None, :]
    return ((r // 128) * (spr // 4) + s // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + s % 4


def unswizzle_scales(buf: np.ndarray, rows: int, spr: int) -> np.ndarray:
    return np.asarray(buf, dtype=np.uint8).reshape(-1)[atom_index(rows, spr)]


def meta_to_idx(buf: np.ndarray, tokens: int, k: int, unit: int) -> np.ndarray:
    """Kept unit indices [tokens, G, 2] from metadata slabs (groups of 4 units)."""
    tp = (tokens + 255) // 256 * 256
    G = k // (4 * unit)
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    g = np.arange(G)
    t = np.arange(tokens)[:, None]
    byte = ((g // 32)[None, :] * tp + t) * 16 + (g % 32)[None, :] // 2
    nib = (b[byte] >> (4 * (g % 2))[None, :]) & 0xF
    return np.stack([nib & 3, nib >> 2], axis=-1).astype(np.int64)


def read_prep(p, block: int) -> dict:
    """Canonical arrays of a library Prep (pattern 2:4) for comparison with oracle.prepare."""
    T, K, unit = p.tokens, p.k, p.unit
    stored = K // 2
    return dict(
        idx=meta_to_idx(to_np(p.sparse_meta), T, K, unit),
        sp_codes=unpack_e2m1(to_np(p.sparse_codes), T, stored),
        sp_scales=unswizzle_scales(to_np(p.sparse_scales), T, stored // block),
        res_codes=unpack_e2m1(to_np(p.resid_codes), T, K),
        res_scales=unswizzle_scales(to_np(p.resid_scales), T, K // block),
        row_scale=to_np(p.row_scale),
    )


def read_wpack(w, block: int) -> dict:
    N, K = w.n_out, w.k
    return dict(
        codes=unpack_e2m1(to_np(w.codes), N, K),
        scales_sparse=unswizzle_scales(to_np(w.scales_sparse), N, K // (2 * block)),
        scales_dense=unswizzle_scales(to_np(w.scales_dense), N, K // block),
        tensor_scale=to_np(w.tensor_scale)[0],
    )
