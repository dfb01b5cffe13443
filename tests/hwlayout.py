"""Readers that turn the library's tiled operands back into the oracle's canonical arrays.

Test infrastructure, written from the layout contract in include/sharq.h ("Tiled
operands"), not from the CUDA sources: chunks of 128 rows x 256 K, chunk-major
[row block][K step]; E2M1 pairs with the lower K index in the low nibble; code rows
with their 16-byte units swizzled by row bits; scale runs of 128x4 atoms; metadata
bit strings of 16 bytes per row per 256 K (pairs), two such halves (elements 2:4) or three
(elements 4:8, 12-bit entries).
"""
from __future__ import annotations

import numpy as np
import torch

KSTEP = 256


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def act_layout(block: int, unit: int, sparse: bool = True, m: int = 4) -> dict:
    """Byte offsets inside one activation chunk and the chunk size C (header table); m = 8
    for the 4:8 element pattern."""
    sf_sp, sf_res = 128 // block, 256 // block  # scales per row per K step
    if not sparse:
        return dict(res=0, sf_res=16384, bytes=_round1k(16384 + 128 * sf_res), spk_res=sf_res)
    meta = 6144 if m == 8 else 2048 if unit == 2 else 4096
    off_sp = 24576 + meta
    off_res = off_sp + 128 * sf_sp
    return dict(res=0, sp=16384, meta=24576, sf_sp=off_sp, sf_res=off_res, bytes=_round1k(off_res + 128 * sf_res),
                spk_sp=sf_sp, spk_res=sf_res)


def w_layout(block: int) -> dict:
    sf_sp, sf_res = 128 // block, 256 // block
    return dict(b=0, sf_sp=16384, sf_res=16384 + 256 * sf_sp, bytes=16384 + 256 * (sf_sp + sf_res),
                spk_sp=sf_sp, spk_res=sf_res)


def _round1k(n: int) -> int:
    return (n + 1023) // 1024 * 1024


def _chunk_base(rows: np.ndarray, ks: np.ndarray, k: int, chunk: int) -> np.ndarray:
    return ((rows // 128) * (k // KSTEP) + ks) * chunk


def code_bytes(buf: np.ndarray, rows: int, k: int, chunk: int, off: int, pitch: int) -> np.ndarray:
    """[rows, pitch * k/256] code bytes of a code region (pitch 128 or 64 bytes per K step)."""
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    r = np.arange(rows)[:, None]
    j = np.arange(pitch * (k // KSTEP))[None, :]  # byte index along the row
    ks, within = j // pitch, j % pitch
    rr = r % 128
    swz = rr % 8 if pitch == 128 else (rr // 2) % 4
    addr = _chunk_base(r, ks, k, chunk) + off + rr * pitch + ((within // 16) ^ swz) * 16 + within % 16
    return b[addr]


def nibbles(byts: np.ndarray) -> np.ndarray:
    out = np.empty((byts.shape[0], 2 * byts.shape[1]), dtype=np.uint8)
    out[:, 0::2] = byts & 0xF
    out[:, 1::2] = byts >> 4
    return out


def scale_run(buf: np.ndarray, rows: int, k: int, chunk: int, off: int, spk: int, row_of=None) -> np.ndarray:
    """[rows, spk * k/256] scale bytes of a scale run (spk scales per row per K step).

    row_of maps a row to (chunk row for the chunk base, row inside the run's 128-row
    atoms, extra byte offset) for the weight's 256-row-block runs."""
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    r = np.arange(rows)[:, None]
    s = np.arange(spk * (k // KSTEP))[None, :]
    ks, sl = s // spk, s % spk
    if row_of is None:
        base_row, rr, extra = r, r % 128, 0
    else:
        base_row, rr, extra = row_of(r)
    addr = (_chunk_base(base_row, ks, k, chunk) + off + extra + (sl // 4) * 512 + (rr % 32) * 16 + (rr // 32) * 4
            + sl % 4)
    return b[addr]


def meta_idx(buf: np.ndarray, tokens: int, k: int, unit: int, chunk: int, off: int) -> np.ndarray:
    """Kept unit indices [tokens, G, 2] (groups of 4 units) from the metadata bit strings."""
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    per_step = KSTEP // (4 * unit)  # groups per K step: 32 (pairs) or 64 (elements)
    g = np.arange(k // (4 * unit))[None, :]
    t = np.arange(tokens)[:, None]
    ks, gg = g // per_step, g % per_step
    half, gh = gg // 32, gg % 32
    addr = _chunk_base(t, ks, k, chunk) + off + half * 2048 + (t % 128) * 16 + gh // 2
    nib = (b[addr] >> (4 * (gh % 2))) & 0xF
    return np.stack([nib & 3, nib >> 2], axis=-1).astype(np.int64)


def meta_idx48(buf: np.ndarray, tokens: int, k: int, chunk: int, off: int) -> np.ndarray:
    """Kept element indices [tokens, k/8, 4] of the 4:8 pattern: 12-bit entries (3 bits per
    index, ascending), group g of a K step at bits 12g.. of the row's 48 bytes, byte b of
    those at (b/16)*2048 + r*16 + b%16."""
    b = np.asarray(buf, dtype=np.uint8).reshape(-1)
    g = np.arange(k // 8)[None, :]
    t = np.arange(tokens)[:, None]
    ks, gg = g // 32, g % 32
    base = _chunk_base(t, ks, k, chunk) + off + (t % 128) * 16
    bit0 = 12 * gg
    val = np.zeros(g.shape[:1] + (tokens, k // 8), dtype=np.int64)[0]
    for d in range(3):  # the three bytes that can hold bits of the entry
        byte = bit0 // 8 + d
        byte_c = np.minimum(byte, 47)
        addr = base + (byte_c // 16) * 2048 + byte_c % 16
        val |= np.where(byte < 48, b[addr].astype(np.int64), 0) << (8 * d)
    entry = (val >> (bit0 % 8)) & 0xFFF
    return np.stack([(entry >> (3 * i)) & 7 for i in range(4)], axis=-1)


def read_prep(p, block: int) -> dict:
    """Canonical arrays of a library Prep (2:4 or 4:8) for comparison with oracle.prepare."""
    T, K, unit = p.tokens, p.k, p.unit
    m = getattr(p, "nm_m", 4)
    L = act_layout(block, unit, m=m)
    buf = to_np(p.tiles)
    return dict(
        idx=(meta_idx48(buf, T, K, L["bytes"], L["meta"]) if m == 8 else
             meta_idx(buf, T, K, unit, L["bytes"], L["meta"])),
        sp_codes=nibbles(code_bytes(buf, T, K, L["bytes"], L["sp"], 64)),
        sp_scales=scale_run(buf, T, K, L["bytes"], L["sf_sp"], L["spk_sp"]),
        res_codes=nibbles(code_bytes(buf, T, K, L["bytes"], L["res"], 128)),
        res_scales=scale_run(buf, T, K, L["bytes"], L["sf_res"], L["spk_res"]),
        row_scale=to_np(p.row_scale),
    )


def read_dense(q, block: int) -> dict:
    """Codes and scales of a dense-quantized activation (sharq_quantize_dense)."""
    T, K = q.tokens, q.k
    L = act_layout(block, 2, sparse=False)
    buf = to_np(q.tiles)
    return dict(codes=nibbles(code_bytes(buf, T, K, L["bytes"], L["res"], 128)),
                scales=scale_run(buf, T, K, L["bytes"], L["sf_res"], L["spk_res"]),
                row_scale=to_np(q.row_scale))


def read_wpack(w, block: int, half: str = "own") -> dict:
    """Canonical arrays of a packed weight. `half` picks which copy of the block's scales
    is read: "own" (the chunk of the row's half), "lo" or "hi" (the block's first or second
    half chunk)."""
    N, K = w.n_out, w.k
    L = w_layout(block)
    buf = to_np(w.tiles)

    def run(off, spk):
        def row_of(r):
            blk_half = (r // 128) % 2
            pick = {"own": blk_half, "lo": np.zeros_like(blk_half), "hi": np.ones_like(blk_half)}[half]
            base_row = (r // 256) * 256 + pick * 128
            extra = blk_half * 128 * spk  # second run of the block for its upper 128 rows
            return base_row, r % 128, extra
        return scale_run(buf, N, K, L["bytes"], off, spk, row_of)

    return dict(
        codes=nibbles(code_bytes(buf, N, K, L["bytes"], L["b"], 128)),
        scales_sparse=run(L["sf_sp"], L["spk_sp"]),
        scales_dense=run(L["sf_res"], L["spk_res"]),
        tensor_scale=to_np(w.tensor_scale)[0],
    )
