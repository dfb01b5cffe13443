"""Self-checks of the test-side layout readers (tests/hwlayout.py), on the CPU: bit strings
packed here from the header's layout contract must read back to the same indices. The GPU
parity tests decode the library's tiled operands with these readers, so a reader that
misplaced a bit would hide (or fake) a kernel mismatch."""
import numpy as np
import pytest

from tests import hwlayout as hw


@pytest.mark.parametrize("T,K", [(130, 512), (3, 256)])
def test_meta_idx48_round_trip(T, K):
    """4:8 over elements: group g of a K step in bits 12g..12g+11 of the row's 48 bytes, byte b of
    those at (b/16)*2048 + r*16 + b%16, four ascending 3-bit indices per entry."""
    rng = np.random.default_rng(T + K)
    L = hw.act_layout(16, 1, m=8)
    chunk, off = L["bytes"], L["meta"]
    assert (chunk, off) == (33792, 24576)
    buf = np.zeros(((T + 255) // 256 * 2) * (K // 256) * chunk, np.uint8)
    idx = np.sort(np.stack([rng.permutation(8)[:4] for _ in range(T * K // 8)]).reshape(T, K // 8, 4), axis=-1)
    for t in range(T):
        for g in range(K // 8):
            ks, gg = g // 32, g % 32
            entry = idx[t, g, 0] | idx[t, g, 1] << 3 | idx[t, g, 2] << 6 | idx[t, g, 3] << 9
            base = ((t // 128) * (K // 256) + ks) * chunk + off + (t % 128) * 16
            for bit in range(12):
                if (entry >> bit) & 1:
                    b = 12 * gg + bit
                    byte = b // 8
                    buf[base + (byte // 16) * 2048 + byte % 16] |= 1 << (b % 8)
    assert np.array_equal(hw.meta_idx48(buf, T, K, chunk, off), idx)


@pytest.mark.parametrize("unit", [2, 1])
def test_meta_idx_2of4_round_trip(unit):
    """2:4: one nibble i0 | i1 << 2 per group; pairs 16 bytes per row per K step, elements two
    16-byte halves 2048 apart."""
    rng = np.random.default_rng(unit)
    T, K = 200, 512
    L = hw.act_layout(16, unit)
    chunk, off = L["bytes"], L["meta"]
    buf = np.zeros(((T + 255) // 256 * 2) * (K // 256) * chunk, np.uint8)
    G = K // (4 * unit)
    idx = np.sort(np.stack([rng.permutation(4)[:2] for _ in range(T * G)]).reshape(T, G, 2), axis=-1)
    per_step = 256 // (4 * unit)
    for t in range(T):
        for g in range(G):
            ks, gg = g // per_step, g % per_step
            half, gh = gg // 32, gg % 32
            addr = ((t // 128) * (K // 256) + ks) * chunk + off + half * 2048 + (t % 128) * 16 + gh // 2
            buf[addr] |= (idx[t, g, 0] | idx[t, g, 1] << 2) << (4 * (gh % 2))
    assert np.array_equal(hw.meta_idx(buf, T, K, unit, chunk, off), idx)
