"""The integer and rounding identities the CUDA kernels rely on, checked on
the CPU by brute force (no GPU, no library call).  Each kernel comment states
one of these as the reason a shortcut gives the same bits as the plain
formula; a wrong constant or bound in that reasoning fails here.

  * top-2 with multiplicity by sorted pairs (the export's full-unit path):
    the four's largest is max(h_xy, h_zw), their second
    max(min(h_xy, h_zw), l_xy, l_zw), and merging sorted pairs (t1, t2),
    (X1, X2) gives max(t1, X1) and max(t2, X2, min(t1, X1));
  * int6 code bytes by multiply-adds: with x_i = 0x4B400000 + m_i and
    m_i in [-32, 31], sum_i (4 x_i) 2^(8i) + C, XOR 0x80808080, is the word
    of the two's-complement bytes 4 m_i (C folds the offset in);
  * the clamp of rne(k / 4) at 31 through the bit pattern: min over
    0x4B400000 + m with 0x4B40001F;
  * the dequantize row index: floor(l / d) = the high 64 bits of
    l * (floor((2^64 - 1) / d) + 1) for l < 2^46 and 2 <= d <= 2^18;
  * the quantizer's tiles: min(S, 8) warps per row of S 512-column segments,
    8 / min(S, 8) rows per block, every row and segment covered once.
"""
import itertools

import numpy as np
import pytest


def _top2(vals):
    s = sorted(vals, reverse=True)
    return s[0], s[1]


def _pairs_push4(v, t1, t2):
    a, b, c, e = (abs(x) for x in v)
    hab, lab = max(a, b), min(a, b)
    hce, lce = max(c, e), min(c, e)
    x1 = max(hab, hce)
    x2 = max(min(hab, hce), lab, lce)
    y = min(t1, x1)
    return max(t1, x1), max(t2, y, x2)


def _merge(t1, t2, u1, u2):
    return max(t1, u1), max(t2, u2, min(t1, u1))


@pytest.mark.parametrize("seed", range(4))
def test_sorted_pair_top2_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    for _ in range(400):
        n4 = int(rng.integers(1, 13))
        # few distinct magnitudes, so ties (with multiplicity) are common
        vals = rng.choice(np.float32([0.0, 0.25, -0.25, 0.5, -0.5, 0.125, 1.0]), size=4 * n4)
        if rng.random() < 0.5:
            vals = (rng.standard_normal(4 * n4) * 0.02).astype(np.float32)
        # three chains over thirds, merged, as for one 1,536-column row
        chains = [(0.0, 0.0)] * 3
        for g in range(n4):
            c = g % 3
            chains[c] = _pairs_push4(vals[4 * g:4 * g + 4], *chains[c])
        t1, t2 = chains[0]
        t1, t2 = _merge(t1, t2, *chains[1])
        t1, t2 = _merge(t1, t2, *chains[2])
        r1, r2 = _top2([abs(float(x)) for x in vals] + [0.0, 0.0])
        assert (t1, t2) == (r1, r2)


def _pack_offset4(xs, mul, base):
    kc = ((128 - mul * base) * 0x01010101) % 2**32
    acc = (xs[3] * ((mul << 24) % 2**32) + kc) % 2**32
    acc = (xs[2] * (mul << 16) + acc) % 2**32
    acc = (xs[1] * (mul << 8) + acc) % 2**32
    acc = (xs[0] * mul + acc) % 2**32
    return acc ^ 0x80808080


def test_int6_code_bytes_by_multiply_adds():
    base = 0x4B400000
    for ms in itertools.product(range(-32, 32, 3), repeat=4):
        xs = [(base + m) % 2**32 for m in ms]
        want = sum(((4 * m) & 0xFF) << (8 * i) for i, m in enumerate(ms))
        assert _pack_offset4(xs, 4, base) == want


def test_int6_top_clamp_on_the_bit_pattern():
    # kOff + rne(k / 4) for k in [-127, 127] (no clamp binds below); the
    # grid's clamp min(4 rne(k / 4), 124) is min on the pattern at +31
    koff = np.float32(12582912.0)
    for k in range(-127, 128):
        t = np.float32(koff + np.float32(k))
        u = np.float32(np.float32(t * np.float32(0.25)) + np.float32(-koff / 4))
        u = np.float32(u + koff)
        bits = int(np.array(u, np.float32).view(np.uint32))
        m = min(bits, 0x4B40001F) - 0x4B400000
        assert 4 * m == min(4 * round(k / 4), 124), k


def test_dequant_row_index_by_multiply_high():
    rng = np.random.default_rng(7)
    for d in [2, 3, 4, 34, 128, 384, 1 << 18] + [int(x) for x in rng.integers(2, 1 << 18, 200)]:
        magic = (2**64 - 1) // d + 1
        for l in [0, 1, d - 1, d, d + 1, 2**31 - 1, 2**46 - 1] + \
                 [int(x) for x in rng.integers(0, 2**46, 30)]:
            assert (l * magic) >> 64 == l // d


@pytest.mark.parametrize("K", [8, 64, 136, 512, 520, 1032, 1536, 2048, 4096, 4104, 9000])
def test_quantizer_tiles_cover_every_row_and_segment(K):
    K4 = K // 4
    S = (K4 + 127) >> 7
    wpr = min(S, 8)
    rpb = 8 // wpr
    for N in [1, 7, 8, 9, 37, 512]:
        tiles = (N + rpb - 1) // rpb
        seen = {}
        for t in range(tiles):
            for warp in range(8):
                rib, wir = divmod(warp, wpr)
                row = t * rpb + rib
                if rib >= rpb or row >= N:
                    continue
                for sg in range(wir, S, wpr):
                    for j in range(sg * 128, min(sg * 128 + 128, K4)):
                        seen[(row, j)] = seen.get((row, j), 0) + 1
        assert len(seen) == N * K4 and set(seen.values()) == {1}
