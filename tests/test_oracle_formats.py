"""Pins for the oracle's E4M3 / E2M1 encoders (CPU only).

The encoders are written from the OCP FP8 (E4M3) and FP4 (E2M1) element
definitions; these tests check the grid facts those definitions fix, the
round-half-to-even rule, saturation, and agree with torch's own float8_e4m3fn
cast (an independent library routine) on the representable range.
"""
import numpy as np
import pytest
import torch

from oracle import rq_oracle as orc


def test_e4m3_grid_facts():
    enc = orc.e4m3_encode
    assert enc(np.float32(448.0)) == 0x7E
    assert enc(np.float32(2.0 ** -9)) == 0x01          # smallest subnormal
    assert enc(np.float32(2.0 ** -6)) == 0x08          # smallest normal
    assert enc(np.float32(1.0)) == 0x38
    assert [int(enc(np.float32(v))) for v in range(1, 8)] == [0x38, 0x40, 0x44, 0x48, 0x4A, 0x4C, 0x4E]
    assert enc(np.float32(-3.0)) == 0xC4
    assert enc(np.float32(0.0)) == 0x00
    assert enc(np.float32(-0.0)) == 0x80


def test_e4m3_ties_and_saturation():
    enc = orc.e4m3_encode
    assert enc(np.float32(1.0625)) == 0x38   # tie 1.0 / 1.125 -> even (1.0)
    assert enc(np.float32(1.1875)) == 0x3A   # tie 1.125 / 1.25 -> even (1.25)
    assert enc(np.float32(2.0 ** -10)) == 0x00  # tie 0 / 2^-9 -> even (0)
    assert enc(np.float32(3 * 2.0 ** -10)) == 0x02  # tie 2^-9 / 2^-8 -> even
    for v in (449.0, 464.0, 480.0, 1e6, 3e38):
        assert enc(np.float32(v)) == 0x7E
        assert enc(np.float32(-v)) == 0xFE


def test_e4m3_matches_torch_cast():
    rng = np.random.default_rng(0)
    v = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(50),
        rng.uniform(-448, 448, 20000).astype(np.float32),
        (rng.standard_normal(20000) * 2.0 ** -7).astype(np.float32),
        orc.E4M3_GRID.astype(np.float32),
        ((orc.E4M3_GRID[1:] + orc.E4M3_GRID[:-1]) / 2).astype(np.float32),
    ])
    v = v[np.abs(v) <= 448]
    ours = orc.e4m3_encode(v)
    theirs = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)
    assert np.array_equal(orc.e4m3_decode(ours), torch.from_numpy(ours).view(torch.float8_e4m3fn).float().numpy())


def test_e2m1_values_ties_saturation():
    enc = orc.e2m1_encode
    assert [int(enc(np.float32(v))) for v in orc.E2M1_GRID] == list(range(8))
    assert [int(enc(np.float32(-v))) for v in orc.E2M1_GRID[1:]] == list(range(9, 16))
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert enc(np.float32(v)) == c, v
        assert enc(np.float32(-v)) == (c | 8) if c else 8
    assert enc(np.float32(7.0)) == 7 and enc(np.float32(100.0)) == 7
    assert enc(np.float32(-1e9)) == 15


def test_e2m1_nearest_brute_force():
    rng = np.random.default_rng(1)
    v = rng.uniform(-6.5, 6.5, 50000).astype(np.float32)
    c = orc.e2m1_encode(v)
    dec = orc.e2m1_decode(c)
    cand = np.concatenate([-orc.E2M1_GRID, orc.E2M1_GRID])
    best = np.min(np.abs(v[:, None].astype(np.float64) - cand[None, :]), axis=1)
    inside = np.abs(v) <= 6
    assert np.all(np.abs(np.abs(v[inside]) - np.abs(dec[inside])) <= best[inside] + 0)


def test_int4_lut():
    lut = orc.int4_e4m3_lut()
    vals = orc.e4m3_decode(lut)
    assert list(vals) == [0, 1, 2, 3, 4, 5, 6, 7, -8, -7, -6, -5, -4, -3, -2, -1]


def test_pack_layout():
    q = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    assert list(orc.pack_nibbles(q)[0]) == [0x21, 0x43, 0x0F]
    assert np.array_equal(orc.unpack_nibbles(orc.pack_nibbles(q)), q)
    # 16 codes per 32-bit word, nibble i = element i (bits 0-1) | element i+8 (bits 2-3)
    c = np.array([[1, 2, 3, 0, 3, 3, 3, 3, 0, 1, 2, 3, 0, 0, 1, 2]], dtype=np.uint8)
    # nibbles: 1|0<<2=1, 2|1<<2=6, 3|2<<2=11, 0|3<<2=12, 3|0=3, 3|0=3, 3|1<<2=7, 3|2<<2=11
    assert list(orc.pack_crumbs(c)[0]) == [0x61, 0xCB, 0x33, 0xB7]
    assert np.array_equal(orc.unpack_crumbs(orc.pack_crumbs(c)), c)
    rng = np.random.default_rng(5)
    c2 = rng.integers(0, 4, size=(3, 64)).astype(np.uint8)
    assert np.array_equal(orc.unpack_crumbs(orc.pack_crumbs(c2)), c2)
    assert list(orc.int4_from_nibble(np.array([0, 7, 8, 9, 15], np.uint8))) == [0, 7, -8, -7, -1]


def test_sign_magnitude16_layout():
    c = np.arange(16, dtype=np.uint8)
    d = orc.sign_magnitude16(c)
    # upper half: distance from the centre; lower half: the mirrored distance with bit 3
    assert list(d) == [15, 14, 13, 12, 11, 10, 9, 8, 0, 1, 2, 3, 4, 5, 6, 7]
    assert sorted(d) == list(range(16))                                   # a bijection
    assert np.array_equal(orc.code_from_sign_magnitude16(d), c)
    q = np.array([[0, 15, 7, 8, 3, 12]], dtype=np.uint8)
    assert list(orc.pack_nibbles(orc.sign_magnitude16(q))[0]) == [0x7F, 0x08, 0x4C]


@pytest.mark.parametrize("K", [1152, 1536, 3072])
def test_codebook_symmetry_behind_sign_magnitude(K):
    # the stored form relies on centroid(c) = +-centroid(8 + m): check it on the
    # FP64 Lloyd-Max solution and on the E4M3 bytes the GEMM multiplies
    cent, bnd = orc.lloyd_max(K, 16)
    assert np.allclose(cent[::-1], -cent, rtol=0, atol=1e-12)
    _, e8 = orc.codebook_tables(K, 16)
    d = orc.sign_magnitude16(np.arange(16))
    mag = e8[8 + (d & 7)]
    assert np.array_equal(e8, np.where(d & 8, mag | 0x80, mag).astype(np.uint8))
