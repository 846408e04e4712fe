"""Pins of the oracle's number formats (CPU only).

The bf16 / E4M3 / E2M1 decoders and encoders are checked against published
format definitions (tests/golden, OCP specifications) and against torch's own
casts, never against a second copy of the oracle's code.
"""
import math
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, b = line.split()
            rows.append((a, float(b)))
    return rows


def test_e2m1_decode_matches_spec_table(orc):
    for code, val in _golden("e2m1_values.txt"):
        got = orc.e2m1_decode(int(code))
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e4m3_corner_points_match_spec(orc):
    for code, val in _golden("e4m3_points.txt"):
        got = orc.e4m3_decode(int(code, 16))
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), (code, got, val)


def test_e4m3_decode_all_codes_match_torch(orc):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got, want = orc.e4m3_decode(c), ref[c].item()
        assert (math.isnan(got) and math.isnan(want)) or got == want, c


def test_e4m3_encode_roundtrip_midpoints_and_saturation(orc):
    vals = sorted({orc.e4m3_decode(c) for c in range(0, 0x7F)})  # non-negative finite values
    for c in range(0, 0x7F):
        v = orc.e4m3_decode(c)
        assert orc.e4m3_decode(orc.e4m3_encode(v)) == v
    # midpoints round to the neighbour with the even code
    for lo, hi in zip(vals[:-1], vals[1:]):
        mid = 0.5 * (lo + hi)
        c = orc.e4m3_encode(mid)
        assert orc.e4m3_decode(c) in (lo, hi) and c % 2 == 0, (lo, hi, c)
        assert orc.e4m3_decode(orc.e4m3_encode(-mid)) == -orc.e4m3_decode(c)
    for big in (448.0, 449.0, 463.9, 464.0, 500.0, 1e9):
        assert orc.e4m3_encode(big) == 0x7E and orc.e4m3_encode(-big) == 0xFE


def test_e4m3_encode_matches_torch_cast_in_range(orc):
    g = torch.Generator().manual_seed(11)
    x = (torch.randn(4000, generator=g, dtype=torch.float64) * 60).clamp(-447, 447)
    x = torch.cat([x, torch.randn(1000, generator=g, dtype=torch.float64) * 1e-3])
    x32 = x.to(torch.float32)  # torch's cast starts from fp32: use fp32-exact inputs
    want = x32.to(torch.float8_e4m3fn).view(torch.uint8)
    for xv, wv in zip(x32.tolist(), want.tolist()):
        got = orc.e4m3_encode(xv)
        assert got == wv or (orc.e4m3_decode(got) == 0.0 and orc.e4m3_decode(wv) == 0.0), (xv, got, wv)


def test_e2m1_encode_rne_and_saturation(orc):
    table = {int(c): v for c, v in _golden("e2m1_values.txt")}
    # exact values
    for c in range(16):
        if c == 8:
            continue
        assert orc.e2m1_encode(table[c]) == c
    # midpoints -> even code
    cases = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for x, want in cases.items():
        assert table[orc.e2m1_encode(x)] == want
        assert table[orc.e2m1_encode(-x)] == -want
    for x in (6.0, 6.5, 7.0, 100.0):
        assert table[orc.e2m1_encode(x)] == 6.0
    # nearest value everywhere else
    for x in np.linspace(0, 6, 601):
        best = min(table[c] for c in range(8) if abs(table[c] - x) == min(abs(table[j] - x) for j in range(8)))
        assert abs(table[orc.e2m1_encode(float(x))] - x) == abs(best - x)


def test_bf16_matches_torch_rne(orc):
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(5000, generator=g) * 10.0 ** torch.randint(-20, 20, (5000,), generator=g).float(),
                   torch.tensor([0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1e-40, 65504.0])])
    want = x.to(torch.bfloat16).view(torch.int16).to(torch.int64) & 0xFFFF
    for xv, wv in zip(x.tolist(), want.tolist()):
        assert orc.bf16_encode(xv) == wv, xv
        assert orc.bf16_decode(wv) == float(torch.tensor(wv & 0xFFFF, dtype=torch.int32).to(torch.int16)
                                            .view(torch.bfloat16).float())


def test_fp8mix_row_layout_and_error_bound(orc):
    dim = 512
    assert orc.row_bytes(orc.FP8MIX, dim) == 608  # 448 + 128 + 28 -> 16-byte multiple
    rng = np.random.default_rng(0)
    x = rng.standard_normal((20, dim)) * rng.uniform(0.01, 100, (20, 1))
    buf, _ = orc.encode_rows(x, orc.FP8MIX)
    assert buf.shape == (20, 608) and (buf[:, 604:] == 0).all()
    y = orc.decode_rows(buf, orc.FP8MIX, dim)
    for r in range(20):
        for b in range(7):
            blk = slice(64 * b, 64 * b + 64)
            amax = np.abs(x[r, blk]).max()
            scale = np.frombuffer(buf[r, 576 + 4 * b:580 + 4 * b].tobytes(), np.float32)[0]
            assert scale == np.float32(amax / 448.0)
            # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above 2^-6*scale,
            # absolute error <= 2^-10*scale below
            err = np.abs(y[r, blk] - x[r, blk])
            bound = np.maximum(np.abs(x[r, blk]) * 2.0 ** -4, 2.0 ** -10 * scale) * (1 + 1e-6)
            assert (err <= bound).all()
        # RoPE dims are plain bf16
        rope = x[r, 448:]
        assert np.array_equal(y[r, 448:], orc.round_bf16(rope))


def test_nvfp4_exact_roundtrip_pins_nibble_order(orc):
    """Values that are exactly e2m1 * scale with the block max at 6*scale survive
    encode/decode bit-exactly; element 2j sits in the low nibble of byte j."""
    rng = np.random.default_rng(1)
    table = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    scales = np.array([0.125, 0.25, 0.375, 0.5, 1.0, 2.0])
    dim = 64
    x = np.zeros((10, dim))
    for r in range(10):
        for b in range(dim // 16):
            s = scales[rng.integers(len(scales))]
            v = table[rng.integers(8, size=16)] * rng.choice([-1, 1], 16)
            v[rng.integers(16)] = 6.0
            x[r, 16 * b:16 * b + 16] = v * s
    codes, sf = orc.encode_rows(x, orc.NVFP4)
    assert codes.shape == (10, 32) and sf.shape == (10, 4)
    assert np.array_equal(orc.decode_rows(codes, orc.NVFP4, dim, sf=sf), x)
    # nibble order: element 0 low nibble, element 1 high nibble
    x2 = np.zeros((1, 16))
    x2[0, 0], x2[0, 1] = 6.0, -0.5
    c2, s2 = orc.encode_rows(x2, orc.NVFP4)
    assert c2[0, 0] == (0x7 | (0x9 << 4)) and orc.e4m3_decode(int(s2[0, 0])) == 1.0


def test_nvfp4_blocked_key_scale_layout(orc):
    """The key-cache scale layout (128-row blocks of 512-byte atoms; byte
    m0*16 + m1*4 + kk of atom a = scale of block row m0 + 32*m1, values
    64a + 16kk ..) agrees between the oracle's permutation, the workload
    generator's torch permutation and a direct evaluation of the definition,
    and decodes to the same values as the row-major layout."""
    from compressed_sparse_attention_hca_b200 import workloads as W
    rng = np.random.default_rng(5)
    for rows, dim in [(1, 64), (127, 128), (128, 128), (300, 128), (257, 256)]:
        sf = rng.integers(0, 256, (rows, dim // 16)).astype(np.uint8)
        blocked = orc.block_scales(sf, dim)
        assert blocked.size == -(-rows // 128) * (dim // 64) * 512
        by_gen = W.block_scales(torch.from_numpy(sf), dim).numpy()
        assert np.array_equal(blocked, by_gen)
        for r in range(0, rows, max(1, rows // 17)):
            for j in range(dim // 16):
                m = r % 128
                off = (r // 128) * (dim // 64) * 512 + (j // 4) * 512 + (m % 32) * 16 + (m // 32) * 4 + j % 4
                assert blocked[off] == sf[r, j]
        assert np.array_equal(orc.unblock_scales(blocked, rows, dim), sf)
        codes = rng.integers(0, 256, (rows, dim // 2)).astype(np.uint8)
        sf_ok = np.full_like(sf, 0x38)  # keep scales finite (E4M3 1.0) for the decode comparison
        sf_ok[:, ::2] = 0x30
        assert np.array_equal(orc.decode_rows(codes, orc.NVFP4, dim, sf=orc.block_scales(sf_ok, dim), sf_blocked=True),
                              orc.decode_rows(codes, orc.NVFP4, dim, sf=sf_ok))
