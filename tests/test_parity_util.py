"""The NVFP4 row check used by the GPU parity tests, on the CPU: rows the
oracle encodes itself pass, and a code or a block scale moved by one step
where the rounding is clear fails (so the check is tight enough to catch a
systematic off-by-one in the GPU encoder)."""
import numpy as np
import pytest

from parity_util import check_nvfp4_rows


def _rows(seed, rows=6, dim=128):
    rng = np.random.default_rng(seed)
    return rng.normal(size=(rows, dim)) * rng.uniform(0.2, 3.0, size=(rows, 1))


def test_oracle_encoding_passes(orc):
    x = _rows(1)
    codes, sf = orc.encode_rows(x, orc.NVFP4)
    check_nvfp4_rows(orc, codes, sf, x, 128)


def test_one_code_off_by_one_step_fails(orc):
    x = _rows(2)
    codes, sf = orc.encode_rows(x, orc.NVFP4)
    # pick a value whose scaled magnitude is clearly inside a rounding cell
    s = np.repeat(np.vectorize(orc.e4m3_decode)(sf.astype(np.int64)), 16, axis=1)
    r = np.abs(x / s)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    mids = (grid[1:] + grid[:-1]) / 2
    dist = np.min(np.abs(r[..., None] - mids), axis=-1)
    i, j = np.unravel_index(np.argmax(np.where(r < 5.5, dist, -1)), r.shape)
    nib = codes[i, j // 2] >> (4 * (j % 2)) & 15
    mag = nib & 7
    new = (nib & 8) | (mag + 1 if mag < 7 else mag - 1)
    bad = codes.copy()
    bad[i, j // 2] = (bad[i, j // 2] & (0xF0 if j % 2 == 0 else 0x0F)) | (new << (4 * (j % 2)))
    with pytest.raises(AssertionError, match="value codes"):
        check_nvfp4_rows(orc, bad, sf, x, 128)


def test_one_scale_off_by_one_step_fails(orc):
    x = _rows(3)
    codes, sf = orc.encode_rows(x, orc.NVFP4)
    bad = sf.copy()
    bad[0, 0] = bad[0, 0] + 1
    with pytest.raises(AssertionError, match="block scales"):
        check_nvfp4_rows(orc, codes, bad, x, 128)
