"""Helpers for the parity tests: move tensors to the oracle's numpy formats and
compare results.  No method arithmetic lives here."""
import numpy as np
import torch


def raw(t: torch.Tensor) -> np.ndarray:
    """A tensor as the oracle's row format: f32 -> float32, bf16 -> uint16 bits,
    uint8 -> uint8 (FP8MIX rows, NVFP4 codes/scales)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float32, torch.uint8, torch.int32, torch.int64):
        return t.numpy()
    raise TypeError(t.dtype)


def f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of an f32 / bf16 tensor."""
    return t.detach().cpu().to(torch.float64).numpy()


def assert_close(got, want, atol, rtol=0.0, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (what, got.shape, want.shape)
    err = np.abs(got - want)
    bad = err > atol + rtol * np.abs(want)
    if bad.any():
        i = np.unravel_index(np.argmax(err - atol - rtol * np.abs(want)), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} / {bad.size} elements off; worst at {i}: "
                             f"got {got[i]!r} want {want[i]!r} (max abs err {err.max():.3g})")


def _enc(fn, a):
    a = np.asarray(a, np.float64)
    return np.vectorize(lambda v: int(fn(float(v))), otypes=[np.int64])(a) if a.size else a.astype(np.int64)


def check_nvfp4_rows(orc, codes, sf_rowmajor, want, dim, rel=1e-5):
    """NVFP4 rows written by the GPU (codes [rows, dim/2], row-major E4M3 scale
    codes [rows, dim/16]) against the oracle's fp64 rows `want`.

    The GPU computes a row in fp32, the oracle in fp64, so the two may only
    disagree where the fp64 value sits within fp32 rounding of an encoder
    decision: each block scale must be the oracle encoder's code for amax/6,
    unless amax/6 moved by delta would change that code; each value code must
    be the oracle encoder's code for value/scale (with the GPU's scale),
    unless the value moved by delta would change it.  delta = rel * (1 + amax
    of the block), far above fp32 error and far below any step of the
    formats, so a code off by one step where the rounding is clear fails."""
    codes = np.asarray(codes, np.uint8)
    sf_rowmajor = np.asarray(sf_rowmajor, np.uint8)
    want = np.asarray(want, np.float64)
    rows = want.shape[0]
    nib = np.stack([codes & 15, codes >> 4], axis=-1).reshape(rows, dim).astype(np.int64)
    blocks = want.reshape(rows, dim // 16, 16)
    amax = np.abs(blocks).max(axis=-1)
    delta = rel * (1.0 + amax)
    s_ref = _enc(orc.e4m3_encode, amax / 6.0)
    s_lo = _enc(orc.e4m3_encode, np.maximum(amax - delta, 0.0) / 6.0)
    s_hi = _enc(orc.e4m3_encode, (amax + delta) / 6.0)
    s_gpu = sf_rowmajor.astype(np.int64)
    bad_s = (s_gpu != s_ref) & ~((s_lo != s_hi) & ((s_gpu == s_lo) | (s_gpu == s_hi)))
    assert not bad_s.any(), f"{bad_s.sum()} block scales differ where the rounding is clear"
    sval = np.vectorize(orc.e4m3_decode, otypes=[np.float64])(s_gpu)
    s_rep = np.repeat(sval, 16, axis=1)
    d_rep = np.repeat(delta, 16, axis=1)
    zero = s_rep == 0
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.where(zero, 0.0, want / np.where(zero, 1.0, s_rep))
        x_lo = np.where(zero, 0.0, (want - d_rep) / np.where(zero, 1.0, s_rep))
        x_hi = np.where(zero, 0.0, (want + d_rep) / np.where(zero, 1.0, s_rep))
    c_ref = _enc(orc.e2m1_encode, x)
    c_lo, c_hi = _enc(orc.e2m1_encode, x_lo), _enc(orc.e2m1_encode, x_hi)

    def mag(c):
        return np.vectorize(orc.e2m1_decode, otypes=[np.float64])(c)

    same = (nib == c_ref) | ((mag(nib) == 0) & (mag(c_ref) == 0))  # +0 and -0
    ok_amb = (c_lo != c_hi) & ((nib == c_lo) | (nib == c_hi))
    bad_c = ~(same | ok_amb)
    assert not bad_c.any(), f"{bad_c.sum()} value codes differ where the rounding is clear"
