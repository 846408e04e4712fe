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


def selection_from_scores(scores: np.ndarray, vis: int, k: int) -> np.ndarray:
    """The top-k set of a score row under (score desc, index asc), ascending."""
    s = scores[:vis]
    order = np.lexsort((np.arange(vis), -s))
    return np.sort(order[:min(k, vis)])
