"""The grouped output projection ("DeepSeek-V4 内部机制" 1.2 Step 3) on the GPU
against the float64 oracle.

Tolerance, derived from the arithmetic: the kernel accumulates in fp32 and
rounds Z = O Wg once to bf16 (relative error <= 2^-8) before Y = Z Wo, then
rounds Y to bf16.  So per output
    |Y_gpu - Y| <= 2^-8 |Y| + 2^-8 S (1 + 2^-4) + 2^-16 S,    S = sum_j |Z_j| |Wo_jo|
(the 2^-4 and 2^-16 terms cover fp32 accumulation over at most 2^16 terms and
the fp32 error of Z itself).  S is taken from a float64 product of the same
inputs: it only sizes the bound, the expected values are the oracle's.  Since
that bound is loose for random signs, the RMS error is also held to
2^-8 RMS(Y), which a dropped group, a transposed tile or a wrong K slice
exceeds by orders of magnitude.
"""
import numpy as np
import pytest
import torch

from compressed_sparse_attention_hca_b200 import csa
from compressed_sparse_attention_hca_b200 import workloads as W
from parity_util import f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    csa.load()


def _check(Y, O, Wg, Wo, want, what):
    got = f64(Y)
    T, n_h, c = O.shape
    g, k1, d_g = Wg.shape
    Z = np.einsum("tgk,gke->tge", f64(O).reshape(T, g, k1), f64(Wg)).reshape(T, g * d_g)
    S = np.abs(Z) @ np.abs(f64(Wo))
    err = np.abs(got - want)
    bound = 2.0 ** -8 * np.abs(want) + 2.0 ** -8 * S * (1 + 2.0 ** -4) + 2.0 ** -16 * S + 1e-30
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} / {bad.size} outside the bound; max err {err.max():.3g}"
    rms_err, rms = np.sqrt((err ** 2).mean()), np.sqrt((want ** 2).mean())
    assert rms_err <= 2.0 ** -8 * rms, f"{what}: rms error {rms_err:.3g} vs rms {rms:.3g}"


@pytest.mark.parametrize("T,n_h,c,g,d_g,d", [
    (5, 16, 64, 4, 128, 256),        # one K slice, one tile
    (3, 32, 128, 2, 256, 384),       # K split 8 ways (group) and 2 ways (output)
    (300, 64, 128, 8, 256, 512),     # prefill: two token tiles, ragged tail of 44
    (1, 8, 512, 1, 128, 128),        # one group, one token
    (37, 128, 64, 16, 128, 640),     # 16 groups, 37 tokens (N = 48)
])
def test_matches_oracle(orc, T, n_h, c, g, d_g, d):
    O, Wg, Wo = W.out_proj_inputs(W.generator(T * 7 + d), T, n_h, c, g, d_g, d)
    Y = csa.grouped_out_proj(O.to(DEV), Wg.to(DEV), Wo.to(DEV))
    torch.cuda.synchronize()
    csa.check_device_status()
    _check(Y, O, Wg, Wo, orc.grouped_out_proj(f64(O), f64(Wg), f64(Wo)), f"T={T} g={g}")


@pytest.mark.parametrize("T", [4, 64])
def test_v4_pro_shape(orc, T):
    """g = 16, d_g = 1024, d = 7168: the plan that splits K over every SM.
    The oracle computes 512 sampled output columns (columns are independent)."""
    s = W.OUT_PROJ_V4_PRO
    O, Wg, Wo = W.out_proj_inputs(W.generator(99 + T), T, s["n_h"], s["c"], s["g"], s["d_g"], s["d"])
    Y = csa.grouped_out_proj(O.to(DEV), Wg.to(DEV), Wo.to(DEV))
    torch.cuda.synchronize()
    csa.check_device_status()
    cols = torch.randperm(s["d"], generator=torch.Generator().manual_seed(T))[:512].sort().values
    Wo_s = Wo[:, cols].contiguous()
    want = orc.grouped_out_proj(f64(O), f64(Wg), f64(Wo_s))
    _check(Y[:, cols.to(DEV)].cpu(), O, Wg, Wo_s, want, f"V4-Pro T={T}")


def test_deterministic_and_workspace_left_zero():
    """Split-K sums add the slices in a fixed order: repeated calls (and a call
    on another stream) give the same bytes, and every call leaves the
    workspace's counters zero, so one workspace serves shapes in turn."""
    s = W.OUT_PROJ_V4_PRO
    O, Wg, Wo = (t.to(DEV) for t in W.out_proj_inputs(W.generator(5), 4, s["n_h"], s["c"], s["g"], s["d_g"], s["d"]))
    need = max(csa.grouped_out_proj_workspace_size(T, **s) for T in (4, 1))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    y0 = csa.grouped_out_proj(O, Wg, Wo, ws=ws)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        y1 = csa.grouped_out_proj(O, Wg, Wo, ws=ws)
    side.synchronize()
    y2 = csa.grouped_out_proj(O[:1].contiguous(), Wg, Wo, ws=ws)
    y3 = csa.grouped_out_proj(O, Wg, Wo, ws=ws)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(y0, y1) and torch.equal(y0, y3)
    # the counters (148 SMs x 16 slots, int32) open the workspace; all zero again
    assert int(ws[:148 * 16 * 4].count_nonzero()) == 0
    assert y2.shape == (1, s["d"])


def test_empty_and_launch_count():
    s = dict(n_h=16, c=64, g=4, d_g=128, d=256)
    O = torch.zeros(0, 16, 64, dtype=torch.bfloat16, device=DEV)
    Wg = torch.zeros(4, 256, 128, dtype=torch.bfloat16, device=DEV)
    Wo = torch.zeros(512, 256, dtype=torch.bfloat16, device=DEV)
    Y = csa.grouped_out_proj(O, Wg, Wo)
    assert Y.shape == (0, 256) and csa.last_launch_count() == 0
    O = torch.randn(2, 16, 64, device=DEV).to(torch.bfloat16)
    csa.grouped_out_proj(O, Wg, Wo)
    assert csa.last_launch_count() == 2
    torch.cuda.synchronize()
    csa.check_device_status()
