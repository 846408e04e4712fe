"""Pins for the oracle's Q / KV-entry RMSNorm and partial RoPE
("DeepSeek-V4 内部机制" 1.4 table; admirer.cn article, RoPE paragraph).

Each check ties the oracle to something other than its own formula: torch's
RMSNorm, complex multiplication, the group law of rotations, the relative-
position property that the page states as the reason for rotating the output
at -i, and the identity at position 0."""
import numpy as np
import pytest
import torch

import oracle as orc

pytestmark = pytest.mark.filterwarnings("ignore")
R = 64


@pytest.fixture(scope="module", autouse=True)
def _built():
    orc.build()


def test_rmsnorm_equals_torch_rms_norm():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(7, 512)) * rng.uniform(0.1, 10, size=(7, 1))
    g = rng.normal(size=512)
    for eps in (1e-6, 1e-2):
        want = torch.nn.functional.rms_norm(torch.from_numpy(x), (512,), weight=torch.from_numpy(g), eps=eps)
        np.testing.assert_allclose(orc.rmsnorm(x, g, eps), want.numpy(), rtol=1e-13, atol=1e-13)


def test_rmsnorm_unit_mean_square_and_scale_invariance():
    rng = np.random.default_rng(1)
    x = rng.normal(size=(5, 448))
    y = orc.rmsnorm(x, None, 0.0)
    np.testing.assert_allclose((y * y).mean(axis=1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(orc.rmsnorm(37.5 * x, None, 0.0), y, rtol=1e-13, atol=1e-15)


def _complex_rope(x, p, base=10000.0):
    """The rotation written as complex multiplication of adjacent pairs."""
    x = np.array(x, np.float64)
    c = x[..., -R::2] + 1j * x[..., -R + 1::2]
    freq = base ** (-np.arange(R // 2) * 2.0 / R)
    c = c * np.exp(1j * np.asarray(p, np.float64)[..., None] * freq)
    out = x.copy()
    out[..., -R::2] = c.real
    out[..., -R + 1::2] = c.imag
    return out


def test_rope_equals_complex_multiplication_and_leaves_other_dims():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(6, 512))
    pos = np.array([0, 1, 7, 1000, 262143, 1048575], np.float64)
    y = orc.rope_tail(x, pos)
    # the two agree up to the rounding of the angle (|p| * 2^-52 radians)
    np.testing.assert_allclose(y, _complex_rope(x, pos), rtol=0, atol=1e-9)
    np.testing.assert_array_equal(y[:, :512 - R], x[:, :512 - R])
    np.testing.assert_array_equal(y[0], x[0])  # position 0: identity
    # pair 0 turns by one radian per position step, the last pair the slowest
    e = np.zeros((1, 512))
    e[0, 512 - R] = 1.0
    np.testing.assert_allclose(orc.rope_tail(e, [1.0])[0, 512 - R:512 - R + 2], [np.cos(1.0), np.sin(1.0)],
                               atol=1e-15)


def test_rope_preserves_pair_norms_and_composes():
    rng = np.random.default_rng(3)
    x = rng.normal(size=(4, 128))
    a, b = np.array([3.0, -5.0, 100.0, 0.5]), np.array([11.0, 5.0, -40.0, 2.0])
    y = orc.rope_tail(x, a)
    pn = lambda v: v[:, -R::2] ** 2 + v[:, -R + 1::2] ** 2  # noqa: E731
    np.testing.assert_allclose(pn(y), pn(x), rtol=1e-12)
    np.testing.assert_allclose(orc.rope_tail(y, b), orc.rope_tail(x, a + b), atol=1e-11)
    np.testing.assert_allclose(orc.rope_tail(y, -a), x, atol=1e-12)


def test_rope_dot_products_depend_on_relative_position_only():
    rng = np.random.default_rng(4)
    q, k = rng.normal(size=(1, 512)), rng.normal(size=(1, 512))
    d0 = (orc.rope_tail(q, [1000.0]) * orc.rope_tail(k, [977.0])).sum()
    d1 = (orc.rope_tail(q, [501023.0]) * orc.rope_tail(k, [501000.0])).sum()
    d2 = (orc.rope_tail(q, [1000.0]) * orc.rope_tail(k, [970.0])).sum()
    assert d0 == pytest.approx(d1, rel=1e-9)
    assert abs(d0 - d2) > 1e-6


def test_output_turned_at_minus_t_is_invariant_to_a_global_shift():
    """Shared-KV attention with q at t and KV rows at p_j, the output turned at
    -t: shifting every position by s leaves the output unchanged, and without
    the output rotation it does not (the page's reason for position -i)."""
    rng = np.random.default_rng(5)
    H, c, n = 4, 512, 9
    q = orc.rmsnorm(rng.normal(size=(H, c)))
    kv = orc.rmsnorm(rng.normal(size=(n, c)))
    sink = rng.normal(size=H)
    t = 5000.0
    p = t - np.array([0, 1, 2, 3, 4, 7, 11, 15, 127], np.float64)

    def out(shift, turn_back=True):
        o = orc.attend(orc.rope_tail(q, np.full(H, t + shift)), orc.rope_tail(kv, p + shift), sink, c ** -0.5)
        return orc.rope_tail(o, np.full(H, -(t + shift))) if turn_back else o

    np.testing.assert_allclose(out(0.0), out(123457.0), atol=1e-9)
    assert np.abs(out(0.0, False) - out(123457.0, False)).max() > 1e-3
