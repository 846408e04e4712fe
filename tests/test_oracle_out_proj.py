"""Pins for the oracle's grouped output projection ("DeepSeek-V4 内部机制" 1.2
Step 3): per group of heads a projection to d_g, then the concatenation
projected to d.  Checked against numpy matrix products (one group; a block-
diagonal matrix), against group locality and against linearity."""
import numpy as np
import pytest
import scipy.linalg

import oracle as orc


@pytest.fixture(scope="module", autouse=True)
def _built():
    orc.build()


def _inputs(rng, T=3, n_h=8, c=16, g=4, d_g=12, d=20):
    O = rng.normal(size=(T, n_h, c))
    Wg = rng.normal(size=(g, n_h // g * c, d_g))
    Wo = rng.normal(size=(g * d_g, d))
    return O, Wg, Wo


def test_one_group_is_two_matrix_products():
    rng = np.random.default_rng(0)
    O, Wg, Wo = _inputs(rng, g=1)
    want = (O.reshape(O.shape[0], -1) @ Wg[0]) @ Wo
    np.testing.assert_allclose(orc.grouped_out_proj(O, Wg, Wo), want, rtol=1e-12, atol=1e-12)


def test_groups_equal_a_block_diagonal_projection():
    rng = np.random.default_rng(1)
    O, Wg, Wo = _inputs(rng, T=5, n_h=16, c=8, g=4, d_g=6, d=11)
    W = scipy.linalg.block_diag(*Wg)  # [n_h c, g d_g]
    want = O.reshape(O.shape[0], -1) @ W @ Wo
    np.testing.assert_allclose(orc.grouped_out_proj(O, Wg, Wo), want, rtol=1e-12, atol=1e-12)


def test_a_group_only_reaches_its_own_block():
    """With W_O the identity, the output is the concatenated group results:
    changing the heads of group 2 changes block 2 only."""
    rng = np.random.default_rng(2)
    O, Wg, _ = _inputs(rng, T=2, n_h=8, c=4, g=4, d_g=5)
    Wo = np.eye(4 * 5)
    y0 = orc.grouped_out_proj(O, Wg, Wo)
    O2 = O.copy()
    O2[:, 4:6] += rng.normal(size=(2, 2, 4))  # heads 4, 5 = group 2
    y1 = orc.grouped_out_proj(O2, Wg, Wo)
    changed = np.abs(y1 - y0).reshape(2, 4, 5).max(axis=(0, 2)) > 0
    assert changed.tolist() == [False, False, True, False]


def test_linear_in_the_head_outputs():
    rng = np.random.default_rng(3)
    O, Wg, Wo = _inputs(rng)
    O2 = rng.normal(size=O.shape)
    lhs = orc.grouped_out_proj(2.5 * O - O2, Wg, Wo)
    rhs = 2.5 * orc.grouped_out_proj(O, Wg, Wo) - orc.grouped_out_proj(O2, Wg, Wo)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-11, atol=1e-11)
