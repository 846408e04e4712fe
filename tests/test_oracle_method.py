"""Pins of the oracle's method arithmetic (CPU only).

Each test checks the oracle against something other than itself: a closed
form, a library routine (numpy matmul, scipy softmax/expit, torch scaled dot
product attention in float64), brute force on tiny inputs, or an invariant
that the pages fix:
  * "DeepSeek-V4 内部机制" 1.2 Step 1: per-channel (Hadamard) softmax weights,
    entry i covers tokens [m(i-1), m(i+1)); 1.3: HCA has no overlap and no
    top-k; 1.2 Step 2: non-negative ReLU-weighted index score, top-k; 1.4: the
    sink adds exp(z') to the denominator only, the window holds raw tokens.
  * yunpan.plus write-up, CSA step 1: every group except the last is covered
    by two entries.
"""
import numpy as np
import pytest
import scipy.special as sps
import torch
import torch.nn.functional as F

RNG = np.random.default_rng(1234)


def _tok(n, d, rng=RNG):
    return rng.standard_normal((n, d))


# ----------------------------------------------------------------- compressor

def _csa_inputs(n, d, m, rng=RNG):
    return dict(Ca=_tok(n, d, rng), Cb=_tok(n, d, rng), Za=_tok(n, d, rng), Zb=_tok(n, d, rng),
                Ba=0.1 * rng.standard_normal((m, d)), Bb=0.1 * rng.standard_normal((m, d)))


def test_compress_weights_sum_to_one(orc):
    n, d, m = 64, 8, 4
    x = _csa_inputs(n, d, m)
    x["Ca"][:] = 1.0
    x["Cb"][:] = 1.0
    out = orc.compress(m=m, **x)
    assert out.shape == (n // m, d)
    assert np.abs(out - 1.0).max() < 1e-14


def test_compress_constant_logits_is_mean_of_2m_tokens(orc):
    n, d, m = 40, 6, 4
    x = _csa_inputs(n, d, m)
    x["Za"][:] = 0.7
    x["Zb"][:] = 0.7
    x["Ba"][:] = 0.0
    x["Bb"][:] = 0.0
    out = orc.compress(m=m, **x)
    for i in range(n // m):
        vals = [x["Ca"][m * i:m * i + m]]
        if i >= 1:
            vals.append(x["Cb"][m * (i - 1):m * i])
        want = np.concatenate(vals).mean(axis=0)
        assert np.abs(out[i] - want).max() < 1e-14, i


def test_compress_m1_closed_form_logistic(orc):
    """m = 1: entry i = sigma(a - b) C^a_i + (1 - sigma(a - b)) C^b_{i-1}."""
    n, d = 30, 5
    x = _csa_inputs(n, d, 1)
    out = orc.compress(m=1, **x)
    for i in range(n):
        if i == 0:
            want = x["Ca"][0]
        else:
            a = x["Za"][i] + x["Ba"][0]
            b = x["Zb"][i - 1] + x["Bb"][0]
            s = sps.expit(a - b)
            want = s * x["Ca"][i] + (1 - s) * x["Cb"][i - 1]
        assert np.abs(out[i] - want).max() < 1e-14


def test_compress_matches_library_softmax(orc):
    n, d, m = 48, 7, 4
    x = _csa_inputs(n, d, m)
    out = orc.compress(m=m, **x)
    for i in range(1, n // m):
        logits = np.concatenate([x["Za"][m * i:m * i + m] + x["Ba"], x["Zb"][m * (i - 1):m * i] + x["Bb"]])
        vals = np.concatenate([x["Ca"][m * i:m * i + m], x["Cb"][m * (i - 1):m * i]])
        S = sps.softmax(logits, axis=0)  # over the 2m positions, per channel
        assert np.abs(out[i] - (S * vals).sum(0)).max() < 1e-14


def test_compress_locality_and_double_coverage(orc):
    """Changing the tokens of group g changes exactly entries g and g+1."""
    n, d, m = 64, 4, 4
    x = _csa_inputs(n, d, m)
    base = orc.compress(m=m, **x)
    E = n // m
    for g in range(E):
        y = {k: v.copy() for k, v in x.items()}
        for key in ("Ca", "Cb", "Za", "Zb"):
            y[key][m * g:m * g + m] += 1.0
        out = orc.compress(m=m, **y)
        changed = [i for i in range(E) if not np.array_equal(out[i], base[i])]
        assert changed == ([g, g + 1] if g + 1 < E else [g]), (g, changed)


def test_compress_one_hot_logit_selects_token(orc):
    n, d, m = 32, 3, 4
    x = _csa_inputs(n, d, m)
    for k in ("Za", "Zb", "Ba", "Bb"):
        x[k][:] = 0.0
    i, j = 5, 2
    x["Za"][m * i + j, :] = 60.0
    out = orc.compress(m=m, **x)
    assert np.abs(out[i] - x["Ca"][m * i + j]).max() < 1e-20 + 1e-12


def test_compress_first_entry_has_no_previous_block(orc):
    n, d, m = 16, 5, 4
    x = _csa_inputs(n, d, m)
    csa = orc.compress(m=m, **x)
    hca = orc.compress(x["Ca"], x["Za"], x["Ba"], m)
    assert np.array_equal(csa[0], hca[0])
    S = sps.softmax(x["Za"][:m] + x["Ba"], axis=0)
    assert np.abs(csa[0] - (S * x["Ca"][:m]).sum(0)).max() < 1e-14


def test_hca_no_overlap_matches_library_softmax(orc):
    n, d, m = 3 * 128 + 17, 4, 128  # trailing partial block is not compressed
    C, Z = _tok(n, d), _tok(n, d)
    B = 0.1 * RNG.standard_normal((m, d))
    out = orc.compress(C, Z, B, m)
    assert out.shape == (3, d)
    for i in range(3):
        S = sps.softmax(Z[m * i:m * i + m] + B, axis=0)
        assert np.abs(out[i] - (S * C[m * i:m * i + m]).sum(0)).max() < 1e-14
    # locality: tokens of other groups do not matter
    C2 = C.copy()
    C2[m:2 * m] += 5
    out2 = orc.compress(C2, Z, B, m)
    assert np.array_equal(out2[0], out[0]) and np.array_equal(out2[2], out[2])
    assert not np.array_equal(out2[1], out[1])


def test_compress_token_offset_equals_full(orc):
    """Computing entries from a slice of token rows (decode: only the last
    2m tokens are kept) gives the same result as from the whole sequence."""
    n, d, m = 64, 6, 4
    x = _csa_inputs(n, d, m)
    full = orc.compress(m=m, **x)
    e0 = 13
    tok0 = m * (e0 - 1)
    part = orc.compress(m=m, tok0=tok0, e0=e0, n_out=3, **{k: (v[tok0:] if k[0] in "CZ" else v)
                                                          for k, v in x.items()})
    assert np.array_equal(part, full[e0:e0 + 3])
    with pytest.raises(ValueError):
        orc.compress(m=m, tok0=tok0 + m, e0=e0, n_out=1, **{k: (v[tok0 + m:] if k[0] in "CZ" else v)
                                                           for k, v in x.items()})


# ------------------------------------------------------------------- indexer

def test_index_score_single_head_is_matmul(orc):
    q = np.abs(_tok(1, 16))
    K = np.abs(_tok(50, 16))
    got = orc.index_scores(q, np.ones(1), K)
    assert np.abs(got - (K @ q[0])).max() < 1e-12


def test_index_score_head_weights_and_relu(orc):
    H, d = 5, 12
    q, K = _tok(H, d), _tok(40, d)
    for h in range(H):
        w = np.zeros(H)
        w[h] = 1.0
        got = orc.index_scores(q, w, K)
        assert np.abs(got - np.maximum(K @ q[h], 0.0)).max() < 1e-12
    w1, w2 = RNG.uniform(0, 1, H), RNG.uniform(0, 1, H)
    s1, s2 = orc.index_scores(q, w1, K), orc.index_scores(q, w2, K)
    s12 = orc.index_scores(q, w1 + 2.5 * w2, K)
    assert np.abs(s12 - (s1 + 2.5 * s2)).max() < 1e-12
    assert (s1 >= 0).all()
    # all dot products negative -> ReLU removes every term
    qn = -np.abs(q)
    assert (orc.index_scores(qn, w1, np.abs(K)) == 0).all()


def _brute_topk(scores, k):
    order = sorted(range(len(scores)), key=lambda i: (-scores[i], i))
    return (order + [-1] * k)[:k]


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (20, 20), (33, 16), (64, 16), (5, 9), (0, 4)])
def test_topk_brute_force_with_ties(orc, n, k):
    for trial in range(20):
        scores = RNG.integers(0, 4, n).astype(np.float64)  # many exact ties
        assert list(orc.topk(scores, k)) == _brute_topk(list(scores), k)


def test_index_topk_visibility_and_padding(orc):
    B, T, H, d, E, m, k = 2, 5, 3, 8, 20, 4, 6
    qI, wI, KI = RNG.standard_normal((B, T, H, d)), RNG.uniform(0, 1, (B, T, H)), RNG.standard_normal((B, E, d))
    q_pos = np.array([[0, 3, 10, 23, 79], [2, 7, 40, 80, 90]])
    scores, idx = orc.index_topk(qI, wI, KI, q_pos, m, k)
    for b in range(B):
        for t in range(T):
            vis = min((q_pos[b, t] + 1) // m, E)
            sel = idx[b, t]
            assert (sel[:min(k, vis)] >= 0).all() and (sel[min(k, vis):] == -1).all()
            assert (sel[sel >= 0] < vis).all()
            assert np.isneginf(scores[b, t, vis:]).all()
            raw = orc.index_scores(qI[b, t], wI[b, t], KI[b, :vis])
            assert np.array_equal(scores[b, t, :vis], orc.round_bf16(raw))
            # every selected score >= every unselected visible score
            chosen = set(sel[sel >= 0].tolist())
            rest = [s for s in range(vis) if s not in chosen]
            if chosen and rest:
                assert min(scores[b, t, list(chosen)]) >= max(scores[b, t, rest])


# ----------------------------------------------------------------- attention

def _sdpa(q, kv, mask, scale):
    """torch float64 scaled_dot_product_attention with K = V shared by all heads."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]  # [1, H, T, c]
    kt = torch.from_numpy(kv)[None, None].expand(1, q.shape[1], -1, -1)
    out = F.scaled_dot_product_attention(qt, kt, kt, attn_mask=torch.from_numpy(mask), scale=scale)
    return out[0].permute(1, 0, 2).numpy()


def test_mqa_reduces_to_dense_causal_attention(orc):
    """m = 1 one-branch compression (weight 1: entry = token), k >= E, no window,
    sink = -inf: CSA sparse MQA is dense causal MQA."""
    n, c, H = 24, 16, 3
    C, Z = _tok(n, c), _tok(n, c)
    entries = orc.compress(C, Z, np.zeros((1, c)), 1)
    assert np.array_equal(entries, C)
    Q = RNG.standard_normal((1, n, H, c))
    q_pos = np.arange(n)[None]
    idx = np.full((1, n, n + 3), -1, np.int32)
    for t in range(n):
        idx[0, t, :t + 1] = RNG.permutation(t + 1)
    ent32 = entries.astype(np.float32)
    sink = np.full(H, -np.inf)
    scale = 0.3
    out = orc.sparse_mqa(Q, ent32[None], orc.F32, idx, ent32[None], [0], q_pos, 0, 1, sink, scale)
    mask = np.tril(np.ones((n, n), bool))
    want = _sdpa(Q[0], ent32.astype(np.float64), mask, scale)
    assert np.abs(out[0] - want).max() < 1e-12
    # HCA dense over the same entries is the same thing
    out2 = orc.hca_dense_mqa(Q, ent32[None], orc.F32, ent32[None], [0], q_pos, 0, 1, sink, scale)
    assert np.abs(out2 - out).max() < 1e-12


def test_mqa_window_only_is_sliding_window_attention(orc):
    n, c, H, W = 30, 8, 2, 5
    kv = _tok(n, c).astype(np.float32)
    Q = RNG.standard_normal((1, n, H, c))
    q_pos = np.arange(n)[None]
    sink = np.full(H, -np.inf)
    out = orc.sparse_mqa(Q, np.zeros((1, 0, c), np.float32), orc.F32, np.full((1, n, 4), -1, np.int32),
                         kv[None], [0], q_pos, W, 4, sink, 0.5)
    i = np.arange(n)
    mask = (i[None, :] <= i[:, None]) & (i[None, :] > i[:, None] - W)
    want = _sdpa(Q[0], kv.astype(np.float64), mask, 0.5)
    assert np.abs(out[0] - want).max() < 1e-12


def test_mqa_sink_closed_form(orc):
    """q = 0: every logit is 0, so o = sum_j KV_j / (n + exp(sink))."""
    c, H, n = 8, 4, 9
    kv = _tok(n, c)
    sink = np.array([-1.0, 0.0, 2.0, np.inf])
    out = orc.attend(np.zeros((H, c)), kv, sink, 1.0)
    for h in range(3):
        assert np.abs(out[h] - kv.sum(0) / (n + np.exp(sink[h]))).max() < 1e-14
    assert (out[3] == 0).all()
    big = orc.attend(np.zeros((1, c)), kv, np.array([700.0]), 1.0)
    assert np.abs(big).max() < 1e-290


def test_mqa_sink_minus_inf_is_plain_softmax(orc):
    c, H, n = 8, 3, 11
    kv, q = _tok(n, c), _tok(H, c)
    out = orc.attend(q, kv, np.full(H, -np.inf), 0.7)
    p = sps.softmax(0.7 * q @ kv.T, axis=1)
    assert np.abs(out - p @ kv).max() < 1e-14
    # a finite sink scales the probabilities by den/(den + e^sink)
    s = np.array([0.3, -2.0, 1.5])
    out2 = orc.attend(q, kv, s, 0.7)
    z = 0.7 * q @ kv.T
    den = np.exp(z).sum(1)
    ratio = den / (den + np.exp(s))
    assert np.abs(out2 - (p @ kv) * ratio[:, None]).max() < 1e-14


def test_mqa_rejects_invisible_entries(orc):
    c = 8
    ent = _tok(10, c).astype(np.float32)[None]
    Q = RNG.standard_normal((1, 1, 1, c))
    # query at t = 7 with m = 4 sees entries 0, 1 only
    with pytest.raises(ValueError):
        orc.sparse_mqa(Q, ent, orc.F32, np.array([[[2]]], np.int32), ent, [0], [[7]], 1, 4, [0.0], 1.0)
    orc.sparse_mqa(Q, ent, orc.F32, np.array([[[1]]], np.int32), ent, [0], [[7]], 1, 4, [0.0], 1.0)


def test_mqa_fp8mix_rows_are_decoded_exactly(orc):
    c, H, E = 512, 2, 6
    x = _tok(E, c)
    buf, _ = orc.encode_rows(x, orc.FP8MIX)
    dec = orc.decode_rows(buf, orc.FP8MIX, c)
    Q = RNG.standard_normal((1, 1, H, c)) * 0.05
    sink = np.array([0.1, -0.4])
    idx = np.array([[[4, 0, 2, -1]]], np.int32)
    out = orc.sparse_mqa(Q, buf[None], orc.FP8MIX, idx, buf[None], [0], [[5]], 3, 1, sink, 0.1)
    want = orc.attend(Q[0, 0], dec[[4, 0, 2, 3, 4, 5]], sink, 0.1)
    assert np.abs(out[0, 0] - want).max() < 1e-13
