"""Parity of the CUDA path (through the C ABI) with the float64 oracle.

Inputs come from the seeded generators in compressed_sparse_attention_hca_b200.workloads
(or are built in the test from plain random draws); expected values come from
the oracle only.  Tolerances (spec contract):
  * index scores: |g - o| <= 1e-2 |o| + 1e-3 rms(row) (BF16 scores);
    bit-exact when every product and sum is exact in fp32 (integer inputs,
    power-of-two weights): then top-k index sets are bit-exact too;
  * attention outputs: 2e-2 max-abs for BF16 outputs, 1e-5 in F32 mode;
  * compressor: F32 1e-5, BF16 one bf16 ulp (2^-8 relative); quantised
    outputs (FP8MIX, NVFP4) within one code step of the oracle's value.
"""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_attention_hca_b200 import csa
from compressed_sparse_attention_hca_b200 import workloads as W
from parity_util import assert_close, check_nvfp4_rows, f64, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    csa.load()


def _cuda(d):
    return {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


# ---------------------------------------------------------------- compressor

def _oracle_compress(orc, x, m, tok0, e0, n_out):
    outs = []
    for b in range(x["Ca"].shape[0]):
        kw = {}
        if x["Cb"] is not None:
            kw = dict(Cb=f64(x["Cb"][b]), Zb=f64(x["Zb"][b]), Bb=f64(x["Bb"]))
        outs.append(orc.compress(f64(x["Ca"][b]), f64(x["Za"][b]), f64(x["Ba"]), m, tok0=tok0, e0=e0,
                                 n_out=n_out, **kw))
    return np.stack(outs)


@pytest.mark.parametrize("case", [
    # batch, n_tok, dim, m, overlap, dtype, out_dt, tok0, e0, n_out
    (1, 256, 64, 4, True, torch.float32, csa.F32, 0, 0, None),          # tiny prefill shape
    (2, 4 * 37 + 3, 512, 4, True, torch.bfloat16, csa.BF16, 0, 0, None),  # ragged tail
    (2, 128 * 5 + 17, 512, 128, False, torch.bfloat16, csa.F32, 0, 0, None),  # HCA
    (3, 8, 512, 4, True, torch.bfloat16, csa.BF16, 4 * 1000, 1001, 1),   # decode: closing block
    (1, 64, 128, 4, True, torch.float32, csa.F32, 0, 0, 16),
    (2, 4 * 4800, 64, 4, True, torch.float32, csa.F32, 0, 0, None),  # many entries: thread per entry
    (1, 4 * 10, 72, 4, True, torch.float32, csa.F32, 0, 0, None),    # dim not a multiple of 64
    (2, 40 * 6, 128, 40, True, torch.bfloat16, csa.BF16, 0, 0, None),  # 2m = 80 positions, 3 blocks
    (1, 100 * 4, 64, 100, True, torch.float32, csa.F32, 0, 0, None),     # 2m = 200: two staged chunks
    (2, 300 * 2 + 5, 128, 300, False, torch.bfloat16, csa.F32, 0, 0, None),  # m' = 300: three chunks
])
def test_compress_matches_oracle(orc, case):
    batch, n_tok, dim, m, overlap, dtype, out_dt, tok0, e0, n_out = case
    g = W.generator(100 + n_tok)
    x = W.compress_inputs(g, batch, n_tok, dim, m, overlap, dtype)
    if n_out is None:
        n_out = (tok0 + n_tok) // m - e0
    gx = _cuda(x)
    out = csa.compress(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], tok0=tok0, e0=e0,
                       n_out=n_out, out_dt=out_dt)
    want = _oracle_compress(orc, x, m, tok0, e0, n_out)
    got = f64(out)
    if out_dt == csa.F32:
        assert_close(got, want, atol=1e-5, what="compress f32")
    else:
        assert_close(got, want, atol=1e-6, rtol=2.0 ** -8, what="compress bf16")


@pytest.mark.parametrize("out_dt", [csa.F32, csa.BF16, csa.KV_FP8MIX, csa.IDX_NVFP4])
def test_compress_forms_write_the_same_bytes(out_dt):
    """One call over many entries (a thread per entry and 8 channels) and
    calls over a few entries each (a block per entry) compute every channel's
    softmax with the same operations in the same order: the bytes agree."""
    batch, dim, m, n_out = 2, 128, 4, 2400  # 2 x 2400 x 16 chunks: the thread-per-entry form
    g = W.generator(4242)
    x = _cuda(W.compress_inputs(g, batch, m * n_out, dim, m, True, torch.bfloat16))
    args = (x["Ca"], x["Za"], x["Ba"], m, x["Cb"], x["Zb"], x["Bb"])
    one = csa.compress(*args, out_dt=out_dt)
    one, one_sf = one if out_dt == csa.IDX_NVFP4 else (one, None)
    many = torch.full_like(one, 0x5A if one.dtype == torch.uint8 else 3.0)
    many_sf = None if one_sf is None else torch.zeros_like(one_sf)
    for e0 in range(0, n_out, 300):
        csa.compress(*args, e0=e0, n_out=300, out_dt=out_dt, out=many, out_sf=many_sf, out_row0=e0)
    assert torch.equal(one, many)
    if one_sf is not None:
        assert torch.equal(one_sf, many_sf)


def test_compress_writes_into_cache_row(orc):
    """Decode: the entry closed by the last token lands at row E-1 of the cache."""
    batch, dim, m, E = 2, 512, 4, 50
    g = W.generator(7)
    x = W.compress_inputs(g, batch, 2 * m, dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    cache = torch.full((batch, E, dim), 7.0, device=DEV, dtype=torch.bfloat16)
    csa.compress(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], tok0=m * (E - 2), e0=E - 1,
                 n_out=1, out=cache, out_row0=E - 1)
    want = _oracle_compress(orc, x, m, m * (E - 2), E - 1, 1)
    assert_close(f64(cache[:, E - 1:]), want, atol=1e-6, rtol=2.0 ** -8)
    assert (cache[:, :E - 1] == 7.0).all()


def test_compress_fp8mix_output(orc):
    batch, n_tok, dim, m = 2, 4 * 40, 512, 4
    x = W.compress_inputs(W.generator(5), batch, n_tok, dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    out = csa.compress(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], out_dt=csa.KV_FP8MIX)
    want = _oracle_compress(orc, x, m, 0, 0, None)
    got_bytes = raw(out)
    assert got_bytes.shape == (batch, 40, 608)
    assert (got_bytes[:, :, 604:] == 0).all()
    for b in range(batch):
        dec = orc.decode_rows(got_bytes[b], orc.FP8MIX, dim)
        ref_bytes, _ = orc.encode_rows(want[b], orc.FP8MIX)
        ref_scale = ref_bytes[:, 576:604].copy().view(np.float32)
        got_scale = got_bytes[b, :, 576:604].copy().view(np.float32)
        assert_close(got_scale, ref_scale, atol=0, rtol=1e-6, what="fp8 scales")
        # one E4M3 step (relative 2^-3) or one subnormal step of the block scale
        scale_per_dim = np.repeat(ref_scale, 64, axis=1)
        bound = 2.0 ** -3 * np.abs(want[b, :, :448]) + 2.0 ** -9 * scale_per_dim + 1e-7
        assert (np.abs(dec[:, :448] - want[b, :, :448]) <= bound).all()
        assert_close(dec[:, 448:], want[b, :, 448:], atol=1e-6, rtol=2.0 ** -8, what="rope bf16")
        codes_differ = (got_bytes[b, :, :448] != ref_bytes[:, :448]).mean()
        assert codes_differ < 0.01, codes_differ


def _check_nvfp4_rows(orc, codes, sf_rowmajor, want, dim):
    """Compressor NVFP4 rows against the oracle's encoding of its own fp64
    entries: codes differ only where fp32 and fp64 straddle a rounding
    boundary of the scale or value encoder."""
    check_nvfp4_rows(orc, codes, sf_rowmajor, want, dim)


def test_compress_nvfp4_output(orc):
    batch, n_tok, dim, m = 2, 4 * 64, 128, 4
    x = W.compress_inputs(W.generator(6), batch, n_tok, dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    codes, sf = csa.compress(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"],
                             out_dt=csa.IDX_NVFP4)
    want = _oracle_compress(orc, x, m, 0, 0, None)
    n = codes.shape[1]
    assert sf.shape == (batch, csa.nvfp4_key_scale_bytes(n, dim))
    for b in range(batch):
        _check_nvfp4_rows(orc, raw(codes[b]), orc.unblock_scales(raw(sf[b]), n, dim), want[b], dim)


def test_compress_nvfp4_into_cache_rows(orc):
    """Entries written at cache rows out_row0.. of a larger cache: the blocked
    scale bytes land in the right 128-row block and atom byte (a run that
    crosses a block boundary), and every other byte of the cache is unchanged."""
    batch, dim, m, E = 2, 128, 4, 300
    e0, n_out, row0 = 37, 120, 100  # rows 100..219 straddle the 128-row block boundary
    tok0 = m * (e0 - 1)
    x = W.compress_inputs(W.generator(8), batch, m * (n_out + 1), dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    codes = torch.full((batch, E, dim // 2), 0xA5, dtype=torch.uint8, device=DEV)
    sf = torch.full((batch, csa.nvfp4_key_scale_bytes(E, dim)), 0x5A, dtype=torch.uint8, device=DEV)
    csa.compress(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], tok0=tok0, e0=e0, n_out=n_out,
                 out_dt=csa.IDX_NVFP4, out=codes, out_sf=sf, out_row0=row0)
    want = _oracle_compress(orc, x, m, tok0, e0, n_out)
    for b in range(batch):
        c = raw(codes[b])
        s = orc.unblock_scales(raw(sf[b]), E, dim)
        rows = slice(row0, row0 + n_out)
        _check_nvfp4_rows(orc, c[rows], s[rows], want[b], dim)
        others = np.ones(E, bool)
        others[rows] = False
        assert (c[others] == 0xA5).all() and (s[others] == 0x5A).all()
        # bytes of the blocked array that belong to no row (past E) are untouched too
        full = raw(sf[b])
        mask = np.ones(full.size, bool)
        mask[orc.block_scales(np.zeros((E, dim // 16), np.uint8) + 1, dim) == 1] = False
        assert (full[mask] == 0x5A).all()


# ------------------------------------------------------------- indexer + top-k

def _exact_index_inputs(B, T, H, d, E, dt, seed):
    """Integer-valued q, K and power-of-two weights: every score is exact in fp32."""
    g = torch.Generator().manual_seed(seed)
    wI = (2.0 ** torch.randint(-1, 2, (B, T, H), generator=g)).to(torch.float32)
    if dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, T, H), d)
        KI, ksf = W.nvfp4_rows(g, (B, E), d)
        p2 = torch.tensor([0.125, 0.25, 0.5, 1.0]).to(torch.float8_e4m3fn).view(torch.uint8)
        qsf = p2[torch.randint(0, 4, qsf.shape, generator=g)]
        ksf = p2[torch.randint(0, 4, ksf.shape, generator=g)]
        return dict(qI=qI, qI_sf=qsf, KI=KI, KI_sf=W.block_scales(ksf, d), wI=wI)
    tdt = torch.float32 if dt == csa.F32 else torch.bfloat16
    qI = torch.randint(-2, 3, (B, T, H, d), generator=g).to(tdt)
    KI = torch.randint(-2, 3, (B, E, d), generator=g).to(tdt)
    return dict(qI=qI, KI=KI, wI=wI, qI_sf=None, KI_sf=None)


def _decode_idx_inputs(orc, x, dt, d):
    if dt == csa.IDX_NVFP4:
        B, T, H = x["wI"].shape
        q = orc.decode_rows(raw(x["qI"]).reshape(-1, d // 2), orc.NVFP4, d,
                            sf=raw(x["qI_sf"]).reshape(-1, d // 16)).reshape(B, T, H, d)
        E = x["KI"].shape[1]
        K = np.stack([orc.decode_rows(raw(x["KI"][b]), orc.NVFP4, d, sf=raw(x["KI_sf"][b]), sf_blocked=True)
                      for b in range(B)]).reshape(B, E, d)
        return q, K
    return f64(x["qI"]), f64(x["KI"])


def _run_index(x, q_pos, m, k, dt):
    gx = _cuda(x)
    return csa.index_topk(gx["qI"], gx["wI"], gx["KI"], q_pos.to(DEV), m, k, dt=dt, qI_sf=gx["qI_sf"],
                          KI_sf=gx["KI_sf"], scores=True)


def _sorted_idx(idx):
    """Oracle idx rows (score order) -> ascending index order, -1 at the end."""
    out = np.full_like(idx, -1)
    for r in np.ndindex(idx.shape[:-1]):
        v = np.sort(idx[r][idx[r] >= 0])
        out[r][:len(v)] = v
    return out


@pytest.mark.parametrize("dt,H,d,E,k,T", [
    (csa.BF16, 64, 128, 3000, 512, 3),      # tensor-core producer, 2 queries per CTA, merge
    (csa.BF16, 64, 128, 20000, 1024, 1),    # tensor-core producer, decode slices, merge
    (csa.BF16, 64, 128, 9000, 512, 16),     # tensor-core producer, prefill-like rows
    (csa.F32, 2, 32, 64, 16, 3),
    (csa.IDX_NVFP4, 64, 128, 2500, 512, 3),   # block-scaled FP4 tensor cores, 2 queries per CTA
    (csa.IDX_NVFP4, 64, 128, 30000, 1024, 1),  # decode slices, cooperative selection
    (csa.IDX_NVFP4, 64, 128, 30000, 1024, 2),  # 2 queries per CTA, several tiles per slice, merge
    (csa.IDX_NVFP4, 64, 128, 2501, 512, 3),   # odd entry count: partial last scale block
    (csa.IDX_NVFP4, 2, 64, 700, 100, 3),      # SIMT producer on blocked key scales
    (csa.BF16, 8, 64, 700, 100, 3),
])
def test_index_topk_bit_exact_on_exact_scores(orc, dt, H, d, E, k, T):
    B, m = 2, 4
    x = _exact_index_inputs(B, T, H, d, E, dt, seed=E)
    base = [[4 * E - 1, 2999, 39], [4 * E + 50, 4 * 512 - 1, 6]]
    q_pos = torch.tensor([[base[b][t % 3] - 13 * (t // 3) for t in range(T)] for b in range(B)],
                         dtype=torch.int64).clamp(min=0)
    idx, sc = _run_index(x, q_pos, m, k, dt)
    csa.check_device_status()
    q, K = _decode_idx_inputs(orc, x, dt, d)
    want_sc, want_idx = orc.index_topk(q, f64(x["wI"]), K, q_pos.numpy(), m, k, round_bf16=(dt != csa.F32))
    got_sc = f64(sc)
    assert np.array_equal(np.isneginf(got_sc), np.isneginf(want_sc))
    fin = ~np.isneginf(want_sc)
    assert np.array_equal(got_sc[fin], want_sc[fin])
    assert np.array_equal(raw(idx), _sorted_idx(want_idx))


@pytest.mark.parametrize("dt,H,d,E,k,T", [
    (csa.BF16, 64, 128, 5000, 512, 2),
    (csa.IDX_NVFP4, 64, 128, 5000, 1024, 1),
    (csa.F32, 2, 32, 64, 16, 256),
])
def test_index_topk_random_inputs(orc, dt, H, d, E, k, T):
    B, m = 2, 4
    g = W.generator(31 + E)
    if dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, T, H), d)
        KI, ksf = W.nvfp4_rows(g, (B, E), d)
        x = dict(qI=qI, qI_sf=qsf, KI=KI, KI_sf=W.block_scales(ksf, d))
    else:
        tdt = torch.float32 if dt == csa.F32 else torch.bfloat16
        x = dict(qI=W.normal(g, (B, T, H, d), 1.0, tdt), KI=W.normal(g, (B, E, d), 1.0, tdt), qI_sf=None,
                 KI_sf=None)
    x["wI"] = W.uniform(g, (B, T, H))
    if T == 256:
        q_pos = torch.arange(T, dtype=torch.int64).repeat(B, 1)
    else:
        q_pos = torch.tensor([[4 * E - 1] * T, [1500 + 4 * t for t in range(T)]], dtype=torch.int64)
    idx, sc = _run_index(x, q_pos, m, k, dt)
    csa.check_device_status()
    q, K = _decode_idx_inputs(orc, x, dt, d)
    want_sc, _ = orc.index_topk(q, f64(x["wI"]), K, q_pos.numpy(), m, k, round_bf16=False)
    got_sc, got_idx = f64(sc), raw(idx)
    for b in range(B):
        for t in range(T):
            vis = orc.visible_entries(int(q_pos[b, t]), m, E)
            o, gsc = want_sc[b, t, :vis], got_sc[b, t, :vis]
            rms = math.sqrt(float(np.mean(o * o))) if vis else 0.0
            if dt == csa.F32:
                assert_close(gsc, o, atol=1e-5 * (1 + rms), rtol=1e-5, what="f32 scores")
            else:
                assert_close(gsc, o, atol=1e-3 * rms, rtol=1e-2, what="scores")
            assert np.isneginf(got_sc[b, t, vis:]).all()
            # the GPU selection is exactly the oracle's top-k of the GPU's own score row ...
            sel = got_idx[b, t][got_idx[b, t] >= 0]
            want_sel = orc.topk(gsc, k)
            assert np.array_equal(sel, np.sort(want_sel[want_sel >= 0]))
            assert (got_idx[b, t][len(sel):] == -1).all()
            # ... and every selected entry is within tolerance of the oracle's k-th best
            if 0 < k < vis:
                kth = np.sort(o)[::-1][k - 1]
                tol = 2e-2 * abs(kth) + 2e-3 * rms
                assert o[sel].min() >= kth - tol


def test_index_workspace_reused_across_shapes():
    """One workspace serves a merge-mode call (candidate lists) and then a
    cooperative decode call (counters and histograms): every call leaves the
    workspace zero, so both select exactly what they select on a fresh one."""
    H, d = 64, 128
    g = W.generator(9090)
    cases = [dict(dt=csa.IDX_NVFP4, B=2, T=2, E=30000, k=1024), dict(dt=csa.BF16, B=3, T=1, E=20000, k=512)]
    ws = torch.zeros(max(csa.index_topk_workspace_size(c["B"], c["T"], c["E"], c["k"], H, d, c["dt"])
                         for c in cases), device=DEV, dtype=torch.uint8)
    for c in cases + cases:
        if c["dt"] == csa.IDX_NVFP4:
            qI, qsf = W.nvfp4_rows(g, (c["B"], c["T"], H), d)
            KI, ksf = W.nvfp4_rows(g, (c["B"], c["E"]), d)
            ksf = W.block_scales(ksf, d)
        else:
            qI, qsf = W.normal(g, (c["B"], c["T"], H, d), 1.0, torch.bfloat16), None
            KI, ksf = W.normal(g, (c["B"], c["E"], d), 1.0, torch.bfloat16), None
        wI = W.uniform(g, (c["B"], c["T"], H))
        q_pos = torch.tensor([[4 * c["E"] - 1 - 37 * t for t in range(c["T"])]] * c["B"], dtype=torch.int64)
        cu = lambda v: None if v is None else v.to(DEV)  # noqa: E731
        args = (cu(qI), cu(wI), cu(KI), cu(q_pos), 4, c["k"])
        kw = dict(dt=c["dt"], qI_sf=cu(qsf), KI_sf=cu(ksf))
        fresh = csa.index_topk(*args, **kw)
        reused = csa.index_topk(*args, **kw, ws=ws)
        torch.cuda.synchronize()
        assert torch.equal(fresh, reused)
        assert int(ws.count_nonzero()) == 0, "the call left the workspace dirty"


# ------------------------------------------------------------------ attention

def _random_selection(g, B, T, k, vis_rows, drop=0.1):
    """Random distinct visible entries per query (some slots -1)."""
    idx = torch.full((B, T, k), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(T):
            vis = int(vis_rows[b][t])
            n = min(k, vis)
            if n:
                sel = torch.randperm(vis, generator=g)[:n].to(torch.int32)
                keep = torch.rand(n, generator=g) >= drop
                sel = torch.where(keep, sel, torch.full_like(sel, -1))
                idx[b, t, torch.randperm(k, generator=g)[:n]] = sel
    return idx


def _mqa_case(orc, cfg_name, B, T, E, k, q0, sink_override=None, dense=False, seed=None):
    cfg = dict(W.CONFIGS[cfg_name])
    x = W.attention_inputs(cfg, "cpu", batch=B, ctx=E * cfg["m"], n_q=T, q0=q0, n_entries=E, seed=seed)
    if sink_override is not None:
        x["sink"] = torch.tensor(sink_override, dtype=torch.float32)
    m, W_ = cfg["m"], cfg["window"]
    scale = 1.0 / math.sqrt(cfg["dim"])
    vis = [[orc.visible_entries(int(x["q_pos"][b, t]), m, E) for t in range(T)] for b in range(B)]
    g = torch.Generator().manual_seed(77)
    gx = _cuda(x)
    if dense:
        out = csa.hca_dense_mqa(gx["Q"], gx["entries"], gx["win"], gx["win_start"], gx["q_pos"], W_, m,
                                gx["sink"], scale, kv_dt=cfg["kv_dt"])
        want = orc.hca_dense_mqa(f64(x["Q"]), raw(x["entries"]), cfg["kv_dt"], raw(x["win"]),
                                 raw(x["win_start"]), raw(x["q_pos"]), W_, m, f64(x["sink"]), scale)
    else:
        idx = _random_selection(g, B, T, k, vis)
        out = csa.sparse_mqa(gx["Q"], gx["entries"], idx.to(DEV), gx["win"], gx["win_start"], gx["q_pos"], W_,
                             m, gx["sink"], scale, kv_dt=cfg["kv_dt"])
        want = orc.sparse_mqa(f64(x["Q"]), raw(x["entries"]), cfg["kv_dt"], raw(idx), raw(x["win"]),
                              raw(x["win_start"]), raw(x["q_pos"]), W_, m, f64(x["sink"]), scale)
    return f64(out), want, cfg


@pytest.mark.parametrize("cfg_name,B,T,E,k,q0", [
    ("tiny_prefill_f32", 1, 256, 64, 16, 0),             # the tiny prefill workload itself
    ("csa_decode_bf16", 2, 1, 4000, 512, 4 * 4000 - 1),   # decode
    ("csa_decode_1m_mixed", 2, 1, 3000, 1024, 4 * 3000 - 1),  # FP8MIX entries, 128 heads
    ("csa_prefill_bf16", 1, 40, 300, 64, 0),              # early queries: t < window, t < m-1
    ("csa_prefill_bf16", 1, 16, 300, 64, 1100),           # chunk of prefill queries
])
def test_sparse_mqa_matches_oracle(orc, cfg_name, B, T, E, k, q0):
    got, want, cfg = _mqa_case(orc, cfg_name, B, T, E, k, q0)
    atol = 1e-5 if cfg["q_dt"] == csa.F32 else 2e-2
    assert_close(got, want, atol=atol, what=cfg_name)


@pytest.mark.parametrize("B,T,E,q0", [(2, 1, 300, 128 * 300 - 1), (1, 8, 40, 128 * 30), (1, 3, 5, 0),
                                      (1, 1, 8192, 128 * 8192 - 1)])  # long rows: split over the GPU
def test_hca_dense_mqa_matches_oracle(orc, B, T, E, q0):
    got, want, _ = _mqa_case(orc, "hca_decode_bf16", B, T, E, 0, q0, dense=True)
    assert_close(got, want, atol=2e-2, what="hca")


def test_mqa_sink_limits(orc):
    H = 4
    got, want, _ = _mqa_case(orc, "tiny_prefill_f32", 1, 20, 64, 16, 10,
                             sink_override=[float("inf"), float("-inf"), 30.0, -30.0])
    assert_close(got, want, atol=1e-5, what="sink limits")
    assert (got[0, :, 0] == 0).all()


def test_mqa_sink_limits_split_rows(orc):
    """Sink +inf / -inf / large values on the tensor-core path whose decode
    rows are split over several CTAs (the per-split maxima and sums are
    combined with the sink after the split partials are written)."""
    sinks = [float("inf"), float("-inf"), 30.0, -30.0] + [0.5] * 60
    got, want, _ = _mqa_case(orc, "csa_decode_bf16", 2, 1, 4000, 512, 4 * 4000 - 1, sink_override=sinks)
    assert_close(got, want, atol=2e-2, what="sink limits, split rows")
    assert (got[:, :, 0] == 0).all()


# ------------------------------------------ fused compressions + indexer

@pytest.mark.parametrize("dt,B,T,E,k,n_new", [
    (csa.IDX_NVFP4, 3, 1, 30000, 1024, 1),   # one launch: the lead CTA compresses while its keys land
    (csa.BF16, 2, 1, 20000, 512, 1),         # one launch (BF16 keys)
    (csa.IDX_NVFP4, 2, 1, 300, 128, 1),      # tiny cache: the new row is in the lead slice's first stage
    (csa.IDX_NVFP4, 2, 3, 5000, 512, 1),     # two queries per CTA: the calls in order
    # two new rows 19967, 19968 across the boundary of 384-entry slices (2 requests on
    # 148 SMs): two CTAs compress a key row each, the lead also both KV entries
    (csa.IDX_NVFP4, 2, 1, 19969, 512, 2),
    (csa.BF16, 2, 1, 19969, 512, 2),
])
def test_compress_index_topk_equals_the_separate_calls(orc, dt, B, T, E, k, n_new):
    """The fused call writes the same key-cache and KV-cache bytes and selects
    the same indices as csa_compress (twice) followed by csa_index_topk, and
    the new key entry matches the oracle's compression."""
    m, dI, H, c = 4, 128, 64, 512
    g = W.generator(500 + E)
    tok = W.compress_inputs(g, B, m * (n_new + 1), dI, m, True, torch.bfloat16)
    ktok = W.compress_inputs(g, B, m * (n_new + 1), c, m, True, torch.bfloat16)
    if dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, T, H), dI)
        KI, ksf = W.nvfp4_rows(g, (B, E), dI)
        ksf = W.block_scales(ksf, dI)
    else:
        qI, qsf = W.normal(g, (B, T, H, dI), 1.0, torch.bfloat16), None
        KI, ksf = W.normal(g, (B, E, dI), 1.0, torch.bfloat16), None
    wI = W.uniform(g, (B, T, H))
    kv = torch.randint(0, 256, (B, E, 608), generator=g, dtype=torch.uint8)
    q_pos = torch.tensor([[m * E - 1 - 13 * t for t in range(T)]] * B, dtype=torch.int64)
    gt, gk, e0 = _cuda(tok), _cuda(ktok), E - n_new
    tok0 = m * (e0 - 1)
    cu = lambda v: None if v is None else v.to(DEV)  # noqa: E731
    # separate calls
    K1, S1, V1 = cu(KI).clone(), (cu(ksf).clone() if ksf is not None else None), cu(kv).clone()
    csa.compress(gt["Ca"], gt["Za"], gt["Ba"], m, gt["Cb"], gt["Zb"], gt["Bb"], tok0=tok0, e0=e0, n_out=n_new,
                 out_dt=dt, out=K1, out_sf=S1, out_row0=e0)
    csa.compress(gk["Ca"], gk["Za"], gk["Ba"], m, gk["Cb"], gk["Zb"], gk["Bb"], tok0=tok0, e0=e0, n_out=n_new,
                 out_dt=csa.KV_FP8MIX, out=V1, out_row0=e0)
    idx1 = csa.index_topk(cu(qI), cu(wI), K1, q_pos.to(DEV), m, k, dt=dt, qI_sf=cu(qsf), KI_sf=S1)
    # fused
    K2, S2, V2 = cu(KI).clone(), (cu(ksf).clone() if ksf is not None else None), cu(kv).clone()
    keys = csa.compress_job(gt["Ca"], gt["Za"], gt["Ba"], m, gt["Cb"], gt["Zb"], gt["Bb"], tok0=tok0, e0=e0,
                            n_out=n_new, out=K2, out_sf=S2, out_dt=dt)
    extra = csa.compress_job(gk["Ca"], gk["Za"], gk["Ba"], m, gk["Cb"], gk["Zb"], gk["Bb"], tok0=tok0, e0=e0,
                             n_out=n_new, out=V2, out_dt=csa.KV_FP8MIX)
    idx2 = csa.compress_index_topk(keys, cu(qI), cu(wI), K2, q_pos.to(DEV), m, k, extra_job=extra, dt=dt,
                                   qI_sf=cu(qsf), KI_sf=S2)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(K1, K2)
    if S1 is not None:
        assert torch.equal(S1, S2)
    assert torch.equal(V1, V2)
    assert torch.equal(idx1, idx2)
    # the new key entry against the oracle's own compression (one quantisation step)
    want = _oracle_compress(orc, tok, m, tok0, e0, n_new)
    for b in range(B):
        if dt == csa.IDX_NVFP4:
            codes = raw(K2[b, e0:e0 + n_new])
            sfr = orc.unblock_scales(raw(S2[b]), E, dI)[e0:e0 + n_new]
            _check_nvfp4_rows(orc, codes, sfr, want[b], dI)
        else:
            assert_close(f64(K2[b, e0:e0 + n_new]), want[b], atol=1e-6, rtol=2.0 ** -8, what="fused bf16 key")


# ------------------------------------------------- Q / KV normalisation + partial RoPE

@pytest.mark.parametrize("case", [
    # rows, dim, rope_dims, rows_per_pos, in, out, with g, pos_sign, max position
    (4 * 128, 512, 64, 128, torch.bfloat16, csa.BF16, True, 1, 1 << 20),   # decode queries: 4 x 128 heads
    (37, 512, 64, 1, torch.bfloat16, csa.BF16, True, 1, 262143),           # ragged cache rows
    (45, 128, 64, 1, torch.float32, csa.F32, False, -1, 1 << 20),          # rotation only, turned back
    (16, 448, 0, 1, torch.float32, csa.BF16, True, 1, 10),                 # normalisation only
    (8, 64, 64, 4, torch.bfloat16, csa.F32, True, 1, 77),                  # every dim rotated
])
def test_rmsnorm_rope_matches_oracle(orc, case):
    n, dim, rope, rpp, dtype, out_dt, with_g, sign, pmax = case
    g = torch.Generator().manual_seed(900 + n + dim)
    x = (torch.randn(n, dim, generator=g) * (1 + 3 * torch.rand(n, 1, generator=g))).to(dtype)
    w = torch.randn(dim, generator=g) if with_g else None
    pos = torch.randint(0, pmax + 1, ((n + rpp - 1) // rpp,), generator=g, dtype=torch.int64)
    pos[0] = pmax
    y = csa.rmsnorm_rope(x.to(DEV), pos.to(DEV), g=None if w is None else w.to(DEV), eps=1e-6, rows_per_pos=rpp,
                         pos_sign=sign, rope_dims=rope, out_dt=out_dt)
    torch.cuda.synchronize()
    want = f64(x)
    if w is not None:
        want = orc.rmsnorm(want, f64(w), 1e-6)
    p_rows = np.repeat(f64(pos), rpp)[:n] * sign
    want = orc.rope_tail(want, p_rows, rope_dims=rope)
    got = f64(y)
    if out_dt == csa.F32:
        assert_close(got, want, atol=2e-5, rtol=2e-5, what="rmsnorm_rope f32")
    else:
        assert_close(got, want, atol=1e-5, rtol=2.0 ** -8, what="rmsnorm_rope bf16")


def test_rmsnorm_rope_in_place_and_turn_back():
    """In place on bf16 rows; turning f32 rows at p and then at -p returns them."""
    g = torch.Generator().manual_seed(77)
    x = torch.randn(64, 512, generator=g).to(torch.bfloat16).to(DEV)
    pos = torch.randint(0, 1 << 20, (64,), generator=g, dtype=torch.int64).to(DEV)
    w = torch.randn(512, generator=g).to(DEV)
    ref = csa.rmsnorm_rope(x, pos, g=w)
    y = x.clone()
    csa.rmsnorm_rope(y, pos, g=w, out=y)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    z = torch.randn(64, 512, generator=g).to(DEV)
    back = csa.rmsnorm_rope(csa.rmsnorm_rope(z, pos), pos, pos_sign=-1)
    torch.cuda.synchronize()
    assert (back - z).abs().max().item() < 1e-5
