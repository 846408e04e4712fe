"""Parity at the benchmark's own shapes, in the launch configuration bench.py
times (the same call sequence on the same seeded inputs).

The decode indexer splits each request's entries into one slice per CTA; at
these shapes a slice streams several times more key stages than its
shared-memory ring holds, so the producer and MMA issuers wrap the ring and
every mbarrier phase is reused.  The tests assert that regime from the call's
own plan before checking results:

  * exact inputs (integer-valued codes, power-of-two scales and weights), where
    every score is exact in fp32: scores and top-k indices bit-exact against
    the float64 oracle's index_topk;
  * the benchmark's own step (compressions fused into the indexer launch, then
    attention) on its realistic inputs: the compressed rows within one
    quantisation step of the oracle's compression, scores within
    1e-2 |o| + 1e-3 rms(row) of the oracle's, the selection bit-exact against
    the oracle's top-k run on the GPU's own score row, and the attention
    output within 2e-2 (max abs, bf16) of the oracle's attention over the
    GPU's selection;
  * the prefill workload on a fixed sample of its queries.
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


def _ring_stages_per_slice(plan):
    return math.ceil(plan["slice_len"] / (128 * plan["tiles_per_stage"]))


def _sorted(idx_row):
    v = np.sort(idx_row[idx_row >= 0])
    out = np.full(idx_row.shape, -1, np.int32)
    out[:len(v)] = v
    return out


def _decode_keys(orc, KI, KI_sf, dt, d):
    """One request's key cache as exact float64 rows."""
    if dt == csa.IDX_NVFP4:
        return orc.decode_rows(raw(KI), orc.NVFP4, d, sf=raw(KI_sf), sf_blocked=True)
    return f64(KI)


def _decode_queries(orc, qI, qI_sf, dt, d):
    """Queries [T, H, ...] of one request as float64 [T, H, d]."""
    T, H = qI.shape[:2]
    if dt == csa.IDX_NVFP4:
        return orc.decode_rows(raw(qI).reshape(-1, d // 2), orc.NVFP4, d,
                               sf=raw(qI_sf).reshape(-1, d // 16)).reshape(T, H, d)
    return f64(qI)


# ------------------------------------------------- exact scores, full decode shapes

def _exact_decode_inputs(cfg, seed):
    """Inputs of the decode indexer with every score exact in fp32: NVFP4 codes
    with power-of-two block scales (or small integers in bf16) and
    power-of-two head weights.  Drawn on the GPU (seeded) for speed."""
    B, E, H, d = cfg["batch"], cfg["ctx"] // cfg["m"], cfg["n_hI"], cfg["dI"]
    g = W.generator(seed, DEV)
    wI = (2.0 ** torch.randint(-1, 2, (B, 1, H), generator=g, device=DEV)).to(torch.float32)
    if cfg["idx_dt"] == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, 1, H), d, device=DEV)
        KI, ksf = W.nvfp4_rows(g, (B, E), d, device=DEV)
        p2 = torch.tensor([0.125, 0.25, 0.5, 1.0], device=DEV).to(torch.float8_e4m3fn).view(torch.uint8)
        qsf = p2[torch.randint(0, 4, qsf.shape, generator=g, device=DEV)]
        ksf = p2[torch.randint(0, 4, ksf.shape, generator=g, device=DEV)]
        return dict(qI=qI, qI_sf=qsf, KI=KI, KI_sf=W.block_scales(ksf, d), wI=wI)
    qI = torch.randint(-2, 3, (B, 1, H, d), generator=g, device=DEV).to(torch.bfloat16)
    KI = torch.randint(-2, 3, (B, E, d), generator=g, device=DEV).to(torch.bfloat16)
    return dict(qI=qI, qI_sf=None, KI=KI, KI_sf=None, wI=wI)


@pytest.mark.parametrize("name", ["csa_decode_1m_mixed", "csa_decode_bf16"])
def test_decode_indexer_full_shape_bit_exact(orc, name):
    cfg = W.CONFIGS[name]
    B, m, k, H, d, dt = cfg["batch"], cfg["m"], cfg["k"], cfg["n_hI"], cfg["dI"], cfg["idx_dt"]
    E = cfg["ctx"] // m
    plan = csa.index_topk_plan(B, 1, E, k, H, d, dt)
    assert plan["tensor_core"] == 1 and plan["coop"] == 1, plan
    # every CTA streams at least three times the ring's stages
    assert _ring_stages_per_slice(plan) >= 3 * plan["ring_stages"], plan
    x = _exact_decode_inputs(cfg, seed=cfg["seed"] + 40)
    q_pos = torch.full((B, 1), m * E - 1, dtype=torch.int64, device=DEV)
    idx = csa.index_topk(x["qI"], x["wI"], x["KI"], q_pos, m, k, dt=dt, qI_sf=x["qI_sf"], KI_sf=x["KI_sf"])
    idx_dbg, sc = csa.index_topk(x["qI"], x["wI"], x["KI"], q_pos, m, k, dt=dt, qI_sf=x["qI_sf"],
                                 KI_sf=x["KI_sf"], scores=True)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(idx, idx_dbg), "the score output changed the selection"
    for b in range(B):
        K = _decode_keys(orc, x["KI"][b], None if x["KI_sf"] is None else x["KI_sf"][b], dt, d)
        q = _decode_queries(orc, x["qI"][b], None if x["qI_sf"] is None else x["qI_sf"][b], dt, d)
        want_sc, want_idx = orc.index_topk(q[None], f64(x["wI"][b:b + 1]), K[None], raw(q_pos[b:b + 1].cpu()), m, k,
                                           round_bf16=True)
        assert np.array_equal(f64(sc[b, 0]), want_sc[0, 0]), f"request {b}: scores differ"
        assert np.array_equal(raw(idx[b, 0]), _sorted(want_idx[0, 0])), f"request {b}: indices differ"


# ------------------------------------------------- the benchmark's decode step

def _step_inputs(name):
    """The benchmark's step inputs (bench.Step draws the same tensors)."""
    cfg = dict(W.CONFIGS[name])
    x = W.attention_inputs(cfg, DEV)
    m, c = cfg["m"], cfg["dim"]
    B, E = x["B"], x["E"]
    g = W.generator(cfg["seed"] + 17, DEV)
    overlap = cfg["kind"].startswith("csa")
    tok0 = E * m - (2 * m if overlap else m)
    rows = m + (m if overlap else 0)
    tok = W.compress_inputs(g, B, rows, c, m, overlap, torch.bfloat16, c_std=cfg["kv_std"], device=DEV)
    itok = W.compress_inputs(g, B, rows, cfg["dI"], m, True, torch.bfloat16, device=DEV) if overlap else None
    return cfg, x, tok, itok, tok0


@pytest.fixture(scope="module", params=["csa_decode_1m_mixed", "csa_decode_bf16"])
def decode_step(request):
    """One benchmark step on the GPU: the fused compressions + indexer call
    (with and without the debug score output, on separate copies of the
    caches), then the sparse attention."""
    name = request.param
    cfg, x, tok, itok, tok0 = _step_inputs(name)
    m, k, E, B = cfg["m"], cfg["k"], x["E"], x["B"]
    e0 = E - 1
    dt = cfg["idx_dt"]
    plan = csa.index_topk_plan(B, 1, E, k, cfg["n_hI"], cfg["dI"], dt)
    kv_before = x["entries"][:, e0].clone()

    def run(KI, KI_sf, entries, scores):
        keys = csa.compress_job(itok["Ca"], itok["Za"], itok["Ba"], m, itok["Cb"], itok["Zb"], itok["Bb"], tok0=tok0,
                                e0=e0, n_out=1, out=KI, out_sf=KI_sf, out_dt=dt)
        kv = csa.compress_job(tok["Ca"], tok["Za"], tok["Ba"], m, tok["Cb"], tok["Zb"], tok["Bb"], tok0=tok0, e0=e0,
                              n_out=1, out=entries, out_dt=cfg["kv_dt"])
        return csa.compress_index_topk(keys, x["qI"], x["wI"], KI, x["q_pos"], m, k, extra_job=kv, dt=dt,
                                       qI_sf=x.get("qI_sf"), KI_sf=KI_sf, scores=scores)

    KI2 = x["KI"].clone()
    sf2 = x["KI_sf"].clone() if "KI_sf" in x else None
    ent2 = x["entries"].clone()
    idx = run(x["KI"], x.get("KI_sf"), x["entries"], False)
    idx_dbg, sc = run(KI2, sf2, ent2, True)
    scale = 1.0 / math.sqrt(cfg["dim"])
    O = csa.sparse_mqa(x["Q"], x["entries"], idx, x["win"], x["win_start"], x["q_pos"], cfg["window"], m, x["sink"],
                       scale, kv_dt=cfg["kv_dt"])
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(idx, idx_dbg), "the score output changed the selection"
    assert torch.equal(x["KI"], KI2) and torch.equal(x["entries"], ent2)
    if sf2 is not None:
        assert torch.equal(x["KI_sf"], sf2)
    assert not torch.equal(x["entries"][:, e0], kv_before), "the KV entry was not written"
    return dict(name=name, cfg=cfg, x=x, tok=tok, itok=itok, tok0=tok0, e0=e0, idx=idx, sc=sc, O=O, plan=plan,
                scale=scale)


def test_decode_step_runs_the_wrapping_regime(decode_step):
    plan = decode_step["plan"]
    assert plan["tensor_core"] == 1 and plan["coop"] == 1, plan
    assert _ring_stages_per_slice(plan) >= 3 * plan["ring_stages"], plan


def _oracle_compress_one(orc, tok, b, m, tok0, e0):
    return orc.compress(f64(tok["Ca"][b]), f64(tok["Za"][b]), f64(tok["Ba"]), m, Cb=f64(tok["Cb"][b]),
                        Zb=f64(tok["Zb"][b]), Bb=f64(tok["Bb"]), tok0=tok0, e0=e0, n_out=1)


def test_decode_step_compressed_rows(orc, decode_step):
    """The new index key and KV entry written by the fused launch, against the
    oracle's compression of the same token rows."""
    s = decode_step
    cfg, x, e0, m = s["cfg"], s["x"], s["e0"], s["cfg"]["m"]
    dI, c = cfg["dI"], cfg["dim"]
    for b in range(x["B"]):
        want_k = _oracle_compress_one(orc, s["itok"], b, m, s["tok0"], e0)
        want_v = _oracle_compress_one(orc, s["tok"], b, m, s["tok0"], e0)
        if cfg["idx_dt"] == csa.IDX_NVFP4:
            codes = raw(x["KI"][b, e0:e0 + 1])
            sfr = orc.unblock_scales(raw(x["KI_sf"][b]), x["E"], dI)[e0:e0 + 1]
            check_nvfp4_rows(orc, codes, sfr, want_k, dI)
        else:
            assert_close(f64(x["KI"][b, e0:e0 + 1]), want_k, atol=1e-6, rtol=2.0 ** -8, what="bf16 key")
        if cfg["kv_dt"] == csa.KV_FP8MIX:
            rowb = raw(x["entries"][b, e0:e0 + 1])
            got = orc.decode_rows(rowb, orc.FP8MIX, c)
            scale = np.repeat(rowb[:, 576:604].copy().view(np.float32), 64, axis=1)
            assert (np.abs(got[:, :448] - want_v[:, :448]) <= 2.0 ** -3 * np.abs(want_v[:, :448])
                    + 2.0 ** -9 * scale + 1e-7).all()
            assert_close(got[:, 448:], want_v[:, 448:], atol=1e-6, rtol=2.0 ** -8, what="rope dims")
        else:
            assert_close(f64(x["entries"][b, e0:e0 + 1]), want_v, atol=1e-6, rtol=2.0 ** -8, what="bf16 entry")


def test_decode_step_scores_and_selection(orc, decode_step):
    """Scores of the whole row against the oracle's, and the selection against
    the oracle's top-k of the GPU's own score row."""
    s = decode_step
    cfg, x, m, k = s["cfg"], s["x"], s["cfg"]["m"], s["cfg"]["k"]
    dI, dt = cfg["dI"], cfg["idx_dt"]
    for b in range(x["B"]):
        K = _decode_keys(orc, x["KI"][b], x["KI_sf"][b] if "KI_sf" in x else None, dt, dI)
        q = _decode_queries(orc, x["qI"][b], x["qI_sf"][b] if "qI_sf" in x else None, dt, dI)
        t = int(x["q_pos"][b, 0])
        vis = orc.visible_entries(t, m, x["E"])
        o = orc.index_scores(q[0], f64(x["wI"][b, 0]), K[:vis])
        gsc = f64(s["sc"][b, 0])
        rms = math.sqrt(float(np.mean(o * o)))
        assert_close(gsc[:vis], o, atol=1e-3 * rms, rtol=1e-2, what=f"scores, request {b}")
        assert np.isneginf(gsc[vis:]).all()
        want = _sorted(orc.topk(gsc[:vis], k))
        assert np.array_equal(raw(s["idx"][b, 0]), want), f"request {b}: selection differs"


def test_decode_step_attention(orc, decode_step):
    s = decode_step
    cfg, x = s["cfg"], s["x"]
    want = orc.sparse_mqa(f64(x["Q"]), raw(x["entries"]), cfg["kv_dt"], raw(s["idx"]), raw(x["win"]),
                          raw(x["win_start"]), raw(x["q_pos"]), cfg["window"], cfg["m"], f64(x["sink"]), s["scale"])
    assert_close(f64(s["O"]), want, atol=2e-2, what=f"{s['name']} attention")


def test_hca_decode_step_full_shape(orc):
    """The HCA benchmark step: compress the closed 128-token block into the
    cache, then dense attention over every entry and the window (8 requests x
    8192 entries)."""
    cfg, x, tok, _, tok0 = _step_inputs("hca_decode_bf16")
    m, E = cfg["m"], x["E"]
    e0 = E - 1
    csa.compress(tok["Ca"], tok["Za"], tok["Ba"], m, tok0=tok0, e0=e0, n_out=1, out_dt=cfg["kv_dt"],
                 out=x["entries"], out_row0=e0)
    scale = 1.0 / math.sqrt(cfg["dim"])
    O = csa.hca_dense_mqa(x["Q"], x["entries"], x["win"], x["win_start"], x["q_pos"], cfg["window"], m, x["sink"],
                          scale, kv_dt=cfg["kv_dt"])
    torch.cuda.synchronize()
    csa.check_device_status()
    for b in range(x["B"]):
        want_v = orc.compress(f64(tok["Ca"][b]), f64(tok["Za"][b]), f64(tok["Ba"]), m, tok0=tok0, e0=e0, n_out=1)
        assert_close(f64(x["entries"][b, e0:e0 + 1]), want_v, atol=1e-6, rtol=2.0 ** -8, what="hca entry")
    want = orc.hca_dense_mqa(f64(x["Q"]), raw(x["entries"]), cfg["kv_dt"], raw(x["win"]), raw(x["win_start"]),
                             raw(x["q_pos"]), cfg["window"], m, f64(x["sink"]), scale)
    assert_close(f64(O), want, atol=2e-2, what="hca attention")


# ------------------------------------------------- prefill, sampled queries

PREFILL_SAMPLE = [0, 1, 2, 127, 128, 129, 1000, 2047, 2048, 4095, 4096, 5555, 6000, 8000, 8190, 8191]


def test_prefill_full_shape_sampled_queries(orc):
    """The chunked-prefill workload (8192 queries on a 72K context) at full
    size; the oracle checks a fixed sample of 16 queries (scores, selection on
    the GPU's score row, attention)."""
    cfg = dict(W.CONFIGS["csa_prefill_bf16"])
    x = W.attention_inputs(cfg, DEV)
    m, k, E, T = cfg["m"], cfg["k"], x["E"], x["T"]
    idx, sc = csa.index_topk(x["qI"], x["wI"], x["KI"], x["q_pos"], m, k, dt=cfg["idx_dt"], scores=True)
    idx_p = csa.index_topk(x["qI"], x["wI"], x["KI"], x["q_pos"], m, k, dt=cfg["idx_dt"])
    scale = 1.0 / math.sqrt(cfg["dim"])
    O = csa.sparse_mqa(x["Q"], x["entries"], idx_p, x["win"], x["win_start"], x["q_pos"], cfg["window"], m,
                       x["sink"], scale, kv_dt=cfg["kv_dt"])
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(idx, idx_p)
    t_s = torch.tensor(PREFILL_SAMPLE)
    K = f64(x["KI"][0])
    sc_s, idx_s = f64(sc[0, t_s]), raw(idx[0, t_s])
    for j, t in enumerate(PREFILL_SAMPLE):
        tp = int(x["q_pos"][0, t])
        vis = orc.visible_entries(tp, m, E)
        o = orc.index_scores(f64(x["qI"][0, t]), f64(x["wI"][0, t]), K[:vis])
        rms = math.sqrt(float(np.mean(o * o)))
        assert_close(sc_s[j, :vis], o, atol=1e-3 * rms, rtol=1e-2, what=f"prefill scores, query {t}")
        assert np.isneginf(sc_s[j, vis:]).all()
        assert np.array_equal(idx_s[j], _sorted(orc.topk(sc_s[j, :vis], k))), f"query {t}: selection"
    # attention of the sampled queries (the oracle's sparse MQA on those rows)
    want = orc.sparse_mqa(f64(x["Q"][:, t_s]), raw(x["entries"]), cfg["kv_dt"], raw(idx_p[:, t_s]), raw(x["win"]),
                          raw(x["win_start"]), raw(x["q_pos"][:, t_s]), cfg["window"], m, f64(x["sink"]), scale)
    assert_close(f64(O[:, t_s]), want, atol=2e-2, what="prefill attention")
