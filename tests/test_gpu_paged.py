"""The paged compressed cache (admirer.cn article, cache paragraph: 128-token
pages, i.e. 32 CSA entries or 1 HCA entry per page; "DeepSeek-V4 内部机制"
section 7) on the GPU.

Every test scatters a contiguous cache into a pool of pages in random order
(plus spare pages of random bytes, and -1 in the table slots past the used
pages), pins that scatter with the oracle's gather_paged (which must give the
contiguous cache back byte for byte), and then checks the paged call:

  * against the oracle run on the gathered cache (attention 2e-2 max abs,
    bf16; indexer scores and indices bit-exact on exact inputs), and
  * bitwise against the same call on the contiguous cache (the kernels differ
    only in where they read rows).

The compressor writing through a block table is checked the same way: the
gathered pool equals the contiguous output byte for byte, and pool rows no
entry maps to are left untouched.
"""
import math

import numpy as np
import pytest
import torch

from compressed_sparse_attention_hca_b200 import csa
from compressed_sparse_attention_hca_b200 import workloads as W
from parity_util import assert_close, f64, raw

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.fail("the gpu tests need a CUDA device")
    csa.load()


def _noise(gen, shape, dtype, device):
    """Seeded filler bytes / values (drawn on the CPU)."""
    if dtype == torch.uint8:
        return torch.randint(0, 256, shape, generator=gen, dtype=torch.uint8).to(device)
    return torch.randn(shape, generator=gen).to(dtype).to(device)


def _scatter(cache, pe, gen, spare=5):
    """cache [B, E, ...] -> (pool [n_pages * pe, ...], table [B, max_pages] int32, n_pages).
    Request b's page j is pool page table[b, j]; unused pool rows are noise."""
    B, E = cache.shape[:2]
    rest = tuple(cache.shape[2:])
    per = -(-E // pe)
    n_pages = B * per + spare
    perm = torch.randperm(n_pages, generator=gen, device="cpu")[:B * per].reshape(B, per)
    padded = _noise(gen, (B, per * pe) + rest, cache.dtype, cache.device)
    padded[:, :E] = cache
    pool = _noise(gen, (n_pages, pe) + rest, cache.dtype, cache.device)
    pool[perm.reshape(-1).to(cache.device)] = padded.reshape((B * per, pe) + rest)
    table = torch.full((B, per + 2), -1, dtype=torch.int32)
    table[:, :per] = perm.to(torch.int32)
    return pool.reshape((n_pages * pe,) + rest), table, n_pages


def _row_bytes(t, rows_shape):
    """A tensor as uint8 rows of shape rows_shape + [row bytes]."""
    b = t.detach().contiguous().cpu().view(torch.uint8)
    return b.reshape(tuple(rows_shape) + (-1,)).numpy()


def _pin_scatter(orc, pool, table, n_pages, pe, cache):
    """The oracle's gather through the table gives the contiguous cache back."""
    B, E = cache.shape[:2]
    got = orc.gather_paged(_row_bytes(pool, (n_pages, pe)), raw(table), E)
    assert np.array_equal(got, _row_bytes(cache, (B, E))), "scatter / gather round trip"
    return got


def _scatter_key_scales(ksf, table, pe, n_pages, dim, gen):
    """Blocked NVFP4 key scales [B, blocks * A] -> the paged scale pool
    [n_pages, A]: block u of request b goes to the pool page holding row 128 u."""
    A = dim // 64 * 512
    B = ksf.shape[0]
    nblk = ksf.shape[1] // A
    pool = _noise(gen, (n_pages, A), torch.uint8, ksf.device)
    pages = table[:, ::128 // pe][:, :nblk].reshape(-1).to(torch.int64)
    pool[pages.to(ksf.device)] = ksf.reshape(B * nblk, A)
    # the test's own regather (block u from the page of row 128 u) is the identity
    assert torch.equal(pool[pages.to(ksf.device)].reshape(B, nblk * A), ksf)
    return pool


# ------------------------------------------------------------------ attention

def _selection(g, B, T, k, vis):
    idx = torch.full((B, T, k), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(T):
            n = min(k, vis[b][t])
            idx[b, t, :n] = torch.randperm(vis[b][t], generator=g)[:n].to(torch.int32)
    return idx


def _attention_case(cfg_name, B, E, T, seed):
    cfg = dict(W.CONFIGS[cfg_name])
    m = cfg["m"]
    q0 = m * E - 1 if T == 1 else m * (E - 8)
    x = W.attention_inputs(cfg, "cpu", batch=B, ctx=E * m, n_q=T, q0=q0, n_entries=E, seed=seed)
    vis = [[min(E, (int(x["q_pos"][b, t]) + 1) // m) for t in range(T)] for b in range(B)]
    if cfg["kind"].startswith("csa"):
        x["idx"] = _selection(torch.Generator().manual_seed(seed), B, T, cfg["k"], vis)
    return cfg, x


def _attend(cfg, x, entries, opt=None, n_entries=None):
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    scale = 1.0 / math.sqrt(cfg["dim"])
    if cfg["kind"].startswith("csa"):
        return csa.sparse_mqa(g["Q"], entries.to(DEV), g["idx"], g["win"], g["win_start"], g["q_pos"],
                              cfg["window"], cfg["m"], g["sink"], scale, kv_dt=cfg["kv_dt"], options=opt,
                              n_entries=n_entries)
    return csa.hca_dense_mqa(g["Q"], entries.to(DEV), g["win"], g["win_start"], g["q_pos"], cfg["window"],
                             cfg["m"], g["sink"], scale, kv_dt=cfg["kv_dt"], options=opt, n_entries=n_entries)


def _oracle_attention(orc, cfg, x, entries_bytes):
    """The oracle's attention over the cache the oracle's gather returned
    (uint8 rows, viewed in the oracle's row format)."""
    scale = 1.0 / math.sqrt(cfg["dim"])
    ent = {csa.KV_FP8MIX: entries_bytes, csa.BF16: entries_bytes.view(np.uint16),
           csa.F32: entries_bytes.view(np.float32)}[cfg["kv_dt"]]
    if cfg["kind"].startswith("csa"):
        return orc.sparse_mqa(f64(x["Q"]), ent, cfg["kv_dt"], raw(x["idx"]), raw(x["win"]), raw(x["win_start"]),
                              raw(x["q_pos"]), cfg["window"], cfg["m"], f64(x["sink"]), scale)
    return orc.hca_dense_mqa(f64(x["Q"]), ent, cfg["kv_dt"], raw(x["win"]), raw(x["win_start"]),
                             raw(x["q_pos"]), cfg["window"], cfg["m"], f64(x["sink"]), scale)


@pytest.mark.parametrize("cfg_name,B,E,T,pe,splits", [
    ("csa_decode_1m_mixed", 2, 3000, 1, 32, 0),   # FP8MIX rows, tensor cores, 32-entry pages
    ("csa_decode_1m_mixed", 3, 2000, 1, 32, 2),   # fixed splits
    ("csa_decode_bf16", 2, 2500, 1, 64, 0),       # BF16 rows, 64-entry pages
    ("hca_decode_bf16", 2, 1500, 1, 1, 0),        # HCA: one entry per 128-token page
    ("csa_prefill_bf16", 1, 400, 24, 32, 0),      # many queries per request
    ("tiny_prefill_f32", 2, 64, 4, 8, 0),         # F32 rows: the SIMT kernel
])
def test_paged_attention(orc, cfg_name, B, E, T, pe, splits):
    cfg, x = _attention_case(cfg_name, B, E, T, seed=E + pe)
    gen = torch.Generator().manual_seed(E * 3 + pe)
    pool, table, n_pages = _scatter(x["entries"], pe, gen)
    gathered = _pin_scatter(orc, pool, table, n_pages, pe, x["entries"])
    opt = csa.mqa_options(splits=splits, entry_pages=csa.pages(table.to(DEV), pe, n_pages))
    paged = _attend(cfg, x, pool, opt, n_entries=E)
    plain = _attend(cfg, x, x["entries"], csa.mqa_options(splits=splits) if splits else None)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(paged, plain), "paged and contiguous calls differ"
    want = _oracle_attention(orc, cfg, x, gathered)
    assert_close(f64(paged), want, atol=1e-5 if cfg["kv_dt"] == csa.F32 else 2e-2, what=f"{cfg_name} pe={pe}")


def test_paged_attention_bad_page_is_reported():
    """A table slot naming a page outside the pool: the row is dropped (no
    memory outside the pool is read) and the status call reports it."""
    cfg, x = _attention_case("csa_decode_bf16", 1, 600, 1, seed=3)
    gen = torch.Generator().manual_seed(4)
    pool, table, n_pages = _scatter(x["entries"], 32, gen)
    j = int(x["idx"][0, 0, 0]) // 32
    table[0, j] = n_pages + 3
    opt = csa.mqa_options(entry_pages=csa.pages(table.to(DEV), 32, n_pages))
    _attend(cfg, x, pool, opt, n_entries=600)
    torch.cuda.synchronize()
    with pytest.raises(csa.CsaError) as e:
        csa.check_device_status()
    assert e.value.status == 1 and "page" in str(e.value)
    csa.check_device_status()  # the status word was cleared


# ------------------------------------------------------------------ indexer

def _exact_index_inputs(B, T, E, dt, seed, H=64, d=128):
    """Indexer inputs with every score exact in fp32 (power-of-two scales and
    weights, small integers), drawn on the GPU."""
    g = W.generator(seed, DEV)
    wI = (2.0 ** torch.randint(-1, 2, (B, T, H), generator=g, device=DEV)).to(torch.float32)
    if dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, T, H), d, device=DEV)
        KI, ksf = W.nvfp4_rows(g, (B, E), d, device=DEV)
        p2 = torch.tensor([0.125, 0.25, 0.5, 1.0], device=DEV).to(torch.float8_e4m3fn).view(torch.uint8)
        qsf = p2[torch.randint(0, 4, qsf.shape, generator=g, device=DEV)]
        ksf = p2[torch.randint(0, 4, ksf.shape, generator=g, device=DEV)]
        return dict(qI=qI, qI_sf=qsf, KI=KI, KI_sf=W.block_scales(ksf, d), wI=wI)
    tdt = torch.float32 if dt == csa.F32 else torch.bfloat16
    qI = torch.randint(-2, 3, (B, T, H, d), generator=g, device=DEV).to(tdt)
    KI = torch.randint(-2, 3, (B, E, d), generator=g, device=DEV).to(tdt)
    return dict(qI=qI, qI_sf=None, KI=KI, KI_sf=None, wI=wI)


def _sorted(row):
    v = np.sort(row[row >= 0])
    out = np.full(row.shape, -1, np.int32)
    out[:len(v)] = v
    return out


@pytest.mark.parametrize("dt,B,T,E,k,pe,H,d", [
    (csa.IDX_NVFP4, 2, 1, 262144, 1024, 32, 64, 128),  # decode, slices wrap the key ring
    (csa.IDX_NVFP4, 3, 1, 30000, 512, 128, 64, 128),   # one page per 128-entry tile
    (csa.BF16, 2, 1, 65536, 512, 64, 64, 128),         # BF16 decode
    (csa.BF16, 1, 6, 8192, 256, 16, 64, 128),          # several queries per CTA
    (csa.F32, 2, 2, 1000, 64, 8, 8, 64),               # F32: the SIMT kernel
])
def test_paged_indexer_bit_exact(orc, dt, B, T, E, k, pe, H, d):
    m = 4
    x = _exact_index_inputs(B, T, E, dt, seed=E + pe, H=H, d=d)
    gen = torch.Generator().manual_seed(pe + 1)
    pool, table, n_pages = _scatter(x["KI"], pe, gen)
    _pin_scatter(orc, pool, table, n_pages, pe, x["KI"])
    sf_pool = None
    if dt == csa.IDX_NVFP4:
        sf_pool = _scatter_key_scales(x["KI_sf"], table, pe, n_pages, d, gen)
    q_pos = torch.tensor([[m * E - 1 - 37 * t for t in range(T)]] * B, dtype=torch.int64, device=DEV)
    kp = csa.pages(table.to(DEV), pe, n_pages)
    idx_p, sc_p = csa.index_topk(x["qI"], x["wI"], pool, q_pos, m, k, dt=dt, qI_sf=x["qI_sf"], KI_sf=sf_pool,
                                 key_pages=kp, n_entries=E, scores=True)
    idx_c, sc_c = csa.index_topk(x["qI"], x["wI"], x["KI"], q_pos, m, k, dt=dt, qI_sf=x["qI_sf"],
                                 KI_sf=x["KI_sf"], scores=True)
    idx_p2 = csa.index_topk(x["qI"], x["wI"], pool, q_pos, m, k, dt=dt, qI_sf=x["qI_sf"], KI_sf=sf_pool,
                            key_pages=kp, n_entries=E)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(idx_p, idx_c) and torch.equal(sc_p, sc_c), "paged and contiguous calls differ"
    assert torch.equal(idx_p2, idx_p), "the score output changed the selection"
    for b in range(B):
        if dt == csa.IDX_NVFP4:
            K = orc.decode_rows(raw(x["KI"][b]), orc.NVFP4, d, sf=raw(x["KI_sf"][b]), sf_blocked=True)
            q = orc.decode_rows(raw(x["qI"][b]).reshape(-1, d // 2), orc.NVFP4, d,
                                sf=raw(x["qI_sf"][b]).reshape(-1, d // 16)).reshape(T, H, d)
        else:
            K, q = f64(x["KI"][b]), f64(x["qI"][b])
        want_sc, want_idx = orc.index_topk(q[None], f64(x["wI"][b:b + 1]), K[None], raw(q_pos[b:b + 1].cpu()), m, k,
                                           round_bf16=dt != csa.F32)
        assert np.array_equal(f64(sc_p[b]), want_sc[0]), f"request {b}: scores differ"
        for t in range(T):
            assert np.array_equal(raw(idx_p[b, t]), _sorted(want_idx[0, t])), f"request {b} query {t}"


def test_paged_indexer_bad_page_is_reported():
    x = _exact_index_inputs(1, 1, 4096, csa.BF16, seed=9)
    pool, table, n_pages = _scatter(x["KI"], 32, torch.Generator().manual_seed(2))
    table[0, 5] = -7
    q_pos = torch.tensor([[4 * 4096 - 1]], dtype=torch.int64, device=DEV)
    csa.index_topk(x["qI"], x["wI"], pool, q_pos, 4, 128, dt=csa.BF16,
                   key_pages=csa.pages(table.to(DEV), 32, n_pages), n_entries=4096)
    torch.cuda.synchronize()
    with pytest.raises(csa.CsaError) as e:
        csa.check_device_status()
    assert e.value.status == 1
    csa.check_device_status()


# ------------------------------------------------------------ compressor writes

@pytest.mark.parametrize("out_dt,dim,m,overlap,pe,E", [
    (csa.KV_FP8MIX, 512, 4, True, 32, 150),   # KV entries, 32 per page
    (csa.IDX_NVFP4, 128, 4, True, 32, 300),   # index keys with their blocked scales
    (csa.BF16, 512, 128, False, 1, 9),        # HCA entries, one per page
])
def test_paged_compress_writes_the_contiguous_bytes(orc, out_dt, dim, m, overlap, pe, E):
    B = 2
    x = W.compress_inputs(W.generator(E + pe), B, m * E, dim, m, overlap, torch.bfloat16)
    gx = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    args = (gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"])
    res = csa.compress(*args, out_dt=out_dt)
    ref, ref_sf = res if out_dt == csa.IDX_NVFP4 else (res, None)
    gen = torch.Generator().manual_seed(11)
    pool, table, n_pages = _scatter(torch.zeros_like(ref), pe, gen)
    pool = pool.to(DEV)
    before = pool.clone()
    sf_pool = None
    if out_dt == csa.IDX_NVFP4:
        sf_pool = _noise(gen, (n_pages, dim // 64 * 512), torch.uint8, DEV)
    sf_before = None if sf_pool is None else sf_pool.clone()
    kp = csa.pages(table.to(DEV), pe, n_pages)
    job = csa.compress_job(*args, tok0=0, e0=0, n_out=E, out=pool, out_sf=sf_pool, out_dt=out_dt, out_pages=kp)
    csa.compress_ex(job, B)
    torch.cuda.synchronize()
    csa.check_device_status()
    got = orc.gather_paged(_row_bytes(pool, (n_pages, pe)), raw(table), E)
    assert np.array_equal(got, _row_bytes(ref, (B, E))), "gathered pool differs from the contiguous output"
    # rows that no entry maps to keep their bytes
    used = torch.zeros(n_pages * pe, dtype=torch.bool)
    for b in range(B):
        for e in range(E):
            used[int(table[b, e // pe]) * pe + e % pe] = True
    assert torch.equal(pool[~used.to(DEV)], before[~used.to(DEV)])
    if out_dt == csa.IDX_NVFP4:
        A = dim // 64 * 512
        nblk = -(-E // 128)
        pages = table[:, ::128 // pe][:, :nblk].reshape(-1).to(torch.int64).to(DEV)
        got_sf = sf_pool[pages].reshape(B, nblk * A)
        # the scales of rows 0 .. E-1 (rows past E in the last block are written by neither form)
        for b in range(B):
            g_rows = orc.unblock_scales(raw(got_sf[b]), nblk * 128, dim)[:E]
            r_rows = orc.unblock_scales(raw(ref_sf[b]), E, dim)[:E]
            assert np.array_equal(g_rows, r_rows), f"request {b}: key scales"
        untouched = torch.ones(n_pages, dtype=torch.bool)
        untouched[pages.cpu()] = False
        assert torch.equal(sf_pool[untouched.to(DEV)], sf_before[untouched.to(DEV)])


@pytest.mark.parametrize("dt,n_new,pe", [(csa.IDX_NVFP4, 2, 32), (csa.BF16, 1, 64)])
def test_paged_compress_index_topk(orc, dt, n_new, pe):
    """The fused decode call on paged key and KV caches writes the bytes and
    selects the indices of the fused call on contiguous caches."""
    B, T, E, k, m, dI, H, c = 2, 1, 19969, 512, 4, 128, 64, 512
    g = W.generator(700 + pe)
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
    q_pos = torch.full((B, T), m * E - 1, dtype=torch.int64, device=DEV)
    cu = lambda v: None if v is None else v.to(DEV)  # noqa: E731
    gt, gk = ({k: cu(v) if isinstance(v, torch.Tensor) else v for k, v in d.items()} for d in (tok, ktok))
    e0 = E - n_new
    tok0 = m * (e0 - 1)
    # contiguous caches
    K1, S1, V1 = cu(KI).clone(), cu(ksf).clone() if ksf is not None else None, cu(kv).clone()
    keys1 = csa.compress_job(gt["Ca"], gt["Za"], gt["Ba"], m, gt["Cb"], gt["Zb"], gt["Bb"], tok0=tok0, e0=e0,
                             n_out=n_new, out=K1, out_sf=S1, out_dt=dt)
    extra1 = csa.compress_job(gk["Ca"], gk["Za"], gk["Ba"], m, gk["Cb"], gk["Zb"], gk["Bb"], tok0=tok0, e0=e0,
                              n_out=n_new, out=V1, out_dt=csa.KV_FP8MIX)
    idx1 = csa.compress_index_topk(keys1, cu(qI), cu(wI), K1, q_pos, m, k, extra_job=extra1, dt=dt,
                                   qI_sf=cu(qsf), KI_sf=S1)
    # paged caches, the same contents before the call
    gen = torch.Generator().manual_seed(pe)
    Kp, kt, kn = _scatter(cu(KI), pe, gen)
    Vp, vt, vn = _scatter(cu(kv), 32, gen)
    Sp = _scatter_key_scales(cu(ksf), kt, pe, kn, dI, gen) if ksf is not None else None
    kpages, vpages = csa.pages(kt.to(DEV), pe, kn), csa.pages(vt.to(DEV), 32, vn)
    keys2 = csa.compress_job(gt["Ca"], gt["Za"], gt["Ba"], m, gt["Cb"], gt["Zb"], gt["Bb"], tok0=tok0, e0=e0,
                             n_out=n_new, out=Kp, out_sf=Sp, out_dt=dt, out_pages=kpages)
    extra2 = csa.compress_job(gk["Ca"], gk["Za"], gk["Ba"], m, gk["Cb"], gk["Zb"], gk["Bb"], tok0=tok0, e0=e0,
                              n_out=n_new, out=Vp, out_dt=csa.KV_FP8MIX, out_pages=vpages)
    idx2 = csa.compress_index_topk(keys2, cu(qI), cu(wI), Kp, q_pos, m, k, extra_job=extra2, dt=dt,
                                   qI_sf=cu(qsf), KI_sf=Sp, n_entries=E)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(idx1, idx2), "paged and contiguous selections differ"
    assert np.array_equal(orc.gather_paged(_row_bytes(Kp, (kn, pe)), raw(kt), E), _row_bytes(K1, (B, E)))
    assert np.array_equal(orc.gather_paged(_row_bytes(Vp, (vn, 32)), raw(vt), E), _row_bytes(V1, (B, E)))
    if Sp is not None:
        A = dI // 64 * 512
        nblk = S1.shape[1] // A
        pages = kt[:, ::128 // pe][:, :nblk].reshape(-1).to(torch.int64).to(DEV)
        assert torch.equal(Sp[pages].reshape(B, nblk * A), S1)
