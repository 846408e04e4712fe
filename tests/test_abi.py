"""The C ABI library loads, exports what include/csa.h declares, and validates
arguments on the host (CPU only: no call here reaches a kernel launch)."""
import ctypes
import subprocess

import pytest

from compressed_sparse_attention_hca_b200 import csa

INVALID, UNSUPPORTED = 1, 2
P = ctypes.c_void_p
A = P(4096)  # a 16-byte aligned non-null address; never dereferenced by these calls


def test_library_exports_every_declared_symbol():
    lib = csa.load()
    declared = csa.header_functions()
    assert {"csa_compress", "csa_index_topk", "csa_sparse_mqa", "hca_dense_mqa"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", csa.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared:
        assert name in exported, name
        getattr(lib, name)


def test_version_and_row_bytes():
    assert csa.load().csa_version() == 201
    assert csa.row_bytes(csa.F32, 512) == 2048
    assert csa.row_bytes(csa.BF16, 512) == 1024
    assert csa.row_bytes(csa.KV_FP8MIX, 512) == 608
    assert csa.row_bytes(csa.IDX_NVFP4, 128) == 64
    assert csa.row_bytes(csa.KV_FP8MIX, 100) == -1
    assert csa.row_bytes(csa.IDX_NVFP4, 40) == -1
    # blocked key scales: 128-row blocks of dim/64 atoms of 512 bytes
    assert csa.nvfp4_key_scale_bytes(1, 128) == 1024
    assert csa.nvfp4_key_scale_bytes(128, 128) == 1024
    assert csa.nvfp4_key_scale_bytes(129, 128) == 2048
    assert csa.nvfp4_key_scale_bytes(262144, 128) == 262144 * 8
    assert csa.nvfp4_key_scale_bytes(0, 128) == 0
    assert csa.nvfp4_key_scale_bytes(10, 96) == -1


def _err():
    return csa.load().csa_last_error().decode()


def test_compress_rejects_bad_arguments():
    lib = csa.load()
    args = dict(Ca=A, Cb=A, Za=A, Zb=A, Ba=A, Bb=A, batch=1, n_tok=64, tok0=0, stride=64, e0=0, n_out=16,
                dim=64, m=4, in_dt=csa.F32, out=A, out_sf=None, out_stride=16, out_row0=0, out_dt=csa.F32)

    def call(**kw):
        a = dict(args, **kw)
        return lib.csa_compress(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["Ba"], a["Bb"], a["batch"], a["n_tok"],
                                a["tok0"], a["stride"], a["e0"], a["n_out"], a["dim"], a["m"], a["in_dt"],
                                a["out"], a["out_sf"], a["out_stride"], a["out_row0"], a["out_dt"], None)
    assert call(m=0) == INVALID and "m=0" in _err()
    assert call(dim=60) == INVALID
    assert call(in_dt=csa.KV_FP8MIX) == INVALID
    assert call(out_dt=csa.KV_FP8MIX) == INVALID  # dim 64 has no FP8 dims
    assert call(out_dt=csa.IDX_NVFP4) == INVALID and "out_sf" in _err()
    assert call(Ca=None) == INVALID and "Ca is NULL" in _err()
    assert call(Za=P(4100)) == INVALID and "aligned" in _err()
    # entries 0..16 need tokens up to 67 but only 64 rows are present
    assert call(n_out=17, out_stride=17) == INVALID and "need tokens" in _err()
    # entry 5 with overlap needs token 16 onward; rows start at token 20
    assert call(tok0=20, e0=5, n_out=1, n_tok=44, stride=44) == INVALID
    assert call(out_stride=8) == INVALID
    assert call(out_stride=20, out_row0=5) == INVALID and "out_row0" in _err()  # 5 + 16 rows > 20
    assert call(out_row0=-1) == INVALID
    assert call(out_dt=csa.IDX_NVFP4, out_sf=P(4104)) == INVALID and "aligned" in _err()
    assert call(out_dt=csa.IDX_NVFP4, out_sf=A, dim=32, n_tok=64) == INVALID and "64" in _err()
    assert call(batch=0) == 0  # empty call is a no-op


def test_index_topk_rejects_bad_arguments():
    lib = csa.load()

    def call(k=16, heads=2, dim=32, dt=csa.F32, ws_bytes=1 << 20, qsf=None, ksf=None, ws=A):
        return lib.csa_index_topk(A, qsf, A, A, ksf, A, 1, 4, 64, 4, heads, dim, k, dt, A, None, ws,
                                  ws_bytes, None)
    assert call(k=0) == INVALID
    assert call(k=4096) == INVALID
    assert call(dim=48) == INVALID
    assert call(heads=200) == INVALID
    assert call(dt=csa.KV_FP8MIX) == INVALID
    assert call(dt=csa.IDX_NVFP4) == INVALID and "NVFP4" in _err()
    assert call(dt=csa.IDX_NVFP4, qsf=A, ksf=A, dim=96) == INVALID and "64" in _err()
    assert call(dt=csa.IDX_NVFP4, qsf=A, ksf=P(4104), dim=128) == INVALID and "KI_sf" in _err()
    assert lib.csa_index_topk_workspace_size(1, 4, 64, 16, 2, 32, csa.F32) >= 256
    big = lib.csa_index_topk_workspace_size(4, 1, 262144, 1024, 64, 128, csa.IDX_NVFP4)
    assert call(ws_bytes=16) == INVALID or big <= 16


def test_mqa_rejects_bad_arguments():
    lib = csa.load()

    def call(dim=64, heads=4, k=16, window=16, kv_dt=csa.F32, q_dt=csa.F32, idx=A):
        return lib.csa_sparse_mqa(A, q_dt, A, 64, idx, k, A, 256, A, A, window, 4, A, 0.125, 1, 4, heads,
                                  dim, kv_dt, A, A, 1 << 20, None)
    assert call(dim=96) == INVALID
    assert call(heads=0) == INVALID
    assert call(k=0) == INVALID
    assert call(window=-1) == INVALID
    assert call(kv_dt=csa.IDX_NVFP4) == INVALID
    assert call(q_dt=csa.KV_FP8MIX) == INVALID
    assert call(idx=None) == INVALID
    assert lib.hca_dense_mqa(A, csa.BF16, A, 64, A, 256, A, A, 16, 4, A, 0.1, 1, 4, 4, 100, csa.BF16,
                             A, A, 1 << 20, None) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        csa.compress(torch.zeros(1, 8, 64), torch.zeros(1, 8, 64), torch.zeros(4, 64), 4)


def test_compress_index_topk_rejects_bad_arguments():
    lib = csa.load()
    KI = P(8192)

    def job(**kw):
        j = dict(Ca=4096, Cb=4096, Za=4096, Zb=4096, Ba=4096, Bb=4096, n_tok=8, tok0=56, in_batch_stride=8, e0=15,
                 n_out=1, dim=32, m=4, in_dt=csa.BF16, out=8192, out_sf=None, out_batch_stride=64, out_row0=15,
                 out_dt=csa.BF16)
        j.update(kw)
        return csa.CompressJob(**j)

    def call(keys, extra=None, dt=csa.BF16, n_entries=64, dim=32):
        return lib.csa_compress_index_topk(ctypes.byref(keys), ctypes.byref(extra) if extra else None, A, None, A,
                                           KI, None, A, 1, 1, n_entries, 4, 2, dim, 16, dt, A, None, A, 1 << 20, None)
    assert call(job(), dt=csa.KV_FP8MIX) == INVALID
    # the key job must write entry i to row i of the indexer's cache
    assert call(job(out_row0=3)) == INVALID and "row i" in _err()
    assert call(job(out=4096)) == INVALID and "row i" in _err()
    # entry 15 with overlap needs tokens 56..63; rows start at token 60
    assert call(job(tok0=60, n_tok=4, in_batch_stride=4)) == INVALID and "need tokens" in _err()
    # the extra job must not write the indexer's cache
    assert call(job(), extra=job()) == INVALID and "extra" in _err()
    assert call(job(), dim=48) == INVALID


def test_rmsnorm_rope_rejects_bad_arguments():
    lib = csa.load()
    F32, BF16 = csa.F32, csa.BF16

    def call(x=A, y=P(8192), n=4, dim=512, g=A, eps=1e-6, pos=A, rpp=1, sign=1, rope=64, base=10000.0,
             idt=BF16, odt=BF16):
        return lib.csa_rmsnorm_rope(x, y, n, dim, g, eps, pos, rpp, sign, rope, base, idt, odt, None)

    assert call(n=0) == 0                        # nothing to do
    assert call(n=-1) == INVALID
    assert call(dim=500) == INVALID              # not a multiple of 8
    assert call(rope=60) == INVALID              # rope_dims not a multiple of 8
    assert call(dim=64, rope=72) == INVALID      # rope_dims > dim
    assert call(rpp=0) == INVALID
    assert call(sign=2) == INVALID
    assert call(eps=-1.0) == INVALID
    assert call(base=0.0) == INVALID
    assert call(idt=csa.KV_FP8MIX) == INVALID
    assert call(odt=csa.IDX_NVFP4) == INVALID
    assert call(y=A, idt=F32, odt=BF16) == INVALID   # in place needs one dtype
    assert call(x=P(4100)) == INVALID            # misaligned
    assert call(x=None) == INVALID
    assert call(pos=None) == INVALID             # rotation needs positions
    assert "pos" in csa.load().csa_last_error().decode()


def test_grouped_out_proj_rejects_bad_arguments():
    lib = csa.load()

    def call(O=A, Wg=A, Wo=A, Y=P(8192), T=4, n_h=16, c=64, g=4, d_g=128, d=256, ws=P(16384), wsb=1 << 30):
        return lib.csa_grouped_out_proj(O, Wg, Wo, Y, T, n_h, c, g, d_g, d, ws, wsb, None)

    assert call(T=0) == 0                       # nothing to do
    assert call(T=-1) == INVALID
    assert call(n_h=16, g=3) == INVALID         # groups must divide the heads
    assert call(c=8) == INVALID                 # n_h/g * c = 32: not a multiple of 64
    assert call(d_g=96) == INVALID              # not a multiple of 128
    assert call(d=200) == INVALID
    assert call(O=None) == INVALID
    assert call(Wo=P(4104)) == INVALID          # misaligned
    assert call(Y=A) == INVALID                 # Y aliases O
    assert call(wsb=256) == INVALID and "workspace too small" in _err()


def test_grouped_out_proj_plan():
    v4 = dict(n_h=128, c=512, g=16, d_g=1024, d=7168)
    for T in (1, 4, 16):
        p = csa.grouped_out_proj_plan(T, **v4)
        # decode reads only weights: K is split until both launches cover the 148 SMs
        for step in ("group", "output"):
            assert p[step]["ctas"] >= 148 and p[step]["splits"] > 1, (T, p)
            assert p[step]["tokens_per_cta"] == 16
    p = csa.grouped_out_proj_plan(4096, **v4)
    assert p["group"] == {"tokens_per_cta": 256, "splits": 1, "ctas": 8 * 16 * 16}
    assert p["output"] == {"tokens_per_cta": 256, "splits": 1, "ctas": 56 * 16}
    # the workspace holds Z (bf16) at least, and grows with T
    sizes = [csa.grouped_out_proj_workspace_size(T, **v4) for T in (1, 4, 64, 4096)]
    assert sizes[-1] >= 4096 * 16 * 1024 * 2 and sizes == sorted(sizes)
    with pytest.raises(csa.CsaError):
        csa.grouped_out_proj_plan(0, **v4)


def test_paged_calls_reject_bad_tables():
    lib = csa.load()
    pg = csa.Pages(table=4096, max_pages=4, page_entries=32, n_pages=100)

    def index(pages, n_entries=100, dt=csa.BF16):
        return lib.csa_index_topk_paged(A, None, A, A, None, ctypes.byref(pages) if pages else None, A, 1, 1,
                                        n_entries, 4, 64, 128, 16, dt, A, None, A, 1 << 30, None)
    assert index(csa.Pages(table=4096, max_pages=4, page_entries=12, n_pages=100)) == INVALID  # 12 does not divide 128
    assert index(csa.Pages(table=4096, max_pages=4, page_entries=4, n_pages=100)) == INVALID   # below 8
    assert index(pg, n_entries=129) == INVALID and "max_pages" in _err()                      # 129 > 4 x 32
    assert index(csa.Pages(table=None, max_pages=4, page_entries=32, n_pages=100)) == INVALID
    assert index(csa.Pages(table=4100, max_pages=4, page_entries=32, n_pages=100)) == INVALID  # misaligned
    assert index(csa.Pages(table=4096, max_pages=4, page_entries=32, n_pages=0)) == INVALID

    def mqa(pages):
        opt = csa.MqaOptions(entry_pages=ctypes.pointer(pages))
        return lib.csa_sparse_mqa_ex(A, csa.BF16, A, 100, A, 16, A, 0, A, A, 0, 4, A, 1.0, 1, 1, 64, 512,
                                     csa.BF16, A, A, 1 << 30, ctypes.byref(opt), None)
    assert mqa(csa.Pages(table=4096, max_pages=0, page_entries=32, n_pages=10)) == INVALID
    assert mqa(csa.Pages(table=4096, max_pages=3, page_entries=32, n_pages=10)) == INVALID  # 100 > 96


def test_compress_job_rejects_bad_epilogue_and_pages():
    lib = csa.load()

    def job(**kw):
        j = csa.CompressJob(Ca=4096, Za=4096, Ba=4096, n_tok=64, tok0=0, in_batch_stride=64, e0=0, n_out=16, dim=128,
                            m=4, in_dt=csa.F32, out=8192, out_sf=8192, out_batch_stride=16, out_row0=0,
                            out_dt=csa.F32, rope_base=10000.0, pos_stride=4, pos_offset=3)
        for k, v in kw.items():
            setattr(j, k, v)
        return lib.csa_compress_ex(ctypes.byref(j), 1, None)
    assert job(rope_dims=12) == INVALID                       # not a multiple of 8
    assert job(rope_dims=136) == INVALID                      # beyond dim
    assert job(norm_g=4096, norm_eps=-1.0) == INVALID
    assert job(rope_dims=64, rope_base=0.0) == INVALID
    pg = csa.Pages(table=4096, max_pages=1, page_entries=48, n_pages=4)
    assert job(out_dt=csa.IDX_NVFP4, out_pages=ctypes.pointer(pg)) == INVALID  # 48 does not divide 128
    pg2 = csa.Pages(table=4096, max_pages=1, page_entries=8, n_pages=4)
    assert job(out_pages=ctypes.pointer(pg2)) == INVALID      # 16 entries > 1 x 8
