"""KV-entry RMSNorm and partial RoPE in the compressor's epilogue
("DeepSeek-V4 内部机制" 1.4 table: the compressed entries are normalised and
their last 64 dims turned by RoPE; reading of the entry position: its last
token, m (i + 1) - 1).

  * the fused BF16 entry is bitwise csa_rmsnorm_rope applied to the F32 entry
    of the plain compressor and rounded, in every compressor form (a CTA per
    entry for prefill, the staged form inside the fused decode indexer);
  * against the float64 oracle's composition rope_tail(rmsnorm(compress)):
    BF16 within one rounding step, FP8MIX within one E4M3 step of the block
    scale, NVFP4 codes the oracle's encoding unless fp32 and fp64 straddle a
    rounding boundary;
  * the fused decode call (keys + normalised KV entries + indexer in one
    launch) writes the bytes of the separate calls.
"""
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


def _weights(dim, seed):
    return (torch.randn(dim, generator=torch.Generator().manual_seed(seed)) * 0.3 + 1.0).to(torch.float32)


def _oracle_entries(orc, x, m, tok0, e0, n_out, g, eps, rope_dims, stride, offset):
    outs = []
    for b in range(x["Ca"].shape[0]):
        kw = {}
        if x["Cb"] is not None:
            kw = dict(Cb=f64(x["Cb"][b]), Zb=f64(x["Zb"][b]), Bb=f64(x["Bb"]))
        e = orc.compress(f64(x["Ca"][b]), f64(x["Za"][b]), f64(x["Ba"]), m, tok0=tok0, e0=e0, n_out=n_out, **kw)
        pos = stride * (e0 + np.arange(e.shape[0], dtype=np.float64)) + offset
        if g is not None:
            e = orc.rmsnorm(e, f64(g), eps)
        outs.append(orc.rope_tail(e, pos, rope_dims=rope_dims) if rope_dims else e)
    return np.stack(outs)


CASES = [
    # batch, n_tok, dim, m, overlap, tok0, e0, n_out, norm, rope_dims
    (2, 4 * 300, 512, 4, True, 0, 0, 300, True, 64),       # CSA prefill: a CTA per entry
    (3, 8, 512, 4, True, 4 * 1000, 1001, 1, True, 64),     # decode: the closing block
    (2, 128 * 6, 512, 128, False, 0, 0, 6, True, 64),      # HCA, m' = 128
    (1, 4 * 50, 128, 4, True, 0, 0, 50, False, 64),        # RoPE only
    (1, 4 * 20, 448, 4, True, 0, 0, 20, True, 0),          # normalisation only
]


@pytest.mark.parametrize("case", CASES)
def test_bf16_entry_equals_the_separate_norm(orc, case):
    B, n_tok, dim, m, overlap, tok0, e0, n_out, norm, rope = case
    x = W.compress_inputs(W.generator(n_tok + dim), B, n_tok, dim, m, overlap, torch.bfloat16)
    gx = _cuda(x)
    g = _weights(dim, 1) if norm else None
    gd = g.to(DEV) if g is not None else None
    args = (gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"])
    out = torch.empty(B, n_out, dim, dtype=torch.bfloat16, device=DEV)
    job = csa.compress_job(*args, tok0=tok0, e0=e0, n_out=n_out, out=out, out_dt=csa.BF16, out_row0=0,
                           norm_g=gd, norm_eps=1e-6, rope_dims=rope, n_tok=n_tok)
    csa.compress_ex(job, B)
    f32 = csa.compress(*args, tok0=tok0, e0=e0, n_out=n_out, out_dt=csa.F32, n_tok=n_tok)
    pos = (m * (e0 + torch.arange(n_out, device=DEV)) + m - 1).to(torch.int64)
    pos = pos.repeat(B)
    sep = csa.rmsnorm_rope(f32.reshape(-1, dim), pos, g=gd, eps=1e-6, rope_dims=rope, out_dt=csa.BF16)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(out.reshape(-1, dim), sep), "fused and separate normalisation differ"
    want = _oracle_entries(orc, x, m, tok0, e0, n_out, g, 1e-6, rope, m, m - 1)
    assert_close(f64(out), want, atol=1e-5, rtol=2.0 ** -8, what="bf16 entries vs oracle")


def test_fp8mix_entry_matches_oracle(orc):
    B, n_tok, dim, m = 2, 4 * 40, 512, 4
    x = W.compress_inputs(W.generator(8), B, n_tok, dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    g = _weights(dim, 2)
    out = torch.empty(B, 40, 608, dtype=torch.uint8, device=DEV)
    job = csa.compress_job(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], tok0=0, e0=0, n_out=40,
                           out=out, out_dt=csa.KV_FP8MIX, norm_g=g.to(DEV), rope_dims=64)
    csa.compress_ex(job, B)
    torch.cuda.synchronize()
    csa.check_device_status()
    want = _oracle_entries(orc, x, m, 0, 0, 40, g, 1e-6, 64, m, m - 1)
    got_bytes = raw(out)
    for b in range(B):
        dec = orc.decode_rows(got_bytes[b], orc.FP8MIX, dim)
        ref_bytes, _ = orc.encode_rows(want[b], orc.FP8MIX)
        ref_scale = ref_bytes[:, 576:604].copy().view(np.float32)
        got_scale = got_bytes[b, :, 576:604].copy().view(np.float32)
        assert_close(got_scale, ref_scale, atol=0, rtol=1e-5, what="fp8 scales")
        scale_per_dim = np.repeat(ref_scale, 64, axis=1)
        bound = 2.0 ** -3 * np.abs(want[b, :, :448]) + 2.0 ** -9 * scale_per_dim + 1e-6
        assert (np.abs(dec[:, :448] - want[b, :, :448]) <= bound).all()
        assert_close(dec[:, 448:], want[b, :, 448:], atol=1e-5, rtol=2.0 ** -8, what="rope dims bf16")


def test_nvfp4_key_matches_oracle(orc):
    B, n_tok, dim, m = 2, 4 * 64, 128, 4
    x = W.compress_inputs(W.generator(9), B, n_tok, dim, m, True, torch.bfloat16)
    gx = _cuda(x)
    g = _weights(dim, 3)
    codes = torch.empty(B, 64, 64, dtype=torch.uint8, device=DEV)
    sf = torch.zeros(B, csa.nvfp4_key_scale_bytes(64, dim), dtype=torch.uint8, device=DEV)
    job = csa.compress_job(gx["Ca"], gx["Za"], gx["Ba"], m, gx["Cb"], gx["Zb"], gx["Bb"], tok0=0, e0=0, n_out=64,
                           out=codes, out_sf=sf, out_dt=csa.IDX_NVFP4, norm_g=g.to(DEV), rope_dims=64)
    csa.compress_ex(job, B)
    torch.cuda.synchronize()
    csa.check_device_status()
    want = _oracle_entries(orc, x, m, 0, 0, 64, g, 1e-6, 64, m, m - 1)
    for b in range(B):
        check_nvfp4_rows(orc, raw(codes[b]), orc.unblock_scales(raw(sf[b]), 64, dim), want[b], dim)


@pytest.mark.parametrize("dt", [csa.IDX_NVFP4, csa.BF16])
def test_fused_decode_with_normalised_entries(dt):
    """Key job plain, KV job normalised and turned: the one-launch decode call
    writes the separate calls' bytes (staged form vs a CTA per entry)."""
    B, T, E, k, m, dI, H, c, n_new = 2, 1, 19969, 512, 4, 128, 64, 512, 2
    g = W.generator(77)
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
    gn = _weights(c, 4).to(DEV)
    gk = _weights(dI, 5).to(DEV)
    cu = lambda v: None if v is None else v.to(DEV)  # noqa: E731
    gt, gkv = _cuda(tok), _cuda(ktok)
    e0 = E - n_new
    tok0 = m * (e0 - 1)

    def jobs(K, S, V):
        keys = csa.compress_job(gt["Ca"], gt["Za"], gt["Ba"], m, gt["Cb"], gt["Zb"], gt["Bb"], tok0=tok0, e0=e0,
                                n_out=n_new, out=K, out_sf=S, out_dt=dt, norm_g=gk, rope_dims=64)
        extra = csa.compress_job(gkv["Ca"], gkv["Za"], gkv["Ba"], m, gkv["Cb"], gkv["Zb"], gkv["Bb"], tok0=tok0,
                                 e0=e0, n_out=n_new, out=V, out_dt=csa.KV_FP8MIX, norm_g=gn, rope_dims=64)
        return keys, extra

    K1, S1, V1 = cu(KI).clone(), cu(ksf).clone() if ksf is not None else None, cu(kv).clone()
    keys1, extra1 = jobs(K1, S1, V1)
    csa.compress_ex(keys1, B)
    csa.compress_ex(extra1, B)
    idx1 = csa.index_topk(cu(qI), cu(wI), K1, q_pos, m, k, dt=dt, qI_sf=cu(qsf), KI_sf=S1)
    K2, S2, V2 = cu(KI).clone(), cu(ksf).clone() if ksf is not None else None, cu(kv).clone()
    keys2, extra2 = jobs(K2, S2, V2)
    idx2 = csa.compress_index_topk(keys2, cu(qI), cu(wI), K2, q_pos, m, k, extra_job=extra2, dt=dt,
                                   qI_sf=cu(qsf), KI_sf=S2)
    assert csa.last_launch_count() == 1, "the decode step is one launch"
    torch.cuda.synchronize()
    csa.check_device_status()
    assert torch.equal(K1, K2) and torch.equal(V1, V2) and torch.equal(idx1, idx2)
    if S1 is not None:
        assert torch.equal(S1, S2)
    assert not torch.equal(V2[:, e0:], cu(kv)[:, e0:]), "the new KV entries were written"
