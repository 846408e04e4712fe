"""The tensor-core attention's modes and options against the float64 oracle.

  * every way the rows of a query are split -- one CTA per (query, 64 heads),
    several splits combined by the combine kernel, one split or several chunks
    per CTA -- gives the oracle's output (2e-2 max abs, bf16);
  * batch-invariant decode ("CSA / HCA: 混合稀疏注意力机制", infrastructure
    section; "DeepSeek-V4 内部机制" 6.3): with a fixed split count a request's
    output is bitwise the same alone and inside batches of 16 and 40, for
    FP8MIX and BF16 rows and for the dense form;
  * the fused query RMSNorm + RoPE and the output turned at -t
    ("DeepSeek-V4 内部机制" 1.4 table) equal the oracle's composition
    rope_tail(attend(rope_tail(rmsnorm(Q), t)), -t), and the fused query
    prologue gives bitwise what csa_rmsnorm_rope followed by the plain call
    gives.
"""
import math

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


def _selection(g, B, T, k, vis):
    idx = torch.full((B, T, k), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(T):
            n = min(k, vis[b][t])
            idx[b, t, :n] = torch.randperm(vis[b][t], generator=g)[:n].to(torch.int32)
    return idx


def _case(cfg_name, B, E, T=1, seed=11, q0=None):
    cfg = dict(W.CONFIGS[cfg_name])
    m = cfg["m"]
    q0 = m * E - 1 if q0 is None else q0
    x = W.attention_inputs(cfg, "cpu", batch=B, ctx=E * m, n_q=T, q0=q0, n_entries=E, seed=seed)
    vis = [[min(E, (int(x["q_pos"][b, t]) + 1) // m) for t in range(T)] for b in range(B)]
    if cfg["kind"].startswith("csa"):
        x["idx"] = _selection(torch.Generator().manual_seed(seed), B, T, cfg["k"], vis)
    return cfg, x


def _run(cfg, x, opt=None, rows=None):
    """The attention call on requests `rows` (all by default) of the case."""
    sl = slice(None) if rows is None else rows
    g = {k: (v[sl].to(DEV) if isinstance(v, torch.Tensor) and v.dim() > 0 and k not in ("sink",) else
             (v.to(DEV) if isinstance(v, torch.Tensor) else v)) for k, v in x.items()}
    scale = 1.0 / math.sqrt(cfg["dim"])
    if cfg["kind"].startswith("csa"):
        return csa.sparse_mqa(g["Q"], g["entries"], g["idx"], g["win"], g["win_start"], g["q_pos"], cfg["window"],
                              cfg["m"], g["sink"], scale, kv_dt=cfg["kv_dt"], options=opt)
    return csa.hca_dense_mqa(g["Q"], g["entries"], g["win"], g["win_start"], g["q_pos"], cfg["window"], cfg["m"],
                             g["sink"], scale, kv_dt=cfg["kv_dt"], options=opt)


def _oracle(orc, cfg, x, Q=None):
    scale = 1.0 / math.sqrt(cfg["dim"])
    Q = f64(x["Q"]) if Q is None else Q
    if cfg["kind"].startswith("csa"):
        return orc.sparse_mqa(Q, raw(x["entries"]), cfg["kv_dt"], raw(x["idx"]), raw(x["win"]), raw(x["win_start"]),
                              raw(x["q_pos"]), cfg["window"], cfg["m"], f64(x["sink"]), scale)
    return orc.hca_dense_mqa(Q, raw(x["entries"]), cfg["kv_dt"], raw(x["win"]), raw(x["win_start"]),
                             raw(x["q_pos"]), cfg["window"], cfg["m"], f64(x["sink"]), scale)


@pytest.mark.parametrize("cfg_name,B,E,T,splits", [
    ("csa_decode_1m_mixed", 1, 3000, 1, 0),    # automatic: 9 splits, one chunk each
    ("csa_decode_1m_mixed", 4, 3000, 1, 0),    # automatic, the benchmark's shape of splits
    ("csa_decode_bf16", 3, 3000, 1, 0),        # BF16 rows, automatic
    ("csa_decode_bf16", 2, 3000, 1, 1),        # one CTA per (query, 64 heads)
    ("csa_decode_1m_mixed", 40, 2000, 1, 3),   # 240 CTAs, three chunks per split
    ("hca_decode_bf16", 2, 1500, 1, 0),        # dense rows, several chunks per split (prefetch)
    ("hca_decode_bf16", 1, 1500, 1, 2),        # dense rows, long splits
    ("csa_prefill_bf16", 1, 300, 40, 0),       # many queries: one CTA per (query, 64 heads)
])
def test_modes_match_oracle(orc, cfg_name, B, E, T, splits):
    cfg, x = _case(cfg_name, B, E, T, q0=None if T == 1 else 600)
    out = _run(cfg, x, csa.mqa_options(splits=splits) if splits else None)
    torch.cuda.synchronize()
    csa.check_device_status()
    assert_close(f64(out), _oracle(orc, cfg, x), atol=2e-2, what=f"{cfg_name} B={B} splits={splits}")


@pytest.mark.parametrize("cfg_name,E,splits", [
    ("csa_decode_1m_mixed", 3000, 3),
    ("csa_decode_1m_mixed", 3000, 1),
    ("csa_decode_bf16", 3000, 4),
    ("hca_decode_bf16", 1200, 3),
])
def test_fixed_splits_are_batch_invariant(cfg_name, E, splits):
    """Requests 0, 7 and 15 of a batch of 16 (and of 40: more CTAs than SMs)
    give bitwise the outputs they give alone."""
    cfg, x = _case(cfg_name, 40, E, seed=23)
    opt = csa.mqa_options(splits=splits)
    o40 = _run(cfg, x, opt)
    o16 = _run(cfg, x, opt, rows=slice(0, 16))
    torch.cuda.synchronize()
    for j in (0, 7, 15):
        o1 = _run(cfg, x, opt, rows=slice(j, j + 1))
        torch.cuda.synchronize()
        assert torch.equal(o1[0], o16[j]), f"request {j}: batch 1 vs 16"
        assert torch.equal(o1[0], o40[j]), f"request {j}: batch 1 vs 40"
    csa.check_device_status()


@pytest.mark.parametrize("cfg_name,B,splits", [("csa_decode_1m_mixed", 2, 0), ("csa_decode_bf16", 3, 0),
                                               ("hca_decode_bf16", 1, 0), ("csa_decode_1m_mixed", 2, 1)])
def test_query_norm_rope_and_output_turn(orc, cfg_name, B, splits):
    cfg, x = _case(cfg_name, B, 700 if cfg_name.startswith("hca") else 2000, seed=31)
    H, c = cfg["n_h"], cfg["dim"]
    gw = torch.randn(c, generator=torch.Generator().manual_seed(5)) * 0.5 + 1.0
    gd = gw.to(DEV)
    opt = csa.mqa_options(splits=splits, q_norm_g=gd, q_norm_eps=1e-6, q_rope_dims=64, out_rope_dims=64)
    out = _run(cfg, x, opt)
    torch.cuda.synchronize()
    csa.check_device_status()
    t = f64(x["q_pos"])[:, :, None]
    Qn = orc.rope_tail(orc.rmsnorm(f64(x["Q"]), f64(gw), 1e-6), t, rope_dims=64)
    want = orc.rope_tail(_oracle(orc, cfg, x, Q=Qn), -t, rope_dims=64)
    assert_close(f64(out), want, atol=2e-2, what=f"{cfg_name}: fused norm + rope")
    # the fused prologue gives the bytes of csa_rmsnorm_rope followed by the plain call
    Q2 = csa.rmsnorm_rope(x["Q"].to(DEV).reshape(-1, c), x["q_pos"].to(DEV).reshape(-1), g=gd, eps=1e-6,
                          rows_per_pos=H, rope_dims=64).reshape(x["Q"].shape)
    x2 = dict(x)
    x2["Q"] = Q2.cpu()
    plain = _run(cfg, x2, csa.mqa_options(splits=splits) if splits else None)
    fused = _run(cfg, x, csa.mqa_options(splits=splits, q_norm_g=gd, q_norm_eps=1e-6, q_rope_dims=64))
    torch.cuda.synchronize()
    assert torch.equal(plain, fused)


def test_options_rejected_off_the_tensor_core_path():
    cfg, x = _case("tiny_prefill_f32", 1, 64, T=4, q0=100)
    with pytest.raises(csa.CsaError) as e:
        _run(cfg, x, csa.mqa_options(q_rope_dims=64))
    assert e.value.status == 2  # CSA_ERR_UNSUPPORTED
