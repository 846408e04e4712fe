"""An HCA decode step in one call: hca_dense_mqa with the step's compression
job as an option ("DeepSeek-V4 内部机制" 1.3: the closed block of m' = 128
tokens becomes the newest entry, then every visible entry is attended).

  * the call writes the cache bytes of csa_compress_ex and returns bitwise the
    output of the attention call that follows it (compression, attention and
    split combine launched in order);
  * against the float64 oracle: the new entry within one bf16 rounding (or
    one FP8 step) of orc.compress, the output within 2e-2 of orc.hca_dense_mqa
    over the GPU's cache.
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


def _case(B, E, kv_dt, n_h, seed):
    cfg = dict(W.CONFIGS["hca_decode_bf16"])
    cfg.update(kv_dt=kv_dt, n_h=n_h)
    m = cfg["m"]
    x = W.attention_inputs(cfg, "cpu", batch=B, ctx=E * m, n_q=1, q0=m * E - 1, n_entries=E, seed=seed)
    tok = W.compress_inputs(W.generator(seed + 1), B, m, cfg["dim"], m, False, torch.bfloat16, c_std=cfg["kv_std"])
    return cfg, x, tok


def _run(cfg, x, tok, fused, ws=None):
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    t = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in tok.items()}
    m, E = cfg["m"], x["entries"].shape[1]
    entries = g["entries"].clone()
    job = csa.compress_job(t["Ca"], t["Za"], t["Ba"], m, tok0=m * (E - 1), e0=E - 1, n_out=1, out=entries,
                           out_dt=cfg["kv_dt"])
    scale = 1.0 / math.sqrt(cfg["dim"])
    if fused:
        O = csa.hca_dense_mqa(g["Q"], entries, g["win"], g["win_start"], g["q_pos"], cfg["window"], m, g["sink"],
                              scale, kv_dt=cfg["kv_dt"], options=csa.mqa_options(compress=job), ws=ws)
    else:
        csa.compress_ex(job, x["Q"].shape[0])
        O = csa.hca_dense_mqa(g["Q"], entries, g["win"], g["win_start"], g["q_pos"], cfg["window"], m, g["sink"],
                              scale, kv_dt=cfg["kv_dt"])
    launches = csa.last_launch_count()
    torch.cuda.synchronize()
    csa.check_device_status()
    return O, entries, launches


@pytest.mark.parametrize("B,E,kv_dt", [
    (8, 8192, csa.BF16),       # the benchmark's shape: 18 splits per query
    (2, 1500, csa.BF16),       # 13 splits per query
    (3, 1200, csa.KV_FP8MIX),  # FP8MIX entries
])
def test_fused_equals_separate_and_oracle(orc, B, E, kv_dt):
    cfg, x, tok = _case(B, E, kv_dt, 64, seed=E + B)
    Of, ent_f, n_f = _run(cfg, x, tok, True)
    Os, ent_s, _ = _run(cfg, x, tok, False)
    assert n_f == 3, f"the step call launched {n_f} kernels (compression, attention, combine expected)"
    assert torch.equal(ent_f, ent_s), "the step call wrote other cache bytes"
    assert torch.equal(Of, Os), "step call and separate calls differ"
    m = cfg["m"]
    want_e = np.stack([orc.compress(f64(tok["Ca"][b]), f64(tok["Za"][b]), f64(tok["Ba"]), m, tok0=m * (E - 1),
                                    e0=E - 1, n_out=1)[0] for b in range(B)])
    got_e = orc.decode_rows(raw(ent_f[:, E - 1]), kv_dt, cfg["dim"]) if kv_dt == csa.KV_FP8MIX else f64(ent_f[:, E - 1])
    if kv_dt == csa.KV_FP8MIX:
        # one E4M3 step of the value (relative 2^-3) plus one of the block scale; RoPE dims bf16
        assert (np.abs(got_e[:, :448] - want_e[:, :448]) <= 2.0 ** -3 * np.abs(want_e[:, :448]) + 1e-3).all()
        assert_close(got_e[:, 448:], want_e[:, 448:], atol=1e-6, rtol=2.0 ** -8, what="rope dims")
    else:
        assert_close(got_e, want_e, atol=1e-6, rtol=2.0 ** -8, what="new entry")
    scale = 1.0 / math.sqrt(cfg["dim"])
    want = orc.hca_dense_mqa(f64(x["Q"]), raw(ent_f), kv_dt, raw(x["win"]), raw(x["win_start"]), raw(x["q_pos"]),
                             cfg["window"], m, f64(x["sink"]), scale)
    assert_close(f64(Of), want, atol=2e-2, what=f"HCA step B={B} E={E}")


def test_two_head_groups():
    cfg, x, tok = _case(2, 1500, csa.BF16, 128, seed=7)
    Of, ent_f, n_f = _run(cfg, x, tok, True)
    Os, ent_s, _ = _run(cfg, x, tok, False)
    assert n_f == 3
    assert torch.equal(ent_f, ent_s) and torch.equal(Of, Os)
