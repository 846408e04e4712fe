"""csa_index_topk_noalloc: the indexer call for callers that cannot allocate.

Callers such as a plugin inside a host that owns all device memory, or a
serving loop that forbids cudaMalloc after start-up, get their scratch from an
array built into the library.  This test calls that entry point through the C
ABI twice in a row and checks that both calls return exactly what the
workspace-taking csa_index_topk returns for the same inputs (selection is
integer work, so the tolerance is bit-exact), and that a shape needing more
than the built-in 4 MiB is refused before anything is launched.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""
import ctypes

import pytest
import torch

from compressed_sparse_attention_hca_b200 import csa
from compressed_sparse_attention_hca_b200 import workloads as W

pytestmark = pytest.mark.gpu
STATIC_SCRATCH_BYTES = 4 << 20


def _noalloc():
    lib = csa.load()
    fn = lib.csa_index_topk_noalloc
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    fn.restype = i32
    fn.argtypes = [P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P, P]
    return fn


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _inputs(dt, B, T, E, seed):
    g = W.generator(seed)
    H, d = 64, 128
    if dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, T, H), d)
        KI, ksf = W.nvfp4_rows(g, (B, E), d)
        ksf = W.block_scales(ksf, d)
    else:
        qI, qsf = W.normal(g, (B, T, H, d), 1.0, torch.bfloat16), None
        KI, ksf = W.normal(g, (B, E, d), 1.0, torch.bfloat16), None
    wI = W.uniform(g, (B, T, H))
    q_pos = torch.tensor([[4 * E - 1 - 37 * t for t in range(T)]] * B, dtype=torch.int64)
    cuda = lambda t: None if t is None else t.cuda()  # noqa: E731
    return dict(qI=cuda(qI), qI_sf=cuda(qsf), KI=cuda(KI), KI_sf=cuda(ksf), wI=cuda(wI), q_pos=cuda(q_pos),
                H=H, d=d)


@pytest.mark.parametrize("dt,B,T,E,k", [(csa.BF16, 3, 1, 20000, 512), (csa.IDX_NVFP4, 2, 2, 30000, 1024)])
def test_noalloc_matches_workspace_entry_point_twice(dt, B, T, E, k):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    x = _inputs(dt, B, T, E, seed=E)
    need = csa.index_topk_workspace_size(B, T, E, k, x["H"], x["d"], dt)
    assert need <= STATIC_SCRATCH_BYTES
    ref = csa.index_topk(x["qI"], x["wI"], x["KI"], x["q_pos"], 4, k, dt=dt, qI_sf=x["qI_sf"],
                         KI_sf=x["KI_sf"])
    torch.cuda.synchronize()
    fn = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        out = torch.full((B, T, k), -7, device="cuda", dtype=torch.int32)
        st = fn(_p(x["qI"]), _p(x["qI_sf"]), _p(x["wI"]), _p(x["KI"]), _p(x["KI_sf"]), _p(x["q_pos"]), B, T, E,
                4, x["H"], x["d"], k, dt, _p(out), None, stream)
        assert st == 0, csa.load().csa_last_error().decode()
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"call {call}: differs from csa_index_topk"


@pytest.mark.parametrize("merge_first", [True, False])
def test_noalloc_merge_and_cooperative_calls_in_turn(merge_first):
    """A call whose rows select through per-slice candidate lists and a merge
    kernel (two queries per request) and a decode call whose slices select
    cooperatively (counters and histograms) share the built-in array; in
    either order each call returns exactly what csa_index_topk returns."""
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    merge = dict(dt=csa.IDX_NVFP4, B=2, T=2, E=30000, k=1024)
    coop = dict(dt=csa.BF16, B=3, T=1, E=20000, k=512)
    cases = [merge, coop] if merge_first else [coop, merge]
    fn = _noalloc()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for rnd in range(2):
        for c in cases:
            x = _inputs(c["dt"], c["B"], c["T"], c["E"], seed=c["E"] + rnd)
            plan = csa.index_topk_plan(c["B"], c["T"], c["E"], c["k"], x["H"], x["d"], c["dt"])
            assert plan["coop"] == (1 if c is coop else 0) and plan["n_slices"] > 1, plan
            ref = csa.index_topk(x["qI"], x["wI"], x["KI"], x["q_pos"], 4, c["k"], dt=c["dt"], qI_sf=x["qI_sf"],
                                 KI_sf=x["KI_sf"])
            out = torch.full((c["B"], c["T"], c["k"]), -7, device="cuda", dtype=torch.int32)
            st = fn(_p(x["qI"]), _p(x["qI_sf"]), _p(x["wI"]), _p(x["KI"]), _p(x["KI_sf"]), _p(x["q_pos"]), c["B"],
                    c["T"], c["E"], 4, x["H"], x["d"], c["k"], c["dt"], _p(out), None, stream)
            assert st == 0, csa.load().csa_last_error().decode()
            torch.cuda.synchronize()
            assert torch.equal(out, ref), f"round {rnd}, {'merge' if c is merge else 'cooperative'} call differs"


def test_noalloc_rejects_shapes_beyond_static_scratch():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    B, T, E, k, H, d = 512, 1, 262144, 2048, 64, 128
    need = csa.index_topk_workspace_size(B, T, E, k, H, d, csa.BF16)
    assert need > STATIC_SCRATCH_BYTES  # so the call must return before any launch
    small = torch.zeros(64, device="cuda", dtype=torch.float32)
    idx = torch.zeros(64, device="cuda", dtype=torch.int32)
    st = _noalloc()(_p(small), None, _p(small), _p(small), None, _p(small), B, T, E, 4, H, d, k, csa.BF16,
                    _p(idx), None, None)
    assert st == csa.CsaError(1, "").status == 1
    assert "built-in scratch" in csa.load().csa_last_error().decode()
