"""The decode path captured in a CUDA graph and replayed gives exactly the
results of the same calls made one by one (GPU only).

A serving loop replays one captured step per token; every launch of the path
(the workspace memset, the cooperative indexer launch, the attention kernels)
must therefore be capture-safe and take all its inputs from device memory.
"""
import pytest
import torch

from compressed_sparse_attention_hca_b200 import csa
from compressed_sparse_attention_hca_b200 import workloads as W

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("idx_dt,n_h", [(csa.IDX_NVFP4, 16), (csa.BF16, 16), (csa.BF16, 128)])
def test_graph_replay_matches_eager(idx_dt, n_h):
    """n_h = 16 runs the SIMT attention, n_h = 128 the tensor-core attention
    (each with its split combine kernel)."""
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    B, E, k, H, dI, m = 2, 30000, 1024, 64, 128, 4
    g = W.generator(77)
    if idx_dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, 1, H), dI)
        KI, ksf = W.nvfp4_rows(g, (B, E), dI)
        ksf = W.block_scales(ksf, dI)
    else:
        qI, qsf = W.normal(g, (B, 1, H, dI), 1.0, torch.bfloat16), None
        KI, ksf = W.normal(g, (B, E, dI), 1.0, torch.bfloat16), None
    wI = W.uniform(g, (B, 1, H))
    q_pos = torch.tensor([[m * E - 1], [m * E - 777]], dtype=torch.int64)
    c, window = 512, 128
    Q = W.normal(g, (B, 1, n_h, c), 1.0, torch.bfloat16)
    entries = W.normal(g, (B, E, c), 1.0, torch.bfloat16)
    win = W.normal(g, (B, window, c), 1.0, torch.bfloat16)
    win_start = (q_pos[:, 0] - window + 1).clamp(min=0)
    sink = W.normal(g, (n_h,), 1.0, torch.float32)
    dev = "cuda"
    t = {n: (v.to(dev) if v is not None else None) for n, v in dict(
        qI=qI, qsf=qsf, KI=KI, ksf=ksf, wI=wI, q_pos=q_pos, Q=Q, entries=entries, win=win,
        win_start=win_start, sink=sink).items()}
    ws_i = torch.zeros(csa.index_topk_workspace_size(B, 1, E, k, H, dI, idx_dt), dtype=torch.uint8, device=dev)
    ws_a = torch.zeros(csa.sparse_mqa_workspace_size(B, 1, n_h, c, k, window, csa.BF16, csa.BF16),
                       dtype=torch.uint8, device=dev)
    idx = torch.empty(B, 1, k, dtype=torch.int32, device=dev)
    O = torch.empty(B, 1, n_h, c, dtype=torch.bfloat16, device=dev)

    def step():
        csa.index_topk(t["qI"], t["wI"], t["KI"], t["q_pos"], m, k, dt=idx_dt, qI_sf=t["qsf"], KI_sf=t["ksf"],
                       idx_out=idx, ws=ws_i)
        csa.sparse_mqa(t["Q"], t["entries"], idx, t["win"], t["win_start"], t["q_pos"], window, m, t["sink"],
                       c ** -0.5, O=O, ws=ws_a)

    step()
    torch.cuda.synchronize()
    idx_eager, O_eager = idx.clone(), O.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        idx.fill_(-7)
        O.zero_()
        graph.replay()
        torch.cuda.synchronize()
        csa.check_device_status()
        assert torch.equal(idx, idx_eager)
        assert torch.equal(O, O_eager)


@pytest.mark.parametrize("idx_dt", [csa.IDX_NVFP4, csa.BF16])
def test_index_workspace_returns_to_zero(idx_dt):
    """Decode rows split over several CTAs select through counters and
    histograms in the workspace; every call must leave it zero-filled so the
    next call (or graph replay) can use it without clearing it."""
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    B, E, k, H, dI, m = 3, 40000, 1024, 64, 128, 4
    g = W.generator(91)
    if idx_dt == csa.IDX_NVFP4:
        qI, qsf = W.nvfp4_rows(g, (B, 1, H), dI)
        KI, ksf = W.nvfp4_rows(g, (B, E), dI)
        ksf = W.block_scales(ksf, dI)
    else:
        qI, qsf = W.normal(g, (B, 1, H, dI), 1.0, torch.bfloat16), None
        KI, ksf = W.normal(g, (B, E, dI), 1.0, torch.bfloat16), None
    wI = W.uniform(g, (B, 1, H))
    q_pos = torch.tensor([[m * E - 1], [m * E - 1001], [m * 3000]], dtype=torch.int64)
    cuda = lambda v: None if v is None else v.cuda()  # noqa: E731
    ws = torch.zeros(csa.index_topk_workspace_size(B, 1, E, k, H, dI, idx_dt), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        outs.append(csa.index_topk(cuda(qI), cuda(wI), cuda(KI), cuda(q_pos), m, k, dt=idx_dt, qI_sf=cuda(qsf),
                                   KI_sf=cuda(ksf), ws=ws))
        torch.cuda.synchronize()
        csa.check_device_status()
        assert int(ws.count_nonzero()) == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


def test_attention_repeated_calls_identical():
    """The tensor-core attention on a decode batch (split rows, combine
    kernel): repeated calls on the same workspace give the same bytes."""
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    B, E, k, n_h, c, window, m = 2, 3000, 1024, 128, 512, 128, 4
    g = W.generator(93)
    q_pos = torch.tensor([[m * E - 1], [m * E - 501]], dtype=torch.int64).cuda()
    Q = W.normal(g, (B, 1, n_h, c), 1.0, torch.bfloat16).cuda()
    entries = W.fp8mix_rows(g, (B, E), c).cuda()
    win = W.fp8mix_rows(g, (B, window), c).cuda()
    win_start = (q_pos[:, 0] - window + 1).clamp(min=0)
    sink = W.normal(g, (n_h,), 1.0, torch.float32).cuda()
    idx = torch.stack([torch.randperm(E - 200, generator=g)[:k] for _ in range(B)]).view(B, 1, k)
    idx = idx.to(torch.int32).cuda()
    ws = torch.empty(csa.sparse_mqa_workspace_size(B, 1, n_h, c, k, window, csa.BF16, csa.KV_FP8MIX),
                     dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        outs.append(csa.sparse_mqa(Q, entries, idx, win, win_start, q_pos, window, m, sink, c ** -0.5, ws=ws))
        torch.cuda.synchronize()
        csa.check_device_status()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])
