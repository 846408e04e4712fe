"""Benchmark of the CSA / HCA decode (and prefill) hot path on B200.

One step = one pass of the whole hot path over one batch:
  csa_* workloads: compress the block closed by the newest token (KV entry and
  indexer key) -> csa_index_topk -> csa_sparse_mqa;
  hca_decode_bf16: compress the closed 128-token block -> hca_dense_mqa.
Default workload: "csa_decode_1m_mixed" (4 requests x 1,048,576 tokens,
262,144 entries each, NVFP4 indexer, FP8/BF16 KV, top-k 1024, 128 heads).

Timing: W warm-up steps, then K timed steps between a barrier + synchronize.
Before every step a 256 MiB buffer is written and then read to flush L2
(outside the step's CUDA events; the read leaves no dirty lines behind); each step is bracketed by CUDA events on the launching stream,
and the dominant kernel call (the indexer) by its own events.  Multi-GPU: one
process per GPU, each rank runs its own independent requests (weak scaling,
no collective on the data path); the step time is the max over ranks.

`--impl reference` times the float64 CPU oracle (the reference for this
method) on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from compressed_sparse_attention_hca_b200 import workloads as W  # noqa: E402

METRIC = "CSA decode query-tokens/s at 1M ctx on 1 B200; % of HBM roofline (GB/s)"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ------------------------------------------------------------------ workload

class Step:
    """Device-resident inputs and outputs of one hot-path step."""

    def __init__(self, name: str, device, seed_offset: int = 0):
        from compressed_sparse_attention_hca_b200 import csa
        self.csa = csa
        self.name = name
        self.cfg = cfg = dict(W.CONFIGS[name])
        cfg["seed"] += 1000 * seed_offset
        self.dev = device
        self.kind = cfg["kind"]
        x = W.attention_inputs(cfg, device)
        self.x = x
        m, c = cfg["m"], cfg["dim"]
        self.scale = 1.0 / math.sqrt(c)
        B, T, E = x["B"], x["T"], x["E"]
        g = W.generator(cfg["seed"] + 17, device)
        # newest tokens: the block closed by the last query token (decode), or
        # every new token of the chunk (prefill)
        if self.kind == "csa_prefill":
            # the chunk's blocks, plus the block before it (overlap) when there is one
            n_new = T
            self.e0 = x["q0"] // m
            self.tok0 = max(0, x["q0"] - m)
            rows = n_new + (x["q0"] - self.tok0)
        else:
            n_new = m
            self.tok0 = E * m - (2 * m if self.kind.startswith("csa") else m)
            self.e0 = E - 1
            rows = n_new + (m if self.kind.startswith("csa") else 0)
        overlap = self.kind.startswith("csa")
        self.n_out = n_new // m if self.kind == "csa_prefill" else 1
        self.tok = W.compress_inputs(g, B, rows, c, m, overlap, torch.bfloat16, c_std=cfg["kv_std"],
                                     device=device)
        if overlap:
            dI = cfg["dI"]
            self.itok = W.compress_inputs(g, B, rows, dI, m, True, torch.bfloat16, device=device)
        self.idx = torch.empty(B, T, cfg.get("k", 1), device=device, dtype=torch.int32)
        self.O = torch.empty_like(x["Q"])
        self.ws_idx = None
        self.ws_mqa = None
        kv_dt = cfg["kv_dt"]
        if overlap:
            idt = cfg["idx_dt"]
            H = cfg["n_hI"]
            self.ws_idx = torch.zeros(csa.index_topk_workspace_size(B, T, E, cfg["k"], H, cfg["dI"], idt),
                                      device=device, dtype=torch.uint8)
            self.ws_mqa = torch.zeros(csa.sparse_mqa_workspace_size(B, T, cfg["n_h"], c, cfg["k"],
                                                                    cfg["window"], cfg["q_dt"], kv_dt),
                                      device=device, dtype=torch.uint8)
        else:
            self.ws_mqa = torch.zeros(csa.hca_dense_mqa_workspace_size(B, T, cfg["n_h"], c, E, cfg["window"],
                                                                       cfg["q_dt"], kv_dt),
                                      device=device, dtype=torch.uint8)
        self.launches = 0

    def _kv_job(self):
        """The step's KV-cache compression as a job (built per call: it holds
        the tensors' current addresses)."""
        csa, x, cfg, t = self.csa, self.x, self.cfg, self.tok
        return csa.compress_job(t["Ca"], t["Za"], t["Ba"], cfg["m"], t["Cb"], t["Zb"], t["Bb"], tok0=self.tok0,
                                e0=self.e0, n_out=self.n_out, out=x["entries"], out_dt=cfg["kv_dt"])

    def attend(self):
        csa, x, cfg = self.csa, self.x, self.cfg
        if self.kind.startswith("csa"):
            csa.sparse_mqa(x["Q"], x["entries"], self.idx, x["win"], x["win_start"], x["q_pos"], cfg["window"],
                           cfg["m"], x["sink"], self.scale, kv_dt=cfg["kv_dt"], O=self.O, ws=self.ws_mqa)
        else:
            csa.hca_dense_mqa(x["Q"], x["entries"], x["win"], x["win_start"], x["q_pos"], cfg["window"],
                              cfg["m"], x["sink"], self.scale, kv_dt=cfg["kv_dt"], O=self.O, ws=self.ws_mqa,
                              options=csa.mqa_options(compress=self._kv_job()))
        return csa.last_launch_count()

    def compress_index(self):
        """The step's compressions (index key and KV entry) fused with the
        indexer call: one launch on the tensor-core path."""
        csa, x, cfg, it, t = self.csa, self.x, self.cfg, self.itok, self.tok
        m = cfg["m"]
        keys = csa.compress_job(it["Ca"], it["Za"], it["Ba"], m, it["Cb"], it["Zb"], it["Bb"], tok0=self.tok0,
                                e0=self.e0, n_out=self.n_out, out=x["KI"], out_sf=x.get("KI_sf"),
                                out_dt=cfg["idx_dt"])
        kv = csa.compress_job(t["Ca"], t["Za"], t["Ba"], m, t["Cb"], t["Zb"], t["Bb"], tok0=self.tok0, e0=self.e0,
                              n_out=self.n_out, out=x["entries"], out_dt=cfg["kv_dt"])
        csa.compress_index_topk(keys, x["qI"], x["wI"], x["KI"], x["q_pos"], m, cfg["k"], extra_job=kv,
                                dt=cfg["idx_dt"], qI_sf=x.get("qI_sf"), KI_sf=x.get("KI_sf"), idx_out=self.idx,
                                ws=self.ws_idx)
        return csa.last_launch_count()

    def run(self, ev=None):
        """One step; ev = (start, after_compress, after_index, end) CUDA events
        (any of them may be None).

        CSA: both compressions (index key, KV entry) run inside the indexer
        call, then attention.  HCA: one dense attention call that launches the
        KV-cache compression first."""
        s = torch.cuda.current_stream()
        if ev and ev[0] is not None:
            ev[0].record(s)
        n = 0
        csa_kind = self.kind.startswith("csa")
        if ev and ev[1] is not None:
            ev[1].record(s)
        if csa_kind:
            n += self.compress_index()
        if ev and ev[2] is not None:
            ev[2].record(s)
        n += self.attend()
        if ev and ev[3] is not None:
            ev[3].record(s)
        self.launches = n

    # per-step host<->device traffic for the end-to-end measurement: the new
    # tokens' projections, the queries (attention + indexer) and the output;
    # the compressed caches and the window are device-resident state.
    def step_inputs(self):
        x = self.x
        ts = [self.tok[k] for k in ("Ca", "Za", "Cb", "Zb") if self.tok[k] is not None]
        if self.kind.startswith("csa"):
            ts += [self.itok[k] for k in ("Ca", "Za", "Cb", "Zb")]
            ts += [x["qI"], x["wI"]] + ([x["qI_sf"]] if "qI_sf" in x else [])
        ts += [x["Q"], x["q_pos"]]
        return ts

    def algorithmic_bytes(self):
        """Minimum HBM bytes of one step (each byte the step must read or write once)."""
        x, cfg = self.x, self.cfg
        B, T, E = x["B"], x["T"], x["E"]
        c, m = cfg["dim"], cfg["m"]
        kvb = W.row_bytes(cfg["kv_dt"], c)
        nb = lambda t: t.numel() * t.element_size()  # noqa: E731
        comp = sum(nb(self.tok[k]) for k in ("Ca", "Za", "Cb", "Zb") if self.tok[k] is not None)
        comp += nb(self.tok["Ba"]) + (nb(self.tok["Bb"]) if self.tok["Bb"] is not None else 0)
        comp += B * self.n_out * kvb
        if self.kind.startswith("csa"):
            comp += sum(nb(self.itok[k]) for k in ("Ca", "Za", "Cb", "Zb"))
            comp += B * self.n_out * (nb(x["KI"][0, 0]) + (cfg["dI"] // 16 if "KI_sf" in x else 0))
        idx_bytes = self.index_bytes() if self.kind.startswith("csa") else 0
        if self.kind.startswith("csa"):
            if self.kind == "csa_prefill":
                # every entry and window row at least once
                att = B * (min(E, T * cfg["k"]) + x["Lw"]) * kvb + nb(self.idx)
            else:
                att = B * T * (cfg["k"] + cfg["window"]) * kvb + nb(self.idx)
        else:
            att = B * (E + cfg["window"]) * kvb
        att += nb(x["Q"]) + nb(self.O)
        return comp + idx_bytes + att

    def index_bytes(self):
        """Algorithmic bytes of one indexer call: every key once, queries, weights, idx."""
        x = self.x
        nb = lambda t: t.numel() * t.element_size()  # noqa: E731
        b = nb(x["KI"]) + nb(x["qI"]) + nb(x["wI"]) + nb(self.idx)
        if "KI_sf" in x:
            b += nb(x["KI_sf"]) + nb(x["qI_sf"])
        return b

    def index_flops(self):
        x, cfg = self.x, self.cfg
        tot = 0
        qp = x["q_pos"].cpu()
        for b in range(x["B"]):
            for t in range(x["T"]):
                tot += min(x["E"], (int(qp[b, t]) + 1) // cfg["m"])
        return 2.0 * tot * cfg["n_hI"] * cfg["dI"]


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# dominant kernel, measured by an ncu capture of that kernel on the same
# workload.  A change to that kernel makes the figure stale: it is then removed
# until the next capture.
NCU_TRAFFIC = {"csa_decode_1m_mixed": 77_410_000,   # 75.76 MB read + 1.65 MB written (ncu, 2 decimals)
               "csa_decode_bf16": 135_100_000}      # 134.97 MB read + 0.13 MB written


def max_over_ranks(x, dist, device):
    """The largest x of all ranks (the job's time is its slowest rank's)."""
    if not dist:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, units_per_rank_step, ms_per_step):
    """Whole-job throughput: every rank processes its own units each step."""
    return world * units_per_rank_step / (ms_per_step / 1e3)


def l2_flush_buffer(device):
    return torch.empty(256 * 1024 * 1024 // 4, device=device, dtype=torch.float32)


def flush_l2(buf):
    """Writes then reads a buffer twice the L2 size: the write evicts the step's
    data, the read evicts (and writes back) the dirty lines of the write, so
    the next step starts with a cold and clean L2 and pays no write-back that
    belongs to the flush."""
    buf.zero_()
    return buf.sum()


DOM_TIMING = ("avg_launch_ms: (graph of 16 x (L2 flush, call) - graph of 16 x L2 flush) / 16, "
              "median of 5 replays each; the phase graph's event nodes add ~2.5 us per phase")


def launch_ms_differential(fn, flush, reps=16, rounds=5):
    """Mean device time one call of fn adds to a graph that starts it from a
    cold, clean L2, without the latency of event nodes between the phases: a
    graph of reps x (L2 flush, fn) and a graph of reps x (L2 flush), each timed
    whole with events around its replay; the difference of their medians over
    reps."""
    g1, g0 = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1):
        for _ in range(reps):
            flush_l2(flush)
            fn()
    with torch.cuda.graph(g0):
        for _ in range(reps):
            flush_l2(flush)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def once(g):
        e0.record()
        g.replay()
        e1.record()
        e1.synchronize()
        return e0.elapsed_time(e1)

    g1.replay()
    g0.replay()
    torch.cuda.synchronize()
    t1 = statistics.median([once(g1) for _ in range(rounds)])
    t0 = statistics.median([once(g0) for _ in range(rounds)])
    del g1, g0
    return (t1 - t0) / reps


# ------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                       "-lms", "20", "-i", str(gpu_index)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        # nvidia-smi takes a moment to start: wait for its first sample so the
        # samples cover the timed region
        t0 = time.time()
        while self.p is not None and time.time() - t0 < 5.0:
            self.f.flush()
            if os.path.getsize(self.f.name) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.seek(0)
        rows = [ln.split(", ") for ln in self.f.read().strip().splitlines() if ln.count(",") >= 8]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.strip() == "Active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ CPU side

def oracle_unit(name: str, sample_entries=None, seed_offset=0):
    """Prepares the oracle's run over one request of workload `name` (a bounded
    sample) and returns (run, description).  run() executes it and returns
    (measured seconds, extrapolated seconds): with sample_entries set, the
    indexer runs on that many entries and its time is scaled to all entries
    of the request (the indexer is linear in the entry count); compression and
    attention run in full."""
    import numpy as np

    import oracle as orc
    cfg = dict(W.CONFIGS[name])
    cfg["seed"] += 1000 * seed_offset
    E_full = cfg["ctx"] // cfg["m"]
    E = E_full if sample_entries is None else min(E_full, sample_entries)
    x = W.attention_inputs(cfg, "cpu", batch=1, n_q=1, n_entries=E_full if cfg["kind"] == "hca_decode" else E,
                           ctx=cfg["ctx"] if cfg["kind"] == "hca_decode" else E * cfg["m"])
    m, c = cfg["m"], cfg["dim"]

    def f64(t):
        return t.detach().cpu().to(torch.float64).numpy()

    def raw(t):
        t = t.detach().cpu().contiguous()
        return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()

    g = W.generator(cfg["seed"] + 17)
    overlap = cfg["kind"].startswith("csa")
    tok = W.compress_inputs(g, 1, 2 * m if overlap else m, c, m, overlap, torch.bfloat16, c_std=cfg["kv_std"])
    kw = dict(Cb=f64(tok["Cb"][0]), Zb=f64(tok["Zb"][0]), Bb=f64(tok["Bb"])) if overlap else {}
    comp_in = (f64(tok["Ca"][0]), f64(tok["Za"][0]), f64(tok["Ba"]))
    scale = 1.0 / math.sqrt(c)
    att = dict(Q=f64(x["Q"]), entries=raw(x["entries"]), win=raw(x["win"]), win_start=raw(x["win_start"]),
               q_pos=raw(x["q_pos"]), sink=f64(x["sink"]))
    idx_in = None
    if overlap:
        dI = cfg["dI"]
        if cfg["idx_dt"] == W.NVFP4:
            idx_in = dict(qI=raw(x["qI"]).reshape(-1, dI // 2), qsf=raw(x["qI_sf"]).reshape(-1, dI // 16),
                          KI=raw(x["KI"][0]), ksf=raw(x["KI_sf"][0]))
        else:
            idx_in = dict(q=f64(x["qI"]), K=f64(x["KI"]))
        idx_in["wI"] = f64(x["wI"])

    def run():
        t0 = time.perf_counter()
        orc.compress(*comp_in, m, tok0=(E - 2) * m if overlap else (E - 1) * m, e0=E - 1, n_out=1, **kw)
        t_comp = time.perf_counter() - t0
        t_idx = 0.0
        if overlap:
            t0 = time.perf_counter()
            if "KI" in idx_in:
                dI = cfg["dI"]
                q = orc.decode_rows(idx_in["qI"], orc.NVFP4, dI, sf=idx_in["qsf"]).reshape(1, 1, -1, dI)
                K = orc.decode_rows(idx_in["KI"], orc.NVFP4, dI, sf=idx_in["ksf"], sf_blocked=True)[None]
            else:
                q, K = idx_in["q"], idx_in["K"]
            _, idx = orc.index_topk(q, idx_in["wI"], K, att["q_pos"], m, cfg["k"], want_scores=False)
            t_idx = time.perf_counter() - t0
            t0 = time.perf_counter()
            orc.sparse_mqa(att["Q"], att["entries"], cfg["kv_dt"], idx, att["win"], att["win_start"], att["q_pos"],
                           cfg["window"], m, att["sink"], scale)
        else:
            t0 = time.perf_counter()
            orc.hca_dense_mqa(att["Q"], att["entries"], cfg["kv_dt"], att["win"], att["win_start"], att["q_pos"],
                              cfg["window"], m, att["sink"], scale)
        t_att = time.perf_counter() - t0
        return t_comp + t_idx + t_att, t_comp + t_idx * (E_full / E) + t_att

    desc = (f"oracle (float64) on 1 request of {name} per unit: compress 1 block, "
            + (f"indexer over {E} of {E_full} entries, its time scaled x{E_full / E:.1f}, " if overlap else "")
            + ("top-k + sparse MQA" if overlap else "dense MQA over all entries"))
    return run, desc, E < E_full


def oracle_throughput(name: str, threads: int, sample_entries=None, seed0=0):
    """Runs `threads` independent one-request units concurrently on host
    threads (the oracle's C code releases the GIL), after preparing their
    inputs.  Returns (query tokens/s, measured wall seconds, desc,
    extrapolated): the units start together, so the job's time is the
    slowest unit's (extrapolated) time."""
    from concurrent.futures import ThreadPoolExecutor
    units = [oracle_unit(name, sample_entries, seed0 + i) for i in range(threads)]
    t0 = time.perf_counter()
    with ThreadPoolExecutor(max_workers=threads) as ex:
        res = list(ex.map(lambda u: u[0](), units))
    wall = time.perf_counter() - t0
    slowest = max(r[1] for r in res)
    return threads / slowest, wall, units[0][1], units[0][2]


def host_threads():
    """Host threads for the all-cores oracle leg (at most 32, so that the
    prepared inputs stay a few GB)."""
    return max(1, min(32, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()))


def cpu_baseline_record(name: str, sample_entries, threads: int):
    """The oracle single-threaded and on `threads` host threads."""
    v1, w1, desc, ext = oracle_throughput(name, 1, sample_entries, seed0=0)
    vn, wn, _, _ = oracle_throughput(name, threads, sample_entries, seed0=100)
    return {"value": vn, "unit": "query-tokens/s", "cores": threads, "kind": "oracle",
            "sample": desc + f"; {threads} independent requests on {threads} host threads",
            "extrapolated": ext, "measured_wall_s": wn,
            "single_thread": {"value": v1, "cores": 1, "measured_wall_s": w1}}


def reference_arm(args):
    """`--impl reference`: the oracle on the host cores, same metric and workload.
    Each step runs the step's requests concurrently, one host thread each."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    name = args.config
    cfg = W.CONFIGS[name]
    sample = 8192 if cfg["kind"].startswith("csa") else None
    threads = min(host_threads(), cfg["batch"])
    per_step, walls = [], []
    for i in range(args.warmup + args.steps):
        v, wall, desc, ext = oracle_throughput(name, threads, sample, seed0=1000 * i)
        if i >= args.warmup:
            per_step.append(threads / v)  # seconds for `threads` query tokens
            walls.append(wall)
    step_s = statistics.mean(per_step) * cfg["batch"] / threads
    value = cfg["batch"] / step_s
    line = {
        "impl": "reference", "metric": METRIC if name == "csa_decode_1m_mixed" else f"{name} query-tokens/s",
        "value": value, "unit": "query-tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": name},
        "extrapolated": ext,
        "measured_ms_per_step": statistics.mean(walls) * 1e3,
        "note": ("ms_per_step and value scale the indexer's sampled time to the full entry count; "
                 "measured_ms_per_step is the wall time of one sampled step") if ext else "measured in full",
        "cpu_baseline": {"value": value, "unit": "query-tokens/s", "cores": threads, "kind": "oracle",
                         "sample": desc + f"; the step's {cfg['batch']} requests on {threads} host threads",
                         "extrapolated": ext, "measured_wall_s": sum(walls)},
        "e2e": {"value": value, "unit": "query-tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------- grouped output projection

def out_proj_bench(args):
    """`--op out_proj`: the grouped output projection ("DeepSeek-V4 内部机制"
    1.2 Step 3) on V4-Pro's shape (n_h = 128, c = 512, g = 16, d_g = 1024,
    d = 7168) for `--tokens` tokens, L2 flushed before every call.  Decode
    (few tokens) reads the weights once: HBM-bound; prefill is tensor-bound."""
    from compressed_sparse_attention_hca_b200 import csa
    csa.load()
    dev = torch.device("cuda", 0)
    s = W.OUT_PROJ_V4_PRO
    T = args.tokens
    O, Wg, Wo = (t.to(dev) for t in W.out_proj_inputs(W.generator(1), T, s["n_h"], s["c"], s["g"], s["d_g"],
                                                         s["d"]))
    ws = torch.zeros(csa.grouped_out_proj_workspace_size(T, **s), dtype=torch.uint8, device=dev)
    Y = torch.empty(T, s["d"], dtype=torch.bfloat16, device=dev)
    flush = l2_flush_buffer(dev)
    for _ in range(args.warmup):
        csa.grouped_out_proj(O, Wg, Wo, out=Y, ws=ws)
    torch.cuda.synchronize()
    clk = ClockSampler(0)
    times = []
    for _ in range(args.steps):
        flush_l2(flush)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        csa.grouped_out_proj(O, Wg, Wo, out=Y, ws=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    clocks = clk.stop()
    csa.check_device_status()
    ms = statistics.mean(times)
    peaks = load_peaks()
    weights = (Wg.numel() + Wo.numel()) * 2
    byts = weights + (O.numel() + Y.numel()) * 2 + 2 * T * s["g"] * s["d_g"] * 2  # + Z written and read
    flops = 2.0 * T * (Wg.numel() + Wo.numel())
    hbm = byts / (ms / 1e3) / 1e9
    tfl = flops / (ms / 1e3) / 1e12
    tensor = flops / peaks["bf16_tflops"] / 1e12 > byts / peaks["hbm_gbs"] / 1e9
    roof = ({"bound": "tensor", "achieved": tfl, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
             "frac": tfl / peaks["bf16_tflops"]} if tensor else
            {"bound": "hbm", "achieved": hbm, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": hbm / peaks["hbm_gbs"]})
    roof.update({"traffic": None, "algorithmic_bytes": byts, "flops": flops, "note": f"peak {peaks['source']}"})
    line = {"metric": "grouped output projection tokens/s (V4-Pro shape)", "value": T / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16, fp32 accumulate",
            "data": "synthetic",
            "config": {"workload": f"out_proj_v4pro_T{T}", "tokens": T, **s,
                       "l2": "flushed before every call (256 MiB write then read)"},
            "plan": csa.grouped_out_proj_plan(T, **s), "roofline": roof, "gpu_launches": 2 * args.steps,
            "clocks": clocks}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU side

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="csa_decode_1m_mixed", choices=sorted(W.CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="step", choices=["step", "out_proj"],
                    help="step: the hot-path step of --config; out_proj: the grouped output projection")
    ap.add_argument("--tokens", type=int, default=4, help="tokens of --op out_proj")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.op == "out_proj":
        out_proj_bench(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from compressed_sparse_attention_hca_b200 import csa
    csa.load()
    peaks = load_peaks()
    step = Step(args.config, dev, seed_offset=rank)
    flush = l2_flush_buffer(dev)
    for _ in range(args.warmup):
        flush_l2(flush)
        step.run()
    torch.cuda.synchronize()

    # The step runs as one CUDA graph (captured once, replayed every step): a
    # decode step is a handful of short kernels, and launching them one by one
    # from Python leaves the GPU idle between them.  Event record nodes inside
    # the graph time the step and its phases on the device.
    gev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step.run((gev[0], None, None, gev[3]))
    launches_per_step = step.launches
    # a second graph with event nodes between the phases times the phases
    pev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)]
    pgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(pgraph):
        step.run(pev)
    for _ in range(3):
        flush_l2(flush)
        graph.replay()
        flush_l2(flush)
        pgraph.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    step_ms = []
    for i in range(args.steps):
        flush_l2(flush)
        graph.replay()
        gev[3].synchronize()
        step_ms.append(gev[0].elapsed_time(gev[3]))
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clk = clocks.stop()
    evs_ms = []
    for i in range(min(args.steps, 100)):
        flush_l2(flush)
        pgraph.replay()
        pev[3].synchronize()
        evs_ms.append([pev[0].elapsed_time(pev[j]) for j in (1, 2, 3)])
    launches = launches_per_step * args.steps
    idx_ms = [e[1] - e[0] for e in evs_ms]
    # the dominant call's own duration inside a graph, L2 cold before it
    dom_ms = launch_ms_differential(step.compress_index if step.kind.startswith("csa") else step.attend, flush)
    eager = measure_eager(step, args, flush)
    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_per_step = total_ms / args.steps
    x = step.x
    tokens_per_step = x["B"] * x["T"]
    value = job_throughput(world, tokens_per_step, ms_per_step)

    # dominant kernel roofline
    kind = step.kind
    if kind.startswith("csa"):
        idx_avg_ms = dom_ms
        if kind == "csa_prefill":
            peak = peaks.get("bf16_tflops", PEAKS_FALLBACK["bf16_tflops"])
            ach = step.index_flops() / (idx_avg_ms / 1e3) / 1e12
            roof = {"kernel": "csa_index_topk", "bound": "tensor", "achieved": ach, "peak": peak,
                    "unit": "TFLOP/s", "frac": ach / peak, "traffic": None, "avg_launch_ms": idx_avg_ms,
                    "note": f"bf16 dense peak, {peaks['source']}", "timing": DOM_TIMING}
        else:
            peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
            ach = step.index_bytes() / (idx_avg_ms / 1e3) / 1e9
            roof = {"kernel": "csa_index_topk", "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak, "traffic": NCU_TRAFFIC.get(args.config),
                    "algorithmic_bytes": step.index_bytes(),
                    "avg_launch_ms": idx_avg_ms, "note": f"HBM copy peak, {peaks['source']}",
                    "timing": DOM_TIMING}
    else:
        att_ms = dom_ms
        peak = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
        b = step.algorithmic_bytes()
        ach = b / (att_ms / 1e3) / 1e9
        roof = {"kernel": "hca_dense_mqa", "bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                "frac": ach / peak, "traffic": None, "avg_launch_ms": att_ms,
                "note": f"HBM copy peak, {peaks['source']}", "timing": DOM_TIMING}
    step_bytes = step.algorithmic_bytes()
    step_gbs = step_bytes / (ms_per_step / 1e3) / 1e9
    # mean device time of each phase of the step (same events as above)
    phases = {"compress": statistics.mean([e[0] for e in evs_ms]),
              "index_topk": statistics.mean(idx_ms),
              "attention": statistics.mean([e[2] - e[1] for e in evs_ms])}

    # end to end through the public API with host buffers
    e2e = measure_e2e(step, args, flush, dev, dist, world)

    line = {
        "metric": METRIC if args.config == "csa_decode_1m_mixed" else f"{args.config} query-tokens/s",
        "value": value, "unit": "query-tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype_label(step.cfg), "data": "synthetic",
        "config": {"workload": args.config, "batch_per_gpu": x["B"], "ctx": step.cfg["ctx"],
                   "entries_per_request": x["E"], "query_tokens_per_request": x["T"],
                   "top_k": step.cfg.get("k"), "n_heads": step.cfg["n_h"], "window": step.cfg["window"],
                   "parallelism": f"replicas x{world} (independent requests per GPU)",
                   "l2": "flushed before every step (256 MiB write then read, outside the step events)"},
        "roofline": roof,
        "step_hbm": {"algorithmic_bytes": step_bytes, "achieved_gbs": step_gbs,
                     "frac": step_gbs / peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])},
        "phases_ms": phases,
        "phases_note": ("index_topk includes both compressions (index key and KV entry, fused into the "
                        "indexer call), so the compress phase is empty" if kind.startswith("csa")
                        else "the dense attention call launches the KV-cache compression first, so the "
                        "compress phase is empty and attention includes it"),
        "phases_timing": "a second graph with event nodes between the phases (each node adds latency)",
        "launch": "one CUDA graph per step",
        "eager": eager,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_record(args.config, 65536 if kind.startswith("csa") else None,
                                                   host_threads())
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def dtype_label(cfg):
    names = {W.F32: "f32", W.BF16: "bf16", W.FP8MIX: "fp8e4m3+bf16", W.NVFP4: "nvfp4"}
    parts = [f"kv {names[cfg['kv_dt']]}"]
    if "idx_dt" in cfg:
        parts.insert(0, f"indexer {names[cfg['idx_dt']]}")
    return ", ".join(parts) + ", fp32 accumulate"


def measure_eager(step, args, flush):
    """The same step launched call by call from Python (no graph): device time
    per step and per phase, host launch gaps included."""
    n = max(3, min(args.steps, 100))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    for i in range(n):
        flush_l2(flush)
        step.run(evs[i])
    torch.cuda.synchronize()
    return {"ms_per_step": statistics.mean([e[0].elapsed_time(e[3]) for e in evs]),
            "phases_ms": {"compress": statistics.mean([e[0].elapsed_time(e[1]) for e in evs]),
                          "index_topk": statistics.mean([e[1].elapsed_time(e[2]) for e in evs]),
                          "attention": statistics.mean([e[2].elapsed_time(e[3]) for e in evs])}}


def measure_e2e(step, args, flush, dev, dist, world):
    """Same step through the public API with host buffers: each step copies its
    inputs from pinned host memory and reads the output back (all inside the
    step's graph)."""
    ins = step.step_inputs()
    # The step's inputs live in one device staging buffer (each input tensor
    # becomes a view of it, 256-byte aligned), filled every step by one copy
    # from one pinned host buffer: a serving loop packs a step's inputs the
    # same way instead of issuing one small copy per tensor.
    offs, size = [], 0
    for t in ins:
        assert t.is_contiguous()
        size = (size + 255) // 256 * 256
        offs.append(size)
        size += t.numel() * t.element_size()
    dev_buf = torch.empty(size, dtype=torch.uint8, device=dev)
    host_buf = torch.empty(size, dtype=torch.uint8, pin_memory=True)
    for t, o in zip(ins, offs):
        nb = t.numel() * t.element_size()
        host_buf[o:o + nb].copy_(t.detach().reshape(-1).view(torch.uint8).cpu())
        t.set_(dev_buf.untyped_storage(), o // t.element_size(), t.shape, t.stride())
    dev_buf.copy_(host_buf)
    out_host = torch.empty(step.O.shape, dtype=step.O.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in ins)
    d2h = out_host.numel() * out_host.element_size()
    n = max(3, min(args.steps, 100))
    # one graph: the pinned host -> device copy of the step's inputs, the step,
    # and the device -> host copy of its output, timed by event nodes
    e0, e1 = (torch.cuda.Event(enable_timing=True, external=True) for _ in range(2))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        s = torch.cuda.current_stream()
        e0.record(s)
        dev_buf.copy_(host_buf, non_blocking=True)
        step.run()
        out_host.copy_(step.O, non_blocking=True)
        e1.record(s)
    for _ in range(2):
        flush_l2(flush)
        graph.replay()
    torch.cuda.synchronize()
    total = 0.0
    for i in range(n):
        flush_l2(flush)
        graph.replay()
        e1.synchronize()
        total += e0.elapsed_time(e1)
    total = max_over_ranks(total, dist, dev)
    ms = total / n
    x = step.x
    return {"value": job_throughput(world, x["B"] * x["T"], ms), "unit": "query-tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms}


if __name__ == "__main__":
    main()
