"""Seeded synthetic workloads for the CSA / HCA forward pass.

This module only draws random numbers and lays them out in the library's
storage formats; it contains none of the method's arithmetic (no compression,
no scoring, no selection, no attention, no quantisation rule).  Both the CUDA
path (benchmark, tests) and the float64 oracle (tests) consume what it makes.

Quantised tensors are drawn directly as codes: FP8 E4M3 codes come from
torch's own float8 cast of scaled normal samples, their fp32 block scales are
random positive numbers, and FP4 E2M1 codes and their E4M3 block scales are
drawn from fixed categorical distributions.  The decoded values therefore have
roughly the spread the workloads ask for (about N(0, 1) per element).

Workload shapes follow DeepSeek-V4 as described in "DeepSeek-V4 内部机制"
(sections 1.2-1.5: m = 4, m' = 128, top-k 512 / 1024, 128-token window,
n_h^I = 64 indexer heads of dim 128) and the admirer.cn article (CSA section:
top-k 512 for Flash, 1024 for Pro).
"""
from __future__ import annotations

import math

import torch

F32, BF16, FP8MIX, NVFP4 = 0, 1, 2, 3

# Workloads.  "tiny_prefill_f32" is small enough for the oracle in seconds;
# the others are the decode / prefill shapes timed by the benchmark.
CONFIGS = {
    "tiny_prefill_f32": dict(
        kind="csa_prefill", seed=0, batch=1, ctx=256, n_q=256, m=4, dim=64, n_h=4,
        n_hI=2, dI=32, k=16, window=16, kv_dt=F32, q_dt=F32, idx_dt=F32,
        q_std=1.0 / 8.0, kv_std=1.0, b_std=0.1),
    "csa_decode_bf16": dict(
        kind="csa_decode", seed=2, batch=16, ctx=131072, n_q=1, m=4, dim=512, n_h=64,
        n_hI=64, dI=128, k=512, window=128, kv_dt=BF16, q_dt=BF16, idx_dt=BF16,
        q_std=1.0 / math.sqrt(512), kv_std=1.0 / math.sqrt(512), b_std=0.1),
    "hca_decode_bf16": dict(
        kind="hca_decode", seed=3, batch=8, ctx=1048576, n_q=1, m=128, dim=512, n_h=64,
        window=128, kv_dt=BF16, q_dt=BF16, q_std=1.0 / math.sqrt(512),
        kv_std=1.0 / math.sqrt(512), b_std=0.1),
    "csa_prefill_bf16": dict(
        kind="csa_prefill", seed=4, batch=1, ctx=73728, q0=65536, n_q=8192, m=4, dim=512,
        n_h=64, n_hI=64, dI=128, k=512, window=128, kv_dt=BF16, q_dt=BF16, idx_dt=BF16,
        q_std=1.0, kv_std=1.0, b_std=0.1),
    "csa_decode_1m_mixed": dict(
        kind="csa_decode", seed=5, batch=4, ctx=1048576, n_q=1, m=4, dim=512, n_h=128,
        n_hI=64, dI=128, k=1024, window=128, kv_dt=FP8MIX, q_dt=BF16, idx_dt=NVFP4,
        q_std=1.0 / math.sqrt(512), kv_std=1.0, b_std=0.1),
}


def row_bytes(dt: int, dim: int) -> int:
    """Bytes per row of a storage format (layout only)."""
    if dt == F32:
        return 4 * dim
    if dt == BF16:
        return 2 * dim
    if dt == FP8MIX:
        n8 = dim - 64
        return (n8 + 128 + 4 * (n8 // 64) + 15) // 16 * 16
    if dt == NVFP4:
        return dim // 2
    raise ValueError(dt)


def generator(seed: int, device="cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal(g, shape, std=1.0, dtype=torch.float32, device="cpu"):
    x = torch.randn(*shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def uniform(g, shape, lo=0.0, hi=1.0, device="cpu"):
    return torch.rand(*shape, generator=g, device=device) * (hi - lo) + lo


def rows(g, dt: int, shape, dim: int, std=1.0, device="cpu"):
    """Random rows of format dt with leading shape `shape` (not NVFP4)."""
    if dt == F32:
        return normal(g, (*shape, dim), std, torch.float32, device)
    if dt == BF16:
        return normal(g, (*shape, dim), std, torch.bfloat16, device)
    if dt == FP8MIX:
        return fp8mix_rows(g, shape, dim, std, device)
    raise ValueError(dt)


def fp8mix_rows(g, shape, dim: int, std=1.0, device="cpu"):
    """Random FP8MIX rows: [E4M3 codes | 64 bf16 | fp32 scales | pad] bytes.

    Codes are torch float8 casts of N(0, 64^2) samples (never beyond 448 in
    magnitude after clamping); each 64-element block gets a random scale in
    [0.75, 1.25] * std / 64, so decoded values have about the requested spread.
    """
    n = int(math.prod(shape)) if len(shape) else 1
    n8 = dim - 64
    nb = n8 // 64
    rb = row_bytes(FP8MIX, dim)
    codes = (torch.randn(n, n8, generator=g, device=device) * 64.0).clamp_(-448.0, 448.0)
    codes = codes.to(torch.float8_e4m3fn).view(torch.uint8)
    rope = normal(g, (n, 64), std, torch.bfloat16, device).view(torch.uint8)
    scales = (uniform(g, (n, nb), 0.75, 1.25, device) * (std / 64.0)).to(torch.float32)
    out = torch.zeros(n, rb, dtype=torch.uint8, device=device)
    out[:, :n8] = codes
    out[:, n8:n8 + 128] = rope
    out[:, n8 + 128:n8 + 128 + 4 * nb] = scales.view(torch.uint8)
    return out.view(*shape, rb)


# Categorical weights over E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}: roughly
# a half-normal of standard deviation 2 sampled on the code grid.
_E2M1_WEIGHTS = torch.tensor([0.12, 0.24, 0.22, 0.16, 0.11, 0.09, 0.04, 0.02])
# Candidate E4M3 block scales (decoded values 0.125 .. 0.5).
_SF_VALUES = torch.tensor([0.125, 0.15625, 0.1875, 0.21875, 0.25, 0.3125, 0.375, 0.4375, 0.5])


def nvfp4_rows(g, shape, dim: int, device="cpu"):
    """Random NVFP4 rows: codes uint8 [*shape, dim/2] and E4M3 scales [*shape, dim/16]."""
    n = int(math.prod(shape)) if len(shape) else 1
    mag = torch.multinomial(_E2M1_WEIGHTS.to(device), n * dim, replacement=True, generator=g)
    sign = (torch.rand(n * dim, generator=g, device=device) < 0.5).to(torch.int64) * 8
    nib = (mag + sign).to(torch.uint8).view(n, dim // 2, 2)
    codes = (nib[..., 0] | (nib[..., 1] << 4)).contiguous()
    pick = torch.randint(0, len(_SF_VALUES), (n, dim // 16), generator=g, device=device)
    sf = _SF_VALUES.to(device)[pick].to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.view(*shape, dim // 2), sf.contiguous().view(*shape, dim // 16)


def block_scales(sf, dim: int):
    """Row-major NVFP4 scales [..., rows, dim/16] -> the key-cache layout
    [..., ceil(rows/128) * (dim/64) * 512]: 128-row blocks of 512-byte atoms,
    byte m0*16 + m1*4 + kk of atom a holding the scale of block row m0 + 32*m1
    for values 64*a + 16*kk .. +15 (a pure index permutation)."""
    *lead, rows, ns = sf.shape
    nb = (rows + 127) // 128
    pad = torch.zeros(*lead, nb * 128, ns, dtype=sf.dtype, device=sf.device)
    pad[..., :rows, :] = sf
    x = pad.view(*lead, nb, 4, 32, dim // 64, 4)           # (block, m1, m0, atom, kk)
    n = len(lead)
    x = x.permute(*range(n), n, n + 3, n + 2, n + 1, n + 4)  # (block, atom, m0, m1, kk)
    return x.contiguous().view(*lead, nb * (dim // 64) * 512)


def compress_inputs(g, batch: int, n_tok: int, dim: int, m: int, overlap: bool, dtype,
                    c_std=1.0, z_std=1.0, b_std=0.1, device="cpu"):
    """Per-token C^a, C^b, Z^a, Z^b [batch, n_tok, dim] and biases B^a, B^b [m, dim] fp32."""
    Ca = normal(g, (batch, n_tok, dim), c_std, dtype, device)
    Za = normal(g, (batch, n_tok, dim), z_std, dtype, device)
    Ba = normal(g, (m, dim), b_std, torch.float32, device)
    if not overlap:
        return dict(Ca=Ca, Za=Za, Ba=Ba, Cb=None, Zb=None, Bb=None)
    Cb = normal(g, (batch, n_tok, dim), c_std, dtype, device)
    Zb = normal(g, (batch, n_tok, dim), z_std, dtype, device)
    Bb = normal(g, (m, dim), b_std, torch.float32, device)
    return dict(Ca=Ca, Za=Za, Ba=Ba, Cb=Cb, Zb=Zb, Bb=Bb)


def _torch_dtype(dt):
    return torch.float32 if dt == F32 else torch.bfloat16


def attention_inputs(cfg: dict, device="cpu", batch=None, ctx=None, n_q=None, q0=None,
                     n_entries=None, seed=None):
    """Inputs of one CSA or HCA attention call shaped like workload `cfg`.

    Returns a dict with Q [B, T, n_h, c], q_pos [B, T] (int64), entries
    [B, E, row], window KV rows win [B, Lw, row] with win_start [B] (absolute
    position of row 0), sink [n_h] fp32, and for CSA the indexer inputs
    qI [B, T, n_hI, dI] (+ qI_sf for NVFP4), wI [B, T, n_hI] fp32,
    KI [B, E, dI] (+ KI_sf).  Optional keyword overrides shrink the shape.
    """
    B = batch or cfg["batch"]
    L = ctx or cfg["ctx"]
    T = n_q or cfg["n_q"]
    m, c, H, W = cfg["m"], cfg["dim"], cfg["n_h"], cfg["window"]
    if q0 is None:
        q0 = cfg.get("q0", L - T)
    E = n_entries if n_entries is not None else L // m
    g = generator(cfg["seed"] if seed is None else seed, device)
    out = {}
    out["Q"] = normal(g, (B, T, H, c), cfg["q_std"], _torch_dtype(cfg["q_dt"]), device)
    out["q_pos"] = (torch.arange(T, dtype=torch.int64, device=device) + q0).repeat(B, 1)
    out["entries"] = rows(g, cfg["kv_dt"], (B, E), c, cfg["kv_std"], device)
    # window rows cover tokens [q0 - W + 1, q0 + T - 1] clipped at 0
    w0 = max(0, q0 - W + 1)
    Lw = q0 + T - w0
    out["win"] = rows(g, cfg["kv_dt"], (B, Lw), c, cfg["kv_std"], device)
    out["win_start"] = torch.full((B,), w0, dtype=torch.int64, device=device)
    out["sink"] = normal(g, (H,), 1.0, torch.float32, device)
    if cfg["kind"].startswith("csa"):
        dI, HI = cfg["dI"], cfg["n_hI"]
        if cfg["idx_dt"] == NVFP4:
            out["qI"], out["qI_sf"] = nvfp4_rows(g, (B, T, HI), dI, device)
            out["KI"], ksf = nvfp4_rows(g, (B, E), dI, device)
            out["KI_sf"] = block_scales(ksf, dI)  # key-cache scale layout
        else:
            out["qI"] = normal(g, (B, T, HI, dI), 1.0, _torch_dtype(cfg["idx_dt"]), device)
            out["KI"] = normal(g, (B, E, dI), 1.0, _torch_dtype(cfg["idx_dt"]), device)
        out["wI"] = uniform(g, (B, T, HI), 0.0, 1.0, device)
    out.update(B=B, T=T, E=E, m=m, c=c, n_h=H, window=W, Lw=Lw, q0=q0)
    return out


# V4-Pro grouped output projection ("DeepSeek-V4 内部机制" 1.2 Step 3: g = 16
# groups, d_g = 1024; model dimension d = 7168 from the page's V4-Pro row).
OUT_PROJ_V4_PRO = dict(n_h=128, c=512, g=16, d_g=1024, d=7168)


def out_proj_inputs(g, T: int, n_h: int, c: int, groups: int, d_g: int, d: int, device="cpu"):
    """Attention output O [T, n_h, c] (about N(0, 1)) and weights Wg
    [groups, n_h/groups * c, d_g], Wo [groups * d_g, d] drawn N(0, 1/fan_in),
    all bf16."""
    k1 = n_h // groups * c
    O = normal(g, (T, n_h, c), device=device).to(torch.bfloat16)
    Wg = normal(g, (groups, k1, d_g), std=1.0 / math.sqrt(k1), device=device).to(torch.bfloat16)
    Wo = normal(g, (groups * d_g, d), std=1.0 / math.sqrt(groups * d_g), device=device).to(torch.bfloat16)
    return O, Wg, Wo

