"""float64 CPU oracle for the CSA / HCA forward pass.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only callers.  The CUDA library never
imports, links or calls anything here, and nothing here imports the CUDA
library.  The arithmetic lives in ``csa_oracle.c`` (plain C, double precision,
single-threaded); this module only marshals numpy arrays into it.

Row formats accepted by the functions below (``dt``):
  F32    -> numpy float32 [rows, dim]
  BF16   -> numpy uint16 (raw bf16 bits) [rows, dim]
  FP8MIX -> numpy uint8 [rows, row_bytes(FP8MIX, dim)]
  NVFP4  -> numpy uint8 codes [rows, dim // 2] plus uint8 scales [rows, dim // 16]
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

F32, BF16, FP8MIX, NVFP4 = 0, 1, 2, 3

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libcsa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into libcsa_oracle.so with gcc (strict IEEE double)."""
    stale = not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "csa_oracle.h")))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    sig = {
        "orc_bf16_decode": (dbl, [ctypes.c_uint16]),
        "orc_bf16_encode": (ctypes.c_uint16, [dbl]),
        "orc_round_bf16": (dbl, [dbl]),
        "orc_e4m3_decode": (dbl, [ctypes.c_uint8]),
        "orc_e4m3_encode": (ctypes.c_uint8, [dbl]),
        "orc_e2m1_decode": (dbl, [ctypes.c_uint8]),
        "orc_e2m1_encode": (ctypes.c_uint8, [dbl]),
        "orc_row_bytes": (i64, [i32, i32]),
        "orc_decode_rows": (i32, [P, P, i32, i32, i64, P]),
        "orc_encode_rows": (i32, [P, i32, i32, i64, P, P]),
        "orc_nvfp4_blocked_bytes": (i64, [i64, i32]),
        "orc_nvfp4_unblock_scales": (i32, [P, i64, i32, P]),
        "orc_nvfp4_block_scales": (i32, [P, i64, i32, P]),
        "orc_compress": (i32, [P, P, P, P, P, P, i64, i64, i64, i64, i32, i32, P]),
        "orc_index_scores": (None, [P, P, P, i32, i32, i64, P]),
        "orc_topk": (i32, [P, i64, i32, P]),
        "orc_visible_entries": (i64, [i64, i32, i64]),
        "orc_index_topk": (i32, [P, P, P, P, i32, i32, i32, i32, i64, i32, i32, i32, P, P]),
        "orc_rmsnorm": (i32, [P, i64, i32, P, dbl, P]),
        "orc_rope_tail": (i32, [P, i64, i32, i32, P, dbl, P]),
        "orc_grouped_out_proj": (i32, [P, i32, i32, i32, i32, i32, P, P, i32, P]),
        "orc_gather_paged": (i32, [P, i64, i64, i32, P, i32, i32, i64, P]),
        "orc_attend": (None, [P, i32, i32, P, i64, P, dbl, P]),
        "orc_sparse_mqa": (i32, [P, P, i32, i64, P, i32, P, i64, P, P, i32, i32, P, dbl,
                                 i32, i32, i32, i32, P]),
        "orc_hca_dense_mqa": (i32, [P, P, i32, i64, P, i64, P, P, i32, i32, P, dbl,
                                    i32, i32, i32, i32, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


# --- scalar formats --------------------------------------------------------------

def bf16_decode(h: int) -> float:
    return _load().orc_bf16_decode(h)


def bf16_encode(x: float) -> int:
    return _load().orc_bf16_encode(x)


def round_bf16(x):
    """Round every element to the nearest bf16 (ties to even), as float64."""
    lib = _load()
    a = np.asarray(x, dtype=np.float64)
    return np.vectorize(lib.orc_round_bf16, otypes=[np.float64])(a) if a.size else a.copy()


def e4m3_decode(c: int) -> float:
    return _load().orc_e4m3_decode(c)


def e4m3_encode(x: float) -> int:
    return _load().orc_e4m3_encode(x)


def e2m1_decode(c: int) -> float:
    return _load().orc_e2m1_decode(c)


def e2m1_encode(x: float) -> int:
    return _load().orc_e2m1_encode(x)


# --- row formats -------------------------------------------------------------------

def row_bytes(dt: int, dim: int) -> int:
    return int(_load().orc_row_bytes(dt, dim))


def unblock_scales(blocked, n_rows: int, dim: int) -> np.ndarray:
    """NVFP4 key-cache scales (128-row blocks of tensor-core atoms) -> [rows, dim/16]."""
    blocked = _c(blocked, np.uint8)
    out = np.zeros((n_rows, dim // 16), np.uint8)
    _check(_load().orc_nvfp4_unblock_scales(_p(blocked), n_rows, dim, _p(out)), "unblock_scales")
    return out


def block_scales(rowmajor, dim: int) -> np.ndarray:
    """Row-major NVFP4 scales [rows, dim/16] -> 128-row blocked key-cache layout."""
    rowmajor = _c(rowmajor, np.uint8)
    n_rows = rowmajor.shape[0]
    out = np.zeros(int(_load().orc_nvfp4_blocked_bytes(n_rows, dim)), np.uint8)
    _check(_load().orc_nvfp4_block_scales(_p(rowmajor), n_rows, dim, _p(out)), "block_scales")
    return out


def decode_rows(buf, dt: int, dim: int, sf=None, sf_blocked=False) -> np.ndarray:
    """Decode rows of format dt into float64 [rows, dim] (exact).  For NVFP4,
    sf holds the scales row-major, or in the blocked key-cache layout when
    sf_blocked is set."""
    buf = np.ascontiguousarray(buf)
    rb = row_bytes(dt, dim)
    n_rows = buf.nbytes // rb
    out = np.empty((n_rows, dim), np.float64)
    if sf is not None and sf_blocked:
        sf = unblock_scales(sf, n_rows, dim)
    sf = _c(sf, np.uint8)
    _check(_load().orc_decode_rows(_p(buf), _p(sf), dt, dim, n_rows, _p(out)), "decode_rows")
    return out


def encode_rows(x, dt: int):
    """Encode float64 rows [rows, dim] into format dt; returns (buf, sf-or-None)."""
    x = _f64(x)
    n_rows, dim = x.shape
    rb = row_bytes(dt, dim)
    buf = np.zeros((n_rows, rb), np.uint8)
    sf = np.zeros((n_rows, dim // 16), np.uint8) if dt == NVFP4 else None
    _check(_load().orc_encode_rows(_p(x), dt, dim, n_rows, _p(buf), _p(sf)), "encode_rows")
    if dt == F32:
        buf = buf.view(np.float32)
    elif dt == BF16:
        buf = buf.view(np.uint16)
    return buf, sf


# --- the method -------------------------------------------------------------------

def compress(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None, tok0=0, e0=0, n_out=None):
    """Token-level compressor: entries e0..e0+n_out-1 from token rows tok0.. (float64).

    Cb/Zb/Bb None selects the HCA form (one branch, no overlap)."""
    Ca, Za, Ba = _f64(Ca), _f64(Za), _f64(Ba)
    Cb, Zb, Bb = _f64(Cb), _f64(Zb), _f64(Bb)
    n_tok, dim = Ca.shape
    if n_out is None:
        n_out = (tok0 + n_tok) // m - e0
    out = np.zeros((max(n_out, 0), dim), np.float64)
    _check(_load().orc_compress(_p(Ca), _p(Cb), _p(Za), _p(Zb), _p(Ba), _p(Bb), tok0, n_tok,
                                e0, n_out, dim, m, _p(out)), "compress")
    return out


def index_scores(q, w, K):
    """I[s] = sum_h w[h] * relu(q[h] . K[s]) for one query (float64, no rounding)."""
    q, w, K = _f64(q), _f64(w), _f64(K)
    n_h, dim = q.shape
    out = np.zeros(K.shape[0], np.float64)
    _load().orc_index_scores(_p(q), _p(w), _p(K), n_h, dim, K.shape[0], _p(out))
    return out


def topk(score, k: int) -> np.ndarray:
    score = _f64(score)
    idx = np.zeros(k, np.int32)
    _check(_load().orc_topk(_p(score), score.shape[0], k, _p(idx)), "topk")
    return idx


def visible_entries(t: int, m: int, n_entries: int) -> int:
    return int(_load().orc_visible_entries(t, m, n_entries))


def index_topk(qI, wI, KI, q_pos, m, k, round_bf16=True, want_scores=True):
    """qI [B, T, H, d], wI [B, T, H], KI [B, E, d] (float64 decoded), q_pos [B, T].

    Returns (scores [B, T, E] or None, idx [B, T, k])."""
    qI, wI, KI = _f64(qI), _f64(wI), _f64(KI)
    q_pos = _c(q_pos, np.int64)
    B, T, H, d = qI.shape
    E = KI.shape[1]
    scores = np.zeros((B, T, E), np.float64) if want_scores else None
    idx = np.zeros((B, T, k), np.int32)
    _check(_load().orc_index_topk(_p(qI), _p(wI), _p(KI), _p(q_pos), B, T, H, d, E, m, k,
                                  int(round_bf16), _p(scores), _p(idx)), "index_topk")
    return scores, idx


def rmsnorm(x, g=None, eps=1e-6):
    """RMSNorm of every row (last axis) of x, with per-channel weight g."""
    x = _f64(x)
    dim = x.shape[-1]
    y = np.zeros_like(x)
    _check(_load().orc_rmsnorm(_p(x), x.size // dim, dim, _p(_f64(g)), eps, _p(y)), "rmsnorm")
    return y


def rope_tail(x, pos, rope_dims=64, base=10000.0):
    """Partial RoPE of every row (last axis) of x; pos holds one position per
    row, numpy-broadcast to x.shape[:-1] (e.g. q_pos[..., None] for heads)."""
    x = _f64(x)
    dim = x.shape[-1]
    n = x.size // dim
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(pos, np.float64), x.shape[:-1])).reshape(n)
    y = np.zeros_like(x)
    _check(_load().orc_rope_tail(_p(x), n, dim, rope_dims, _p(pos), base, _p(y)), "rope_tail")
    return y


def grouped_out_proj(O, Wg, Wo):
    """O [T, n_h, c]; Wg [g, n_h/g * c, d_g]; Wo [g * d_g, d] -> Y [T, d]."""
    O, Wg, Wo = _f64(O), _f64(Wg), _f64(Wo)
    T, n_h, c = O.shape
    g, _, d_g = Wg.shape
    d = Wo.shape[1]
    Y = np.zeros((T, d), np.float64)
    _check(_load().orc_grouped_out_proj(_p(O), T, n_h, c, g, d_g, _p(Wg), _p(Wo), d, _p(Y)), "grouped_out_proj")
    return Y


def gather_paged(pool, table, n_entries):
    """pool [n_pages, per_page, row_bytes] uint8; table [B, max_pages] int32 ->
    the contiguous cache [B, n_entries, row_bytes] uint8."""
    pool = np.ascontiguousarray(pool, dtype=np.uint8)
    table = _c(table, np.int32)
    n_pages, per_page, rb = pool.shape
    B, max_pages = table.shape
    out = np.zeros((B, n_entries, rb), np.uint8)
    _check(_load().orc_gather_paged(_p(pool), n_pages, rb, per_page, _p(table), max_pages, B, n_entries, _p(out)),
           "gather_paged")
    return out


def attend(q, KV, sink, scale):
    q, KV = _f64(q), _f64(KV)
    n_h, dim = q.shape
    sink = _f64(sink)
    out = np.zeros((n_h, dim), np.float64)
    _load().orc_attend(_p(q), n_h, dim, _p(KV), KV.shape[0], _p(sink), scale, _p(out))
    return out


def _kv(a):
    return np.ascontiguousarray(a)


def sparse_mqa(Q, entries, kv_dt, idx, win, win_start, q_pos, window, m, sink, scale):
    """Q [B, T, H, c] float64; entries [B, E, ...] and win [B, Lw, ...] in kv_dt rows;
    idx [B, T, k] int32; win_start [B]; q_pos [B, T]; sink [H].  Returns O float64."""
    Q = _f64(Q)
    B, T, H, c = Q.shape
    entries, win = _kv(entries), _kv(win)
    rb = row_bytes(kv_dt, c)
    E = entries.nbytes // (B * rb)
    Lw = win.nbytes // (B * rb)
    idx = _c(idx, np.int32)
    k = idx.shape[-1]
    O = np.zeros_like(Q)
    _check(_load().orc_sparse_mqa(_p(Q), _p(entries), kv_dt, E, _p(idx), k, _p(win), Lw,
                                  _p(_c(win_start, np.int64)), _p(_c(q_pos, np.int64)), window, m,
                                  _p(_f64(sink)), scale, B, T, H, c, _p(O)), "sparse_mqa")
    return O


def hca_dense_mqa(Q, entries, kv_dt, win, win_start, q_pos, window, m, sink, scale):
    Q = _f64(Q)
    B, T, H, c = Q.shape
    entries, win = _kv(entries), _kv(win)
    rb = row_bytes(kv_dt, c)
    E = entries.nbytes // (B * rb)
    Lw = win.nbytes // (B * rb)
    O = np.zeros_like(Q)
    _check(_load().orc_hca_dense_mqa(_p(Q), _p(entries), kv_dt, E, _p(win), Lw,
                                     _p(_c(win_start, np.int64)), _p(_c(q_pos, np.int64)), window,
                                     m, _p(_f64(sink)), scale, B, T, H, c, _p(O)), "hca_dense_mqa")
    return O
