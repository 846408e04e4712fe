"""Thin ctypes binding of libcsa_b200 (include/csa.h): argument marshalling only.

Every function takes torch tensors that already live on the CUDA device,
passes their data pointers and the current CUDA stream to the C ABI, and
returns the output tensors.  All arithmetic runs in the library's kernels;
there is no CPU fallback: if the shared library is missing or a call fails,
an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

F32, BF16, KV_FP8MIX, IDX_NVFP4 = 0, 1, 2, 3
_STATUS = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
           4: "CSA_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa_b200.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "csa.h")
_lib = None


class CsaError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def header_functions():
    """Names of the functions declared in include/csa.h."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(csa_\w+|hca_\w+)\s*\(", src)))


def load():
    """Load libcsa_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: run `python -m compressed_sparse_attention_hca_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    sigs = {
        "csa_last_error": (ctypes.c_char_p, []),
        "csa_version": (i32, []),
        "csa_last_launch_count": (i32, []),
        "csa_check_device_status": (i32, []),
        "csa_row_bytes": (i64, [i32, i32]),
        "csa_nvfp4_key_scale_bytes": (i64, [i64, i32]),
        "csa_compress": (i32, [P, P, P, P, P, P, i32, i64, i64, i64, i64, i64, i32, i32, i32, P, P,
                               i64, i64, i32, P]),
        "csa_rmsnorm_rope": (i32, [P, P, i64, i32, P, f32, P, i32, i32, i32, ctypes.c_double, i32, i32, P]),
        "csa_index_topk_workspace_size": (sz, [i32, i32, i64, i32, i32, i32, i32]),
        "csa_index_topk_plan": (i32, [i32, i32, i64, i32, i32, i32, i32, P]),
        "csa_compress_index_topk": (i32, [ctypes.POINTER(CompressJob), ctypes.POINTER(CompressJob),
                                          P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32,
                                          P, P, P, sz, P]),
        "csa_index_topk": (i32, [P, P, P, P, P, P, i32, i32, i64, i32, i32, i32, i32, i32, P, P, P,
                                 sz, P]),
        "csa_sparse_mqa_workspace_size": (sz, [i32, i32, i32, i32, i32, i32, i32, i32]),
        "csa_sparse_mqa": (i32, [P, i32, P, i64, P, i32, P, i64, P, P, i32, i32, P, f32, i32, i32,
                                 i32, i32, i32, P, P, sz, P]),
        "hca_dense_mqa_workspace_size": (sz, [i32, i32, i32, i32, i64, i32, i32, i32]),
        "hca_dense_mqa": (i32, [P, i32, P, i64, P, i64, P, P, i32, i32, P, f32, i32, i32, i32, i32,
                                i32, P, P, sz, P]),
        "csa_mqa_workspace_size": (sz, [i32, i32, i32, i32, i64, i32, i32, ctypes.POINTER(MqaOptions)]),
        "csa_sparse_mqa_ex": (i32, [P, i32, P, i64, P, i32, P, i64, P, P, i32, i32, P, f32, i32, i32,
                                    i32, i32, i32, P, P, sz, ctypes.POINTER(MqaOptions), P]),
        "hca_dense_mqa_ex": (i32, [P, i32, P, i64, P, i64, P, P, i32, i32, P, f32, i32, i32, i32, i32,
                                   i32, P, P, sz, ctypes.POINTER(MqaOptions), P]),
        "csa_compress_ex": (i32, [ctypes.POINTER(CompressJob), i32, P]),
        "csa_index_topk_paged": (i32, [P, P, P, P, P, ctypes.POINTER(Pages), P, i32, i32, i64, i32, i32, i32, i32,
                                       i32, P, P, P, sz, P]),
        "csa_grouped_out_proj_workspace_size": (sz, [i32, i32, i32, i32, i32, i32]),
        "csa_grouped_out_proj_plan": (i32, [i32, i32, i32, i32, i32, i32, P]),
        "csa_grouped_out_proj": (i32, [P, P, P, P, i32, i32, i32, i32, i32, i32, P, sz, P]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(status):
    if status != 0:
        raise CsaError(status, load().csa_last_error().decode())


def _dt_of(t):
    return F32 if t.dtype == torch.float32 else BF16


def check_device_status():
    """Synchronises the device; raises CsaError if a kernel wait timed out."""
    _check(load().csa_check_device_status())


def last_launch_count():
    """Kernels launched by this thread's last library call."""
    return int(load().csa_last_launch_count())


def row_bytes(dt, dim):
    return int(load().csa_row_bytes(dt, dim))


def nvfp4_key_scale_bytes(n_rows, dim):
    """Bytes of one request's blocked NVFP4 key-scale array."""
    return int(load().csa_nvfp4_key_scale_bytes(n_rows, dim))


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


# ------------------------------------------------------------------ paged cache

class Pages(ctypes.Structure):
    """csa_pages_t: the block table of a paged cache."""
    _fields_ = [("table", ctypes.c_void_p), ("max_pages", ctypes.c_int32), ("page_entries", ctypes.c_int32),
                ("n_pages", ctypes.c_int64)]


def pages(table, page_entries, n_pages):
    """A block table: table [batch, max_pages] int32 (CUDA) of pool pages of
    page_entries rows each; n_pages pages in the pool."""
    _need_cuda(table)
    if table.dtype != torch.int32 or table.dim() != 2:
        raise ValueError("table must be a [batch, max_pages] int32 tensor")
    p = Pages(table=table.data_ptr(), max_pages=table.shape[1], page_entries=page_entries, n_pages=n_pages)
    p._keep = table  # the struct holds a raw pointer: keep the tensor alive with it
    return p


# --------------------------------------------------------------------- compress

def compress(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None, *, tok0=0, e0=0, n_out=None, out_dt=None,
             out=None, out_sf=None, out_row0=0, n_tok=None):
    """Token-level compressor.  Ca/Za [batch, rows, dim] (F32 or BF16), Ba [m, dim] fp32.

    Entry e0 + j of request b goes to row out_row0 + j of out[b] (out:
    [batch, rows, ...]; NVFP4 out_sf: the blocked key scales [batch,
    nvfp4_key_scale_bytes(rows, dim)]; allocated when not given).  Returns out
    (and out_sf for NVFP4)."""
    _need_cuda(Ca, Za, Ba, Cb, Zb, Bb)
    batch, rows, dim = Ca.shape
    n_tok = rows if n_tok is None else n_tok
    in_dt = _dt_of(Ca)
    out_dt = in_dt if out_dt is None else out_dt
    if n_out is None:
        n_out = (tok0 + n_tok) // m - e0
    if out is None:
        stride = n_out + out_row0
        if out_dt in (F32, BF16):
            out = torch.empty(batch, stride, dim, device=Ca.device,
                              dtype=torch.float32 if out_dt == F32 else torch.bfloat16)
        else:
            out = torch.empty(batch, stride, row_bytes(out_dt, dim), device=Ca.device, dtype=torch.uint8)
        if out_dt == IDX_NVFP4:
            out_sf = torch.zeros(batch, nvfp4_key_scale_bytes(stride, dim), device=Ca.device, dtype=torch.uint8)
    _need_cuda(out, out_sf)
    stride = out.shape[1]
    if out_dt == IDX_NVFP4 and out_sf.numel() < batch * nvfp4_key_scale_bytes(stride, dim):
        raise ValueError("out_sf smaller than the blocked key-scale arrays of the cache")
    _check(load().csa_compress(_ptr(Ca), _ptr(Cb), _ptr(Za), _ptr(Zb), _ptr(Ba), _ptr(Bb), batch, n_tok,
                               tok0, rows, e0, n_out, dim, m, in_dt, _ptr(out), _ptr(out_sf), stride,
                               out_row0, out_dt, _stream()))
    return (out, out_sf) if out_dt == IDX_NVFP4 else out


# ------------------------------------------------------ normalisation + partial RoPE

def rmsnorm_rope(x, pos, *, g=None, eps=1e-6, rows_per_pos=1, pos_sign=1, rope_dims=64, base=10000.0,
                 out=None, out_dt=None):
    """RMSNorm (when g is given) and RoPE of the last rope_dims dims of every
    row (last axis) of x; row r uses pos[r // rows_per_pos] (pos int64,
    flattened).  out defaults to a new tensor of out_dt (x's dtype); out=x
    works in place."""
    _need_cuda(x, pos, g, out)
    dim = x.shape[-1]
    n_rows = x.numel() // dim
    in_dt = _dt_of(x)
    out_dt = in_dt if out_dt is None else out_dt
    if out is None:
        out = torch.empty(x.shape, device=x.device, dtype=torch.float32 if out_dt == F32 else torch.bfloat16)
    _check(load().csa_rmsnorm_rope(_ptr(x), _ptr(out), n_rows, dim, _ptr(g), eps, _ptr(pos), rows_per_pos,
                                   pos_sign, rope_dims, base, in_dt, out_dt, _stream()))
    return out


# ------------------------------------------------------------------- index top-k

def index_topk_workspace_size(batch, n_q, n_entries, k, n_heads, dim, dt):
    return int(load().csa_index_topk_workspace_size(batch, n_q, n_entries, k, n_heads, dim, dt))


def index_topk_plan(batch, n_q, n_entries, k, n_heads, dim, dt):
    """How csa_index_topk splits a call of this shape on the current device:
    dict(slice_len, n_slices, coop, tensor_core, ring_stages, tiles_per_stage)."""
    out = (ctypes.c_int32 * 6)()
    _check(load().csa_index_topk_plan(batch, n_q, n_entries, k, n_heads, dim, dt, ctypes.cast(out, ctypes.c_void_p)))
    keys = ("slice_len", "n_slices", "coop", "tensor_core", "ring_stages", "tiles_per_stage")
    return dict(zip(keys, [int(v) for v in out]))


def index_topk(qI, wI, KI, q_pos, m, k, *, dt=None, qI_sf=None, KI_sf=None, n_heads=None,
               scores=False, idx_out=None, ws=None, key_pages=None, n_entries=None):
    """Lightning indexer + top-k.  qI [B, T, H, d] (or NVFP4 codes [B, T, H, d/2]),
    wI [B, T, H] fp32, KI [B, E, d] (codes [B, E, d/2]), q_pos [B, T] int64.
    Paged keys: key_pages a Pages (pages()), KI / KI_sf the pool, n_entries = E.

    Returns idx [B, T, k] int32 (and the score tensor when scores=True)."""
    _need_cuda(qI, wI, KI, q_pos, qI_sf, KI_sf)
    if dt is None:
        dt = IDX_NVFP4 if qI.dtype == torch.uint8 else _dt_of(qI)
    B, T, H = wI.shape
    if key_pages is not None and n_entries is None:
        raise ValueError("paged keys need n_entries (logical keys per request)")
    E = KI.shape[1] if n_entries is None else n_entries
    dim = qI.shape[-1] * (2 if dt == IDX_NVFP4 else 1)
    dev = qI.device
    if idx_out is None:
        idx_out = torch.empty(B, T, k, device=dev, dtype=torch.int32)
    sc = None
    if scores:
        sc = torch.empty(B, T, E, device=dev, dtype=torch.float32 if dt == F32 else torch.bfloat16)
    need = index_topk_workspace_size(B, T, E, k, H, dim, dt)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, device=dev, dtype=torch.uint8)  # zero before first use
    _check(load().csa_index_topk_paged(_ptr(qI), _ptr(qI_sf), _ptr(wI), _ptr(KI), _ptr(KI_sf),
                                       ctypes.byref(key_pages) if key_pages is not None else None, _ptr(q_pos),
                                       B, T, E, m, H, dim, k, dt, _ptr(idx_out), _ptr(sc), _ptr(ws),
                                       ws.numel(), _stream()))
    return (idx_out, sc) if scores else idx_out


class CompressJob(ctypes.Structure):
    """csa_compress_job_t: one compressor call's arguments (see compress())."""
    _fields_ = [("Ca", ctypes.c_void_p), ("Cb", ctypes.c_void_p), ("Za", ctypes.c_void_p), ("Zb", ctypes.c_void_p),
                ("Ba", ctypes.c_void_p), ("Bb", ctypes.c_void_p), ("n_tok", ctypes.c_int64),
                ("tok0", ctypes.c_int64), ("in_batch_stride", ctypes.c_int64), ("e0", ctypes.c_int64),
                ("n_out", ctypes.c_int64), ("dim", ctypes.c_int32), ("m", ctypes.c_int32), ("in_dt", ctypes.c_int32),
                ("out", ctypes.c_void_p), ("out_sf", ctypes.c_void_p), ("out_batch_stride", ctypes.c_int64),
                ("out_row0", ctypes.c_int64), ("out_dt", ctypes.c_int32), ("out_pages", ctypes.POINTER(Pages)),
                ("norm_g", ctypes.c_void_p), ("norm_eps", ctypes.c_float), ("rope_dims", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("pos_stride", ctypes.c_int64), ("pos_offset", ctypes.c_int64)]


def compress_job(Ca, Za, Ba, m, Cb=None, Zb=None, Bb=None, *, tok0, e0, n_out, out, out_dt, out_sf=None,
                 out_row0=None, n_tok=None, out_pages=None, norm_g=None, norm_eps=1e-6, rope_dims=0,
                 rope_base=10000.0, pos_stride=None, pos_offset=None):
    """A compressor call's arguments as a CompressJob (entries e0.. written to
    rows out_row0.. of `out`, out_row0 defaulting to e0; with out_pages (a
    Pages) `out` / `out_sf` are the pool and rows are logical rows).  norm_g /
    rope_dims: RMSNorm and RoPE of each entry before it is stored, entry i at
    position pos_stride * i + pos_offset (default m * i + m - 1)."""
    _need_cuda(Ca, Za, Ba, Cb, Zb, Bb, out, out_sf, norm_g)
    batch, rows, dim = Ca.shape
    job = CompressJob(
        Ca=Ca.data_ptr(), Cb=Cb.data_ptr() if Cb is not None else None, Za=Za.data_ptr(),
        Zb=Zb.data_ptr() if Zb is not None else None, Ba=Ba.data_ptr(), Bb=Bb.data_ptr() if Bb is not None else None,
        n_tok=rows if n_tok is None else n_tok, tok0=tok0, in_batch_stride=rows, e0=e0, n_out=n_out, dim=dim, m=m,
        in_dt=_dt_of(Ca), out=out.data_ptr(), out_sf=out_sf.data_ptr() if out_sf is not None else None,
        out_batch_stride=out.shape[1], out_row0=e0 if out_row0 is None else out_row0, out_dt=out_dt,
        out_pages=ctypes.pointer(out_pages) if out_pages is not None else None,
        norm_g=norm_g.data_ptr() if norm_g is not None else None, norm_eps=norm_eps, rope_dims=rope_dims,
        rope_base=rope_base, pos_stride=m if pos_stride is None else pos_stride,
        pos_offset=m - 1 if pos_offset is None else pos_offset)
    job._keep = (out_pages, norm_g)  # the struct holds raw pointers: keep what they point to alive with it
    return job


def compress_ex(job, batch):
    """Runs one CompressJob (compress_job()) on `batch` requests."""
    _check(load().csa_compress_ex(ctypes.byref(job), batch, _stream()))


def compress_index_topk(keys_job, qI, wI, KI, q_pos, m, k, *, extra_job=None, dt=None, qI_sf=None, KI_sf=None,
                        idx_out=None, ws=None, scores=False, n_entries=None):
    """Run the compressor job `keys_job` (index keys into KI / KI_sf) and, if
    given, `extra_job` (e.g. the KV cache), then index + top-k over KI: one
    launch when the tensor-core indexer takes the shape.  Returns idx
    [B, T, k] int32 (and the score tensor when scores=True)."""
    _need_cuda(qI, wI, KI, q_pos, qI_sf, KI_sf)
    if dt is None:
        dt = IDX_NVFP4 if qI.dtype == torch.uint8 else _dt_of(qI)
    B, T, H = wI.shape
    if keys_job.out_pages and n_entries is None:
        raise ValueError("a paged key cache needs n_entries (logical keys per request)")
    E = KI.shape[1] if n_entries is None else n_entries
    dim = qI.shape[-1] * (2 if dt == IDX_NVFP4 else 1)
    dev = qI.device
    if idx_out is None:
        idx_out = torch.empty(B, T, k, device=dev, dtype=torch.int32)
    sc = None
    if scores:
        sc = torch.empty(B, T, E, device=dev, dtype=torch.float32 if dt == F32 else torch.bfloat16)
    need = index_topk_workspace_size(B, T, E, k, H, dim, dt)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, device=dev, dtype=torch.uint8)  # zero before first use
    _check(load().csa_compress_index_topk(ctypes.byref(keys_job),
                                          ctypes.byref(extra_job) if extra_job is not None else None,
                                          _ptr(qI), _ptr(qI_sf), _ptr(wI), _ptr(KI), _ptr(KI_sf), _ptr(q_pos), B, T,
                                          E, m, H, dim, k, dt, _ptr(idx_out), _ptr(sc), _ptr(ws), ws.numel(),
                                          _stream()))
    return (idx_out, sc) if scores else idx_out


# -------------------------------------------------------------------- attention

class MqaOptions(ctypes.Structure):
    """csa_mqa_options_t: fixed split count (batch-invariant decode), query
    RMSNorm weights and eps, RoPE dims of the query (at q_pos) and of the
    output (at -q_pos), RoPE base, block table of a paged entry cache."""
    _fields_ = [("splits", ctypes.c_int32), ("q_norm_g", ctypes.c_void_p), ("q_norm_eps", ctypes.c_float),
                ("q_rope_dims", ctypes.c_int32), ("out_rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_double),
                ("entry_pages", ctypes.POINTER(Pages)), ("compress", ctypes.POINTER(CompressJob))]


def mqa_options(*, splits=0, q_norm_g=None, q_norm_eps=1e-6, q_rope_dims=0, out_rope_dims=0, rope_base=10000.0,
                entry_pages=None, compress=None):
    """Options of the attention calls; entry_pages: a Pages (pages()) when
    `entries` is the pool of a paged cache; compress: a CompressJob
    (compress_job()) launched before the entries are attended."""
    _need_cuda(q_norm_g)
    o = MqaOptions(splits=splits, q_norm_g=q_norm_g.data_ptr() if q_norm_g is not None else None,
                   q_norm_eps=q_norm_eps, q_rope_dims=q_rope_dims, out_rope_dims=out_rope_dims,
                   rope_base=rope_base, entry_pages=ctypes.pointer(entry_pages) if entry_pages is not None else None,
                   compress=ctypes.pointer(compress) if compress is not None else None)
    o._keep = (q_norm_g, entry_pages, compress)  # raw pointers: keep what they point to alive with the struct
    return o


def _n_entries(entries, n_entries, options):
    if options is not None and options.entry_pages:
        if n_entries is None:
            raise ValueError("a paged call needs n_entries (logical entries per request)")
        return n_entries
    return entries.shape[1] if n_entries is None else n_entries


def _opt_ref(options):
    return ctypes.byref(options) if options is not None else None


def mqa_workspace_size(batch, n_q, n_heads, dim, rows_per_query, q_dt, kv_dt, options=None):
    return int(load().csa_mqa_workspace_size(batch, n_q, n_heads, dim, rows_per_query, q_dt, kv_dt,
                                             _opt_ref(options)))


def _kv_dt(entries, kv_dt):
    if kv_dt is not None:
        return kv_dt
    return KV_FP8MIX if entries.dtype == torch.uint8 else _dt_of(entries)


def sparse_mqa_workspace_size(batch, n_q, n_heads, dim, k, window, q_dt, kv_dt):
    return int(load().csa_sparse_mqa_workspace_size(batch, n_q, n_heads, dim, k, window, q_dt, kv_dt))


def hca_dense_mqa_workspace_size(batch, n_q, n_heads, dim, n_entries, window, q_dt, kv_dt):
    return int(load().hca_dense_mqa_workspace_size(batch, n_q, n_heads, dim, n_entries, window, q_dt,
                                                   kv_dt))


def sparse_mqa(Q, entries, idx, win, win_start, q_pos, window, m, sink, scale, *, kv_dt=None, O=None,
               ws=None, options=None, n_entries=None):
    """CSA shared-KV MQA.  Q [B, T, H, c]; entries [B, E, row] (paged: the
    pool, with n_entries = E); idx [B, T, k] int32; win [B, Lw, row];
    win_start [B] int64; q_pos [B, T] int64; sink [H] fp32.
    options: an MqaOptions (mqa_options()) or None."""
    _need_cuda(Q, entries, idx, win, win_start, q_pos, sink)
    B, T, H, c = Q.shape
    kv_dt = _kv_dt(entries, kv_dt)
    q_dt = _dt_of(Q)
    k = idx.shape[-1]
    if O is None:
        O = torch.empty_like(Q)
    need = mqa_workspace_size(B, T, H, c, k + window, q_dt, kv_dt, options)
    if ws is None or ws.numel() < need:
        ws = torch.empty(need, device=Q.device, dtype=torch.uint8)
    _check(load().csa_sparse_mqa_ex(_ptr(Q), q_dt, _ptr(entries), _n_entries(entries, n_entries, options), _ptr(idx),
                                    k, _ptr(win),
                                    win.shape[1], _ptr(win_start), _ptr(q_pos), window, m, _ptr(sink),
                                    float(scale), B, T, H, c, kv_dt, _ptr(O), _ptr(ws), ws.numel(),
                                    _opt_ref(options), _stream()))
    return O


def hca_dense_mqa(Q, entries, win, win_start, q_pos, window, m, sink, scale, *, kv_dt=None, O=None,
                  ws=None, options=None, n_entries=None):
    """HCA dense shared-KV MQA over every visible entry plus the window
    (paged: entries is the pool, n_entries the logical entries)."""
    _need_cuda(Q, entries, win, win_start, q_pos, sink)
    B, T, H, c = Q.shape
    kv_dt = _kv_dt(entries, kv_dt)
    q_dt = _dt_of(Q)
    if O is None:
        O = torch.empty_like(Q)
    E = _n_entries(entries, n_entries, options)
    need = mqa_workspace_size(B, T, H, c, E + window, q_dt, kv_dt, options)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, device=Q.device, dtype=torch.uint8)
    _check(load().hca_dense_mqa_ex(_ptr(Q), q_dt, _ptr(entries), E, _ptr(win), win.shape[1],
                                   _ptr(win_start), _ptr(q_pos), window, m, _ptr(sink), float(scale), B, T,
                                   H, c, kv_dt, _ptr(O), _ptr(ws), ws.numel(), _opt_ref(options), _stream()))
    return O


# ------------------------------------------------------ grouped output projection

def grouped_out_proj_workspace_size(T, n_h, c, g, d_g, d):
    return int(load().csa_grouped_out_proj_workspace_size(T, n_h, c, g, d_g, d))


def grouped_out_proj_plan(T, n_h, c, g, d_g, d):
    """How csa_grouped_out_proj divides a call of this shape: per projection
    (group, then output) the tokens per CTA, K slices per tile and CTAs."""
    out = (ctypes.c_int32 * 6)()
    _check(load().csa_grouped_out_proj_plan(T, n_h, c, g, d_g, d, ctypes.cast(out, ctypes.c_void_p)))
    v = [int(x) for x in out]
    keys = ("tokens_per_cta", "splits", "ctas")
    return {"group": dict(zip(keys, v[:3])), "output": dict(zip(keys, v[3:]))}


def grouped_out_proj(O, Wg, Wo, *, out=None, ws=None):
    """Grouped output projection.  O [T, n_h, c] bf16, Wg [g, n_h/g * c, d_g]
    bf16, Wo [g * d_g, d] bf16 -> Y [T, d] bf16.  ws: a workspace of
    grouped_out_proj_workspace_size bytes whose counters are zero (a fresh
    zeroed one is made when not given; every call leaves it zero)."""
    _need_cuda(O, Wg, Wo, out, ws)
    T, n_h, c = O.shape
    g, _, d_g = Wg.shape
    d = Wo.shape[1]
    if Wg.shape[1] * g != n_h * c or Wo.shape[0] != g * d_g:
        raise ValueError("Wg must be [g, n_h/g * c, d_g] and Wo [g * d_g, d]")
    if out is None:
        out = torch.empty(T, d, device=O.device, dtype=torch.bfloat16)
    need = grouped_out_proj_workspace_size(T, n_h, c, g, d_g, d)
    if ws is None:
        ws = torch.zeros(need, device=O.device, dtype=torch.uint8)
    _check(load().csa_grouped_out_proj(_ptr(O), _ptr(Wg), _ptr(Wo), _ptr(out), T, n_h, c, g, d_g, d, _ptr(ws),
                                       ws.numel() * ws.element_size(), _stream()))
    return out
