"""Python binding of libcsa.so, the CSA/HCA attention-layer core for B200.

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  PyTorch supplies device memory and streams.  The functions carry the
names of the C entry points (include/csa.h):

    csa_compress, hca_compress, csa_compress_append, hca_compress_append,
    indexer_scores_topk, sparse_mqa_attn, dense_hca_attn, grouped_output_projection,
    csa_workspace_bytes, csa_check_status

Importing succeeds without a GPU; calling any op without the built library or
without a CUDA device raises ``CSAError``.  There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcsa.so")

CSA_OK, CSA_E_ARG, CSA_E_UNSUPPORTED, CSA_E_CUDA, CSA_E_DEVICE, CSA_E_WORKSPACE = range(6)
CSA_F32, CSA_BF16 = 0, 1
CSA_F_NO_NORM, CSA_F_NO_ROPE, CSA_F_PORTABLE, CSA_F_MIXED = 1, 2, 4, 8
(CSA_OP_INDEXER, CSA_OP_SPARSE_ATTN, CSA_OP_DENSE_ATTN, CSA_OP_COMPRESS, CSA_OP_OUT_PROJ,
 CSA_OP_INDEXER_MX) = 1, 2, 3, 4, 5, 6
CSA_DEV_TIMEOUT, CSA_DEV_RANGE, CSA_DEV_BAD_INDEX, CSA_DEV_STREAM = 1, 2, 3, 4

EXPORTED = (
    "csa_compress", "hca_compress", "csa_stream_state_bytes", "csa_compress_append",
    "hca_compress_append", "indexer_scores_topk", "indexer_scores_topk_noalloc",
    "indexer_mxfp8_quantize", "indexer_scores_topk_mxfp8", "indexer_mxfp4_quantize",
    "indexer_scores_topk_mxfp4", "csa_mixed_record_bytes",
    "csa_store_mixed", "sparse_mqa_attn", "dense_hca_attn",
    "grouped_output_projection", "csa_workspace_bytes",
    "csa_check_status",
    "csa_status_string", "csa_launch_count", "csa_selftest_wait",
)


class CSAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = _status_name(status)
        super().__init__(f"{what}: {name} ({status})" if what else f"{name} ({status})")


def _status_name(s: int) -> str:
    try:
        return lib().csa_status_string(s).decode()
    except Exception:
        return {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error",
                4: "device-side error", 5: "workspace"}.get(s, "unknown")


class _CFmt(ctypes.Structure):
    _fields_ = [("c", ctypes.c_int32), ("rope_dims", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("norm_eps", ctypes.c_float), ("flags", ctypes.c_uint32)]


@dataclass(frozen=True)
class Fmt:
    """Entry format: dim c, RoPE on the last ``rope_dims`` dims."""

    c: int = 512
    rope_dims: int = 64
    rope_base: float = 10000.0
    norm_eps: float = 1e-6
    flags: int = 0

    def _c(self):
        return _CFmt(self.c, self.rope_dims, self.rope_base, self.norm_eps, self.flags)


_lib = None


def lib():
    """The loaded libcsa.so (ctypes), with argument types declared."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise CSAError(CSA_E_CUDA, f"{LIB_PATH} is missing; run "
                       "`python -m long_context_attention_csa_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float
    sz = ctypes.c_size_t
    FP = ctypes.POINTER(_CFmt)
    L.csa_compress.argtypes = [i32, i64, i64, i32, FP, P, P, P, P, i32, i64, P, P, P, sz, P]
    L.hca_compress.argtypes = [i32, i64, i64, i32, FP, P, P, i32, i64, P, P, P, sz, P]
    L.indexer_scores_topk.argtypes = [i32, i64, i64, i32, i32, P, P, P, i64, P, i32, i32, P, P,
                                      P, sz, P]
    L.indexer_scores_topk_noalloc.argtypes = [i32, i64, i64, i32, i32, P, P, P, i64, P, i32, i32,
                                              P, P, P]
    L.sparse_mqa_attn.argtypes = [i32, i64, i64, i32, FP, P, P, P, i64, P, i32, P, i64, P, i32,
                                  P, f32, P, P, sz, P]
    L.dense_hca_attn.argtypes = [i32, i64, i64, i32, FP, P, P, P, i64, i32, P, i64, P, i32, P,
                                 f32, P, P, sz, P]
    L.csa_stream_state_bytes.argtypes = [i32, i32, i32, i32, i32]
    L.csa_stream_state_bytes.restype = sz
    L.csa_compress_append.argtypes = [i32, i64, i32, FP, P, P, P, P, i32, i64, P, sz, P, i64, P,
                                      P, sz, P]
    L.hca_compress_append.argtypes = [i32, i64, i32, FP, P, P, i32, i64, P, sz, P, i64, P, P, sz,
                                      P]
    L.indexer_mxfp8_quantize.argtypes = [i32, i64, i64, i32, P, P, P, P]
    L.indexer_mxfp4_quantize.argtypes = [i32, i64, i64, i32, P, P, P, P]
    L.indexer_scores_topk_mxfp4.argtypes = [i64, i64, i32, i32, P, P, P, P, P, i64, P, i32, i32,
                                            P, P, P, sz, P]
    L.csa_mixed_record_bytes.argtypes = [i32, i32]
    L.csa_mixed_record_bytes.restype = sz
    L.csa_store_mixed.argtypes = [i32, i64, i64, FP, P, P, P]
    L.indexer_scores_topk_mxfp8.argtypes = [i64, i64, i32, i32, P, P, P, P, P, i64, P, i32, i32,
                                            P, P, P, sz, P]
    L.grouped_output_projection.argtypes = [i32, i64, i32, i32, i32, i32, i32, P, P, P, P, P, sz,
                                            P]
    L.csa_workspace_bytes.argtypes = [i32, i32, i64, i64, i32, i32, i64, i32, i32]
    L.csa_workspace_bytes.restype = sz
    L.csa_check_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
    L.csa_status_string.argtypes = [i32]
    L.csa_status_string.restype = ctypes.c_char_p
    L.csa_selftest_wait.argtypes = [i64, P, sz, P]
    L.csa_launch_count.argtypes = []
    L.csa_launch_count.restype = ctypes.c_ulonglong
    for fn in ("csa_compress", "hca_compress", "csa_compress_append", "hca_compress_append",
               "indexer_scores_topk",
               "indexer_scores_topk_noalloc", "sparse_mqa_attn", "dense_hca_attn",
               "grouped_output_projection", "indexer_mxfp8_quantize", "csa_store_mixed",
               "indexer_mxfp4_quantize", "indexer_scores_topk_mxfp4",
               "indexer_scores_topk_mxfp8", "csa_check_status", "csa_selftest_wait"):
        getattr(L, fn).restype = i32
    _lib = L
    return L


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return CSA_BF16
    if t.dtype == torch.float32:
        return CSA_F32
    raise CSAError(CSA_E_ARG, f"unsupported dtype {t.dtype}")


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise CSAError(CSA_E_ARG, "tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise CSAError(CSA_E_ARG, "tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(st: int, what: str):
    if st != CSA_OK:
        raise CSAError(st, what)


def csa_workspace_bytes(op, dtype, B, Tq, H=0, c=0, N=0, k=0, n_win=0) -> int:
    dtype = dtype if isinstance(dtype, int) else (CSA_BF16 if dtype == torch.bfloat16 else CSA_F32)
    return int(lib().csa_workspace_bytes(op, dtype, B, Tq, H, c, N, k, n_win))


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zero-filled workspace buffer (the status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def csa_check_status(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    """(status, device code); synchronises the stream."""
    d = ctypes.c_uint32(0)
    st = lib().csa_check_status(_p(ws), _s(stream), ctypes.byref(d))
    return int(st), int(d.value)


def csa_selftest_wait(limit_ns: int, ws: torch.Tensor, stream=None) -> None:
    """Failure-path self test: a device wait that nothing satisfies runs out
    after limit_ns and records CSA_DEV_TIMEOUT in ws's status word."""
    st = lib().csa_selftest_wait(int(limit_ns), _p(ws), ws.numel() * ws.element_size(), _s(stream))
    if st != CSA_OK:
        raise CSAError(st, "csa_selftest_wait")


def csa_launch_count() -> int:
    return int(lib().csa_launch_count())


def csa_compress(kv_a, kv_b, z_a, z_b, m: int, fmt: Fmt, pos0: int = 0, entries=None,
                 win_out=None, want_win=False, ws=None, stream=None):
    """CSA compression of [B, T, c] token groups -> entries [B, T//m, c]
    (and window rows [B, T, c] when ``want_win``)."""
    B, T, c = kv_a.shape
    if entries is None:
        entries = torch.empty((B, T // m, c), dtype=kv_a.dtype, device=kv_a.device)
    if want_win and win_out is None:
        win_out = torch.empty_like(kv_a)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_COMPRESS, _dt(kv_a), B, T), kv_a.device)
    f = fmt._c()
    st = lib().csa_compress(_dt(kv_a), B, T, m, ctypes.byref(f), _p(kv_a), _p(kv_b), _p(z_a),
                            _p(z_b), z_a.shape[-1], pos0, _p(entries), _p(win_out), _p(ws),
                            ws.numel(), _s(stream))
    _check(st, "csa_compress")
    return (entries, win_out) if win_out is not None else entries


def hca_compress(kv, z, m_prime: int, fmt: Fmt, pos0: int = 0, entries=None, win_out=None,
                 want_win=False, ws=None, stream=None):
    """HCA compression of [B, T, c] tokens -> entries [B, T//m', c] (+ window rows)."""
    B, T, c = kv.shape
    if entries is None:
        entries = torch.empty((B, T // m_prime, c), dtype=kv.dtype, device=kv.device)
    if want_win and win_out is None:
        win_out = torch.empty_like(kv)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_COMPRESS, _dt(kv), B, T), kv.device)
    f = fmt._c()
    st = lib().hca_compress(_dt(kv), B, T, m_prime, ctypes.byref(f), _p(kv), _p(z), z.shape[-1],
                            pos0, _p(entries), _p(win_out), _p(ws), ws.numel(), _s(stream))
    _check(st, "hca_compress")
    return (entries, win_out) if win_out is not None else entries


def csa_stream_state_bytes(dtype, m: int, overlap: bool, c: int, z_cols: int) -> int:
    dtype = dtype if isinstance(dtype, int) else (CSA_BF16 if dtype == torch.bfloat16 else CSA_F32)
    return int(lib().csa_stream_state_bytes(dtype, m, int(bool(overlap)), c, z_cols))


def stream_state(B: int, m: int, overlap: bool, c: int, z_cols: int, dtype, device=None):
    """Zero-filled stream states of B sequences: a [B, stride] uint8 tensor."""
    n = csa_stream_state_bytes(dtype, m, overlap, c, z_cols)
    if n == 0:
        raise CSAError(CSA_E_ARG, "csa_stream_state_bytes")
    return torch.zeros((B, n), dtype=torch.uint8, device=device or "cuda")


def csa_compress_append(kv_a, kv_b, z_a, z_b, m: int, fmt: Fmt, state, entries, pos0: int = 0,
                        win_out=None, want_win=False, ws=None, stream=None):
    """Appends one token per sequence (kv_a, kv_b: [B, c]; z_a, z_b: [B, z_cols])
    to the CSA stream states ``state`` [B, stride]; a completed block's entry
    goes to ``entries`` [B, n_cap, c].  Returns the window rows [B, c] when
    asked (or given)."""
    B, c = kv_a.shape
    if want_win and win_out is None:
        win_out = torch.empty_like(kv_a)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_COMPRESS, _dt(kv_a), B, 1), kv_a.device)
    f = fmt._c()
    st = lib().csa_compress_append(_dt(kv_a), B, m, ctypes.byref(f), _p(kv_a), _p(kv_b), _p(z_a),
                                   _p(z_b), z_a.shape[-1], pos0, _p(state), state.shape[1],
                                   _p(entries), entries.shape[1], _p(win_out), _p(ws), ws.numel(),
                                   _s(stream))
    _check(st, "csa_compress_append")
    return win_out


def hca_compress_append(kv, z, m_prime: int, fmt: Fmt, state, entries, pos0: int = 0,
                        win_out=None, want_win=False, ws=None, stream=None):
    """Appends one token per sequence to the HCA stream states (see
    csa_compress_append)."""
    B, c = kv.shape
    if want_win and win_out is None:
        win_out = torch.empty_like(kv)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_COMPRESS, _dt(kv), B, 1), kv.device)
    f = fmt._c()
    st = lib().hca_compress_append(_dt(kv), B, m_prime, ctypes.byref(f), _p(kv), _p(z),
                                   z.shape[-1], pos0, _p(state), state.shape[1], _p(entries),
                                   entries.shape[1], _p(win_out), _p(ws), ws.numel(), _s(stream))
    _check(st, "hca_compress_append")
    return win_out


def indexer_scores_topk(q_I, w, k_I, m: int, k: int, q_pos=None, idx_out=None, score_out=None,
                        want_scores=False, ws=None, stream=None):
    """Indexer scores + causal top-k: q_I [B, Tq, H_I, d_I], w [B, Tq, H_I] fp32,
    k_I [B, N, d_I] -> idx [B, Tq, k] int32 (and scores [B, Tq, k])."""
    B, Tq, HI, dI = q_I.shape
    N = k_I.shape[1]
    dev = q_I.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    if want_scores and score_out is None:
        score_out = torch.empty((B, Tq, k), dtype=torch.float32, device=dev)
    need = csa_workspace_bytes(CSA_OP_INDEXER, _dt(q_I), B, Tq, 0, 0, N, k, 0)
    if ws is None:
        ws = workspace(need, dev)
    st = lib().indexer_scores_topk(_dt(q_I), B, Tq, HI, dI, _p(q_I), _p(w), _p(k_I), N,
                                   _p(q_pos), m, k, _p(idx_out), _p(score_out), _p(ws),
                                   ws.numel(), _s(stream))
    _check(st, "indexer_scores_topk")
    return (idx_out, score_out) if score_out is not None else idx_out


def csa_mixed_record_bytes(c: int, rope_dims: int) -> int:
    return int(lib().csa_mixed_record_bytes(c, rope_dims))


def csa_store_mixed(entries, fmt: Fmt, records=None, stream=None):
    """Mixed BF16 / MX-FP8 records [B, N, record bytes] uint8 of entries
    [B, N, c]; the attention calls read them under CSA_F_MIXED."""
    B, N, c = entries.shape
    rb = csa_mixed_record_bytes(c, fmt.rope_dims)
    if records is None:
        records = torch.empty((B, N, rb), dtype=torch.uint8, device=entries.device)
    f = fmt._c()
    st = lib().csa_store_mixed(_dt(entries), B, N, ctypes.byref(f), _p(entries), _p(records),
                               _s(stream))
    _check(st, "csa_store_mixed")
    return records


def indexer_mxfp8_quantize(x, codes=None, scales=None, per_token=False, stream=None, fp4=False):
    """MX-FP8 (or, with ``fp4``, packed MX-FP4) codes and scale tiles of x
    [B, ..., 128]: codes uint8 with x's shape (the last dim 64 for FP4);
    scales [B, ceil(rows/128), 512] with rows = the middle dims flattened, or,
    with ``per_token`` (q_I [B, Tq, 64, 128]), one tile per token: [B, Tq, 512]."""
    d = x.shape[-1]
    B = x.shape[0] * x.shape[1] if per_token else x.shape[0]
    rows = x.numel() // d // B if B else 0
    if codes is None:
        shape = tuple(x.shape[:-1]) + ((d // 2,) if fp4 else (d,))
        codes = torch.empty(shape, dtype=torch.uint8, device=x.device)
    if scales is None:
        shape = (x.shape[0], x.shape[1], 512) if per_token else (B, (rows + 127) // 128, 512)
        scales = torch.empty(shape, dtype=torch.uint8, device=x.device)
    fn = lib().indexer_mxfp4_quantize if fp4 else lib().indexer_mxfp8_quantize
    st = fn(_dt(x), B, rows, d, _p(x), _p(codes), _p(scales), _s(stream))
    _check(st, "indexer_mxfp4_quantize" if fp4 else "indexer_mxfp8_quantize")
    return codes, scales


def indexer_mxfp4_quantize(x, codes=None, scales=None, per_token=False, stream=None):
    """Packed MX-FP4 codes [..., 64] and scale tiles of x [B, ..., 128]."""
    return indexer_mxfp8_quantize(x, codes, scales, per_token, stream, fp4=True)


def indexer_scores_topk_mxfp8(q_codes, q_scales, w, k_codes, k_scales, m: int, k: int,
                              q_pos=None, idx_out=None, score_out=None, want_scores=False,
                              ws=None, stream=None):
    """indexer_scores_topk on MX-FP8 operands: q_codes [B, Tq, 64, 128] and
    k_codes [B, N, 128] uint8 with their scale tiles; packed MX-FP4 codes
    (last dim 64) take the FP4 kernel."""
    B, Tq, HI, dI = q_codes.shape
    fp4 = dI == 64
    dI = 128
    N = k_codes.shape[1]
    dev = q_codes.device
    if idx_out is None:
        idx_out = torch.empty((B, Tq, k), dtype=torch.int32, device=dev)
    if want_scores and score_out is None:
        score_out = torch.empty((B, Tq, k), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_INDEXER_MX, CSA_BF16, B, Tq, 0, 0, N, k), dev)
    fn = lib().indexer_scores_topk_mxfp4 if fp4 else lib().indexer_scores_topk_mxfp8
    st = fn(B, Tq, HI, dI, _p(q_codes), _p(q_scales), _p(w),
                                         _p(k_codes), _p(k_scales), N, _p(q_pos), m, k,
                                         _p(idx_out), _p(score_out), _p(ws), ws.numel(),
                                         _s(stream))
    _check(st, "indexer_scores_topk_mxfp8")
    return (idx_out, score_out) if score_out is not None else idx_out


def sparse_mqa_attn(q, entries, idx, win, fmt: Fmt, n_win: int, sink=None, q_pos=None,
                    win_pos0=None, scale: float = 0.0, out=None, ws=None, stream=None):
    """Sparse shared-KV MQA: q [B, Tq, H, c], entries [B, N, c], idx [B, Tq, k],
    win [B, Tw, c] -> out [B, Tq, H, c]."""
    B, Tq, H, c = q.shape
    N = entries.shape[1]
    k = idx.shape[-1] if idx is not None else 0
    Tw = win.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = csa_workspace_bytes(CSA_OP_SPARSE_ATTN, _dt(q), B, Tq, H, c, N, k, n_win)
    if ws is None:
        ws = workspace(need, q.device)
    f = fmt._c()
    st = lib().sparse_mqa_attn(_dt(q), B, Tq, H, ctypes.byref(f), _p(q), _p(q_pos), _p(entries),
                               N, _p(idx), k, _p(win), Tw, _p(win_pos0), n_win, _p(sink),
                               float(scale), _p(out), _p(ws), ws.numel(), _s(stream))
    _check(st, "sparse_mqa_attn")
    return out


def dense_hca_attn(q, entries, m_prime: int, win, fmt: Fmt, n_win: int, sink=None, q_pos=None,
                   win_pos0=None, scale: float = 0.0, out=None, ws=None, stream=None):
    """Dense shared-KV MQA over every visible entry (HCA) plus the window."""
    B, Tq, H, c = q.shape
    N = entries.shape[1]
    Tw = win.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = csa_workspace_bytes(CSA_OP_DENSE_ATTN, _dt(q), B, Tq, H, c, N, 0, n_win)
    if ws is None:
        ws = workspace(need, q.device)
    f = fmt._c()
    st = lib().dense_hca_attn(_dt(q), B, Tq, H, ctypes.byref(f), _p(q), _p(q_pos), _p(entries), N,
                              m_prime, _p(win), Tw, _p(win_pos0), n_win, _p(sink), float(scale),
                              _p(out), _p(ws), ws.numel(), _s(stream))
    _check(st, "dense_hca_attn")
    return out


def grouped_output_projection(o, w_group, w_out, y=None, ws=None, stream=None):
    """Grouped output projection: o [T, H, c], w_group [g, d_g, (H/g) c],
    w_out [d, g d_g] -> y [T, d] (bf16)."""
    T, H, c = o.shape
    g, dg, _ = w_group.shape
    d = w_out.shape[0]
    if y is None:
        y = torch.empty((T, d), dtype=o.dtype, device=o.device)
    if ws is None:
        ws = workspace(csa_workspace_bytes(CSA_OP_OUT_PROJ, _dt(o), 1, T, 0, 0, g * dg), o.device)
    st = lib().grouped_output_projection(_dt(o), T, H, c, g, dg, d, _p(o), _p(w_group),
                                         _p(w_out), _p(y), _p(ws), ws.numel(), _s(stream))
    _check(st, "grouped_output_projection")
    return y

