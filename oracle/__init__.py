"""Float64 CPU oracle for the CSA/HCA attention-layer core.

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path never
imports this package.  It shares no code with the CUDA library; the arithmetic
lives in ``csa_oracle.c`` (plain C, double precision, OpenMP over query rows)
and this module only marshals numpy arrays to it.

Functions mirror the method's steps as restated from the page
"DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3 (CSA and HCA hybrid
attention) and the page "DeepSeek V4 完整技术报告", section "混合注意力：CSA +
HCA".  Each function's docstring names the reading it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

NO_NORM = 1
NO_ROPE = 2


def build(force: bool = False) -> str:
    """Compile the oracle's C source into ``liboracle.so`` beside it."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Fmt(ctypes.Structure):
    _fields_ = [
        ("c", ctypes.c_int32),
        ("rope_dims", ctypes.c_int32),
        ("rope_base", ctypes.c_double),
        ("norm_eps", ctypes.c_double),
        ("flags", ctypes.c_uint32),
    ]


@dataclass(frozen=True)
class Fmt:
    """Entry format: dim c, RoPE on the last ``rope_dims`` dims."""

    c: int
    rope_dims: int = 64
    rope_base: float = 10000.0
    norm_eps: float = 1e-6
    flags: int = 0

    def _c(self) -> _Fmt:
        return _Fmt(self.c, self.rope_dims, self.rope_base, self.norm_eps, self.flags)


_lib = None


def _L():
    global _lib
    if _lib is None:
        # CSA_ORACLE_LIB: a build of a modified copy of csa_oracle.c, used by
        # the test that plants mistakes in the oracle to show the pins catch them
        _lib = ctypes.CDLL(os.environ.get("CSA_ORACLE_LIB") or build())
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        FP = ctypes.POINTER(_Fmt)
        _lib.orc_rmsnorm.argtypes = [i32, f64, P, P]
        _lib.orc_rope.argtypes = [i32, i32, f64, f64, P, P]
        _lib.orc_visible.argtypes = [i64, i32, i64]
        _lib.orc_visible.restype = i64
        _lib.orc_csa_compress.argtypes = [i64, i32, FP, P, P, P, P, i32, i64, P, P]
        _lib.orc_hca_compress.argtypes = [i64, i32, FP, P, P, i32, i64, P, P]
        _lib.orc_window_rows.argtypes = [i64, FP, P, i64, P]
        _lib.orc_indexer_scores.argtypes = [i64, i32, i32, i64, P, P, P, P, i32, P]
        _lib.orc_topk.argtypes = [i64, i64, P, P, i32, i32, P]
        _lib.orc_attention.argtypes = [
            i64, i32, FP, P, P, P, i64, P, i32, i32, P, i64, i64, i32, P, f64, P, P,
        ]
        _lib.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        _lib.orc_e4m3_value.restype = f64
        _lib.orc_e4m3_encode.argtypes = [f64]
        _lib.orc_e4m3_encode.restype = ctypes.c_uint8
        _lib.orc_mxfp8_quantize.argtypes = [i64, P, P, P]
        _lib.orc_mxfp8_dequantize.argtypes = [i64, P, P, P]
        _lib.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        _lib.orc_e2m1_value.restype = f64
        _lib.orc_e2m1_encode.argtypes = [f64]
        _lib.orc_e2m1_encode.restype = ctypes.c_uint8
        _lib.orc_mxfp4_quantize.argtypes = [i64, P, P, P]
        _lib.orc_mxfp4_dequantize.argtypes = [i64, P, P, P]
        _lib.orc_nvfp4_quantize.argtypes = [i64, P, P, P, P]
        _lib.orc_nvfp4_quantize.restype = None
        _lib.orc_nvfp4_dequantize.argtypes = [i64, P, P, f64, P]
        _lib.orc_nvfp4_dequantize.restype = None
        _lib.orc_bf16_round.argtypes = [f64]
        _lib.orc_bf16_round.restype = f64
        _lib.orc_mixed_store.argtypes = [i64, i32, i32, P, P, P, P]
        _lib.orc_mixed_store.restype = None
        _lib.orc_mixed_load.argtypes = [i64, i32, i32, P, P, P, P]
        _lib.orc_mixed_load.restype = None
        _lib.orc_stream_state_len.argtypes = [i32, i32, i32]
        _lib.orc_stream_state_len.restype = i64
        _lib.orc_stream_append.argtypes = [i32, i32, FP, i64, P, P, P, P, i32, P, P, P]
        _lib.orc_stream_append.restype = i32
        for fn in (
            "orc_rmsnorm", "orc_rope", "orc_csa_compress", "orc_hca_compress",
            "orc_window_rows", "orc_indexer_scores", "orc_topk", "orc_attention",
            "orc_mxfp8_quantize", "orc_mxfp8_dequantize", "orc_mxfp4_quantize",
            "orc_mxfp4_dequantize",
        ):
            getattr(_lib, fn).restype = None
    return _lib


def _f64(a) -> np.ndarray:
    a = np.asarray(a)
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def rmsnorm(x, eps: float = 1e-6) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _L().orc_rmsnorm(x.shape[-1], eps, _ptr(x), _ptr(y))
    return y


def rope(x, pos: float, rope_dims: int, base: float = 10000.0) -> np.ndarray:
    x = _f64(x)
    y = np.empty_like(x)
    _L().orc_rope(x.shape[-1], rope_dims, base, float(pos), _ptr(x), _ptr(y))
    return y


def visible(pos: int, m: int, n_entries: int) -> int:
    """Entries visible at query position ``pos`` (an entry is visible once its
    last token is at or before the query: s < floor((pos+1)/m))."""
    return int(_L().orc_visible(int(pos), int(m), int(n_entries)))


def csa_compress(kv_a, kv_b, z_a, z_b, m: int, fmt: Fmt, pos0: int = 0, want_weights=False):
    """Overlapped softmax-gated compression, rate exactly 1/m.

    kv_a, kv_b: [T, c]; z_a, z_b: [T, c] or [T, 1].  Returns entries [T//m, c]
    (and the softmax weights [T//m, 2m, c] when asked; slot order a then b).
    """
    kv_a, kv_b, z_a, z_b = map(_f64, (kv_a, kv_b, z_a, z_b))
    T, c = kv_a.shape
    assert c == fmt.c and 2 * m <= 512
    n = T // m
    ent = np.zeros((n, c))
    wts = np.zeros((n, 2 * m, c)) if want_weights else None
    f = fmt._c()
    _L().orc_csa_compress(T, m, ctypes.byref(f), _ptr(kv_a), _ptr(kv_b), _ptr(z_a), _ptr(z_b),
                          z_a.shape[1], pos0, _ptr(ent), _ptr(wts))
    return (ent, wts) if want_weights else ent


def hca_compress(kv, z, m_prime: int, fmt: Fmt, pos0: int = 0, want_weights=False):
    """Non-overlapped softmax-gated compression, rate 1/m'."""
    kv, z = _f64(kv), _f64(z)
    T, c = kv.shape
    assert c == fmt.c
    n = T // m_prime
    ent = np.zeros((n, c))
    wts = np.zeros((n, m_prime, c)) if want_weights else None
    f = fmt._c()
    _L().orc_hca_compress(T, m_prime, ctypes.byref(f), _ptr(kv), _ptr(z), z.shape[1], pos0,
                          _ptr(ent), _ptr(wts))
    return (ent, wts) if want_weights else ent


def window_rows(kv, fmt: Fmt, pos0: int = 0) -> np.ndarray:
    """Stored window rows: RoPE at pos0+j of RMSNorm(kv[j])."""
    kv = _f64(kv)
    out = np.zeros_like(kv)
    f = fmt._c()
    _L().orc_window_rows(kv.shape[0], ctypes.byref(f), _ptr(kv), pos0, _ptr(out))
    return out


def _pos(q_pos, Tq):
    if q_pos is None:
        q_pos = np.arange(Tq)
    return np.ascontiguousarray(np.asarray(q_pos, dtype=np.int64).reshape(Tq))


def indexer_scores(q_I, w, k_I, m: int, q_pos=None) -> np.ndarray:
    """Lightning-indexer scores [Tq, N]; -inf where the entry is not visible."""
    q_I, w, k_I = _f64(q_I), _f64(w), _f64(k_I)
    Tq, HI, dI = q_I.shape
    N = k_I.shape[0]
    qp = _pos(q_pos, Tq)
    sc = np.empty((Tq, N))
    _L().orc_indexer_scores(Tq, HI, dI, N, _ptr(q_I), _ptr(w), _ptr(k_I), _ptr(qp), m, _ptr(sc))
    return sc


def topk(scores, k: int, m: int, q_pos=None) -> np.ndarray:
    """Causal top-k of each row: [Tq, k] int32, ascending, -1 padded."""
    scores = _f64(scores)
    Tq, N = scores.shape
    qp = _pos(q_pos, Tq)
    idx = np.empty((Tq, k), dtype=np.int32)
    _L().orc_topk(Tq, N, _ptr(scores), _ptr(qp), m, k, _ptr(idx))
    return idx


def attention(q, entries, win, fmt: Fmt, n_win: int, idx=None, m_dense: int = 0, sink=None,
              q_pos=None, win_pos0: int = 0, scale: float = 0.0, want_lse=False):
    """Shared-KV MQA over selected (idx) or all visible (m_dense) entries plus the
    window, with sink.  q: [Tq, H, c]; returns out [Tq, H, c] (and lse [Tq, H])."""
    q = _f64(q)
    Tq, H, c = q.shape
    entries = _f64(entries).reshape(-1, c)
    win = _f64(win).reshape(-1, c)
    qp = _pos(q_pos, Tq)
    if idx is not None:
        idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(Tq, -1))
        k = idx.shape[1]
    else:
        k = 0
        assert m_dense > 0
    sk = None if sink is None else _f64(sink).reshape(H)
    out = np.zeros((Tq, H, c))
    lse = np.zeros((Tq, H)) if want_lse else None
    f = fmt._c()
    _L().orc_attention(Tq, H, ctypes.byref(f), _ptr(q), _ptr(qp), _ptr(entries), entries.shape[0],
                       _ptr(idx), k, m_dense, _ptr(win), win.shape[0], win_pos0, n_win, _ptr(sk),
                       float(scale), _ptr(out), _ptr(lse))
    return (out, lse) if want_lse else out


def csa_layer(inp: dict, fmt: Fmt, m: int, k: int, n_win: int, rows=None):
    """The whole CSA prefill path for one sequence: compress, indexer, top-k,
    attention.  ``rows`` restricts the attention (and indexer) to those query
    rows.  Returns dict(entries, win, idx, out)."""
    ent = csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], m, fmt)
    win = window_rows(inp["kv_a"], fmt)
    T = inp["kv_a"].shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    sc = indexer_scores(np.asarray(inp["q_I"])[rows], np.asarray(inp["w"])[rows], inp["k_I"], m,
                        q_pos=rows)
    idx = topk(sc, k, m, q_pos=rows)
    out = attention(np.asarray(inp["q"])[rows], ent, win, fmt, n_win, idx=idx, sink=inp.get("sink"),
                    q_pos=rows)
    return dict(entries=ent, win=win, idx=idx, scores=sc, out=out)


# ---- (next) block-scaled FP8 indexer inputs --------------------------------

def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 (FN) code."""
    return float(_L().orc_e4m3_value(int(code)))


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code (ties to the even code, saturating at +-448)."""
    return int(_L().orc_e4m3_encode(float(x)))


def mxfp8_quantize(x):
    """OCP MX quantization along the last axis (a multiple of 32): returns
    (codes uint8 with x's shape, scale exponents int32 [..., n/32])."""
    x = _f64(x)
    assert x.shape[-1] % 32 == 0
    codes = np.empty(x.shape, dtype=np.uint8)
    exps = np.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=np.int32)
    _L().orc_mxfp8_quantize(x.size, _ptr(x), _ptr(codes), _ptr(exps))
    return codes, exps


def mxfp8_dequantize(codes, exps) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exps = np.ascontiguousarray(exps, dtype=np.int32)
    y = np.empty(codes.shape)
    _L().orc_mxfp8_dequantize(codes.size, _ptr(codes), _ptr(exps), _ptr(y))
    return y


def mxfp8_indexer_scores(q_I, w, k_I, m: int, q_pos=None) -> np.ndarray:
    """Indexer scores with q_I and K_I passed through MX-FP8 (blocks of 32
    along the indexer dim); the products and sums stay in float64."""
    qd = mxfp8_dequantize(*mxfp8_quantize(q_I))
    kd = mxfp8_dequantize(*mxfp8_quantize(k_I))
    return indexer_scores(qd, w, kd, m, q_pos=q_pos)


def e2m1_value(code: int) -> float:
    """Value of an FP4 E2M1 code (4 bits)."""
    return float(_L().orc_e2m1_value(int(code)))


def e2m1_encode(x: float) -> int:
    """Nearest E2M1 code (ties to the even code, saturating at +-6)."""
    return int(_L().orc_e2m1_encode(float(x)))


def mxfp4_quantize(x):
    """OCP MX quantization with E2M1 elements along the last axis (a multiple
    of 32): (codes uint8 holding 4-bit codes, scale exponents int32)."""
    x = _f64(x)
    assert x.shape[-1] % 32 == 0
    codes = np.empty(x.shape, dtype=np.uint8)
    exps = np.empty(x.shape[:-1] + (x.shape[-1] // 32,), dtype=np.int32)
    _L().orc_mxfp4_quantize(x.size, _ptr(x), _ptr(codes), _ptr(exps))
    return codes, exps


def mxfp4_dequantize(codes, exps) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exps = np.ascontiguousarray(exps, dtype=np.int32)
    y = np.empty(codes.shape)
    _L().orc_mxfp4_dequantize(codes.size, _ptr(codes), _ptr(exps), _ptr(y))
    return y


def nvfp4_quantize(x):
    """FP4 with E4M3 scales per 16 elements and one float scale for the whole
    array: (codes uint8 [x.shape], block scales uint8 [n/16], tensor scale)."""
    x = _f64(x)
    assert x.size % 16 == 0
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.size // 16, dtype=np.uint8)
    g = ctypes.c_double(0.0)
    _L().orc_nvfp4_quantize(x.size, _ptr(x), _ptr(codes), _ptr(scales), ctypes.byref(g))
    return codes, scales, g.value


def nvfp4_dequantize(codes, scales, gscale) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.empty(codes.shape)
    _L().orc_nvfp4_dequantize(codes.size, _ptr(codes), _ptr(scales), float(gscale), _ptr(y))
    return y


def nvfp4_indexer_scores(q_I, w, k_I, m: int, q_pos=None) -> np.ndarray:
    """Indexer scores with q_I and K_I passed through the 16-element-block FP4
    layout (one tensor scale each); float64 products and sums."""
    qd = nvfp4_dequantize(*nvfp4_quantize(q_I))
    kd = nvfp4_dequantize(*nvfp4_quantize(k_I))
    return indexer_scores(qd, w, kd, m, q_pos=q_pos)


def mxfp4_indexer_scores(q_I, w, k_I, m: int, q_pos=None) -> np.ndarray:
    """Indexer scores with q_I and K_I passed through MX-FP4 (blocks of 32
    along the indexer dim); the products and sums stay in float64."""
    qd = mxfp4_dequantize(*mxfp4_quantize(q_I))
    kd = mxfp4_dequantize(*mxfp4_quantize(k_I))
    return indexer_scores(qd, w, kd, m, q_pos=q_pos)


# ---- (next) streaming compression for decode ---------------------------------

class Stream:
    """One sequence's compression state for decode: tokens arrive one at a
    time; each yields its window row, and the token that completes block s
    also yields entry s.  ``overlap`` selects CSA (two groups, the previous
    block's group b) or HCA (one group)."""

    def __init__(self, m: int, fmt: Fmt, z_cols: int, overlap: bool = True, pos0: int = 0):
        self.m, self.fmt, self.z_cols, self.overlap, self.pos0 = m, fmt, z_cols, overlap, pos0
        self.state = np.zeros(_L().orc_stream_state_len(m, fmt.c, z_cols))

    def append(self, kv_a, z_a, kv_b=None, z_b=None):
        kv_a, z_a = _f64(kv_a).reshape(-1), _f64(z_a).reshape(-1)
        if self.overlap:
            kv_b, z_b = _f64(kv_b).reshape(-1), _f64(z_b).reshape(-1)
        win = np.empty(self.fmt.c)
        ent = np.empty(self.fmt.c)
        f = self.fmt._c()
        done = _L().orc_stream_append(self.m, int(self.overlap), ctypes.byref(f), self.pos0,
                                      _ptr(kv_a), _ptr(kv_b), _ptr(z_a), _ptr(z_b), self.z_cols,
                                      _ptr(self.state), _ptr(win), _ptr(ent))
        return win, (ent if done else None)


# ---- (next) mixed BF16 / FP8 storage of KV entries ----------------------------

def bf16_round(x: float) -> float:
    """Nearest BF16 value (ties to even)."""
    return float(_L().orc_bf16_round(float(x)))


def mixed_store(entries, rope_dims: int):
    """Entries [n, c] -> (FP8 codes [n, c-r], MX exponents [n, (c-r)/32],
    BF16 RoPE dims [n, r] as float64)."""
    x = _f64(entries)
    n, c = x.shape
    cq = c - rope_dims
    assert cq % 32 == 0
    codes = np.empty((n, cq), dtype=np.uint8)
    exps = np.empty((n, cq // 32), dtype=np.int32)
    rope_part = np.empty((n, rope_dims))
    _L().orc_mixed_store(n, c, rope_dims, _ptr(x), _ptr(codes), _ptr(exps), _ptr(rope_part))
    return codes, exps, rope_part


def mixed_load(codes, exps, rope_part) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    exps = np.ascontiguousarray(exps, dtype=np.int32)
    rope_part = _f64(rope_part)
    n, cq = codes.shape
    r = rope_part.shape[1]
    out = np.empty((n, cq + r))
    _L().orc_mixed_load(n, cq + r, r, _ptr(codes), _ptr(exps), _ptr(rope_part), _ptr(out))
    return out


# ---- (next) grouped output projection ----------------------------------------

def grouped_output_projection(o, w_group, w_out) -> np.ndarray:
    """The attention output's grouped projection (page "DeepSeek-V4：迈向高效
    百万 Token 上下文智能", §3.3, CSA paragraph: c n_h is large, so the heads'
    outputs are first projected group by group to an intermediate dim d_g,
    then concatenated and projected back to d).  Reading taken: the H heads
    split into g consecutive groups of H/g heads.

    o: [T, H, c]; w_group: [g, d_g, (H/g) c]; w_out: [d, g d_g].  Returns
    [T, d] = w_out . concat_j(w_group[j] . concat(o[:, heads of group j]))."""
    o, w_group, w_out = _f64(o), _f64(w_group), _f64(w_out)
    T, H, c = o.shape
    g, dg, gin = w_group.shape
    assert H % g == 0 and gin == (H // g) * c and w_out.shape[1] == g * dg
    u = o.reshape(T, g, (H // g) * c)                     # each group's heads, concatenated
    v = np.einsum("tgi,gdi->tgd", u, w_group)            # [T, g, d_g]
    return v.reshape(T, g * dg) @ w_out.T
