"""Brute-force restatements for TINY inputs, used only to pin the oracle.

Written independently of ``oracle/csa_oracle.c`` and in a different form:
vectorised numpy over whole tensors, RoPE as multiplication by complex
exponentials, compression weights from one stacked softmax, attention as one
dense masked softmax over explicitly materialised compressed entries plus all
window rows (a [T, 1 + N + T] logit matrix with a sink column).  Source: page
"DeepSeek-V4：迈向高效百万 Token 上下文智能", §3.3, and page "DeepSeek V4 完整技术
报告", section "混合注意力：CSA + HCA" (window, sink, partial RoPE).
"""
import numpy as np


def rmsnorm(x, eps=1e-6):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope(x, pos, r, base=10000.0):
    """Rotate the last r dims, pairs as complex numbers, by pos * base^(-2i/r).
    ``pos`` broadcasts against x's leading dims."""
    x = np.array(x, dtype=np.float64, copy=True)
    c = x.shape[-1]
    pos = np.asarray(pos, dtype=np.float64)
    freqs = base ** (-np.arange(0, r, 2, dtype=np.float64) / r)  # [r/2]
    z = x[..., c - r::2] + 1j * x[..., c - r + 1::2]
    ang = pos[..., None] * freqs
    z = z * np.exp(1j * ang)
    x[..., c - r::2] = z.real
    x[..., c - r + 1::2] = z.imag
    return x


def transform(x, pos, c, r, base, eps, norm=True, rot=True):
    y = rmsnorm(x, eps) if norm else np.asarray(x, dtype=np.float64)
    return rope(y, pos, r, base) if rot else y


def csa_entries(ca, cb, za, zb, m, r, base=10000.0, eps=1e-6, pos0=0, norm=True, rot=True):
    """Stack the 2m slots of every entry, softmax over the slot axis."""
    ca, cb, za, zb = (np.asarray(a, dtype=np.float64) for a in (ca, cb, za, zb))
    T, c = ca.shape
    n = T // m
    za = np.broadcast_to(za, (T, c))
    zb = np.broadcast_to(zb, (T, c))
    va = ca[: n * m].reshape(n, m, c)
    la = za[: n * m].reshape(n, m, c)
    # group b of entry s is block s-1; entry 0 gets a -inf (absent) block
    vb = np.concatenate([np.zeros((1, m, c)), cb[: (n - 1) * m].reshape(n - 1, m, c)], axis=0)
    lb = np.concatenate([np.full((1, m, c), -np.inf), zb[: (n - 1) * m].reshape(n - 1, m, c)],
                        axis=0)
    v = np.concatenate([va, vb], axis=1)
    lg = np.concatenate([la, lb], axis=1)
    wts = np.exp(lg - lg.max(axis=1, keepdims=True))
    wts = wts / wts.sum(axis=1, keepdims=True)
    ent = (wts * v).sum(axis=1)
    pos = pos0 + m * np.arange(n)
    return transform(ent, pos, c, r, base, eps, norm, rot), wts


def hca_entries(kv, z, mp, r, base=10000.0, eps=1e-6, pos0=0, norm=True, rot=True):
    kv, z = np.asarray(kv, dtype=np.float64), np.asarray(z, dtype=np.float64)
    T, c = kv.shape
    n = T // mp
    z = np.broadcast_to(z, (T, c))
    v = kv[: n * mp].reshape(n, mp, c)
    lg = z[: n * mp].reshape(n, mp, c)
    wts = np.exp(lg - lg.max(axis=1, keepdims=True))
    wts = wts / wts.sum(axis=1, keepdims=True)
    ent = (wts * v).sum(axis=1)
    return transform(ent, pos0 + mp * np.arange(n), c, r, base, eps, norm, rot), wts


def indexer_scores(qI, w, kI, m):
    qI, w, kI = (np.asarray(a, dtype=np.float64) for a in (qI, w, kI))
    T = qI.shape[0]
    N = kI.shape[0]
    dots = np.einsum("thd,sd->ths", qI, kI)
    sc = np.einsum("th,ths->ts", w, np.maximum(dots, 0.0))
    vis = np.minimum((np.arange(T) + 1) // m, N)
    mask = np.arange(N)[None, :] < vis[:, None]
    return np.where(mask, sc, -np.inf)


def topk(scores, k):
    """Full lexicographic sort per row: key (-score, index)."""
    T, N = scores.shape
    out = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        row = scores[t]
        vis = int(np.isfinite(row).sum())
        order = np.lexsort((np.arange(vis), -row[:vis]))
        sel = np.sort(order[: min(k, vis)])
        out[t, : len(sel)] = sel
    return out


def attention_dense(q, ent, win, idx, n_win, sink, c, r, base=10000.0, eps=1e-6, scale=None,
                    m_dense=None, norm=True, rot=True):
    """One dense masked softmax per (t, h) over [sink | all entries | all window rows]."""
    q = np.asarray(q, dtype=np.float64)
    T, H, _ = q.shape
    N = ent.shape[0]
    scale = 1.0 / np.sqrt(c) if scale is None else scale
    t = np.arange(T)
    qh = transform(q, t[:, None] * np.ones((1, H)), c, r, base, eps, norm, rot)
    keys = np.concatenate([ent.reshape(N, c), win.reshape(-1, c)], axis=0)  # [N+T, c]
    mask = np.zeros((T, N + win.shape[0]), dtype=bool)
    if idx is not None:
        for tt in range(T):
            sel = idx[tt][idx[tt] >= 0]
            mask[tt, sel] = True
    else:
        vis = np.minimum((t + 1) // m_dense, N)
        mask[:, :N] = np.arange(N)[None, :] < vis[:, None]
    j = np.arange(win.shape[0])
    mask[:, N:] = (j[None, :] <= t[:, None]) & (j[None, :] > t[:, None] - n_win)
    lg = scale * np.einsum("thc,kc->thk", qh, keys)
    lg = np.where(mask[:, None, :], lg, -np.inf)
    zs = np.full((H,), -np.inf) if sink is None else np.asarray(sink, dtype=np.float64)
    full = np.concatenate([np.broadcast_to(zs[None, :, None], (T, H, 1)), lg], axis=2)
    mx = full.max(axis=2, keepdims=True)
    e = np.exp(full - mx)
    p = e / e.sum(axis=2, keepdims=True)
    o = np.einsum("thk,kc->thc", p[:, :, 1:], keys)
    if rot:
        o = rope(o, -t[:, None] * np.ones((1, H)), r, base)
    return o
