"""Seeded synthetic inputs for the CSA/HCA attention-layer core.

This module only DRAWS numbers: it holds none of the method's arithmetic, so
that both the CUDA path and the float64 oracle can take the same tensors.  Each
tensor is drawn as float32 N(0,1) (or uniform integers) from its own seeded
``torch.Generator`` on the requested device, scaled, and rounded once to the
workload's dtype (round to nearest even).  Full-size workloads are drawn on the
GPU; the oracle then receives host copies of exactly those drawn values.

The five workloads follow the shapes and value distributions of the pages'
models: V4-Flash-like (64 query heads, top-k 512) and V4-Pro-like (128 query
heads, top-k 1024) attention layers, entry dim 512 with RoPE on the last 64
dims, CSA rate 1/4 and HCA rate 1/128, a 128-token window.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

# tensor ids: each tensor of a workload gets its own stream seed_base + id
_TID = dict(kv_a=1, kv_b=2, z_a=3, z_b=4, q=5, q_I=6, k_I=7, w=8, sink=9, entries=10, win=11,
            kv=12, z=13, idx=14, hca_entries=15, hca_win=16, hca_q=17, hca_sink=18,
            o=19, w_group=20, w_out=21)

# Grouped output projection of the 64-head (V4-Flash-like) layer: model dim
# d = 4096 (the pages' model table); g = 8 groups of 8 heads and d_g = 1024
# are the reading taken (the pages give the map's shape, not its sizes).
PROJ = dict(g=8, d_g=1024, d=4096)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # csa_prefill | hca_prefill | csa_decode | decode_pair
    dtype: torch.dtype
    B: int
    T: int                    # prefill tokens, or context length L for decode
    H: int                    # query heads
    c: int = 512              # entry dim
    r: int = 64               # RoPE dims (the last r of c)
    rope_base: float = 10000.0
    m: int = 4                # CSA rate
    m_prime: int = 128        # HCA rate
    HI: int = 64              # indexer heads
    dI: int = 128             # indexer dim
    k: int = 512              # top-k
    n_win: int = 128
    sink: bool = True
    q_scale: float = 1.0
    qI_scale: float = 1.0
    kI_scale: float = 1.0
    w_scale: float = 1.0 / 8
    seed: int = 0
    per_sequence_seeds: bool = False
    note: str = ""

    @property
    def n_csa(self) -> int:
        return self.T // self.m

    @property
    def n_hca(self) -> int:
        return self.T // self.m_prime


WORKLOADS = {
    # Tiny CSA layer, fp32: every dotted input scaled by 1/sqrt(its dim).
    "tiny_csa_fp32": Workload(
        "tiny_csa_fp32", "csa_prefill", torch.float32, B=1, T=256, H=4, c=64, r=32, m=4, HI=2,
        dI=32, k=16, n_win=16, q_scale=1 / 8, qI_scale=1 / math.sqrt(32),
        kI_scale=1 / math.sqrt(32), w_scale=1.0, seed=0),
    # CSA prefill, V4-Flash-like head count and top-k.
    "csa_prefill_8k": Workload(
        "csa_prefill_8k", "csa_prefill", torch.bfloat16, B=1, T=8192, H=64, k=512, seed=0),
    # HCA prefill at 64K tokens: 512 entries, dense.
    "hca_prefill_64k": Workload(
        "hca_prefill_64k", "hca_prefill", torch.bfloat16, B=1, T=65536, H=64, w_scale=1.0, seed=0),
    # CSA decode: 32 sequences of 128K context, one query each.
    "csa_decode_b32_128k": Workload(
        "csa_decode_b32_128k", "csa_decode", torch.bfloat16, B=32, T=131072, H=64, k=1024,
        seed=0, per_sequence_seeds=True),
    # 1M-context decode layer pair (one CSA layer then one HCA layer), 128 heads.
    "decode_pair_b4_1m": Workload(
        "decode_pair_b4_1m", "decode_pair", torch.bfloat16, B=4, T=1 << 20, H=128, k=1024,
        seed=0, per_sequence_seeds=True),
}


def scaled(w: Workload, **kw) -> Workload:
    """A smaller or altered copy of a workload (for parity tests)."""
    return replace(w, **kw)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn(shape, seed, device="cpu", scale=1.0, dtype=torch.float32):
    """float32 N(0,1) draws times ``scale``, rounded once to ``dtype``."""
    x = torch.randn(shape, generator=_gen(device, seed), device=device, dtype=torch.float32)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def randint_like_float(shape, seed, lo, hi, device="cpu", dtype=torch.float32):
    """Integer values in [lo, hi) stored as floats (exact in bf16 and fp32)."""
    x = torch.randint(lo, hi, shape, generator=_gen(device, seed), device=device)
    return x.to(dtype)


def _seed(w: Workload, name: str, b: int = 0) -> int:
    base = w.seed * 1000 + _TID[name] * 100003
    return base + (b if w.per_sequence_seeds else 0)


def _draw(w: Workload, name, shape, device, scale=1.0, dtype=None):
    dtype = w.dtype if dtype is None else dtype
    if not w.per_sequence_seeds:
        return randn(shape, _seed(w, name), device, scale, dtype)
    parts = [randn(shape[1:], _seed(w, name, b), device, scale, dtype) for b in range(shape[0])]
    return torch.stack(parts)


def csa_prefill_inputs(w: Workload, device="cpu"):
    """Token KV groups a/b, their compression logits, queries, indexer inputs,
    head weights and sinks for a CSA layer over T tokens (batch B)."""
    B, T, H, c = w.B, w.T, w.H, w.c
    n = w.n_csa
    return dict(
        kv_a=_draw(w, "kv_a", (B, T, c), device),
        kv_b=_draw(w, "kv_b", (B, T, c), device),
        z_a=_draw(w, "z_a", (B, T, c), device),
        z_b=_draw(w, "z_b", (B, T, c), device),
        q=_draw(w, "q", (B, T, H, c), device, w.q_scale),
        q_I=_draw(w, "q_I", (B, T, w.HI, w.dI), device, w.qI_scale),
        k_I=_draw(w, "k_I", (B, n, w.dI), device, w.kI_scale),
        w=_draw(w, "w", (B, T, w.HI), device, w.w_scale, dtype=torch.float32),
        sink=randn((H,), _seed(w, "sink"), device) if w.sink else None,
    )


def hca_prefill_inputs(w: Workload, device="cpu"):
    """Per-token KV, its compression logits, queries and sinks for an HCA layer."""
    B, T, H, c = w.B, w.T, w.H, w.c
    return dict(
        kv=_draw(w, "kv", (B, T, c), device),
        z=_draw(w, "z", (B, T, c), device),
        q=_draw(w, "q", (B, T, H, c), device, w.q_scale),
        sink=randn((H,), _seed(w, "sink"), device) if w.sink else None,
    )


def csa_decode_inputs(w: Workload, device="cpu"):
    """Decode: one query per sequence at position L-1 over a filled cache of
    stored compressed entries, indexer keys and the last n_win window rows."""
    B, L, H, c = w.B, w.T, w.H, w.c
    n = w.n_csa
    return dict(
        entries=_draw(w, "entries", (B, n, c), device),
        k_I=_draw(w, "k_I", (B, n, w.dI), device, w.kI_scale),
        win=_draw(w, "win", (B, w.n_win, c), device),
        q=_draw(w, "q", (B, 1, H, c), device, w.q_scale),
        q_I=_draw(w, "q_I", (B, 1, w.HI, w.dI), device, w.qI_scale),
        w=_draw(w, "w", (B, 1, w.HI), device, w.w_scale, dtype=torch.float32),
        sink=randn((H,), _seed(w, "sink"), device) if w.sink else None,
        q_pos=torch.full((B, 1), L - 1, dtype=torch.int64, device=device),
        win_pos0=torch.full((B,), L - w.n_win, dtype=torch.int64, device=device),
    )


def hca_decode_inputs(w: Workload, device="cpu"):
    """Decode cache of the HCA layer of a layer pair (its own entries, window,
    queries and sinks)."""
    B, L, H, c = w.B, w.T, w.H, w.c
    n = w.n_hca
    return dict(
        entries=_draw(w, "hca_entries", (B, n, c), device),
        win=_draw(w, "hca_win", (B, w.n_win, c), device),
        q=_draw(w, "hca_q", (B, 1, H, c), device, w.q_scale),
        sink=randn((H,), _seed(w, "hca_sink"), device) if w.sink else None,
        q_pos=torch.full((B, 1), L - 1, dtype=torch.int64, device=device),
        win_pos0=torch.full((B,), L - w.n_win, dtype=torch.int64, device=device),
    )


def random_index_sets(counts, k: int, seed: int, device="cpu"):
    """For each row r, a uniformly random subset of min(k, counts[r]) of
    range(counts[r]), ascending, padded with -1: valid top-k shaped index sets
    that do not depend on any scorer.  ``counts`` is a 1-D int tensor."""
    counts = torch.as_tensor(counts, dtype=torch.int64).cpu()
    g = _gen("cpu", seed)
    R = counts.numel()
    nmax = int(counts.max().item()) if R else 0
    out = torch.full((R, k), -1, dtype=torch.int32)
    if nmax == 0:
        return out.to(device)
    # random keys per (row, entry); invisible entries pushed to the end
    keys = torch.rand((R, nmax), generator=g)
    ar = torch.arange(nmax).unsqueeze(0)
    keys = torch.where(ar < counts.unsqueeze(1), keys, torch.full_like(keys, 2.0))
    kk = min(k, nmax)
    sel = torch.topk(keys, kk, dim=1, largest=False).indices
    big = 1 << 40
    sel = torch.where(sel < counts.unsqueeze(1), sel, torch.full_like(sel, big))
    sel = torch.sort(sel, dim=1).values
    sel = torch.where(sel == big, torch.full_like(sel, -1), sel)
    out[:, :kk] = sel.to(torch.int32)
    return out.to(device)


def projection_inputs(w: Workload, g: int, d_g: int, d: int, device="cpu"):
    """Attention output o [T, H, c] (N(0,1), a stand-in for the attention's
    output rows) and random synthetic projection weights scaled by
    1/sqrt(fan_in): w_group [g, d_g, (H/g) c], w_out [d, g d_g]."""
    T, H, c = w.T, w.H, w.c
    kg = (H // g) * c
    return dict(
        o=randn((T, H, c), _seed(w, "o"), device, 1.0, w.dtype),
        w_group=randn((g, d_g, kg), _seed(w, "w_group"), device, kg ** -0.5, w.dtype),
        w_out=randn((d, g * d_g), _seed(w, "w_out"), device, (g * d_g) ** -0.5, w.dtype),
    )

