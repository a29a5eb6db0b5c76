"""GPU parity of the streaming compression calls (csa_compress_append,
hca_compress_append) against the oracle's streaming compression, which is
itself pinned to reproduce the batch compression bit for bit.  Tokens arrive
one per sequence per call; window rows every call, an entry on every block's
last token."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_close, f64
import long_context_attention_csa_b200 as csa
from long_context_attention_csa_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _fmts(c, r):
    return csa.Fmt(c=c, rope_dims=r), oracle.Fmt(c=c, rope_dims=r)


def _per_token(x):
    """[B, T, n] -> [T, B, n] so that token t of every sequence is one
    contiguous [B, n] slice."""
    return x.transpose(0, 1).contiguous()


def _run_stream(overlap, B, T, m, c, r, dtype, zc, pos0, n_cap=None, seed=0):
    gf, of = _fmts(c, r)
    kv_a = wl.randn((B, T, c), seed + 1, DEV, dtype=dtype)
    z_a = wl.randn((B, T, zc), seed + 2, DEV, dtype=dtype)
    kv_b = wl.randn((B, T, c), seed + 3, DEV, dtype=dtype) if overlap else None
    z_b = wl.randn((B, T, zc), seed + 4, DEV, dtype=dtype) if overlap else None
    n_cap = T // m if n_cap is None else n_cap
    state = csa.stream_state(B, m, overlap, c, zc, dtype)
    entries = torch.full((B, max(n_cap, 1), c), float("nan"), dtype=dtype, device=DEV)[:, :n_cap]
    entries = entries.contiguous()
    ta, tz = _per_token(kv_a), _per_token(z_a)
    tb, tzb = (_per_token(kv_b), _per_token(z_b)) if overlap else (None, None)
    wins = torch.empty((T, B, c), dtype=dtype, device=DEV)
    ws = csa.workspace(256)
    for t in range(T):
        if overlap:
            csa.csa_compress_append(ta[t], tb[t], tz[t], tzb[t], m, gf, state, entries, pos0=pos0,
                                    win_out=wins[t], ws=ws)
        else:
            csa.hca_compress_append(ta[t], tz[t], m, gf, state, entries, pos0=pos0,
                                    win_out=wins[t], ws=ws)
    torch.cuda.synchronize()
    return dict(kv_a=kv_a, kv_b=kv_b, z_a=z_a, z_b=z_b, state=state, entries=entries,
                wins=wins.transpose(0, 1), ws=ws, fmt=of)


def _oracle_stream(d, b, m, overlap, zc, pos0, T):
    s = oracle.Stream(m, d["fmt"], zc, overlap=overlap, pos0=pos0)
    wins, ents = [], []
    for t in range(T):
        w_, e_ = s.append(f64(d["kv_a"][b, t]), f64(d["z_a"][b, t]),
                          f64(d["kv_b"][b, t]) if overlap else None,
                          f64(d["z_b"][b, t]) if overlap else None)
        wins.append(w_)
        if e_ is not None:
            ents.append(e_)
    return np.stack(wins), (np.stack(ents) if ents else np.zeros((0, d["fmt"].c)))


@pytest.mark.parametrize("B,T,m,c,r,dtype,zc,pos0", [
    (3, 203, 4, 512, 64, torch.bfloat16, 512, 0),     # the workloads' CSA format, ragged tail
    (2, 130, 4, 512, 64, torch.bfloat16, 1, 7),       # per-token scalar logits, pos0 != 0
    (1, 77, 4, 64, 32, torch.float32, 64, 0),         # the tiny float32 format
])
def test_csa_stream_matches_the_oracle(B, T, m, c, r, dtype, zc, pos0):
    d = _run_stream(True, B, T, m, c, r, dtype, zc, pos0)
    assert csa.csa_check_status(d["ws"]) == (csa.CSA_OK, 0)
    st = d["state"][:, :8].contiguous().view(torch.int64).cpu()
    assert torch.equal(st[:, 0], torch.full((B,), T, dtype=torch.int64))
    for b in range(B):
        rw, re = _oracle_stream(d, b, m, True, zc, pos0, T)
        assert re.shape[0] == T // m
        assert_close(d["wins"][b], rw, dtype, f"stream window rows b={b}")
        assert_close(d["entries"][b], re, dtype, f"stream entries b={b}")
        # the batch compression of the whole sequence gives the same entries
        ref = oracle.csa_compress(f64(d["kv_a"][b]), f64(d["kv_b"][b]), f64(d["z_a"][b]),
                                  f64(d["z_b"][b]), m, d["fmt"], pos0=pos0)
        assert_close(d["entries"][b], ref, dtype, f"stream vs batch entries b={b}")


@pytest.mark.parametrize("B,T,mp,zc", [(2, 300, 128, 512), (2, 100, 16, 512), (1, 70, 32, 1)])
def test_hca_stream_matches_the_oracle(B, T, mp, zc):
    d = _run_stream(False, B, T, mp, 512, 64, torch.bfloat16, zc, 0, seed=10)
    assert csa.csa_check_status(d["ws"]) == (csa.CSA_OK, 0)
    for b in range(B):
        rw, re = _oracle_stream(d, b, mp, False, zc, 0, T)
        assert_close(d["wins"][b], rw, torch.bfloat16, f"hca stream window rows b={b}")
        assert_close(d["entries"][b], re, torch.bfloat16, f"hca stream entries b={b}")


def test_stream_rows_do_not_depend_on_the_batch():
    """Sequence 1 streamed alone gives bitwise the entries and window rows it
    gets inside a batch of three."""
    full = _run_stream(True, 3, 41, 4, 512, 64, torch.bfloat16, 512, 0, seed=20)
    gf, _ = _fmts(512, 64)
    state = csa.stream_state(1, 4, True, 512, 512, torch.bfloat16)
    ent = torch.empty((1, 10, 512), dtype=torch.bfloat16, device=DEV)
    ws = csa.workspace(256)
    for t in range(41):
        w_ = csa.csa_compress_append(full["kv_a"][1:2, t].contiguous(),
                                     full["kv_b"][1:2, t].contiguous(),
                                     full["z_a"][1:2, t].contiguous(),
                                     full["z_b"][1:2, t].contiguous(), 4, gf, state, ent,
                                     want_win=True, ws=ws)
        assert torch.equal(w_[0], full["wins"][1, t])
    assert torch.equal(ent[0], full["entries"][1])
    assert csa.csa_check_status(ws) == (csa.CSA_OK, 0)


def test_stream_full_cache_and_bad_state_are_flagged():
    """An entry beyond the cache's capacity is dropped and a state with a
    negative token count is skipped; both record CSA_DEV_STREAM, and the
    entries that fit are still right."""
    d = _run_stream(True, 2, 21, 4, 512, 64, torch.bfloat16, 512, 0, n_cap=3, seed=30)
    assert csa.csa_check_status(d["ws"]) == (csa.CSA_E_DEVICE, csa.CSA_DEV_STREAM)
    for b in range(2):
        _, re = _oracle_stream(d, b, 4, True, 512, 0, 21)
        assert_close(d["entries"][b], re[:3], torch.bfloat16, f"capped entries b={b}")
    gf, _ = _fmts(512, 64)
    state = csa.stream_state(2, 4, True, 512, 512, torch.bfloat16)
    state[1, :8] = torch.tensor([-5], dtype=torch.int64).view(torch.uint8).to(DEV)
    before = state[1].clone()
    ent = torch.zeros((2, 4, 512), dtype=torch.bfloat16, device=DEV)
    x = wl.randn((2, 512), 40, DEV, dtype=torch.bfloat16)
    win = torch.zeros((2, 512), dtype=torch.bfloat16, device=DEV)
    ws = csa.workspace(256)
    csa.csa_compress_append(x, x, x, x, 4, gf, state, ent, win_out=win, ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_E_DEVICE, csa.CSA_DEV_STREAM)
    assert torch.equal(state[1], before)               # the bad sequence untouched
    assert torch.count_nonzero(win[1]) == 0
    assert int(state[0, :8].contiguous().view(torch.int64)[0]) == 1


def _prefilled(overlap, B, L, m, c, dtype, seed):
    """Stream states positioned at token L - 1 (the last of a block when m
    divides L), tail rows drawn N(0,1): a decode step at the end of an
    L-token context."""
    st = csa.stream_state(B, m, overlap, c, c, dtype)
    groups = 3 if overlap else 1
    n = groups * m * 2 * c
    rows = wl.randn((B, n), seed, DEV, dtype=dtype)
    st[:, 16:16 + n * 2] = rows.view(torch.uint8).view(B, n * 2)
    st[:, :8] = torch.tensor([L - 1] * B, dtype=torch.int64).view(torch.uint8).view(B, 8).to(DEV)
    return st


def _oracle_state(gpu_state_row, t, m, c, overlap):
    """The oracle's stream state (t, cur_a, cur_b, prev_b, cur_za, cur_zb,
    prev_zb as float64) holding the same tail rows as a GPU state."""
    x = f64(gpu_state_row[16:].view(torch.bfloat16))
    s = np.zeros(1 + 6 * m * c)
    s[0] = t
    s0 = s[1:]
    if overlap:
        par = (t // m) & 1
        ra = x[:m * c]
        rb = x[m * c:3 * m * c].reshape(2, m * c)
        za = x[3 * m * c:4 * m * c]
        zb = x[4 * m * c:6 * m * c].reshape(2, m * c)
        s0[0:m * c] = ra
        s0[m * c:2 * m * c] = rb[par]
        s0[2 * m * c:3 * m * c] = rb[par ^ 1]
        s0[3 * m * c:4 * m * c] = za
        s0[4 * m * c:5 * m * c] = zb[par]
        s0[5 * m * c:6 * m * c] = zb[par ^ 1]
    else:
        s0[0:m * c] = x[:m * c]
        s0[3 * m * c:4 * m * c] = x[m * c:2 * m * c]
    return s


@pytest.mark.parametrize("overlap,B,L,m", [(True, 32, 131072, 4), (False, 4, 1 << 20, 128)])
def test_stream_decode_step_at_full_context(overlap, B, L, m):
    """The decode workloads' step: each sequence's token L - 1 completes a
    block (CSA: entry 32767 of a 128K context at position 131068; HCA: entry
    8191 of a 1M context at position 2^20 - 128), pooled from a filled tail
    buffer; window row at position L - 1."""
    c, dt = 512, torch.bfloat16
    gf, of = _fmts(c, 64)
    st = _prefilled(overlap, B, L, m, c, dt, 50)
    host_states = [st[b].cpu() for b in range(B)]
    x = [wl.randn((B, c), 51 + i, DEV, dtype=dt) for i in range(4)]
    n_cap = L // m
    ent = torch.zeros((B, n_cap, c), dtype=dt, device=DEV)
    win = torch.empty((B, c), dtype=dt, device=DEV)
    ws = csa.workspace(256)
    if overlap:
        csa.csa_compress_append(x[0], x[1], x[2], x[3], m, gf, st, ent, win_out=win, ws=ws)
    else:
        csa.hca_compress_append(x[0], x[2], m, gf, st, ent, win_out=win, ws=ws)
    assert csa.csa_check_status(ws) == (csa.CSA_OK, 0)
    for b in range(B):
        s = oracle.Stream(m, of, c, overlap=overlap)
        s.state = _oracle_state(host_states[b], L - 1, m, c, overlap)
        rw, re = s.append(f64(x[0][b]), f64(x[2][b]), f64(x[1][b]) if overlap else None,
                          f64(x[3][b]) if overlap else None)
        assert re is not None
        assert_close(win[b], rw, dt, f"decode window row b={b}")
        assert_close(ent[b, n_cap - 1], re, dt, f"decode entry b={b}")
    assert torch.count_nonzero(ent[:, :n_cap - 1]) == 0
