"""Benchmark of the CSA layer prefill step on B200.

One step = the whole CSA hot path over one batch of synthetic input at the
csa_prefill_8k workload (batch 1, 8192 tokens, 64 query heads, entry dim 512
with RoPE on the last 64 dims, m = 4 -> 2048 entries, indexer 64 x 128 with
w ~ N(0,1)/8, top-k 512, window 128, per-head sinks):
    csa_compress (entries + window rows) -> indexer_scores_topk -> sparse_mqa_attn.
Prints one JSON line (see the keys below).  ``--impl reference`` times the
float64 CPU oracle on a bounded sample of the same workload instead.

Multi-GPU: one process per GPU (torchrun); the path has no exchange step, so
every rank runs its own replica of the step and ``value`` sums all ranks'
tokens over the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import long_context_attention_csa_b200 as csa  # noqa: E402
from long_context_attention_csa_b200 import workloads as wl  # noqa: E402

WORKLOAD = "csa_prefill_8k"
METRIC = "CSA/HCA layer prefill tokens/s & decode queries/s on 1 B200; % of roofline"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def attn_useful_flops(w) -> float:
    """Algorithmic FLOPs of sparse_mqa_attn: 4 * H * c per (query, key) pair,
    keys = min(k, visible entries) + window rows present."""
    t = np.arange(w.T, dtype=np.int64)
    vis = np.minimum((t + 1) // w.m, w.n_csa)
    pairs = np.minimum(w.k, vis) + np.minimum(w.n_win, t + 1)
    return float(4.0 * w.H * w.c * pairs.sum()) * w.B


def indexer_useful_flops(w) -> float:
    t = np.arange(w.T, dtype=np.int64)
    vis = np.minimum((t + 1) // w.m, w.n_csa)
    return float(2.0 * w.HI * w.dI * vis.sum()) * w.B


def compress_bytes(w) -> float:
    e = 2 if w.dtype == torch.bfloat16 else 4
    # read kv_a, kv_b, z_a, z_b; write entries and window rows
    return float(w.B * (4 * w.T * w.c + w.n_csa * w.c + w.T * w.c) * e)


class Clocks:
    """nvidia-smi sampler over the timed region."""

    def __init__(self, index: int):
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_rank{index}.csv")
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={index}",
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,"
                 "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
                 "clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        torch.distributed.init_process_group(
            "nccl" if torch.cuda.is_available() else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def allmax(x: float, ws: int) -> float:
    if ws == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        torch.distributed.barrier()


# ------------------------------------------------------------------ GPU arm

class Step:
    """Device buffers and the three calls of one CSA prefill step."""

    def __init__(self, w, device):
        self.w = w
        inp = wl.csa_prefill_inputs(w, device)
        self.inp = inp
        self.fmt = csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
        B, T, c = w.B, w.T, w.c
        self.entries = torch.empty((B, w.n_csa, c), dtype=w.dtype, device=device)
        self.win = torch.empty((B, T, c), dtype=w.dtype, device=device)
        self.idx = torch.empty((B, T, w.k), dtype=torch.int32, device=device)
        self.out = torch.empty((B, T, w.H, c), dtype=w.dtype, device=device)
        self.ws_idx = csa.workspace(csa.csa_workspace_bytes(
            csa.CSA_OP_INDEXER, w.dtype, B, T, 0, 0, w.n_csa, w.k, 0), device)
        self.ws_attn = csa.workspace(csa.csa_workspace_bytes(
            csa.CSA_OP_SPARSE_ATTN, w.dtype, B, T, w.H, c, w.n_csa, w.k, w.n_win), device)

    def run(self, inp=None, ev=None):
        inp = inp or self.inp
        w = self.w
        s = torch.cuda.current_stream()
        if ev:
            ev[0].record(s)
        csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, self.fmt,
                         entries=self.entries, win_out=self.win)
        if ev:
            ev[1].record(s)
        csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, idx_out=self.idx,
                                ws=self.ws_idx)
        if ev:
            ev[2].record(s)
        csa.sparse_mqa_attn(inp["q"], self.entries, self.idx, self.win, self.fmt, w.n_win,
                            sink=inp["sink"], out=self.out, ws=self.ws_attn)
        if ev:
            ev[3].record(s)
        return self.out


def run_gpu(args):
    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[WORKLOAD]
    step = Step(w, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # > 126 MB L2
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    st, d = csa.csa_check_status(step.ws_idx)
    st2, d2 = csa.csa_check_status(step.ws_attn)
    if st or st2:
        raise RuntimeError(f"device status after warm-up: indexer {st}/{d}, attention {st2}/{d2}")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    clocks = Clocks(local) if rank == 0 or ws > 1 else None
    launches0 = csa.csa_launch_count()
    barrier(ws)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()                       # L2 flushed between timed steps (not timed)
        step.run(ev=evs[i])
    torch.cuda.synchronize()
    barrier(ws)
    launches = csa.csa_launch_count() - launches0
    ck = clocks.stop() if clocks else None
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]),
                     e[0].elapsed_time(e[3])] for e in evs])     # ms
    step_ms = allmax(float(per[:, 3].mean()), ws)
    t_compress, t_index, t_attn = (float(per[:, i].mean()) for i in range(3))

    # e2e through the public API: pinned host inputs -> device, step, result -> host
    host = {k: (v.to("cpu").pin_memory() if v is not None else None) for k, v in step.inp.items()}
    dev_in = {k: (torch.empty_like(v, device=dev) if v is not None else None)
              for k, v in host.items()}
    out_host = torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_host.numel() * out_host.element_size()
    e2e_steps = max(1, min(K, 5))
    for _ in range(2):
        for kk, v in host.items():
            if v is not None:
                dev_in[kk].copy_(v, non_blocking=True)
        step.run(dev_in)
        out_host.copy_(step.out, non_blocking=True)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        for kk, v in host.items():
            if v is not None:
                dev_in[kk].copy_(v, non_blocking=True)
        step.run(dev_in)
        out_host.copy_(step.out, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = allmax(e0.elapsed_time(e1) / e2e_steps, ws)
    st, d = csa.csa_check_status(step.ws_attn)
    if st:
        raise RuntimeError(f"device status after timing: {st}/{d}")

    hbm, bf16, src = peaks()
    tokens = w.B * w.T
    fl_attn = attn_useful_flops(w)
    fl_idx = indexer_useful_flops(w)
    achieved = fl_attn / (t_attn * 1e-3) / 1e12
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": tokens * ws / (step_ms * 1e-3),
            "unit": "tokens/s",
            "n_gpus": ws,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": step_ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) activations, w~N(0,1)/8, sinks~N(0,1))",
            "config": {
                "workload": WORKLOAD, "batch": w.B, "seq_len": w.T, "heads": w.H,
                "entry_dim": w.c, "rope_dims": w.r, "m": w.m, "entries": w.n_csa,
                "indexer": f"{w.HI}x{w.dI}", "top_k": w.k, "n_win": w.n_win, "sink": True,
                "parallelism": f"replica x{ws}" if ws > 1 else "single GPU",
                "l2": "flushed between timed steps (256 MiB write, outside the step events)",
            },
            "stages_ms": {"csa_compress": t_compress, "indexer_scores_topk": t_index,
                          "sparse_mqa_attn": t_attn},
            "stage_roofline": {
                "csa_compress": {"bound": "hbm", "achieved_GBps":
                                 compress_bytes(w) / (t_compress * 1e-3) / 1e9, "peak": hbm},
                "indexer_scores_topk": {"bound": "tensor", "achieved_TFLOPs":
                                        fl_idx / (t_index * 1e-3) / 1e12, "peak": bf16},
            },
            "roofline": {"bound": "tensor", "kernel": "sparse_mqa_attn",
                         "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                         "frac": achieved / bf16, "traffic": None,
                         "peak_source": f"{src} bf16 burst (MEASURED_PEAKS.json)"
                         if src == "measured" else "fallback 1.59 PFLOP/s",
                         "algorithmic_flops_per_launch": fl_attn},
            "e2e": {"value": tokens * ws / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": ck,
        }
        if ws == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w, args.cpu_rows)
        print(json.dumps(line), flush=True)
    if ws > 1:
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------------ oracle arm

def cpu_baseline(w, rows: int):
    """The float64 oracle, as it stands, on a bounded sample of the workload:
    the whole CSA layer (compression of every entry and window row, then indexer,
    top-k and attention) for `rows` query rows spread evenly over the sequence.
    Reported in query tokens per second."""
    import oracle

    inp = wl.csa_prefill_inputs(w, "cpu")
    x = {k: (None if v is None else (v[0] if v.dim() > 1 else v).double().numpy())
         for k, v in inp.items()}
    sel = np.linspace(0, w.T - 1, rows).astype(np.int64)
    t0 = time.perf_counter()
    oracle.csa_layer(x, oracle.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base), w.m, w.k,
                     w.n_win, rows=sel)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows} of {w.T} query rows evenly spaced (whole layer for those rows, "
                      f"compression of the full sequence), float64, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = wl.WORKLOADS[WORKLOAD]
    import oracle

    oracle.build()
    vals = []
    rows = min(args.cpu_rows, 1024)   # per step: the K + W steps end within a few minutes
    for _ in range(max(1, args.steps)):
        vals.append(cpu_baseline(w, rows))
    args.cpu_rows = rows
    v = float(np.mean([x["value"] for x in vals]))
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * args.cpu_rows / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": os.cpu_count(),
                         "kind": "oracle", "sample": vals[0]["sample"]},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_only(args):
    """One stage of the step alone on the csa_prefill workload at --seq-len
    tokens (for kernel profiles): warm-up, then --steps timed launches."""
    torch.cuda.set_device(0)
    w = wl.scaled(wl.WORKLOADS[WORKLOAD], T=args.seq_len) if args.seq_len else wl.WORKLOADS[WORKLOAD]
    step = Step(w, torch.device("cuda", 0))
    inp = step.inp
    if args.only == "attn":
        import oracle   # valid index sets only: s < visible entries, ascending

        counts = torch.tensor([oracle.visible(t, w.m, w.n_csa) for t in range(w.T)])
        step.idx.copy_(wl.random_index_sets(counts, w.k, 5).unsqueeze(0))
        step.entries.copy_(wl.randn(step.entries.shape, 2, "cuda", dtype=w.dtype))
        step.win.copy_(wl.randn(step.win.shape, 3, "cuda", dtype=w.dtype))

    def once():
        if args.only == "compress":
            csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, step.fmt,
                             entries=step.entries, win_out=step.win)
        elif args.only == "indexer":
            csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k,
                                    idx_out=step.idx, ws=step.ws_idx)
        else:
            csa.sparse_mqa_attn(inp["q"], step.entries, step.idx, step.win, step.fmt, w.n_win,
                                sink=inp["sink"], out=step.out, ws=step.ws_attn)

    for _ in range(args.warmup):
        once()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        once()
    e1.record()
    torch.cuda.synchronize()
    print(json.dumps({"only": args.only, "seq_len": w.T, "ms": e0.elapsed_time(e1) / args.steps}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--only", choices=["compress", "indexer", "attn"], default=None,
                    help="time one stage alone (kernel profiling)")
    ap.add_argument("--seq-len", type=int, default=0, help="tokens for --only (default 8192)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=8192)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.only:
        run_only(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args)
        return
    run_gpu(args)


if __name__ == "__main__":
    main()
