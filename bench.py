"""Benchmark of the CSA layer prefill step on B200.

One step = the whole CSA hot path over one batch of synthetic input at the
csa_prefill_8k workload (batch 1, 8192 tokens, 64 query heads, entry dim 512
with RoPE on the last 64 dims, m = 4 -> 2048 entries, indexer 64 x 128 with
w ~ N(0,1)/8, top-k 512, window 128, per-head sinks):
    csa_compress (entries + window rows) -> indexer_scores_topk -> sparse_mqa_attn.
Prints one JSON line (see the keys below).  Beside the headline it carries
the HCA layer prefill step at hca_prefill_64k (hca_compress -> dense_hca_attn,
65536 tokens, 512 entries), the two decode workloads and the compression
kernels alone at 2^20 tokens, each with its roofline and a float64-oracle
baseline.  ``--impl reference`` times the float64 CPU oracle on a bounded
sample of the headline workload instead.

Multi-GPU: one process per GPU (torchrun); the path has no exchange step, so
every rank runs its own replica of the step and ``value`` sums all ranks'
tokens over the slowest rank's time ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import os
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


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one attention
# launch at 8192 query rows, from an ncu capture of the kernel source whose
# SHA-256 is given.  Reported as the roofline's `traffic` only while the
# kernel source still has that hash; otherwise null.
ATTN_TRAFFIC = {"source": "long_context_attention_csa_b200/csrc/attn_tc.cu",
                "sha256": "71432149def5493f370ffca271d31a7bb5e7127d10eacd89d6c86f35604781b0",
                "bytes_per_launch": 564.28e6 + 492.45e6}


def attn_traffic():
    import hashlib

    try:
        with open(os.path.join(ROOT, ATTN_TRAFFIC["source"]), "rb") as fh:
            h = hashlib.sha256(fh.read()).hexdigest()
    except OSError:
        return None, "kernel source not found"
    if ATTN_TRAFFIC["sha256"] is None or h != ATTN_TRAFFIC["sha256"]:
        return None, "no ncu capture of the current kernel source"
    return ATTN_TRAFFIC["bytes_per_launch"], "ncu capture of this kernel source"


class Clocks:
    """SM clock and clock-event-reason sampler over the timed region.

    NVML is read from a background thread every 2 ms (the timed region of a
    default run lasts only tens of milliseconds); the device is matched to
    torch's by UUID.  Only reads the GPU's state."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, index: int):
        import threading
        self.samples = []
        self.stop_evt = threading.Event()
        self.thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(index).uuid)
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
            self.masks = [(n, getattr(pynvml, c, 0)) for n, c in self.REASONS]
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self.stop_evt.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), float(sm), int(rs)))
            except Exception:
                pass
            self.stop_evt.wait(0.002)

    def start(self):
        import threading
        if self.nv is not None:
            self.thread = threading.Thread(target=self._run, daemon=True)
            self.thread.start()

    def stop(self, t0: float, t1: float):
        """Stops sampling; summarises the samples taken in [t0, t1] (the timed
        region), or the one nearest to it when the region is shorter than the
        sampling period."""
        if self.thread is None:
            return None
        self.stop_evt.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        inside = [x for x in self.samples if t0 <= x[0] <= t1]
        if not inside:
            inside = [min(self.samples, key=lambda x: min(abs(x[0] - t0), abs(x[0] - t1)))]
        reasons = sorted({n for _, _, rs in inside for n, m in self.masks if m and rs & m})
        return {"sm_mhz": float(np.median([sm for _, sm, _ in inside])),
                "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(inside), "source": "NVML sampled every 2 ms over the timed region"}


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
    """Max over ranks (every rank calls it, in the same order)."""
    if ws == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
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
        self.ws_comp = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_COMPRESS, w.dtype, B, T),
                                     device)

    def run(self, inp=None, ev=None, out=None):
        inp = inp or self.inp
        out = self.out if out is None else out
        w = self.w
        s = torch.cuda.current_stream()
        if ev:
            ev[0].record(s)
        csa.csa_compress(inp["kv_a"], inp["kv_b"], inp["z_a"], inp["z_b"], w.m, self.fmt,
                         entries=self.entries, win_out=self.win, ws=self.ws_comp)
        if ev:
            ev[1].record(s)
        csa.indexer_scores_topk(inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, idx_out=self.idx,
                                ws=self.ws_idx)
        if ev:
            ev[2].record(s)
        csa.sparse_mqa_attn(inp["q"], self.entries, self.idx, self.win, self.fmt, w.n_win,
                            sink=inp["sink"], out=out, ws=self.ws_attn)
        if ev:
            ev[3].record(s)
        return out


def run_gpu(args):
    ws, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.WORKLOADS[WORKLOAD]
    step = Step(w, dev)
    flush = L2Flush(dev)
    clocks = Clocks(local) if rank == 0 or ws > 1 else None
    if clocks:
        clocks.start()   # running through warm-up, so samples exist when timing starts
    for _ in range(args.warmup):
        step.run()
    torch.cuda.synchronize()
    st, d = csa.csa_check_status(step.ws_idx)
    st2, d2 = csa.csa_check_status(step.ws_attn)
    if st or st2:
        raise RuntimeError(f"device status after warm-up: indexer {st}/{d}, attention {st2}/{d2}")

    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    launches0 = csa.csa_launch_count()
    barrier(ws)
    torch.cuda.synchronize()
    t_begin = time.time()
    for i in range(K):
        flush()                       # L2 flushed between timed steps (not timed)
        step.run(ev=evs[i])
    torch.cuda.synchronize()
    barrier(ws)
    launches = csa.csa_launch_count() - launches0
    ck = clocks.stop(t_begin, time.time()) if clocks else None
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3]),
                     e[0].elapsed_time(e[3])] for e in evs])     # ms
    step_ms = allmax(float(per[:, 3].mean()), ws)
    t_compress, t_index, t_attn = (float(per[:, i].mean()) for i in range(3))

    # e2e through the public API: every step copies its inputs from pinned host
    # memory to the device, runs, and copies its output back to pinned host
    # memory.  Steps are pipelined over three streams with two sets of device
    # inputs and outputs: step i+1's inputs upload while step i computes and
    # step i-1's output downloads (the copy engines of the two directions
    # work at once); every buffer is reused only after the event of its last
    # user.  Timed from the first upload to the last download.
    host = {k: (v.to("cpu").pin_memory() if v is not None else None) for k, v in step.inp.items()}
    dev_in = [{k: (torch.empty_like(v, device=dev) if v is not None else None)
               for k, v in host.items()} for _ in range(2)]
    dev_out = [step.out, torch.empty_like(step.out)]
    out_host = [torch.empty(step.out.shape, dtype=step.out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = out_host[0].numel() * out_host[0].element_size()
    e2e_steps = max(2, K)   # the pipeline fills and drains once: K steps amortise it
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def pipelined(n):
        ev_up = [torch.cuda.Event() for _ in range(n)]
        ev_comp = [torch.cuda.Event() for _ in range(n)]
        ev_down = [torch.cuda.Event() for _ in range(n)]
        for i in range(n):
            j = i & 1
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_comp[i - 2])      # dev_in[j] no longer read
                for kk, v in host.items():
                    if v is not None:
                        dev_in[j][kk].copy_(v, non_blocking=True)
                ev_up[i].record(up)
            comp.wait_event(ev_up[i])
            if i >= 2:
                comp.wait_event(ev_down[i - 2])        # dev_out[j] downloaded
            step.run(dev_in[j], out=dev_out[j])
            ev_comp[i].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[i])
                out_host[j].copy_(dev_out[j], non_blocking=True)
                ev_down[i].record(down)
        return ev_down[n - 1]

    pipelined(2)
    torch.cuda.synchronize()
    barrier(ws)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(up)
    last = pipelined(e2e_steps)
    down.wait_event(last)
    e1.record(down)
    torch.cuda.synchronize()
    e2e_ms = allmax(e0.elapsed_time(e1) / e2e_steps, ws)
    st, d = csa.csa_check_status(step.ws_attn)
    if st:
        raise RuntimeError(f"device status after timing: {st}/{d}")

    del step, dev_in, dev_out, host, out_host
    torch.cuda.empty_cache()
    decode = {} if args.no_decode else {
        n: measure_decode(n, dev, K, args.warmup, flush, ws, ws == 1 and not args.no_cpu_baseline)
        for n in DECODE_WORKLOADS}
    proj = None if args.no_hca else measure_projection(
        dev, K, args.warmup, flush, ws, ws == 1 and not args.no_cpu_baseline)
    hca = None if args.no_hca else measure_hca_prefill(
        dev, K, args.warmup, flush, ws, ws == 1 and not args.no_cpu_baseline)
    comp_1m = None if args.no_decode else measure_compress_1m(dev, min(K, 10), args.warmup)

    hbm, bf16, src = peaks()
    tokens = w.B * w.T
    fl_attn = attn_useful_flops(w)
    fl_idx = indexer_useful_flops(w)
    achieved = fl_attn / (t_attn * 1e-3) / 1e12
    traffic, traffic_src = attn_traffic()
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
                "l2": "flushed between timed steps (256 MiB write + 256 MiB read, "
                      "outside the step events)",
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
                         "frac": achieved / bf16, "traffic": traffic,
                         "traffic_source": traffic_src,
                         "peak_source": f"{src} bf16 burst (MEASURED_PEAKS.json)"
                         if src == "measured" else "fallback 1.59 PFLOP/s",
                         "algorithmic_flops_per_launch": fl_attn},
            "e2e": {"value": tokens * ws / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps,
                    "schedule": "pinned host <-> device copies every step, pipelined over three "
                                "streams (uploads of step i+1 and the download of step i-1 "
                                "overlap step i)"},
            "gpu_launches": int(launches),
            "clocks": ck,
        }
        if decode:
            line["decode"] = decode
        if hca:
            line["hca_prefill_64k"] = hca
        if proj:
            line["out_proj_8k"] = proj
        if comp_1m:
            line["compress_1m_tokens"] = comp_1m
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


def run_only_hca(args):
    """HCA compression or dense HCA attention alone on the hca_prefill_64k
    workload at --seq-len tokens (for kernel profiles)."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w0 = wl.WORKLOADS["hca_prefill_64k"]
    w = wl.scaled(w0, T=args.seq_len) if args.seq_len else w0
    inp = wl.hca_prefill_inputs(w, dev)
    fmt = csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
    entries = torch.empty((w.B, w.n_hca, w.c), dtype=w.dtype, device=dev)
    win = torch.empty((w.B, w.T, w.c), dtype=w.dtype, device=dev)
    ws_c = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_COMPRESS, 1, w.B, w.T), dev)
    csa.hca_compress(inp["kv"], inp["z"], w.m_prime, fmt, entries=entries, win_out=win, ws=ws_c)
    out = torch.empty_like(inp["q"])
    ws = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_DENSE_ATTN, 1, w.B, w.T, w.H, w.c,
                                               w.n_hca, 0, w.n_win), dev)

    def once():
        if args.only == "hca_compress":
            csa.hca_compress(inp["kv"], inp["z"], w.m_prime, fmt, entries=entries, win_out=win,
                             ws=ws_c)
        else:
            csa.dense_hca_attn(inp["q"], entries, w.m_prime, win, fmt, w.n_win, sink=inp["sink"],
                               out=out, ws=ws)

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


def hca_attn_flops(w) -> float:
    """Algorithmic FLOPs of dense_hca_attn: 4 * H * c per (query, key) pair,
    keys = every visible entry + the window rows present."""
    t = np.arange(w.T, dtype=np.int64)
    vis = np.minimum((t + 1) // w.m_prime, w.n_hca)
    pairs = vis + np.minimum(w.n_win, t + 1)
    return float(4.0 * w.H * w.c * pairs.sum()) * w.B


def hca_compress_bytes(w) -> float:
    # read kv and z; write entries and window rows
    return float(w.B * (2 * w.T * w.c + w.n_hca * w.c + w.T * w.c) * 2)


def hca_cpu_baseline(w, inp, rows: int):
    """The float64 oracle on a stratified sample of the HCA prefill workload:
    compression of the whole sequence (entries and window rows), then dense
    attention for `rows` query rows evenly spaced over the sequence (first and
    last included).  Query tokens per second."""
    import oracle

    fmt = oracle.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
    kv, z = inp["kv"][0].double().cpu().numpy(), inp["z"][0].double().cpu().numpy()
    sel = np.linspace(0, w.T - 1, rows).astype(np.int64)
    q = inp["q"][0][torch.from_numpy(sel).to(inp["q"].device)].double().cpu().numpy()
    sink = inp["sink"].double().cpu().numpy()
    t0 = time.perf_counter()
    ent = oracle.hca_compress(kv, z, w.m_prime, fmt)
    win = oracle.window_rows(kv, fmt)
    oracle.attention(q, ent, win, fmt, w.n_win, m_dense=w.m_prime, sink=sink, q_pos=sel)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{rows} of {w.T} query rows evenly spaced (compression of the whole "
                      f"sequence, dense attention for those rows), float64, {dt:.1f} s"}


def measure_hca_prefill(dev, steps: int, warmup: int, flush, ws_n: int, cpu: bool,
                        cpu_rows: int = 4096):
    """The HCA layer prefill step at hca_prefill_64k (65536 tokens, m' = 128 ->
    512 entries, 64 heads, entry dim 512, window 128, sinks):
    hca_compress (entries + window rows) -> dense_hca_attn.  Tokens/s of the
    whole step (max over ranks), each stage's time from CUDA events on the
    launching stream, and the dense attention kernel's tensor roofline."""
    w = wl.WORKLOADS["hca_prefill_64k"]
    inp = wl.hca_prefill_inputs(w, dev)
    fmt = csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
    entries = torch.empty((w.B, w.n_hca, w.c), dtype=w.dtype, device=dev)
    win = torch.empty((w.B, w.T, w.c), dtype=w.dtype, device=dev)
    out = torch.empty_like(inp["q"])
    ws_c = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_COMPRESS, 1, w.B, w.T), dev)
    ws_a = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_DENSE_ATTN, 1, w.B, w.T, w.H, w.c,
                                                 w.n_hca, 0, w.n_win), dev)
    s = torch.cuda.current_stream()

    def run(ev=None):
        if ev:
            ev[0].record(s)
        csa.hca_compress(inp["kv"], inp["z"], w.m_prime, fmt, entries=entries, win_out=win,
                         ws=ws_c)
        if ev:
            ev[1].record(s)
        csa.dense_hca_attn(inp["q"], entries, w.m_prime, win, fmt, w.n_win, sink=inp["sink"],
                           out=out, ws=ws_a)
        if ev:
            ev[2].record(s)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    for ws in (ws_c, ws_a):
        st, d = csa.csa_check_status(ws)
        if st:
            raise RuntimeError(f"hca_prefill_64k: device status {st}/{d}")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    for i in range(steps):
        flush()          # L2 flushed between timed steps (not timed)
        run(evs[i])
    torch.cuda.synchronize()
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[0].elapsed_time(e[2])]
                    for e in evs])
    step_ms = allmax(float(per[:, 2].mean()), ws_n)
    t_comp, t_attn = float(per[:, 0].mean()), float(per[:, 1].mean())
    st, d = csa.csa_check_status(ws_a)
    if st:
        raise RuntimeError(f"hca_prefill_64k: device status {st}/{d}")
    hbm, bf16, src = peaks()
    fl = hca_attn_flops(w)
    achieved = fl / (t_attn * 1e-3) / 1e12
    res = {
        "value": w.B * w.T * ws_n / (step_ms * 1e-3), "unit": "tokens/s", "ms_per_step": step_ms,
        "config": {"workload": w.name, "batch": w.B, "seq_len": w.T, "heads": w.H,
                   "entry_dim": w.c, "rope_dims": w.r, "m_prime": w.m_prime,
                   "entries": w.n_hca, "n_win": w.n_win, "sink": True,
                   "l2": "flushed between timed steps (256 MiB write + 256 MiB read, "
                         "outside the step events)"},
        "stages_ms": {"hca_compress": t_comp, "dense_hca_attn": t_attn},
        "stage_roofline": {"hca_compress": {
            "bound": "hbm", "achieved_GBps": hca_compress_bytes(w) / (t_comp * 1e-3) / 1e9,
            "peak": hbm}},
        "roofline": {"bound": "tensor", "kernel": "dense_hca_attn", "achieved": achieved,
                     "peak": bf16, "unit": "TFLOP/s", "frac": achieved / bf16, "traffic": None,
                     "algorithmic_flops_per_launch": fl,
                     "peak_source": f"{src} bf16 burst (MEASURED_PEAKS.json)"
                     if src == "measured" else "fallback 1.59 PFLOP/s"},
    }
    if cpu:
        res["cpu_baseline"] = hca_cpu_baseline(w, inp, cpu_rows)
    del inp, entries, win, out
    torch.cuda.empty_cache()
    return res


def measure_projection(dev, steps: int, warmup: int, flush, ws_n: int, cpu: bool,
                       cpu_rows: int = 64):
    """The grouped output projection of the csa_prefill_8k layer's attention
    output (8192 rows, 64 heads x 512, g = 8 groups -> d_g = 1024, then
    g d_g = 8192 -> d = 4096): two tcgen05 GEMMs, bf16 in and out.  Rows/s of
    the call and its tensor roofline over 2 T (H c d_g + g d_g d) FLOPs."""
    w = wl.WORKLOADS[WORKLOAD]
    p = wl.PROJ
    x = wl.projection_inputs(w, p["g"], p["d_g"], p["d"], dev)
    y = torch.empty((w.T, p["d"]), dtype=w.dtype, device=dev)
    ws = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_OUT_PROJ, 1, 1, w.T, 0, 0,
                                               p["g"] * p["d_g"]), dev)

    def run():
        csa.grouped_output_projection(x["o"], x["w_group"], x["w_out"], y=y, ws=ws)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    st, d = csa.csa_check_status(ws)
    if st:
        raise RuntimeError(f"projection: device status {st}/{d}")
    ms = allmax(float(np.mean([a.elapsed_time(b) for a, b in evs])), ws_n)
    fl = 2.0 * w.T * (w.H * w.c * p["d_g"] + p["g"] * p["d_g"] * p["d"])
    _, bf16, src = peaks()
    achieved = fl / (ms * 1e-3) / 1e12
    res = {"value": w.T * ws_n / (ms * 1e-3), "unit": "tokens/s", "ms": ms,
           "config": {"workload": w.name, "rows": w.T, "heads": w.H, "head_dim": w.c, **p,
                      "weights": "random synthetic, N(0,1)/sqrt(fan_in)",
                      "l2": "flushed between timed calls (256 MiB write + 256 MiB read, "
                            "outside the events)"},
           "roofline": {"bound": "tensor", "kernel": "gemm_bf16_tc_kernel (two launches)",
                        "achieved": achieved, "peak": bf16, "unit": "TFLOP/s",
                        "frac": achieved / bf16, "algorithmic_flops_per_call": fl,
                        "peak_source": f"{src} bf16 burst (MEASURED_PEAKS.json)"
                        if src == "measured" else "fallback 1.59 PFLOP/s"}}
    if cpu:
        import oracle

        sel = np.linspace(0, w.T - 1, cpu_rows).astype(np.int64)
        o = x["o"][torch.from_numpy(sel).to(dev)].double().cpu().numpy()
        wg, wo = x["w_group"].double().cpu().numpy(), x["w_out"].double().cpu().numpy()
        t0 = time.perf_counter()
        oracle.grouped_output_projection(o, wg, wo)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": cpu_rows / dt, "unit": "tokens/s",
                               "cores": os.cpu_count(), "kind": "oracle",
                               "sample": f"{cpu_rows} of {w.T} rows evenly spaced, float64 "
                                         f"numpy matmuls, {dt:.2f} s"}
    del x, y, ws
    torch.cuda.empty_cache()
    return res


DECODE_WORKLOADS = ("csa_decode_b32_128k", "decode_pair_b4_1m")


def decode_bytes(w) -> float:
    """Bytes one decode step must move: the indexer keys of every visible entry
    (all of them: the query sits at the end of its context), q_I and w, the
    selected entries and the window rows gathered once, the queries read and
    the outputs written; for the layer pair also the HCA layer's entries,
    window, queries and outputs."""
    e = 2
    nb = w.B * w.n_csa * w.dI * e + w.B * w.HI * (w.dI * e + 4)
    nb += w.B * (min(w.k, w.n_csa) + w.n_win) * w.c * e + 2 * w.B * w.H * w.c * e
    if w.kind == "decode_pair":
        nb += w.B * (w.n_hca + w.n_win) * w.c * e + 2 * w.B * w.H * w.c * e
    return float(nb)


class DecodeStep:
    """One decode step of a decode workload through the public API, into
    preallocated outputs: indexer + top-k over the cached indexer keys, then
    sparse MQA over the selected entries and the window; for the 1M layer
    pair also the HCA layer's dense MQA."""

    def __init__(self, w, dev):
        self.w = w
        inp = wl.csa_decode_inputs(w, dev)
        fmt = csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
        self.idx = torch.empty((w.B, 1, w.k), dtype=torch.int32, device=dev)
        self.ws = [csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_INDEXER, 1, w.B, 1, 0, 0,
                                                         w.n_csa, w.k, 0), dev),
                   csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_SPARSE_ATTN, 1, w.B, 1, w.H,
                                                         w.c, w.n_csa, w.k, w.n_win), dev)]
        self.out = torch.empty_like(inp["q"])
        ws_i, ws_a = self.ws
        self.stages = [
            ("indexer_scores_topk", lambda: csa.indexer_scores_topk(
                inp["q_I"], inp["w"], inp["k_I"], w.m, w.k, q_pos=inp["q_pos"], idx_out=self.idx,
                ws=ws_i), w.B * w.n_csa * w.dI * 2),
            ("sparse_mqa_attn", lambda: csa.sparse_mqa_attn(
                inp["q"], inp["entries"], self.idx, inp["win"], fmt, w.n_win, sink=inp["sink"],
                q_pos=inp["q_pos"], win_pos0=inp["win_pos0"], out=self.out, ws=ws_a),
                w.B * (min(w.k, w.n_csa) + w.n_win) * w.c * 2 + 2 * w.B * w.H * w.c * 2),
        ]
        if w.kind == "decode_pair":
            h = wl.hca_decode_inputs(w, dev)
            n_h = h["entries"].shape[1]
            ws_h = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_DENSE_ATTN, 1, w.B, 1, w.H,
                                                         w.c, n_h, 0, w.n_win), dev)
            self.ws.append(ws_h)
            self.out_h = torch.empty_like(h["q"])
            self.stages.append(("dense_hca_attn", lambda: csa.dense_hca_attn(
                h["q"], h["entries"], w.m_prime, h["win"], fmt, w.n_win, sink=h["sink"],
                q_pos=h["q_pos"], win_pos0=h["win_pos0"], out=self.out_h, ws=ws_h),
                w.B * (n_h + w.n_win) * w.c * 2 + 2 * w.B * w.H * w.c * 2))
        self.inp = inp

        # streaming compression of the step's new token (one per sequence), the
        # states positioned at token L - 1 so the token completes a block: CSA
        # entry L/m - 1 (and for the pair HCA entry L/m' - 1) is pooled from a
        # filled tail buffer.  Timed beside the step, not inside it.
        self.append = []
        c = w.c

        def state_at_end(overlap, m):
            st = csa.stream_state(w.B, m, overlap, c, c, w.dtype, dev)
            n = (3 if overlap else 1) * m * 2 * c
            rows = wl.randn((w.B, n), 300 + m, dev, dtype=w.dtype)
            st[:, 16:16 + 2 * n] = rows.view(torch.uint8).view(w.B, 2 * n)
            st[:, :8] = torch.tensor([w.T - 1] * w.B, dtype=torch.int64).view(
                torch.uint8).view(w.B, 8).to(dev)
            return st

        tok = [wl.randn((w.B, c), 310 + i, dev, dtype=w.dtype) for i in range(4)]
        self.tok = tok
        ent_c = torch.empty((w.B, w.n_csa, c), dtype=w.dtype, device=dev)
        win_c = torch.empty((w.B, c), dtype=w.dtype, device=dev)
        st_c = state_at_end(True, w.m)
        ws_s = csa.workspace(256, dev)
        self.ws.append(ws_s)
        self.st_c = st_c
        self.append.append(("csa_compress_append", lambda: csa.csa_compress_append(
            tok[0], tok[1], tok[2], tok[3], w.m, fmt, st_c, ent_c, win_out=win_c, ws=ws_s),
            st_c.shape[1] * w.B))
        if w.kind == "decode_pair":
            ent_h = torch.empty((w.B, w.n_hca, c), dtype=w.dtype, device=dev)
            st_h = state_at_end(False, w.m_prime)
            self.st_h = st_h
            self.append.append(("hca_compress_append", lambda: csa.hca_compress_append(
                tok[0], tok[2], w.m_prime, fmt, st_h, ent_h, win_out=win_c, ws=ws_s),
                st_h.shape[1] * w.B))
        self.ent_c = ent_c

        # the same step with the indexer on MX-FP8 operands: the cache's K_I
        # quantized once (as the cache writer would store it), q_I every step
        self.kc, self.ks = csa.indexer_mxfp8_quantize(inp["k_I"])
        self.qc = torch.empty(inp["q_I"].shape, dtype=torch.uint8, device=dev)
        self.qs = torch.empty((w.B, 1, 512), dtype=torch.uint8, device=dev)
        ws_mx = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_INDEXER_MX, 1, w.B, 1, 0, 0,
                                                      w.n_csa, w.k, 0), dev)
        self.ws.append(ws_mx)
        self.mx_stages = [
            ("indexer_mxfp8_quantize", lambda: csa.indexer_mxfp8_quantize(
                inp["q_I"], self.qc, self.qs, per_token=True), w.B * w.HI * w.dI * 3),
            ("indexer_scores_topk_mxfp8", lambda: csa.indexer_scores_topk_mxfp8(
                self.qc, self.qs, inp["w"], self.kc, self.ks, w.m, w.k, q_pos=inp["q_pos"],
                idx_out=self.idx, ws=ws_mx), w.B * w.n_csa * (w.dI + w.dI // 32)),
        ] + self.stages[1:]
        # and on MX-FP4 operands (packed E2M1: 64 code bytes + 4 scale bytes an entry)
        self.kc4, self.ks4 = csa.indexer_mxfp4_quantize(inp["k_I"])
        self.qc4 = torch.empty(tuple(inp["q_I"].shape[:-1]) + (w.dI // 2,), dtype=torch.uint8,
                               device=dev)
        self.qs4 = torch.empty((w.B, 1, 512), dtype=torch.uint8, device=dev)
        self.mx4_stages = [
            ("indexer_mxfp4_quantize", lambda: csa.indexer_mxfp4_quantize(
                inp["q_I"], self.qc4, self.qs4, per_token=True), w.B * w.HI * w.dI * 5 // 2),
            ("indexer_scores_topk_mxfp4", lambda: csa.indexer_scores_topk_mxfp8(
                self.qc4, self.qs4, inp["w"], self.kc4, self.ks4, w.m, w.k, q_pos=inp["q_pos"],
                idx_out=self.idx, ws=ws_mx), w.B * w.n_csa * (w.dI // 2 + w.dI // 32)),
        ] + self.stages[1:]

        # the same step with the entry caches stored mixed (RoPE dims bf16,
        # the rest MX-FP8: 592 instead of 1024 bytes an entry), written once
        fm = csa.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base, flags=csa.CSA_F_MIXED)
        self.rec = csa.csa_store_mixed(inp["entries"], fmt)
        rb = self.rec.shape[-1]
        self.mixed_stages = [self.stages[0], ("sparse_mqa_attn_mixed", lambda: csa.sparse_mqa_attn(
            inp["q"], self.rec, self.idx, inp["win"], fm, w.n_win, sink=inp["sink"],
            q_pos=inp["q_pos"], win_pos0=inp["win_pos0"], out=self.out, ws=ws_a),
            w.B * (min(w.k, w.n_csa) * rb + w.n_win * w.c * 2) + 2 * w.B * w.H * w.c * 2)]
        if w.kind == "decode_pair":
            self.rec_h = csa.csa_store_mixed(h["entries"], fmt)
            self.mixed_stages.append(("dense_hca_attn_mixed", lambda: csa.dense_hca_attn(
                h["q"], self.rec_h, w.m_prime, h["win"], fm, w.n_win, sink=h["sink"],
                q_pos=h["q_pos"], win_pos0=h["win_pos0"], out=self.out_h, ws=ws_h),
                w.B * (n_h * rb + w.n_win * w.c * 2) + 2 * w.B * w.H * w.c * 2))

    def run_mixed(self):
        for _, fn, _ in self.mixed_stages:
            fn()

    def run_mx(self):
        for _, fn, _ in self.mx_stages:
            fn()

    def run_mx4(self):
        for _, fn, _ in self.mx4_stages:
            fn()

    def rewind(self):
        """Puts every stream state back at token L - 1 (each append advances it)."""
        self.st_c[:, :8] = torch.tensor([self.w.T - 1] * self.w.B, dtype=torch.int64).view(
            torch.uint8).view(self.w.B, 8).to(self.st_c.device)
        if hasattr(self, "st_h"):
            self.st_h[:, :8] = self.st_c[:, :8]

    def run(self):
        for _, fn, _ in self.stages:
            fn()

    def check(self):
        for ws in self.ws:
            st, d = csa.csa_check_status(ws)
            if st:
                raise RuntimeError(f"{self.w.name}: device status {st}/{d}")


class L2Flush:
    """Empties the 126 MB L2 between timed steps, outside the events: a 256 MiB
    write, then a 256 MiB read of a second buffer, so that the cache holds only
    clean lines and the write-back of the flush's own dirty lines does not land
    in the next timed region."""

    def __init__(self, dev):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.zeros(64 << 20, dtype=torch.int32, device=dev)

    def __call__(self):
        self.w.zero_()
        self.r.sum()


def graph_ms(fn, steps: int, flush, before=None) -> float:
    """Mean device time of `fn` captured once in a CUDA graph and replayed
    `steps` times, with the L2 flushed (and `before` run) before each replay,
    outside the events, as a decode server replays its step."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        fn()
    if before:
        before()
    g.replay()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        if before:
            before()
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        evs.append((e0, e1))
    torch.cuda.synchronize()
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    del g
    return ms


def measure_compress_1m(dev, steps: int, warmup: int, T: int = 1 << 20):
    """CSA (m = 4) and HCA (m' = 128) compression alone at 2^20 tokens, c = 512
    bf16, window rows written: inputs of 2-4 GiB (far larger than L2), so
    the kernels' HBM bandwidth shows without launch overhead (the 8192-token
    workload moves only 42 MB).  Algorithmic bytes: every input read once,
    entries and window rows written once."""
    c = 512
    fmt = csa.Fmt(c=c, rope_dims=64)
    hbm, _, src = peaks()
    res = {}

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    x = [wl.randn((1, T, c), 100 + i, dev, dtype=torch.bfloat16) for i in range(4)]
    ent = torch.empty((1, T // 4, c), dtype=torch.bfloat16, device=dev)
    win = torch.empty((1, T, c), dtype=torch.bfloat16, device=dev)
    ws_c = csa.workspace(csa.csa_workspace_bytes(csa.CSA_OP_COMPRESS, 1, 1, T), dev)
    ms = timed(lambda: csa.csa_compress(x[0], x[1], x[2], x[3], 4, fmt, entries=ent, win_out=win,
                                        ws=ws_c))
    nb = (4 * T + T // 4 + T) * c * 2
    res["csa_compress"] = {"ms": ms, "bytes": nb, "GBps": nb / ms / 1e6, "frac": nb / ms / 1e6 / hbm}
    del x, ent
    x = [wl.randn((1, T, c), 110 + i, dev, dtype=torch.bfloat16) for i in range(2)]
    ent = torch.empty((1, T // 128, c), dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: csa.hca_compress(x[0], x[1], 128, fmt, entries=ent, win_out=win,
                                        ws=ws_c))
    nb = (2 * T + T // 128 + T) * c * 2
    res["hca_compress"] = {"ms": ms, "bytes": nb, "GBps": nb / ms / 1e6, "frac": nb / ms / 1e6 / hbm}
    del x, ent, win
    torch.cuda.empty_cache()
    res["config"] = {"tokens": T, "entry_dim": c, "dtype": "bf16", "window_rows": True,
                     "peak": f"{src} HBM copy {hbm} GB/s"}
    return res


def decode_cpu_baseline(w, queries: int):
    """The float64 oracle on `queries` decode queries of the workload (indexer
    scores over the whole cache, top-k, sparse MQA; for the layer pair also the
    HCA layer's dense MQA), in queries per second."""
    import oracle

    inp = wl.csa_decode_inputs(w, "cpu")
    fmt = oracle.Fmt(c=w.c, rope_dims=w.r, rope_base=w.rope_base)
    h = wl.hca_decode_inputs(w, "cpu") if w.kind == "decode_pair" else None
    sink = None if inp["sink"] is None else inp["sink"].double().numpy()
    t0 = time.perf_counter()
    for b in range(queries):
        pos = inp["q_pos"][b].numpy()
        sc = oracle.indexer_scores(inp["q_I"][b].double().numpy(), inp["w"][b].double().numpy(),
                                   inp["k_I"][b].double().numpy(), w.m, q_pos=pos)
        idx = oracle.topk(sc, w.k, w.m, q_pos=pos)
        oracle.attention(inp["q"][b].double().numpy(), inp["entries"][b].double().numpy(),
                         inp["win"][b].double().numpy(), fmt, w.n_win, idx=idx, sink=sink,
                         q_pos=pos, win_pos0=int(inp["win_pos0"][b]))
        if h is not None:
            oracle.attention(h["q"][b].double().numpy(), h["entries"][b].double().numpy(),
                             h["win"][b].double().numpy(), fmt, w.n_win, m_dense=w.m_prime,
                             sink=h["sink"].double().numpy(), q_pos=pos,
                             win_pos0=int(h["win_pos0"][b]))
    dt = time.perf_counter() - t0
    return {"value": queries / dt, "unit": "queries/s", "cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{queries} of {w.B} queries (the whole decode step for each), float64, "
                      f"{dt:.1f} s"}


def measure_decode(name: str, dev, steps: int, warmup: int, flush, ws_n: int, cpu: bool):
    """Decode queries/s of one decode workload: the whole step as one CUDA-graph
    replay (max over ranks), each stage also alone, and the step's HBM
    roofline over the bytes it must move."""
    w = wl.WORKLOADS[name]
    d = DecodeStep(w, dev)
    for _ in range(warmup):
        d.run()
    torch.cuda.synchronize()
    d.check()
    step_ms = allmax(graph_ms(d.run, steps, flush), ws_n)
    stages = {n: graph_ms(fn, steps, flush) for n, fn, _ in d.stages}
    d.check()
    mixed_ms = allmax(graph_ms(d.run_mixed, steps, flush), ws_n)
    mixed_stages = {n: graph_ms(fn, steps, flush) for n, fn, _ in d.mixed_stages[1:]}
    mx_ms = allmax(graph_ms(d.run_mx, steps, flush), ws_n)
    mx_stages = {n: graph_ms(fn, steps, flush) for n, fn, _ in d.mx_stages[:2]}
    mx4_ms = allmax(graph_ms(d.run_mx4, steps, flush), ws_n)
    mx4_stages = {n: graph_ms(fn, steps, flush) for n, fn, _ in d.mx4_stages[:2]}
    d.check()
    append = {}
    for n, fn, nb in d.append:
        # a state rewind (outside the events) before every timed append, so
        # each one completes a block
        ms = graph_ms(fn, steps, flush, before=d.rewind)
        append[n] = {"ms": ms, "state_bytes_read": nb, "GBps": nb / ms / 1e6}
    d.check()
    hbm, _, src = peaks()
    nb = decode_bytes(w)
    achieved = nb / (step_ms * 1e-3) / 1e9
    # MX-FP8 indexer operands: 128 code bytes + 4 scale bytes per entry instead of 256
    nb_mx = nb - w.B * w.n_csa * w.dI * 2 + w.B * w.n_csa * (w.dI + w.dI // 32)
    mx_achieved = nb_mx / (mx_ms * 1e-3) / 1e9
    # MX-FP4: 64 packed code bytes + 4 scale bytes per entry
    nb_mx4 = nb - w.B * w.n_csa * w.dI * 2 + w.B * w.n_csa * (w.dI // 2 + w.dI // 32)
    mx4_achieved = nb_mx4 / (mx4_ms * 1e-3) / 1e9
    res = {
        "value": w.B * ws_n / (step_ms * 1e-3), "unit": "queries/s", "ms_per_step": step_ms,
        "config": {"workload": w.name, "batch": w.B, "context": w.T, "heads": w.H,
                   "entries": w.n_csa, "top_k": w.k, "n_win": w.n_win, "sink": True,
                   **({"hca_entries": w.n_hca} if w.kind == "decode_pair" else {}),
                   "l2": "flushed before every replay (256 MiB write + 256 MiB read, "
                         "outside the events)",
                   "timing": "whole step captured once in a CUDA graph, replayed"},
        "stages_ms": stages,
        "mixed_entries": {
            "value": w.B * ws_n / (mixed_ms * 1e-3), "unit": "queries/s",
            "ms_per_step": mixed_ms, "stages_ms": mixed_stages,
            "stage_bytes": {n: nb_ for n, _, nb_ in d.mixed_stages[1:]},
            "note": "the same step with the entry caches stored mixed (RoPE dims bf16, the rest "
                    "MX-FP8 with a scale per 32 dims: 592 bytes an entry instead of 1024)"},
        "mxfp8_indexer": {
            "value": w.B * ws_n / (mx_ms * 1e-3), "unit": "queries/s", "ms_per_step": mx_ms,
            "stages_ms": mx_stages,
            "note": "the same step with q_I quantized each step and the indexer on MX-FP8 "
                    "operands (K_I cached as E4M3 codes + UE8M0 scales per 32)",
            "roofline": {"bound": "hbm", "achieved": mx_achieved, "peak": hbm, "unit": "GB/s",
                         "frac": mx_achieved / hbm, "algorithmic_bytes_per_step": nb_mx}},
        "mxfp4_indexer": {
            "value": w.B * ws_n / (mx4_ms * 1e-3), "unit": "queries/s", "ms_per_step": mx4_ms,
            "stages_ms": mx4_stages,
            "note": "the same step with the indexer on MX-FP4 operands (K_I cached as packed "
                    "E2M1 codes + UE8M0 scales per 32: 68 bytes an entry instead of 256)",
            "roofline": {"bound": "hbm", "achieved": mx4_achieved, "peak": hbm, "unit": "GB/s",
                         "frac": mx4_achieved / hbm, "algorithmic_bytes_per_step": nb_mx4}},
        "stream_append": {**append, "note": "the step's new token appended to each sequence's "
                          "compression state (completing a block: entry pooled from the tail "
                          "buffer); latency-bound, timed beside the step"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "algorithmic_bytes_per_step": nb,
                     "peak_source": f"{src} HBM copy (MEASURED_PEAKS.json)"
                     if src == "measured" else "fallback 6.65 TB/s"},
    }
    if cpu:
        res["cpu_baseline"] = decode_cpu_baseline(w, 1)
    del d
    torch.cuda.empty_cache()
    return res


def run_only_decode(args):
    """The decode step of --decode-workload (--decode-batch rows, default the
    workload's), each stage replayed alone from a CUDA graph, with its
    bandwidth over the bytes it must read; also the MX-FP8 indexer, the
    mixed-entry attention and the streaming compression stages."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = wl.WORKLOADS[args.decode_workload]
    if args.decode_batch:
        w = wl.scaled(w, B=args.decode_batch)
    d = DecodeStep(w, dev)
    for _ in range(args.warmup):
        d.run()
    torch.cuda.synchronize()
    d.check()
    flush = L2Flush(dev)
    res = {}
    for name, fn, nbytes in d.stages + d.mx_stages[:2] + d.mx4_stages[:2] + d.mixed_stages[1:]:
        ms = graph_ms(fn, args.steps, flush)
        res[name] = {"ms": ms, "bytes": nbytes, "GBps": nbytes / ms / 1e6}
    for name, fn, nbytes in d.append:
        ms = graph_ms(fn, args.steps, flush, before=d.rewind)
        res[name] = {"ms": ms, "bytes": nbytes, "GBps": nbytes / ms / 1e6}
    step = graph_ms(d.run, args.steps, flush)
    d.check()
    print(json.dumps({"only": "decode", "workload": w.name, "stages": res, "step_ms": step,
                      "queries_per_s": w.B / (step * 1e-3),
                      "step_GBps": decode_bytes(w) / step / 1e6}))


def run_only(args):
    """One stage of the step alone on the csa_prefill workload at --seq-len
    tokens (for kernel profiles): warm-up, then --steps timed launches."""
    if args.only == "compress_stream":   # CSA then HCA compression alone, inputs only
        torch.cuda.set_device(0)
        res = measure_compress_1m(torch.device("cuda", 0), args.steps, args.warmup,
                                  T=args.seq_len or (1 << 20))
        print(json.dumps({"only": args.only, **res}))
        return
    if args.only.startswith("hca_"):
        return run_only_hca(args)
    if args.only == "proj":
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        flush = L2Flush(dev)
        print(json.dumps({"only": "proj", **measure_projection(dev, args.steps, args.warmup,
                                                               flush, 1, False)}))
        return
    if args.only == "decode":
        return run_only_decode(args)
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
                             entries=step.entries, win_out=step.win, ws=step.ws_comp)
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
    ap.add_argument("--only", choices=["compress", "compress_stream", "indexer", "attn",
                                       "hca_compress", "hca_attn", "proj",
                                       "decode"],
                    default=None,
                    help="time one stage alone (kernel profiling)")
    ap.add_argument("--seq-len", type=int, default=0, help="tokens for --only (default 8192)")
    ap.add_argument("--decode-workload", default="csa_decode_b32_128k",
                    choices=["csa_decode_b32_128k", "decode_pair_b4_1m"], help="for --only decode")
    ap.add_argument("--decode-batch", type=int, default=0,
                    help="for --only decode: rows of the workload (a smaller case for profiles)")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=8192)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode workloads")
    ap.add_argument("--no-hca", action="store_true", help="skip the HCA prefill workload")
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
