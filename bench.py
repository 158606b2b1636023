"""Benchmark of the HATA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = one hata_decode_step: append the step's key code (and K/V rows),
hash the queries, Hamming-score every cached code, select the top-k per
query head, gather the selected K/V rows and run softmax attention over them.
Each step appends one token, so step t attends over N + t + 1 keys.

Timing: W untimed warm-up steps, then exactly K timed steps bracketed by a
barrier and torch.cuda.synchronize(); every step is timed on the launching
stream with CUDA events (recorded by the library between its kernels), and L2
is flushed before every step, outside the timed intervals, by reading a
512 MiB buffer: that evicts every line and leaves L2 clean, so no write-back
of flush data lands inside the timed step.
Multi-GPU: one process per GPU (torchrun), each rank decodes its own batch
(weak scaling, no collective on the data path); rank 0 prints the max over
ranks.  `--impl reference` times the CPU oracle instead, on a bounded sample
of heads of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hash_aware_top_hata_b200 import hata as H  # noqa: E402
from hash_aware_top_hata_b200 import workloads as wl  # noqa: E402

METRIC = "µs per decode step & achieved HBM GB/s (score+top-k+sparse attn) vs roofline"
UNIT = "us/step"
DEFAULT_CONFIG = "llama31_8b_gqa_128k"
FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class L2Flush:
    """Evicts L2 by reading a buffer 4x its size (clean lines only)."""

    def __init__(self, buf: torch.Tensor):
        self.buf = buf

    def __call__(self):
        torch.sum(self.buf)


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no samples
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set() and self._nv is not None:
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                mask = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if not self._t.is_alive() and not self._stop.is_set():
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "hata" and torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, x: float) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ oracle (CPU) --

def oracle_step(cfg, w, workers=None):
    """The CPU oracle on whole decode steps of the workload over the host
    cores (oracle/pool.py): the prompt caches (generator values, never
    written by the CUDA path) copied to the host, their key codes hashed by
    the oracle's pool beforehand (untimed)."""
    from oracle import pool
    N = cfg.N
    K = np.zeros((cfg.B, cfg.H_kv, w.n_cap, 128), wl.to_numpy_kv(w.K[:1, :1, :1]).dtype)
    V = np.zeros_like(K)
    K[:, :, :N] = wl.to_numpy_kv(w.K[:, :, :N])
    V[:, :, :N] = wl.to_numpy_kv(w.V[:, :, :N])
    ops = pool.OracleStep(K, V, w.W_H.cpu().numpy(), cfg.H_q, workers=workers)
    del K, V
    t_hash = ops.hash_prefix(N)
    return ops, t_hash


def oracle_step_time(cfg, w, ops, t: int):
    """One oracle decode step t (append of the step's key and value at
    position N + t, then every query head at context N + t + 1); seconds."""
    t0 = time.perf_counter()
    ops.append(wl.to_numpy_kv(w.k_new[t]), wl.to_numpy_kv(w.v_new[t]), cfg.N + t)
    t_append = time.perf_counter() - t0
    dt, _ = ops.step(w.q[t].cpu().numpy(), cfg.N + t + 1, cfg.topk, 1.0 / math.sqrt(128))
    return t_append + dt


def oracle_desc(cfg, ops) -> str:
    from oracle import pool
    return (f"CPU oracle, whole decode steps (append, then hash q, Hamming over "
            f"{cfg.N + 1} codes, sorted top-{cfg.topk} and fp64 attention for all "
            f"{cfg.B * cfg.H_q} query heads), one task per head on {ops.workers} processes "
            f"({pool.cpu_model()}); prompt key codes hashed by the oracle beforehand, untimed")


def bench_config(args):
    """The named workload, optionally at another context / batch (profiling
    and sweeps; the default run uses the named workload unchanged)."""
    cfg = wl.CONFIGS[args.config]
    if args.context or args.batch:
        cfg = wl.scaled(cfg, N=args.context or cfg.N, B=args.batch or cfg.B,
                        topk=max(1, round(cfg.topk * (args.context or cfg.N) / cfg.N)))
    if getattr(args, "topk", 0):
        cfg = wl.scaled(cfg, N=cfg.N, topk=args.topk, name=f"{cfg.name}@k{args.topk}")
    return cfg


def run_reference(args, world, rank):
    """--impl reference: the CPU oracle on whole decode steps of the same
    workload, over all host cores (rank 0 only)."""
    if rank != 0:
        return
    cfg = bench_config(args)
    steps = args.warmup + args.steps
    w = wl.make_workload(cfg, wl.SEED_BASE + wl.CONFIG_ORDER.index(args.config),
                         device="cuda" if torch.cuda.is_available() else "cpu", steps=steps)
    ops, _ = oracle_step(cfg, w)
    try:
        for t in range(args.warmup):
            oracle_step_time(cfg, w, ops, t)
        times = [oracle_step_time(cfg, w, ops, args.warmup + i) for i in range(args.steps)]
        desc = oracle_desc(cfg, ops)
        cores = ops.workers
    finally:
        ops.close()
    us = statistics.mean(times) * 1e6
    line = {
        "impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(us / 1e3, 3), "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(cfg, "none (CPU)"),
        "cpu_baseline": {"value": round(us, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def profiled_traffic(cfg, kernel: str, src: str):
    """DRAM bytes per launch of `kernel` from its committed ncu summary under
    profiles/, or None when there is none for this workload or the kernel's
    source has changed since the capture (hash recorded in the summary)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"{kernel}_{cfg.name}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"sha256\[:16\] = `([0-9a-f]+)`", text)
    m_traffic = re.search(r"traffic_mb: ([0-9.]+)", text)
    if not (m_hash and m_traffic):
        return None
    now = hashlib.sha256(open(os.path.join(ROOT, src), "rb").read()).hexdigest()[:16]
    return round(float(m_traffic.group(1)) * 1e6) if now == m_hash.group(1) else None


def config_dict(cfg, l2: str, rbit: int = 128) -> dict:
    return {"workload": cfg.name, "B": cfg.B, "H_q": cfg.H_q, "H_kv": cfg.H_kv,
            "context": cfg.N, "topk": cfg.topk, "head_dim": 128, "rbit": rbit,
            "kv_dtype": cfg.kv_dtype, "tokens_appended_per_step": 1, "l2": l2}


# ---------------------------------------------------------------- GPU arm --

def _num(x, nd):
    """x rounded, or None (JSON null) when it was not measured."""
    return None if x != x else round(x, nd)


def extras(args, cfg, w, codes, ws, out, seq, flush, stream, W_steps, K_steps, world):
    """e2e (host buffers in, host result out, through the same C ABI) and the
    dense decode attention at the same shape."""
    dev = out.device
    B, Hq, Hkv, N = cfg.B, cfg.H_q, cfg.H_kv, cfg.N
    scale = 1.0 / math.sqrt(128)
    kv_elt = 2 if cfg.kv_dtype == "bf16" else 4
    t0 = W_steps + 2 * K_steps  # steps after the timed and the breakdown passes
    q_h = w.q[t0:t0 + K_steps].cpu().pin_memory()
    kn_h = w.k_new[t0:t0 + K_steps].cpu().pin_memory()
    vn_h = w.v_new[t0:t0 + K_steps].cpu().pin_memory()
    out_h = torch.empty((K_steps, B, Hq, 128)).pin_memory()
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K_steps)]
    # the step's inputs and its output stay in pinned host memory: the caller
    # keeps one pinned staging buffer per tensor and fills it on the CPU
    # before each step; inside the timed region the library's kernels read
    # q, k_new, v_new over the bus and write out back (the public call with
    # host pointers, no separate copy operations)
    q_st, kn_st, vn_st = (torch.empty_like(x[0]).pin_memory() for x in (q_h, kn_h, vn_h))
    out_st = torch.empty_like(out_h[0]).pin_memory()
    for i in range(K_steps):
        q_st.copy_(q_h[i])
        kn_st.copy_(kn_h[i])
        vn_st.copy_(vn_h[i])
        flush()
        e2e_ev[i][0].record(stream)
        H.hata_decode_step(q_st, w.W_H, codes, w.K, w.V, seq[t0 + i], w.n_cap, cfg.topk, scale,
                           ws, out_st, k_new=kn_st, v_new=vn_st)
        e2e_ev[i][1].record(stream)
        e2e_ev[i][1].synchronize()  # a caller reads each step's output before the next
        out_h[i].copy_(out_st)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(world, statistics.mean(a.elapsed_time(b) for a, b in e2e_ev))
    h2d = q_h[0].numel() * 4 + (kn_h[0].numel() + vn_h[0].numel()) * kv_elt
    d2h = out_h[0].numel() * 4

    # ---- dense decode attention at the same shape (context for the speedup) ----
    dws = torch.empty(H.hata_dense_workspace_size(B, Hq, Hkv, w.n_cap), dtype=torch.uint8,
                      device=dev)
    dout = torch.empty_like(out)
    dseq = torch.full((B,), N, dtype=torch.int32, device=dev)
    dense_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(10)]
    for i in range(13):
        flush()
        if i >= 3:
            dense_ev[i - 3][0].record(stream)
        H.hata_dense_decode(w.q[0], w.K, w.V, dseq, N, scale, dws, dout)
        if i >= 3:
            dense_ev[i - 3][1].record(stream)
    torch.cuda.synchronize()
    dense_ms = statistics.median(a.elapsed_time(b) for a, b in dense_ev)

    return e2e_ms, h2d, d2h, dense_ms


def more_legs(cfg, w, codes, ws, out, seq, flush, stream, t0, K_steps):
    """Labelled side measurements of the same workload: warm-L2 step time,
    needle recall, the step with the K/V caches in host memory, the step
    with 64- and 32-bit codes, prefill key encoding against the FP32 peak,
    torch SDPA dense decode, and K_steps consecutive decode steps replayed
    from one CUDA Graph."""
    B, Hq, Hkv, N, G = cfg.B, cfg.H_q, cfg.H_kv, cfg.N, cfg.G
    scale = 1.0 / math.sqrt(128)
    dev = out.device
    res = {}

    def ev_pair():
        return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    # ---- warm L2: the same step with no flush in between ----
    evs = [ev_pair() for _ in range(K_steps)]
    for i in range(K_steps):
        evs[i][0].record(stream)
        H.hata_decode_step(w.q[t0 + i], w.W_H, codes, w.K, w.V, seq[t0 + i], w.n_cap, cfg.topk,
                           scale, ws, out, k_new=w.k_new[t0 + i], v_new=w.v_new[t0 + i])
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    res["warm_l2_us"] = round(statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3, 2)

    # ---- needle recall: needles kept in the selected set of each group's
    # first query head (the head the needles point at) ----
    if cfg.needles > 0:
        sel = torch.empty((B, Hq, cfg.topk), dtype=torch.int32, device=dev)
        H.hata_decode_step(w.q[0], w.W_H, codes, w.K, w.V, seq[t0 + K_steps], w.n_cap,
                           cfg.topk, scale, ws, out, sel_idx=sel)
        torch.cuda.synchronize()
        sel_c = sel.cpu()
        hits = total = 0
        for b in range(B):
            for h in range(Hkv):
                nd = set(x for x in w.planted[b, h].tolist() if x >= 0)
                got = set(sel_c[b, h * G].tolist())
                hits += len(nd & got)
                total += len(nd)
        res["needle_recall"] = round(hits / max(total, 1), 4)

    # ---- HATA-off: the K/V caches in pinned host memory; a step reads only
    # the selected rows over the bus (the codes stay on the device) ----
    try:
        Kh, Vh = w.K.cpu().pin_memory(), w.V.cpu().pin_memory()
        kh_ev = [ev_pair() for _ in range(3)]
        for i in range(5):
            flush()
            if i >= 2:
                kh_ev[i - 2][0].record(stream)
            H.hata_decode_step(w.q[t0 + i], w.W_H, codes, Kh, Vh, seq[t0 + i], w.n_cap, cfg.topk,
                               scale, ws, out, k_new=w.k_new[t0 + i], v_new=w.v_new[t0 + i])
            if i >= 2:
                kh_ev[i - 2][1].record(stream)
        torch.cuda.synchronize()
        t_kh = statistics.median(a.elapsed_time(b) for a, b in kh_ev) / 1e3
        row_bytes = B * Hq * cfg.topk * 2 * w.K.shape[-1] * w.K.element_size()
        res["kv_host"] = {"us_per_step": round(t_kh * 1e6, 1),
                          "selected_row_gbs": round(row_bytes / t_kh / 1e9, 2),
                          "selected_row_bytes": row_bytes}
        del Kh, Vh
    except RuntimeError as e:  # pinned host memory unavailable
        res["kv_host"] = {"unavailable": str(e).splitlines()[0][:120]}

    # ---- narrower codes (the page's r = 64 / 32 ablation): the same step
    # with r-bit codes from the leading r columns of W_H ----
    res["narrow_codes"] = {}
    for r in (64, 32):
        Wr = w.W_H[:, :, :r].contiguous()
        codes_r = torch.empty((B, Hkv, w.n_cap, r // 32), dtype=torch.int32, device=dev)
        H.hata_hash_keys(w.K, Wr, codes_r, 0, N)
        nr_ev = [ev_pair() for _ in range(3)]
        for i in range(5):
            flush()
            if i >= 2:
                nr_ev[i - 2][0].record(stream)
            H.hata_decode_step(w.q[t0 + i], Wr, codes_r, w.K, w.V, seq[t0 + i], w.n_cap,
                               cfg.topk, scale, ws, out, k_new=w.k_new[t0 + i],
                               v_new=w.v_new[t0 + i])
            if i >= 2:
                nr_ev[i - 2][1].record(stream)
        torch.cuda.synchronize()
        res["narrow_codes"][f"r{r}_us_per_step"] = round(
            statistics.median(a.elapsed_time(b) for a, b in nr_ev) * 1e3, 1)
        del codes_r

    # ---- prefill key encoding (hata_hash_keys over the whole cache) ----
    pe = [ev_pair() for _ in range(3)]
    for i in range(4):
        flush()
        if i >= 1:
            pe[i - 1][0].record(stream)
        H.hata_hash_keys(w.K, w.W_H, codes, 0, N)
        if i >= 1:
            pe[i - 1][1].record(stream)
    torch.cuda.synchronize()
    t = statistics.median(a.elapsed_time(b) for a, b in pe) / 1e3
    flops = 2.0 * B * Hkv * N * 128 * 128
    fp32_peak = 148 * 128 * 2 * 1.965e9  # nominal: SMs x FP32 lanes x FMA x max clock
    res["prefill_hash"] = {"us": round(t * 1e6, 1), "keys_per_s": round(B * Hkv * N / t, 0),
                           "tflops": round(flops / t / 1e12, 2),
                           "frac_of_fp32_nominal": round(flops / t / fp32_peak, 3)}

    # ---- torch SDPA dense decode at the same shape (context) ----
    try:
        qs = w.q[0].to(w.K.dtype)[:, :, None, :]
        Kd, Vd = w.K[:, :, :N], w.V[:, :, :N]
        torch.nn.functional.scaled_dot_product_attention(qs, Kd, Vd, enable_gqa=True)
        se = [ev_pair() for _ in range(5)]
        for i in range(5):
            flush()
            se[i][0].record(stream)
            torch.nn.functional.scaled_dot_product_attention(qs, Kd, Vd, enable_gqa=True)
            se[i][1].record(stream)
        torch.cuda.synchronize()
        res["sdpa_dense_us"] = round(statistics.median(a.elapsed_time(b) for a, b in se) * 1e3, 1)
    except Exception as e:  # an older torch without enable_gqa: not measured
        res["sdpa_dense_us"] = None
        res["sdpa_note"] = type(e).__name__

    # ---- K_steps consecutive decode steps captured once and replayed ----
    g = torch.cuda.CUDAGraph()
    gs = torch.cuda.Stream()
    gs.wait_stream(stream)
    with torch.cuda.stream(gs):
        with torch.cuda.graph(g, stream=gs):
            for i in range(K_steps):
                H.hata_decode_step(w.q[t0 + i], w.W_H, codes, w.K, w.V, seq[t0 + i], w.n_cap,
                                   cfg.topk, scale, ws, out, k_new=w.k_new[t0 + i],
                                   v_new=w.v_new[t0 + i])
    stream.wait_stream(gs)
    g.replay()  # warm
    torch.cuda.synchronize()
    gr = [ev_pair() for _ in range(3)]
    for i in range(3):
        flush()
        gr[i][0].record(stream)
        g.replay()
        gr[i][1].record(stream)
    torch.cuda.synchronize()
    res["graph_us_per_step"] = round(
        statistics.median(a.elapsed_time(b) for a, b in gr) * 1e3 / K_steps, 2)
    res["graph_steps"] = K_steps
    del g
    return res


OTHER_WORKLOADS = ("llama2_7b_mha_32k", "qwen_gqa_b32_32k", "needle_gqa_1m")


def other_workloads(args, dev):
    """The other large workloads, each on its own (flushed L2 before every
    step): microseconds per decode step and the step's roofline fraction;
    the batched Qwen-shaped workload runs its 16 consecutive appending steps
    (per-step figure), the million-token workload reports needle recall."""
    res = {}
    peak, _ = measured_peaks()
    scale = 1.0 / math.sqrt(128)
    flush_buf = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()
    for name in OTHER_WORKLOADS:
        if name == args.config:
            continue
        cfg = wl.CONFIGS[name]
        B, Hq, Hkv, N = cfg.B, cfg.H_q, cfg.H_kv, cfg.N
        warm = 3
        timed = cfg.steps if cfg.steps > 1 else 10
        w = wl.make_workload(cfg, wl.SEED_BASE + wl.CONFIG_ORDER.index(name), device=dev,
                             steps=warm + timed)
        codes = torch.zeros((B, Hkv, w.n_cap, 4), dtype=torch.int32, device=dev)
        H.hata_hash_keys(w.K, w.W_H, codes, 0, N)
        ws = torch.empty(H.hata_decode_workspace_size(B, Hq, Hkv, w.n_cap, cfg.topk),
                         dtype=torch.uint8, device=dev)
        out = torch.empty((B, Hq, 128), device=dev)
        sel = torch.empty((B, Hq, cfg.topk), dtype=torch.int32, device=dev)
        seq = (N + 1 + torch.arange(warm + timed, dtype=torch.int32, device=dev))[:, None] \
            .expand(warm + timed, B).contiguous()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(timed)]
        for t in range(warm + timed):
            torch.sum(flush_buf)
            if t >= warm:
                evs[t - warm][0].record(stream)
            H.hata_decode_step(w.q[t], w.W_H, codes, w.K, w.V, seq[t], w.n_cap, cfg.topk, scale,
                               ws, out, k_new=w.k_new[t], v_new=w.v_new[t], sel_idx=sel)
            if t >= warm:
                evs[t - warm][1].record(stream)
        torch.cuda.synchronize()
        H.hata_workspace_check(ws)
        us = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3
        step_bytes = B * Hkv * (N + warm + timed // 2) * 16 + B * Hq * cfg.topk * 2 * 256
        entry = {"us_per_step": round(us, 2), "steps": timed,
                 "launches_per_step": H.hata_decode_kernel_launches(B, Hq, Hkv, w.n_cap, cfg.topk,
                                                                     w.K.dtype),
                 "step_roofline_bytes": step_bytes,
                 "step_frac_of_measured": round(step_bytes / (us * 1e-6) / 1e9 / peak, 4),
                 "shape": f"B {B}, {Hq}/{Hkv} heads, context {N}, top-{cfg.topk}"}
        if cfg.steps > 1:
            entry["note"] = f"{timed} consecutive decode steps, each appending one key"
        if cfg.needles > 0:
            # needles kept in the last step's selection of each group's first
            # query head (the head the needles point at)
            sel_c = sel.cpu()
            hits = total = 0
            for b in range(B):
                for h in range(Hkv):
                    nd = set(x for x in w.planted[b, h].tolist() if x >= 0)
                    hits += len(nd & set(sel_c[b, h * cfg.G].tolist()))
                    total += len(nd)
            entry["needle_recall"] = round(hits / max(total, 1), 4)
        res[name] = entry
        del w, codes, ws, out, sel
        torch.cuda.empty_cache()
    return res


def wide_code_leg(dev, name="llama31_8b_gqa_128k"):
    """The headline workload with 256-bit codes (the widest width of the
    page's ablation): microseconds per decode step (flushed L2) and the
    step's roofline fraction, whose code bytes double to 32 per key."""
    cfg = wl.CONFIGS[name]
    B, Hq, Hkv, N = cfg.B, cfg.H_q, cfg.H_kv, cfg.N
    warm, timed = 3, 10
    peak, _ = measured_peaks()
    w = wl.make_workload(cfg, wl.SEED_BASE + wl.CONFIG_ORDER.index(name), device=dev,
                         steps=warm + timed)
    W = wl.projection(w.W_H, 256)
    codes = torch.zeros((B, Hkv, w.n_cap, 8), dtype=torch.int32, device=dev)
    H.hata_hash_keys(w.K, W, codes, 0, N)
    ws = torch.empty(H.hata_decode_workspace_size(B, Hq, Hkv, w.n_cap, cfg.topk),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((B, Hq, 128), device=dev)
    flush_buf = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()
    seq = (N + 1 + torch.arange(warm + timed, dtype=torch.int32, device=dev))[:, None] \
        .expand(warm + timed, B).contiguous()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(timed)]
    for t in range(warm + timed):
        torch.sum(flush_buf)
        if t >= warm:
            evs[t - warm][0].record(stream)
        H.hata_decode_step(w.q[t], W, codes, w.K, w.V, seq[t], w.n_cap, cfg.topk,
                           1.0 / math.sqrt(128), ws, out, k_new=w.k_new[t], v_new=w.v_new[t])
        if t >= warm:
            evs[t - warm][1].record(stream)
    torch.cuda.synchronize()
    H.hata_workspace_check(ws)
    us = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3
    # per-kernel breakdown: one more (untimed) step with events between kernels
    kev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in kev:  # torch creates the CUDA event on first record; the library needs handles
        e.record(stream)
    torch.sum(flush_buf)
    H.hata_decode_step(w.q[warm + timed - 1], W, codes, w.K, w.V, seq[warm + timed - 1], w.n_cap,
                       cfg.topk, 1.0 / math.sqrt(128), ws, out, events=kev)
    torch.cuda.synchronize()
    names = ("prep", "score", "select", "attend", "combine")
    kernels = {n: round(kev[i].elapsed_time(kev[i + 1]) * 1e3, 2) for i, n in enumerate(names)}
    step_bytes = B * Hkv * (N + warm + timed // 2) * 32 + B * Hq * cfg.topk * 2 * 256
    res = {"us_per_step": round(us, 2), "steps": timed, "r": 256, "kernels_us": kernels,
           "step_roofline_bytes": step_bytes,
           "step_frac_of_measured": round(step_bytes / (us * 1e-6) / 1e9 / peak, 4),
           "shape": f"{name} with 256-bit codes: B {B}, {Hq}/{Hkv} heads, context {N}, "
                    f"top-{cfg.topk}"}
    del w, codes, ws, out, flush_buf
    torch.cuda.empty_cache()
    return res


def seqpar_leg(dev, ranks=8, name="needle_gqa_1m"):
    """The million-token workload as a sequence-parallel step over `ranks`
    emulated ranks on this one GPU: every rank's two local phases are timed
    on its own contiguous shard (flushed L2 before each), the exchanges are
    stacks of the ranks' buffers.  Reported: each phase's slowest rank and
    the merge -- the kernel part of one sharded step's latency; the two
    all-gathers of a few KB per head between GPUs are not in it (one GPU
    here).  Needle recall of the union of the shard selections."""
    cfg = wl.CONFIGS[name]
    B, Hq, Hkv, N, k = cfg.B, cfg.H_q, cfg.H_kv, cfg.N, cfg.topk
    scale = 1.0 / math.sqrt(128)
    w = wl.make_workload(cfg, wl.SEED_BASE + wl.CONFIG_ORDER.index(name), device=dev, steps=1)
    flush_buf = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    stream = torch.cuda.current_stream()
    n = N // ranks
    shards = []
    for r in range(ranks):
        K = w.K[:, :, r * n:(r + 1) * n].contiguous()
        V = w.V[:, :, r * n:(r + 1) * n].contiguous()
        codes = torch.zeros((B, Hkv, n, 4), dtype=torch.int32, device=dev)
        H.hata_hash_keys(K, w.W_H, codes, 0, n)
        ws = torch.empty(H.hata_decode_workspace_size(B, Hq, Hkv, n, k), dtype=torch.uint8,
                         device=dev)
        sl = torch.full((B,), n, dtype=torch.int32, device=dev)
        shards.append((K, V, codes, ws, sl))
    hist = torch.empty((ranks, B, Hq, H.HATA_SP_HIST_WORDS), dtype=torch.int32, device=dev)
    part = torch.empty((ranks, B, Hq, H.HATA_SP_PART_WORDS), device=dev)
    sel = torch.empty((ranks, B, Hq, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, 128), device=dev)

    def ev():
        return torch.cuda.Event(enable_timing=True)

    t1, t2, tm = [], [], []
    for it in range(8):
        e1 = [(ev(), ev()) for _ in range(ranks)]
        e2 = [(ev(), ev()) for _ in range(ranks)]
        em = (ev(), ev())
        for r, (K, V, codes, ws, sl) in enumerate(shards):
            torch.sum(flush_buf)
            e1[r][0].record(stream)
            H.hata_sp_score(w.q[0], w.W_H, codes, K, V, sl, n, k, ws, hist[r])
            e1[r][1].record(stream)
        for r, (K, V, codes, ws, sl) in enumerate(shards):
            torch.sum(flush_buf)
            e2[r][0].record(stream)
            H.hata_sp_attend(hist, r, codes, K, V, sl, n, Hq, 128, k, scale, ws, part[r],
                             sel_idx=sel[r])
            e2[r][1].record(stream)
        em[0].record(stream)
        H.hata_sp_merge(part, out)
        em[1].record(stream)
        torch.cuda.synchronize()
        if it >= 3:
            t1.append(max(a.elapsed_time(b) for a, b in e1))
            t2.append(max(a.elapsed_time(b) for a, b in e2))
            tm.append(em[0].elapsed_time(em[1]))
    for _, _, _, ws, _ in shards:
        H.hata_workspace_check(ws)
    sel_c = sel.cpu()
    hits = total = 0
    for b in range(B):
        for h in range(Hkv):
            got = set()
            for r in range(ranks):
                got |= {x + r * n for x in sel_c[r, b, h * cfg.G].tolist() if x >= 0}
            nd = set(x for x in w.planted[b, h].tolist() if x >= 0)
            hits += len(nd & got)
            total += len(nd)
    res = {"ranks_emulated": ranks, "tokens_per_rank": n,
           "score_us_slowest_rank": round(statistics.mean(t1) * 1e3, 2),
           "attend_us_slowest_rank": round(statistics.mean(t2) * 1e3, 2),
           "merge_us": round(statistics.mean(tm) * 1e3, 2),
           "kernel_us_per_step": round((statistics.mean(t1) + statistics.mean(t2)
                                        + statistics.mean(tm)) * 1e3, 2),
           "needle_recall": round(hits / max(total, 1), 4),
           "note": "one GPU: shards run one after another, exchanges are buffer stacks; the "
                   "NCCL all-gathers between GPUs are not timed"}
    del w, shards, hist, part, sel, out, flush_buf
    torch.cuda.empty_cache()
    return res


def run_hata(args, world, rank, local):
    cfg = bench_config(args)
    K_steps, W_steps = args.steps, args.warmup
    G_steps = min(K_steps, 16)  # side legs: warm-L2 steps and the CUDA Graph
    total_steps = W_steps + 3 * K_steps + G_steps + 6  # + the host-cache leg's 5 steps
    seed = wl.SEED_BASE + wl.CONFIG_ORDER.index(args.config) + 1000 * rank
    dev = torch.device("cuda", torch.cuda.current_device())
    w = wl.make_workload(cfg, seed, device=dev, steps=total_steps)
    B, Hq, Hkv, N = cfg.B, cfg.H_q, cfg.H_kv, cfg.N
    scale = 1.0 / math.sqrt(128)
    r = args.rbit
    W = wl.projection(w.W_H, r)  # r = 128: the workload's W_H itself
    codes = torch.zeros((B, Hkv, w.n_cap, r // 32), dtype=torch.int32, device=dev)
    H.hata_hash_keys(w.K, W, codes, 0, N)
    ws = torch.empty(H.hata_decode_workspace_size(B, Hq, Hkv, w.n_cap, cfg.topk),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((B, Hq, 128), device=dev)
    seq = (N + 1 + torch.arange(total_steps, dtype=torch.int32, device=dev))[:, None] \
        .expand(total_steps, B).contiguous()
    flush_buf = torch.zeros(FLUSH_BYTES // 8, dtype=torch.int64, device=dev)
    flush = L2Flush(flush_buf)
    stream = torch.cuda.current_stream()
    kv_elt = 2 if cfg.kv_dtype == "bf16" else 4

    def step(t, events=None):
        H.hata_decode_step(w.q[t], W, codes, w.K, w.V, seq[t], w.n_cap, cfg.topk, scale,
                           ws, out, k_new=w.k_new[t], v_new=w.v_new[t], events=events)

    # clocks are sampled from the warm-up on, through the timed region
    clk = ClockSampler(local).__enter__()
    for t in range(W_steps):
        flush()
        step(t)
    torch.cuda.synchronize()
    H.hata_workspace_check(ws)

    # timed region: the step alone (no events between its kernels, so each
    # kernel's launch overlaps its predecessor), bracketed by two events
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K_steps)]
    with clk:
        barrier(world)
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        for i in range(K_steps):
            flush()
            evs[i][0].record(stream)
            step(W_steps + i)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        barrier(world)
    H.hata_workspace_check(ws)
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]

    # per-kernel breakdown (untimed pass): events between the five kernels
    kevs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(K_steps)]
    for e6 in kevs:  # torch creates the CUDA event on first record; the library needs handles
        for e in e6:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(K_steps):
        flush()
        step(W_steps + K_steps + i, kevs[i])
        H.hata_workspace_check(ws)  # every step of this untimed pass is checked
    torch.cuda.synchronize()
    prep_ms = [e[0].elapsed_time(e[1]) for e in kevs]
    score_ms = [e[1].elapsed_time(e[2]) for e in kevs]
    select_ms = [e[2].elapsed_time(e[3]) for e in kevs]
    attend_ms = [e[3].elapsed_time(e[4]) for e in kevs]
    combine_ms = [e[4].elapsed_time(e[5]) for e in kevs]
    n_launch = H.hata_decode_kernel_launches(cfg.B, cfg.H_q, cfg.H_kv, w.n_cap, cfg.topk, w.K.dtype,
                                             r)
    fused = n_launch == 3
    cluster = n_launch == 1
    # four launches: one CTA per head, merged in shared memory
    attend_kernel = ("cluster_step_kernel" if cluster else
                     "fused_select_attend_kernel" if fused else
                     "attend_head_kernel" if n_launch == 4 else "attend_tc_kernel")
    split_ms = [e[0].elapsed_time(e[5]) for e in kevs]
    ms = statistics.mean(step_ms)
    ms_max = max_over_ranks(world, ms)

    e2e_ms, h2d, d2h, dense_ms = float("nan"), 0, 0, float("nan")
    side = None
    if not args.no_extras:
        e2e_ms, h2d, d2h, dense_ms = extras(args, cfg, w, codes, ws, out, seq, flush, stream,
                                            W_steps, K_steps, world)
        if rank == 0:  # no collectives inside; only rank 0 prints the line
            side = more_legs(cfg, w, codes, ws, out, seq, flush, stream, W_steps + 3 * K_steps,
                             G_steps)
    # ---- roofline ----
    peak, peak_kind = measured_peaks()
    kv_row = 128 * kv_elt
    attend_bytes = B * Hq * cfg.topk * 2 * kv_row           # selected K and V rows
    code_bytes = B * Hkv * (N + W_steps + K_steps // 2) * (r // 8)  # every code once per KV head
    attend_s = statistics.mean(attend_ms) / 1e3
    score_s = statistics.mean(score_ms) / 1e3
    step_bytes = attend_bytes + code_bytes
    fused_s = statistics.mean(select_ms) / 1e3  # fused step: the selection + attention kernel
    cluster_s = statistics.mean(prep_ms) / 1e3  # cluster step: its one kernel
    if cluster:
        # the one kernel of the step moves every code and the selected K/V rows
        roof_bytes, roof_s = step_bytes, cluster_s
        roof_src = "hash_aware_top_hata_b200/csrc/k_cluster.cu"
        roof_what = "cluster_step_kernel (hash + score + top-k + gather + softmax)"
    elif fused:
        # the selection + attention kernel moves the selected K/V rows
        roof_bytes, roof_s = attend_bytes, fused_s
        roof_src = "hash_aware_top_hata_b200/csrc/k_fused.cu"
        roof_what = "fused_select_attend_kernel (top-k + gather + softmax)"
    else:
        roof_bytes, roof_s = attend_bytes, attend_s
        roof_src = "hash_aware_top_hata_b200/csrc/k_attend.cu"
        roof_what = f"{attend_kernel} (gather + softmax)"
    achieved = roof_bytes / roof_s / 1e9
    line = {
        "metric": METRIC, "value": round(ms_max * 1e3, 2), "unit": UNIT, "n_gpus": world,
        "steps": K_steps, "warmup": W_steps, "ms_per_step": round(ms_max, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded Gaussian q/K/V, 2% planted keys, N(0,1/128) W_H)",
        "config": config_dict(cfg, "flushed before every timed step (512 MiB read)", r),
        "roofline": {"bound": "hbm", "kernel": roof_what,
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": profiled_traffic(cfg, attend_kernel, roof_src),
                     "peak_kind": peak_kind, "algorithmic_bytes_per_launch": roof_bytes},
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": round(step_bytes / (ms / 1e3) / 1e9, 1),
                          "frac_of_measured": round(step_bytes / (ms / 1e3) / 1e9 / peak, 4),
                          "frac_of_8000": round(step_bytes / (ms / 1e3) / 1e9 / 8000.0, 4)},
        "kernels_us": ({"cluster_step": round(cluster_s * 1e6, 2)} if cluster else
                       {"prep": round(statistics.mean(prep_ms) * 1e3, 2),
                        "score": round(score_s * 1e6, 2),
                        "select_attend": round(fused_s * 1e6, 2),
                        "sum_with_events": round(statistics.mean(split_ms) * 1e3, 2),
                        "score_gbs": round(code_bytes / score_s / 1e9, 1)}
                       if fused else
                       {"prep": round(statistics.mean(prep_ms) * 1e3, 2),
                        "score": round(score_s * 1e6, 2),
                        "select": round(statistics.mean(select_ms) * 1e3, 2),
                        "attend": round(attend_s * 1e6, 2),
                        # null: the heads were merged inside the attention CTAs
                        "combine": (round(statistics.mean(combine_ms) * 1e3, 2)
                                    if n_launch == 5 else None),
                        "sum_with_events": round(statistics.mean(split_ms) * 1e3, 2),
                        "score_gbs": round(code_bytes / score_s / 1e9, 1)}),
        "dense_us": _num(dense_ms * 1e3, 1),
        "speedup_vs_dense": None,
        "e2e": {"value": _num(e2e_ms * 1e3, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "side": side,
        # prep, score, select, attend (+ combine unless merged in the attention CTAs)
        "gpu_launches": n_launch * K_steps,
        "clocks": clk.summary(),
        "wall_s_timed_region": round(wall, 4),
    }
    # the speedup over dense decode attention at the same shape divides by
    # the faster of this library's dense kernel and torch SDPA
    sdpa_us = (side or {}).get("sdpa_dense_us")
    dense_cands = [(dense_ms * 1e3, "hata_dense_decode")]
    if sdpa_us:
        dense_cands.append((sdpa_us, "torch SDPA (enable_gqa)"))
    dense_cands = [c for c in dense_cands if c[0] == c[0]]
    if dense_cands:
        best_us, best_name = min(dense_cands)
        line["speedup_vs_dense"] = round(best_us / (ms * 1e3), 2)
        line["dense_baseline"] = {"us": round(best_us, 1), "impl": best_name}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle on one whole step over every host core, and whole heads
        # on one core (scaled to a step)
        ops, t_hash = oracle_step(cfg, w)
        try:
            t_all = oracle_step_time(cfg, w, ops, 0)
            heads = [(0, 0), (B - 1, Hq - 1)]
            per_head = ops.one_core_seconds_per_head(w.q[1].cpu().numpy(), N + 1, cfg.topk,
                                                     scale, heads)
            line["cpu_baseline"] = {"value": round(t_all * 1e6, 1), "unit": UNIT,
                                    "cores": ops.workers, "kind": "oracle",
                                    "sample": oracle_desc(cfg, ops),
                                    "one_core_us_per_step": round(per_head * B * Hq * 1e6, 1),
                                    "one_core_sample": f"{len(heads)} whole heads on one core, "
                                                       f"scaled to {B * Hq} heads",
                                    "prompt_hash_s": round(t_hash, 2)}
        finally:
            ops.close()
    if rank == 0 and world == 1 and not args.no_extras and not args.no_other_configs:
        del w, codes, ws, flush_buf
        torch.cuda.empty_cache()
        line["other_workloads"] = other_workloads(args, dev)
        line["other_workloads"]["llama31_8b_gqa_128k_r256"] = wide_code_leg(dev)
        line["other_workloads"]["needle_gqa_1m_seqpar8"] = seqpar_leg(dev)
    if rank == 0:
        from hash_aware_top_hata_b200 import build as hb
        line["build"] = hb.build_record()  # the library that ran, and its sources
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=wl.CONFIG_ORDER)
    ap.add_argument("--impl", default="hata", choices=["hata", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--context", type=int, default=0, help="override the context length")
    ap.add_argument("--batch", type=int, default=0, help="override the batch size")
    ap.add_argument("--topk", type=int, default=0, help="override the top-k budget")
    ap.add_argument("--rbit", type=int, default=128, choices=[32, 64, 128, 256],
                    help="hash width of the timed steps (other than 128: with --no-extras)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the e2e, dense and CPU legs (profiling runs)")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="skip the side measurements of the other large workloads")
    ap.add_argument("--decode-mode", default="auto",
                    choices=["auto", "multi_kernel", "fused", "cluster"],
                    help="step implementation: auto (the library's choice), the multi-kernel "
                         "step or the fused step")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.rbit != 128 and not args.no_extras:
        ap.error("--rbit other than 128 runs the timed steps only: add --no-extras")
    world, rank, local = dist_setup(args)
    if args.impl == "hata":
        H.hata_set_decode_mode({"auto": H.HATA_MODE_AUTO, "fused": H.HATA_MODE_FUSED,
                                "multi_kernel": H.HATA_MODE_MULTI_KERNEL,
                                "cluster": H.HATA_MODE_CLUSTER}[args.decode_mode])
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_hata(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
