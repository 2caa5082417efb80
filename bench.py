"""Benchmark of the DSA hot path (indexer + top-k + sparse MLA) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = the three kernels of one layer -- Lightning-Indexer scores, top-k, sparse MLA -- over one
batch of the workload through the C ABI (dsa_index_scores, dsa_topk, dsa_sparse_mla), inputs resident
in HBM, with the batch plan computed once per batch (it depends only on the batch's lengths, so a
model computes it once per forward pass for all its layers). `layer_with_plan_us` is the whole
`dsa_layer` call, plan included, and `plan_us` the plan alone. Each timed step is bracketed by CUDA
events on the launching stream, with a 256 MiB L2 flush (untimed) between steps. Under torchrun every rank runs
its own batch (weak scaling, no collective on the data path); rank 0 prints one JSON line with the
max-over-ranks time.

The JSON line also carries
  roofline      the dominant kernel's achieved algorithmic bytes/s against the measured HBM peak,
                from per-stage CUDA-event timings of the same kernels;
  e2e           the same metric through the public API with host (pinned) inputs: per step the
                queries and batch metadata go host->device and the output comes back; the paged
                caches stay resident (they are the cache, not per-step inputs);
  cpu_baseline  the CPU oracle (float64 numpy) timed on this host on a bounded sample of rows;
  short_prefill the masked MHA mode (the dense fallback for short prefill) on two shapes of its
                own, L = 2048 with 16 heads and k = 512, and L = 4096 with 128 heads and k = 2048:
                mask + attention kernels, event-timed, in TFLOP/s of the dense causal work
                against the measured bf16 peak.
`--impl reference` times that oracle alone as the reference arm.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA layer µs (indexer+top-k+sparse MLA), query tok/s; % of HBM/FP8 roofline"
UNIT = "query tok/s"
DEFAULT_WORKLOAD = "decode_64x16k"
L2_FLUSH_BYTES = 256 << 20


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu record, or None when there is no
    record for this workload or the kernel's source changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        if rec["workload"] != workload:
            return None
        with open(os.path.join(ROOT, rec["source"]), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
                return None
        return int(rec["dram_bytes_per_launch"])
    except Exception:
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ---------------------------------------------------------------------------------------------
# algorithmic work per step (what the method must move / compute), from the workload's sizes

def algorithmic(hb):
    """Bytes each kernel must move and FLOPs it must do for one step of this batch."""
    req, pos = _positions(hb)
    T = hb.total_q
    nhI = hb.qI.shape[1]
    H = hb.q.shape[1]
    k = hb.wl.topk
    vis = pos + 1                                   # visible positions per query row
    sel = np.minimum(vis, k)                        # selected positions per row
    # indexer: every request's visible keys once per query group (decode: once per request), the
    # queries, weights and scales, and the score rows written
    keys_per_req = np.zeros(len(hb.seq_lens), np.int64)
    for b in range(len(hb.seq_lens)):
        m = int(hb.cu_q[b + 1] - hb.cu_q[b])
        if m:
            keys_per_req[b] = int(hb.seq_lens[b])
    idx_bytes = int(keys_per_req.sum()) * (128 + 4) + T * (nhI * 128 + 4 + nhI * 4) + int(vis.sum()) * 4
    idx_flops = int(vis.sum()) * 2 * nhI * 128
    topk_bytes = int(vis.sum()) * 4 + T * k * 4
    mla_bytes = int(sel.sum()) * (576 * 2 + 4) + T * H * 576 * 2 + T * H * 512 * 2
    mla_flops = int(sel.sum()) * (2 * H * 576 + 2 * H * 512)
    return dict(index_scores=(idx_bytes, idx_flops), topk=(topk_bytes, 0), sparse_mla=(mla_bytes, mla_flops))


def _positions(hb):
    req, pos = hb.row_positions()
    return req, pos


# ---------------------------------------------------------------------------------------------
# multi-rank plumbing: every rank runs its own batch (weak scaling by request), no data exchange

def rank_seed(rank: int) -> int:
    """Seed of the synthetic batch a rank runs: ranks own disjoint, equally shaped batches."""
    return rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest per-rank value (timings are reported as the slowest rank's)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(rows_per_rank: int, world: int, ms: float) -> float:
    """Whole-job query tokens per second: all ranks' rows over the slowest rank's step time."""
    return world * rows_per_rank / (ms / 1e3)


# ---------------------------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    """Samples SM clock and clock-event reasons every few ms while the timed region runs (NVML reads
    only; nothing is set). Falls back to nvidia-smi's loop mode when NVML is unavailable."""

    # NVML clocks-event reason bits
    REASONS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None

    def _run(self, pynvml, h):
        while not self._stop.is_set():
            try:
                mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                try:
                    bits = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    bits = pynvml.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                self.samples.append((mhz, bits))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(pynvml, h), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "source": "nvml"}
        mhz = [m for m, _ in self.samples]
        reasons = sorted({n for _, b in self.samples for n, bit in self.REASONS.items() if b & bit})
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples), "source": "nvml"}


# ---------------------------------------------------------------------------------------------
# oracle timing (CPU baseline / reference arm)

def short_prefill_mha(dev, timed_mean, n, tf_peak, wl, label):
    """The masked MHA mode (expanded heads, the DSA mask) on one whole-prefill request of workload
    `wl` (its length, heads and k). The index sets are random valid sets (the dense tiles' work does
    not depend on which positions are selected). Algorithmic work: the causal pairs L(L+1)/2 times
    2H(192 + 128) FLOPs."""
    import torch
    import sparse_attention_12_b200 as dsa
    from sparse_attention_12_b200 import synth
    L, H, k = int(wl.seq_lens[0]), wl.n_heads, wl.topk
    x = synth.make_mha_inputs(wl, seed=0)
    S = torch.from_numpy(synth.random_index_sets(wl.seq_lens, wl.q_per_req, k, seed=0)).to(dev)
    i32 = lambda v: torch.tensor(v, dtype=torch.int32, device=dev)
    bt = torch.arange((L + 63) // 64, dtype=torch.int32, device=dev)[None].contiguous()
    batch = dsa.Batch(i32([L]), i32([0, L]), bt, int(bt.shape[1]), L, L, L)
    plan = dsa.plan(batch, 16)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    q, kk, v = bf(x.q), bf(x.k), bf(x.v)
    out = torch.empty((L, H, 128), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(16, dsa.load().dsa_masked_mha_workspace_size(batch.ref(), H, k)), dtype=torch.uint8,
                     device=dev)
    fn = lambda: dsa.masked_mha(batch, plan, q, kk, v, S, wl.softmax_scale, out=out, ws=ws)
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    status = dsa.status_read(plan)
    if status != 0:
        raise RuntimeError(f"device status {status} in the masked MHA mode")
    ms = timed_mean(fn, n)
    flops = L * (L + 1) / 2 * 2 * H * (192 + 128)
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": label, "us": 1e3 * ms, "algorithmic_flops": flops,
            "TFLOPs": tf, "peak_TFLOPs": tf_peak, "frac": tf / tf_peak, "launches": 2,
            "note": "mask kernel + attention kernel, one call, event-timed; random valid index sets"}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count() or 1


def time_oracle(hb, budget_s: float = 12.0, max_rows: int = 64):
    """Run the oracle on a bounded sample of query rows; returns (rows/s, rows, seconds)."""
    from oracle import dsa_oracle as O
    req, pos = O.query_positions(hb.seq_lens, hb.cu_q)
    T = hb.total_q
    tau = hb.wl.softmax_scale
    k = hb.wl.topk
    order = np.random.default_rng(0).permutation(T)
    done, t0 = 0, time.perf_counter()
    for t in order[:max_rows]:
        I = O.index_scores_row(int(t), req, pos, hb.block_table, hb.qI, hb.qI_scale, hb.wI, hb.kI_cache,
                               hb.kI_scale)
        S = O.topk_select(I, k)
        O.sparse_mla_row(int(t), req, S, hb.block_table, hb.q, hb.kv_cache, tau)
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done / dt, done, dt


# ---------------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-short-prefill", action="store_true")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    from sparse_attention_12_b200 import synth
    wl = synth.workload(args.workload)

    if args.impl == "reference":
        if rank != 0:
            return 0
        hb = synth.make_batch(wl, seed=0)
        budget = max(2.0, min(60.0, 8.0 * max(args.steps, 1) / max(args.steps + args.warmup, 1)))
        for _ in range(args.warmup):
            time_oracle(hb, budget_s=0.5, max_rows=1)
        per_step = []
        rows_total, secs_total = 0, 0.0
        for _ in range(args.steps):
            rate, rows, dt = time_oracle(hb, budget_s=budget / max(args.steps, 1), max_rows=hb.total_q)
            per_step.append(hb.total_q / rate)   # seconds a full step would take at this rate
            rows_total += rows
            secs_total += dt
        value = rows_total / secs_total
        ms = 1e3 * hb.total_q / value
        cores = blas_threads()
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": wl.name, "requests": wl.batch, "query_rows": wl.total_q,
                           "context": max(wl.seq_lens), "topk": wl.topk, "index_heads": wl.n_heads_index,
                           "heads": wl.n_heads},
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                                 "sample": f"{rows_total} query rows of {wl.name}, full path per row, "
                                           f"extrapolated to the {hb.total_q}-row step"},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    import torch
    import sparse_attention_12_b200 as dsa

    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    torch.cuda.set_device(dev)
    dsa.load()

    hb = synth.make_batch(wl, seed=rank_seed(rank))
    db = dsa.DeviceBatch(hb, device=dev)
    T = hb.total_q
    stream = torch.cuda.current_stream()
    out = torch.empty((T, db.H, 512), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(16, dsa.layer_workspace_size(db.batch, db.nhI, db.H, db.k)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # the batch plan, once per batch; the layer's three kernels per step
    plan_t = dsa.plan(db.batch, db.nhI)
    ld = (hb.max_seq_len + 127) // 128 * 128
    scores = torch.empty((T, ld), dtype=torch.float32, device=dev)
    S = torch.empty((T, db.k), dtype=torch.int32, device=dev)
    mla_ws_n = dsa.load().dsa_sparse_mla_workspace_size(db.batch.ref(), db.H, db.k)
    mla_ws = torch.empty(max(16, mla_ws_n), dtype=torch.uint8, device=dev)
    topk_ws_n = dsa.load().dsa_topk_workspace_size(db.batch.ref(), db.k)
    topk_ws = torch.empty(max(16, topk_ws_n), dtype=torch.uint8, device=dev) if topk_ws_n else None
    stages = {
        "index_scores": lambda: dsa.index_scores(db.batch, plan_t, db.qI, db.qI_scale, db.wI, db.kI_cache,
                                                 db.kI_scale, scores=scores, ld=ld),
        "topk": lambda: dsa.topk(db.batch, plan_t, scores, db.k, S=S, ws=topk_ws),
        "sparse_mla": lambda: dsa.sparse_mla(db.batch, plan_t, db.q, db.kv_cache, S, db.softmax_scale, out=out,
                                             ws=mla_ws),
    }

    def step():
        for fn in stages.values():
            fn()

    def layer_call():
        dsa.layer(db.batch, db.qI, db.qI_scale, db.wI, db.kI_cache, db.kI_scale, db.q, db.kv_cache, db.k,
                  db.softmax_scale, out=out, ws=ws)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(max(args.warmup, 0)):
        step()
        layer_call()
    torch.cuda.synchronize()
    for plan_ws in (plan_t, ws):  # the layer call keeps its plan at the start of its workspace
        status = dsa.status_read(plan_ws)
        if status != 0:
            raise RuntimeError(f"device status {status} after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    barrier()
    with sampler:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        barrier()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = max_over_ranks(statistics.mean(times), dist, dev)
    value = job_throughput(T, world, ms)

    # the whole dsa_layer call (plan included) and the plan alone, same protocol
    def timed_mean(fn, n):
        ts = []
        for i in range(n):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.mean(ts)

    n_extra = max(3, min(args.steps, 50))
    layer_plan_ms = max_over_ranks(timed_mean(layer_call, n_extra), dist, dev)
    plan_ms = max_over_ranks(timed_mean(lambda: dsa.plan(db.batch, db.nhI, plan_t), n_extra), dist, dev)

    # per-stage timings of the same kernels (roofline of the dominant one)
    stage_ms = {n: [] for n in stages}
    for i in range(max(3, min(args.steps, 20))):
        for name, fn in stages.items():
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            stage_ms[name].append(a.elapsed_time(b))
    stage_ms = {n: statistics.mean(v) for n, v in stage_ms.items()}
    work = algorithmic(hb)
    hbm_peak, tf_peak, peak_src = measured_peaks()
    dominant = max(stage_ms, key=stage_ms.get)
    dom_bytes = work[dominant][0]
    achieved = dom_bytes / (stage_ms[dominant] / 1e3) / 1e9
    stage_report = {n: {"us": 1e3 * stage_ms[n], "GBps": work[n][0] / (stage_ms[n] / 1e3) / 1e9,
                        "TFLOPs": work[n][1] / (stage_ms[n] / 1e3) / 1e12 if work[n][1] else 0.0}
                    for n in stages}
    total_bytes = sum(w[0] for w in work.values())

    # the step before the layer: writing every query row's new key and latent row into the caches
    # (not part of the step; timed after the layer measurements because it rewrites those slots)
    g = torch.Generator(device=dev).manual_seed(7)
    k_new = torch.randn((T, 128), generator=g, device=dev, dtype=torch.float32)
    c_new = torch.randn((T, 576), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    cw_ms = timed_mean(lambda: dsa.cache_write(db.batch, plan_t, k_new, c_new, db.kI_cache, db.kI_scale,
                                               db.kv_cache), max(3, min(args.steps, 20)))
    cw_bytes = T * (128 * 4 + 576 * 2 + 128 + 4 + 576 * 2)

    short = None
    if not args.no_short_prefill:
        reps = max(3, min(args.steps, 20))
        short = [short_prefill_mha(dev, timed_mean, reps, tf_peak, synth.workload("prefill_2048"),
                                   "prefill_2048 (masked MHA mode): L 2048, 16 heads, k 512"),
                 short_prefill_mha(dev, timed_mean, reps, tf_peak,
                                   synth.custom("prefill_4k_128h", [4096], [4096], n_heads=128, topk=2048),
                                   "masked MHA mode at the model's head count: L 4096, 128 heads, k 2048")]

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.cpu().pin_memory()
        h_in = {"qI": pin(db.qI.view(torch.uint8)), "qI_scale": pin(db.qI_scale), "wI": pin(db.wI),
                "q": pin(db.q), "seq_lens": pin(db.batch.seq_lens), "cu_q": pin(db.batch.cu_q),
                "block_table": pin(db.batch.block_table)}
        d_in = {n: torch.empty_like(t, device=dev) for n, t in h_in.items()}
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in h_in.values())
        d2h = h_out.numel() * h_out.element_size()
        batch2 = dsa.Batch(d_in["seq_lens"], d_in["cu_q"], d_in["block_table"], hb.num_pages, T, db.batch.c.max_q,
                           hb.max_seq_len)
        qI_d = d_in["qI"].view(torch.float8_e4m3fn)

        def e2e_step():
            for n in h_in:
                d_in[n].copy_(h_in[n], non_blocking=True)
            dsa.layer(batch2, qI_d, d_in["qI_scale"], d_in["wI"], db.kI_cache, db.kI_scale, d_in["q"],
                      db.kv_cache, db.k, db.softmax_scale, out=out, ws=ws)
            h_out.copy_(out, non_blocking=True)

        for _ in range(max(args.warmup, 1)):
            e2e_step()
        barrier()
        es, ee = [], []
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            es.append(a)
            ee.append(b)
        barrier()
        e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in zip(es, ee)), dist, dev)
        e2e = {"value": job_throughput(T, world, e_ms), "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "ms_per_step": e_ms}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, rows, dt = time_oracle(hb, budget_s=12.0)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{rows} of the {T} query rows of {wl.name} through the whole path in "
                         f"{dt:.1f} s (float64 numpy, BLAS threads)"}
        try:  # the same oracle on one thread, a smaller sample
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                r1, n1, d1 = time_oracle(hb, budget_s=4.0)
            cpu["single_thread"] = {"value": r1, "unit": UNIT, "cores": 1,
                                    "sample": f"{n1} query rows in {d1:.1f} s"}
        except ImportError:
            pass

    launches_per_step = 3 + (1 if mla_ws_n > 0 else 0) + (1 if topk_ws_n > 0 else 0)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "layer_us": 1e3 * ms,
        "layer_with_plan_us": 1e3 * layer_plan_ms, "plan_us": 1e3 * plan_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp8e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
        "config": {"workload": wl.name, "requests": wl.batch, "query_rows": T, "context": max(wl.seq_lens),
                   "topk": wl.topk, "index_heads": wl.n_heads_index, "heads": wl.n_heads, "page_size": 64,
                   "l2": "256 MiB flush between timed steps", "parallelism": f"{world} independent ranks",
                   "step": "dsa_index_scores + dsa_topk + dsa_sparse_mla, batch plan computed once per batch"},
        "roofline": {"bound": "hbm", "kernel": dominant, "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "algorithmic_bytes": dom_bytes,
                     "traffic": recorded_traffic(dominant + "_kernel", wl.name), "peak_source": peak_src},
        "layer_roofline": {"algorithmic_bytes": total_bytes,
                           "achieved_GBps": total_bytes / (ms / 1e3) / 1e9,
                           "frac": total_bytes / (ms / 1e3) / 1e9 / hbm_peak},
        "stages": stage_report,
        "cache_write": {"us": 1e3 * cw_ms, "GBps": cw_bytes / (cw_ms / 1e3) / 1e9, "algorithmic_bytes": cw_bytes,
                        "note": "the step before the layer, not in the step; one launch, event-timed"},
        "short_prefill": short,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
