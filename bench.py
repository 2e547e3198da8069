#!/usr/bin/env python
"""Benchmark of the paged-KV attention library on B200.

Headline: the paged GQA bf16 decode workload (batch 64 per GPU, context lengths uniform in
[512, 8192], Hq 32, Hkv 8, D 128, pages of 16 shuffled over a shared pool, N(0,1) inputs
rounded to bf16, scale 1/sqrt(128), causal). One step = one pa_forward over the whole batch
(split-KV decode kernel + merge kernel). Metric: algorithmic KV bytes per second (each
visible K/V row read once per sequence) -- GB/s.

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

Under torchrun each rank runs its own batch (seed + rank) on its own GPU: weak scaling, no
collective on the data path. Rank 0 prints one JSON line.

The reference arm (--impl reference) times the fp64 CPU oracle on the host cores, one bounded
sample of the same workload per step.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "decode KV GB/s & prefill TFLOPS, paged GQA attention (% of B200 roofline)"
L2_BYTES = 126 * 1024 * 1024


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def allreduce_max(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def allreduce_sum(x: float, ws: int) -> float:
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(ws: int) -> None:
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.15)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


_E2E = None


def e2e_library():
    """libpa_e2e.so (the end-to-end decode loop in C over the public C ABI), built beside libpa.so."""
    global _E2E
    if _E2E is None:
        P, I = ctypes.c_void_p, ctypes.c_int32
        lib = ctypes.CDLL(os.path.join(ROOT, "paged_kv_attention_39_b200", "libpa_e2e.so"))
        lib.pa_e2e_create.restype = P
        lib.pa_e2e_create.argtypes = [P, P, I, P, I, I, I, ctypes.c_int, P, ctypes.c_size_t, P, P, P, ctypes.c_int,
                                      I, I, I, I, ctypes.c_float, ctypes.c_int, I, P, P, ctypes.c_size_t,
                                      ctypes.c_size_t]
        lib.pa_e2e_run.restype = ctypes.c_int
        lib.pa_e2e_run.argtypes = [P, ctypes.c_int, P]
        lib.pa_e2e_destroy.restype = None
        lib.pa_e2e_destroy.argtypes = [P]
        lib.pa_e2e_uploaded_bytes.restype = ctypes.c_longlong
        lib.pa_e2e_uploaded_bytes.argtypes = [P]
        lib.pa_e2e_host_times.restype = None
        lib.pa_e2e_host_times.argtypes = [P, ctypes.POINTER(ctypes.c_double)]
        lib.pa_e2e_gpu_times.restype = None
        lib.pa_e2e_gpu_times.argtypes = [P, ctypes.POINTER(ctypes.c_double)]
        _E2E = lib
    return _E2E


def kernel_traffic(kernel_file: str, key: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)[key]
        src = open(os.path.join(ROOT, "paged_kv_attention_39_b200", "csrc", kernel_file), "rb").read()
        if d.get("source_sha256") != hashlib.sha256(src).hexdigest():
            return None
        return d
    except Exception:
        return None


def kernel_names(bits: int):
    """The PA_KERNEL_* bits of a call as names."""
    names = ["decode_tc", "prefill_tcgen05", "mla_tcgen05", "cuda_core", "merge", "sparse", "append",
             "backward_tc", "backward_cuda_core"]
    return [n for i, n in enumerate(names) if bits >> i & 1]


def time_forward(pa, plan, args_fn, steps, warmup, trace=True, sampler=None, ws=1):
    """W untimed calls, then K calls bracketed by barrier + synchronize; per-call trace events."""
    for _ in range(warmup):
        args_fn(None)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)] if trace else None
    trs = [pa.trace_events(e) for e in evs] if trace else None
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(ws)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    start.record()
    for i in range(steps):
        args_fn(trs[i] if trace else None)
    end.record()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    barrier(ws)
    ms = start.elapsed_time(end) / steps
    kern = comb = None
    if trace:
        kern = statistics.fmean(e[0].elapsed_time(e[1]) for e in evs)
        comb = statistics.fmean(e[1].elapsed_time(e[2]) for e in evs)
    return ms, kern, comb, clocks


def run_ours(args, ws, rank, local):
    import paged_kv_attention_39_b200 as pa
    from paged_kv_attention_39_b200 import workloads as W

    pa.load_library()
    hbm, tf_burst, tf_sust, peak_src = peaks()
    dev = torch.device("cuda", local)
    wl = W.c2_bf16_decode(args.seed + rank)
    kv_bytes = W.algorithmic_kv_bytes(wl)
    q = wl.q.to(dev)
    k = wl.k_cache.to(dev)
    v = wl.v_cache.to(dev)
    nq, hq, d = q.shape
    out = torch.empty(nq, hq, d, dtype=q.dtype, device=dev)
    lse = torch.empty(nq, hq, dtype=torch.float32, device=dev)
    plan = pa.plan_for(wl, device=local)
    pa.pa_plan_prepare(plan, q.dtype, hq, wl.num_kv_heads, d, d, wl.causal, wl.window)

    def step(tr):
        pa.pa_forward(plan, q, k, v, out, lse, wl.scale, wl.causal, wl.window, trace=tr)

    sampler = ClockSampler(local) if rank == 0 else None
    # the timed steps carry no instrumentation; a second, traced pass (events between the kernels of
    # each call) splits a step into the attention kernel and the merge for the roofline
    ms, _, _, clocks = time_forward(pa, plan, step, args.steps, args.warmup, False, sampler, ws)
    _, kern_ms, comb_ms, _ = time_forward(pa, plan, step, max(1, min(args.steps, 200)), 3, True, None, ws)
    launches_per_step = pa.pa_plan_get_info(plan)["last_launches"]
    ms_max = allreduce_max(ms, ws)
    total_bytes = allreduce_sum(kv_bytes, ws)
    value = total_bytes / (ms_max * 1e-3) / 1e9
    achieved = kv_bytes / (kern_ms * 1e-3) / 1e9
    traffic = kernel_traffic("decode.cu", "decode_mma_kernel")

    # ---- end to end through the public API with host buffers -------------------------------
    # A decode loop as a serving engine with asynchronous scheduling runs it, written in C over the
    # public C ABI (paged_kv_attention_39_b200/e2e/e2e_loop.cu, libpa_e2e.so): every step builds and
    # uploads its own plan (pa_plan_create + pa_plan_prepare: a new schedule per step, as lengths grow
    # and pages move) and copies its queries in from pinned host memory on an upload stream, runs
    # pa_forward, and copies out and lse back into pinned host memory on a download stream; two
    # steps are in flight, and the host waits for step i's result before it issues step i+2. The K
    # steps are timed as one region on the compute stream (the call returns once every result is on
    # the host), so every copy, upload and host gap is inside it.
    s = wl.sched
    lib = e2e_library()
    q_dev = [q, torch.empty_like(q)]
    out_dev = [out, torch.empty_like(out)]
    lse_dev = [lse, torch.empty_like(lse)]
    e2e_steps = 0 if args.no_e2e else max(3, min(args.steps, 200))
    sl, qo, bt = pa._i32(s.seq_lens), pa._i32(s.query_offsets), pa._i32(s.block_tables)
    q_src = wl.q.contiguous()
    main = torch.cuda.current_stream(dev)
    ptr2 = lambda ts: (ctypes.c_void_p * 2)(*(t.data_ptr() for t in ts))
    out_bytes, lse_bytes = out.numel() * out.element_size(), lse.numel() * 4
    loop = lib.pa_e2e_create(sl.data_ptr(), qo.data_ptr(), sl.numel(), bt.data_ptr(), bt.shape[1], s.page_size,
                             s.num_pages, local, q_src.data_ptr(), q_src.numel() * q_src.element_size(), ptr2(q_dev),
                             k.data_ptr(), v.data_ptr(), pa._DTYPES[q.dtype], hq, wl.num_kv_heads, d, d, wl.scale,
                             int(wl.causal), wl.window, ptr2(out_dev), ptr2(lse_dev), out_bytes, lse_bytes)
    if not loop:
        raise RuntimeError("end-to-end loop set-up failed")

    def e2e_loop(n):
        rc = lib.pa_e2e_run(loop, n, main.cuda_stream)
        if rc != 0:
            raise RuntimeError(f"end-to-end loop failed with code {rc}")

    e2e_ms = float("nan")
    if e2e_steps:
        e2e_loop(args.warmup)
        torch.cuda.synchronize()
        barrier(ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        e2e_loop(e2e_steps)
        e1.record()
        torch.cuda.synchronize()
        barrier(ws)
        e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = allreduce_max(e2e_ms, ws)
    e2e_val = total_bytes / (e2e_ms * 1e-3) / 1e9
    host_us = (ctypes.c_double * 6)()
    lib.pa_e2e_host_times(loop, host_us)
    gpu_us = (ctypes.c_double * 2)()
    lib.pa_e2e_gpu_times(loop, gpu_us)
    uploaded = lib.pa_e2e_uploaded_bytes(loop)
    lib.pa_e2e_destroy(loop)
    plan.close()

    extra = {}
    if not args.no_extra and rank == 0:
        extra = run_extra(args, pa, W, dev, hbm, tf_burst, peak_src)

    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) rounded to bf16; shuffled page pool)",
        "config": {
            "workload": f"paged GQA bf16 decode: batch {wl.sched.num_seqs}/GPU, context U[512,8192], "
                        "Hq 32, Hkv 8, D 128, page 16, causal",
            "kv_bytes_per_gpu_step": kv_bytes,
            "tokens_per_gpu_step": int(wl.sched.seq_lens.sum()),
            "l2": "inputs larger than L2 (%.2f GB of visible K/V vs 126 MB L2); no flush" % (kv_bytes / 1e9),
            "parallelism": f"replicas x{ws} (independent batches, no collective)",
        },
        "roofline": {
            "bound": "hbm",
            "kernel": "decode_mma_kernel",
            "achieved": round(achieved, 1),
            "peak": hbm,
            "peak_source": f"hbm_gbs {peak_src}",
            "unit": "GB/s",
            "frac": round(achieved / hbm, 4),
            "frac_note": f"of {peak_src}",
            "kernel_ms": round(kern_ms, 5),
            "merge_ms": round(comb_ms, 5),
            "traffic": (traffic["dram_bytes_per_launch"] * kv_bytes / traffic["kv_bytes_per_launch"]) if traffic else None,
            "traffic_source": traffic.get("source") if traffic else None,
            "frac_of_8tbs": round(achieved / 8000.0, 4),
        },
        "e2e": {
            "value": round(e2e_val, 2),
            "unit": "GB/s",
            "h2d_bytes_per_step": int(q_src.numel() * q_src.element_size() + uploaded),
            "d2h_bytes_per_step": int(out_bytes + lse_bytes),
            "host_us_per_step": {name: round(host_us[i] / max(1, e2e_steps), 1) for i, name in enumerate(
                ("plan_create", "plan_prepare", "copies", "forward", "plan_release", "wait"))},
            # device side of the same steps: the forward's kernels, and the compute stream idle
            # before each forward (waiting for the step's uploads or for the host to issue it)
            "gpu_us_per_step": {"forward": round(gpu_us[0] / max(1, e2e_steps - 1), 1),
                                "idle_before_forward": round(gpu_us[1] / max(1, e2e_steps - 2), 1)},
            "ms_per_step": round(e2e_ms, 4),
            "includes": "a C loop over the public C ABI (libpa_e2e.so); per step: a new plan (pa_plan_create + "
                        "pa_plan_prepare: schedule and work-list uploads) and the H2D of Q from pinned memory on "
                        "an upload stream, pa_forward, the D2H of out and lse into pinned memory on a download "
                        "stream; two steps in flight (step i+1's plan and upload overlap step i, step i's "
                        "download overlaps step i+1; the host waits for step i's result before issuing step "
                        "i+2); K steps timed as one region",
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if extra:
        result["extra"] = extra
    if rank == 0 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, kv_bytes)
    return result


def run_extra(args, pa, W, dev, hbm, tf_burst, peak_src, only=None):
    """The other configurations, timed the same way (few steps): context for the headline."""
    res = {}
    cfgs = [("bf16_chunked_prefill", W.c3_chunked_prefill), ("bf16_window_mixed", W.c4_window_mixed),
            ("bf16_window_mixed_decode_part", W.c4_decode_part), ("bf16_window_mixed_prefill_part", W.c4_prefill_part),
            ("bf16_mla_decode", W.c5_mla_decode), ("bf16_sparse_topk_decode", W.sparse_bf16_decode),
            ("fp16_decode", lambda sd: W.c2_decode_variant(sd, torch.float16, 128)),
            ("bf16_decode_d64", lambda sd: W.c2_decode_variant(sd, torch.bfloat16, 64)),
            ("bf16_decode_d256", lambda sd: W.c2_decode_variant(sd, torch.bfloat16, 256)),
            ("bf16_chunked_prefill_d256", lambda sd: W.c3_prefill_variant(sd, torch.bfloat16, 256)),
            ("bf16_append_chunk", W.append_chunk), ("bf16_backward_chunk", W.backward_chunk),
            ("bf16_mla_backward", W.mla_backward_small),
            ("bf16_mla_backward_decode_batch", W.mla_backward_decode_batch)]
    if only is not None:
        cfgs = [only]
    for name, fn in cfgs:
        if name == "bf16_sparse_topk_decode":
            res[name] = run_sparse(args, pa, W, dev, hbm, peak_src, only is not None)
            continue
        if name == "bf16_append_chunk":
            res[name] = run_append(args, pa, W, dev, hbm, peak_src)
            continue
        if name == "bf16_backward_chunk":
            res[name] = run_backward(args, pa, W, dev, tf_burst, peak_src)
            continue
        if name in ("bf16_mla_backward", "bf16_mla_backward_decode_batch"):
            res[name] = run_mla_backward(args, pa, W, dev, tf_burst, peak_src,
                                         "small" if name == "bf16_mla_backward" else "decode_batch")
            continue
        try:
            wl = fn(args.seed)
            flops = W.algorithmic_flops(wl)
            kvb = W.algorithmic_kv_bytes(wl)
            plan = pa.plan_for(wl, device=dev.index)
            if wl.kind == "mla":
                ql, qr = wl.q_latent.to(dev), wl.q_rope.to(dev)
                lat, rope = wl.latent_cache.to(dev), wl.rope_cache.to(dev)
                out = torch.empty(ql.shape, dtype=ql.dtype, device=dev)
                lse = torch.empty(ql.shape[:2], dtype=torch.float32, device=dev)

                def step(tr):
                    pa.pa_mla_forward(plan, ql, qr, lat, rope, out, lse, wl.scale, wl.causal, wl.window, trace=tr)
            else:
                q, k, v = wl.q.to(dev), wl.k_cache.to(dev), wl.v_cache.to(dev)
                out = torch.empty(q.shape[0], q.shape[1], wl.v_head_dim, dtype=q.dtype, device=dev)
                lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)

                def step(tr):
                    pa.pa_forward(plan, q, k, v, out, lse, wl.scale, wl.causal, wl.window, trace=tr)
            ms, _, _, _ = time_forward(pa, plan, step, args.extra_steps, args.warmup if only else 3, False, None, 1)
            _, kern, comb, _ = time_forward(pa, plan, step, args.extra_steps, 1, True, None, 1)
            res[name] = {
                "ms_per_step": round(ms, 4),
                "attention_kernels_ms": round(kern, 4),
                "merge_ms": round(comb, 4),
                "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                "kv_gbs": round(kvb / (ms * 1e-3) / 1e9, 1),
                "frac_tensor_of_%s" % peak_src: round(flops / (ms * 1e-3) / 1e12 / tf_burst, 4),
                "frac_hbm_of_%s" % peak_src: round(kvb / (ms * 1e-3) / 1e9 / hbm, 4),
                "algorithmic_gflop": round(flops / 1e9, 2),
                "algorithmic_kv_mb": round(kvb / 1e6, 1),
                "launches": pa.pa_plan_get_info(plan)["last_launches"],
                "kernels": kernel_names(pa.pa_plan_get_info(plan)["last_kernels"]),
            }
            plan.close()
            del wl
        except Exception as e:  # a failing extra must not hide the headline
            res[name] = {"error": str(e)[:300]}
    return res


def run_sparse(args, pa, W, dev, hbm, peak_src, alone):
    """Sparse top-K decode: one step = proxy scores + top-K selection + attention over the
    selected blocks + merge (pa_sparse_select then pa_sparse_forward)."""
    try:
        wl, bs, topk = W.sparse_bf16_decode(args.seed)
        plan = pa.plan_for(wl, device=dev.index)
        q, k, v = wl.q.to(dev), wl.k_cache.to(dev), wl.v_cache.to(dev)
        out = torch.empty(q.shape[0], q.shape[1], wl.v_head_dim, dtype=q.dtype, device=dev)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
        sel = torch.empty(q.shape[0], wl.num_kv_heads, topk, dtype=torch.int32, device=dev)

        def step(tr):
            pa.pa_sparse_select(plan, q, k, sel, wl.scale, bs, topk, wl.causal, wl.window)
            pa.pa_sparse_forward(plan, q, k, v, sel, out, lse, wl.scale, bs, wl.causal, wl.window)
        ms, _, _, _ = time_forward(pa, plan, step, args.extra_steps, args.warmup if alone else 3, False, None, 1)
        launches = pa.pa_plan_get_info(plan)["last_launches"] + 2
        nbytes = W.sparse_bytes(wl, bs, sel)
        plan.close()
        return {"ms_per_step": round(ms, 4), "block_size": bs, "topk": topk,
                "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac_hbm_of_%s" % peak_src: round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4),
                "algorithmic_mb": round(nbytes / 1e6, 1),
                "dense_kv_mb": round(W.algorithmic_kv_bytes(wl) / 1e6, 1), "launches": launches}
    except Exception as e:  # a failing extra must not hide the headline
        return {"error": str(e)[:300]}


def event_median(fn, before, steps, warmup):
    """Median device time of fn() over `steps` calls, each timed alone with CUDA events; before()
    runs untimed ahead of every call (an L2 flush, zeroing an accumulator)."""
    for _ in range(warmup):
        before()
        fn()
    ts = []
    for _ in range(steps):
        before()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def run_append(args, pa, W, dev, hbm, peak_src):
    """Paged append of the chunked-prefill batch's 4096 new K/V rows (33.6 MB read and written).
    The data is smaller than L2, so a 256 MB write flushes L2 before every timed call."""
    try:
        wl, nk, nv = W.append_chunk(args.seed)
        plan = pa.plan_for(wl, device=dev.index)
        k, v = wl.k_cache.to(dev), wl.v_cache.to(dev)
        nk, nv = nk.to(dev), nv.to(dev)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        ms = event_median(lambda: pa.pa_append(plan, nk, nv, k, v), flush.zero_, max(args.extra_steps, 10), 3)
        nbytes = W.append_bytes(wl)
        plan.close()
        return {"ms_per_step": round(ms, 4), "rows": wl.sched.num_queries * wl.num_kv_heads,
                "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                "frac_hbm_of_%s" % peak_src: round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4),
                "algorithmic_mb": round(nbytes / 1e6, 1), "launches": 1, "l2": "flushed before each call"}
    except Exception as e:  # a failing extra must not hide the headline
        return {"error": str(e)[:300]}


def run_backward(args, pa, W, dev, tf_burst, peak_src):
    """Recompute-based backward of a chunked-prefill batch (4 sequences, history U[0, 2048] plus
    256 queries): d_q written, d_k / d_v caches (float32) zeroed before and accumulated by each
    timed call."""
    try:
        wl, d_out = W.backward_chunk(args.seed)
        plan = pa.plan_for(wl, device=dev.index)
        q, k, v = wl.q.to(dev), wl.k_cache.to(dev), wl.v_cache.to(dev)
        d_out = d_out.to(dev)
        out = torch.empty(q.shape[0], q.shape[1], wl.v_head_dim, dtype=q.dtype, device=dev)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
        pa.pa_forward(plan, q, k, v, out, lse, wl.scale, wl.causal, wl.window)
        d_q = torch.empty(q.shape, dtype=torch.float32, device=dev)
        d_k = torch.empty(k.shape, dtype=torch.float32, device=dev)
        d_v = torch.empty(v.shape, dtype=torch.float32, device=dev)

        def zero():
            d_k.zero_()
            d_v.zero_()
        ms = event_median(lambda: pa.pa_backward(plan, q, k, v, out, lse, d_out, d_q, d_k, d_v, wl.scale,
                                                 wl.causal, wl.window), zero, max(args.extra_steps, 3), 2)
        flops = W.backward_flops(wl)
        launches = pa.pa_plan_get_info(plan)["last_launches"]
        plan.close()
        return {"ms_per_step": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                "frac_tensor_of_%s" % peak_src: round(flops / (ms * 1e-3) / 1e12 / tf_burst, 4),
                "algorithmic_gflop": round(flops / 1e9, 2), "launches": launches,
                "note": "Drow kernel, key-major dK/dV and query-major dQ on tcgen05 (no per-key atomics)"}
    except Exception as e:  # a failing extra must not hide the headline
        return {"error": str(e)[:300]}


def run_mla_backward(args, pa, W, dev, tf_burst, peak_src, batch="small"):
    """MLA backward of a decode batch: 4 sequences with context U[256, 1024] ("small"), or the MLA
    decode batch (32 sequences, context U[1024, 16384]); 128 heads, latent 512, rope 64. The gradient
    caches are zeroed before each timed call, outside the timed region."""
    try:
        wl, d_out = W.mla_backward_small(args.seed) if batch == "small" else W.mla_backward_decode_batch(args.seed)
        plan = pa.plan_for(wl, device=dev.index)
        ql, qr = wl.q_latent.to(dev), wl.q_rope.to(dev)
        lat, rope = wl.latent_cache.to(dev), wl.rope_cache.to(dev)
        d_out = d_out.to(dev)
        out = torch.empty(ql.shape, dtype=ql.dtype, device=dev)
        lse = torch.empty(ql.shape[:2], dtype=torch.float32, device=dev)
        pa.pa_mla_forward(plan, ql, qr, lat, rope, out, lse, wl.scale, wl.causal, wl.window)
        dql = torch.empty(ql.shape, dtype=torch.float32, device=dev)
        dqr = torch.empty(qr.shape, dtype=torch.float32, device=dev)
        dlat = torch.empty(lat.shape, dtype=torch.float32, device=dev)
        drope = torch.empty(rope.shape, dtype=torch.float32, device=dev)

        def zero():
            dlat.zero_()
            drope.zero_()
        ms = event_median(lambda: pa.pa_mla_backward(plan, ql, qr, lat, rope, out, lse, d_out, dql, dqr, dlat, drope,
                                                     wl.scale, wl.causal, wl.window), zero, max(args.extra_steps, 3), 2)
        flops = W.mla_backward_flops(wl)
        info = pa.pa_plan_get_info(plan)
        plan.close()
        tc = bool(info["last_kernels"] & pa.PA_KERNEL_BACKWARD_TC)
        return {"ms_per_step": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 2),
                "frac_tensor_of_%s" % peak_src: round(flops / (ms * 1e-3) / 1e12 / tf_burst, 4),
                "algorithmic_gflop": round(flops / 1e9, 2), "launches": info["last_launches"],
                "kernels": kernel_names(info["last_kernels"]),
                "note": ("Drow kernel, key tiles on tcgen05 (CTA pairs over the latent's column halves, TMA "
                         "reduce-adds), dQ per 64-column chunk on tcgen05" if tc else
                         "CUDA-core float32 kernel with atomics")}
    except Exception as e:  # a failing extra must not hide the headline
        return {"error": str(e)[:300]}


def run_single(args, ws, rank, local):
    """One of the other configurations as the only workload (profiling and tuning runs)."""
    import paged_kv_attention_39_b200 as pa
    from paged_kv_attention_39_b200 import workloads as W
    pa.load_library()
    hbm, tf_burst, _, peak_src = peaks()
    dev = torch.device("cuda", local)
    args.extra_steps = args.steps
    fns = {"bf16_chunked_prefill": W.c3_chunked_prefill, "bf16_window_mixed": W.c4_window_mixed,
           "bf16_mla_decode": W.c5_mla_decode, "tiny_fp32_decode": W.c1_tiny_fp32_decode,
           "bf16_sparse_topk_decode": W.sparse_bf16_decode, "bf16_window_mixed_decode_part": W.c4_decode_part,
           "bf16_window_mixed_prefill_part": W.c4_prefill_part,
           "fp16_decode": lambda sd: W.c2_decode_variant(sd, torch.float16, 128),
           "bf16_decode_d64": lambda sd: W.c2_decode_variant(sd, torch.bfloat16, 64),
           "bf16_decode_d256": lambda sd: W.c2_decode_variant(sd, torch.bfloat16, 256),
           "bf16_chunked_prefill_d256": lambda sd: W.c3_prefill_variant(sd, torch.bfloat16, 256),
           "bf16_append_chunk": W.append_chunk, "bf16_backward_chunk": W.backward_chunk,
           "bf16_mla_backward": W.mla_backward_small,
           "bf16_mla_backward_decode_batch": W.mla_backward_decode_batch}
    res = run_extra(args, pa, W, dev, hbm, tf_burst, peak_src, only=(args.workload, fns[args.workload]))
    r = res[args.workload]
    if args.workload in ("bf16_sparse_topk_decode", "bf16_append_chunk"):
        return {"metric": METRIC, "workload": args.workload, "value": r.get("gbs"), "unit": "GB/s",
                "steps": args.steps, "warmup": args.warmup, "detail": r}
    if args.workload in ("fp16_decode", "bf16_decode_d64", "bf16_decode_d256"):
        return {"metric": METRIC, "workload": args.workload, "value": r.get("kv_gbs"), "unit": "GB/s",
                "steps": args.steps, "warmup": args.warmup, "detail": r}
    return {"metric": METRIC, "workload": args.workload, "value": r.get("tflops"), "unit": "TFLOP/s",
            "steps": args.steps, "warmup": args.warmup, "detail": r}


def cpu_baseline(wl, kv_bytes, budget_s: float = 10.0):
    """The fp64 oracle, as it stands, on the host cores: whole workload, repeated ~budget_s."""
    import oracle
    from paged_kv_attention_39_b200 import workloads as W  # noqa: F401
    orc = oracle.get()
    cores = os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:
        orc.run(wl, nthreads=cores)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(kv_bytes * reps / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"the full headline workload (one GPU's batch), {reps} run(s) in {dt:.1f} s"}


def run_reference(args, ws, rank):
    """The oracle arm: each step runs the fp64 CPU oracle on a bounded sample of the workload."""
    import oracle
    from paged_kv_attention_39_b200 import workloads as W
    if rank != 0:
        return None
    orc = oracle.get()
    cores = os.cpu_count() or 1
    wl = W.c2_bf16_decode(args.seed)
    s = wl.sched
    # a sample of whole sequences sized so that warmup + steps fit about two minutes
    t0 = time.perf_counter()
    orc.run(wl, nthreads=cores, rows=list(range(0, wl.num_q_heads)))  # one sequence's rows
    one = max(time.perf_counter() - t0, 1e-4)
    budget = 120.0 / max(1, args.steps + args.warmup)
    nseq = int(max(1, min(s.num_seqs, budget / one)))
    rows = list(range(0, nseq * wl.num_q_heads))
    sub_bytes = 0
    per_tok = wl.num_kv_heads * (wl.head_dim + wl.v_head_dim) * 2
    for i in range(nseq):
        sub_bytes += int(s.seq_lens[i]) * per_tok
    for _ in range(args.warmup):
        orc.run(wl, nthreads=cores, rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.run(wl, nthreads=cores, rows=rows)
    dt = (time.perf_counter() - t0) / args.steps
    val = sub_bytes / dt / 1e9
    return {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) rounded to bf16; shuffled page pool)",
        "config": {"workload": "paged GQA bf16 decode: batch 64, context U[512,8192], Hq 32, Hkv 8, D 128, "
                               "page 16, causal", "parallelism": "host cores"},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {nseq} sequence(s) of the batch per step, all heads"},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-extra", action="store_true", help="skip the other configurations")
    ap.add_argument("--extra-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffer) leg")
    ap.add_argument("--workload", default="bf16_decode",
                    choices=["bf16_decode", "bf16_chunked_prefill", "bf16_window_mixed", "bf16_mla_decode", "bf16_sparse_topk_decode",
                             "bf16_window_mixed_decode_part", "bf16_window_mixed_prefill_part",
                             "tiny_fp32_decode", "fp16_decode", "bf16_decode_d64", "bf16_decode_d256",
                             "bf16_chunked_prefill_d256",
                             "bf16_append_chunk", "bf16_backward_chunk", "bf16_mla_backward",
                             "bf16_mla_backward_decode_batch"],
                    help="the headline is bf16_decode; the others run alone for profiling")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    ws, rank, local = dist_setup()
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
    elif args.workload != "bf16_decode":
        res = run_single(args, ws, rank, local)
    else:
        res = run_ours(args, ws, rank, local)
    if rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
