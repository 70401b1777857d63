"""Benchmark of pa_decode on B200: µs per call and KV HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config 2] [--no-extra]

One step is one pa_decode call (plan, partition kernel, reduce) over the GQA
decode workload (B=32, H_q=32, H_kv=8, D=128, 16-token blocks,
S~U[1024,8192], queryLen 1, window 0).  Its KV is 0.6 GB, larger than L2, so
steps run back to back.  The JSON line's value is whole-job KV GB/s: bytes of
K and V inside every row's visible span, plus q and dst, summed over ranks,
over the max-over-ranks device time.  The other named workloads are timed
per call (L2 flushed between calls; an event-bracketed launch alone costs
about 6 us on B200) and in steady state (back-to-back calls over several
copies of the KV pool, one per model layer), reported under "configs".

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload (the only reference this path has), on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged-attn decode µs/call and KV HBM GB/s (% of B200 peak) per config"
VARIANTS = {"auto": 0, "fma": 1, "mma": 2, "tc": 3}   # pa_params.force_variant values
FALLBACK_HBM_GBS = 6650.0


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(wl):
    """Bytes a call must move: K and V of every row's visible union span for
    every kv head, plus q and dst.  Union span of a row: positions
    [max(0, S-L+1-w), S) for w > 0, [0, S) otherwise.  Elements are 2 bytes
    (bf16) or 1 (FP8 codes); dst is always bf16."""
    s, l, w = wl.host_lists()
    kv_elem = wl.k_cache.element_size()
    kv = 0
    for S, L, W in zip(s, l, w):
        if L <= 0:
            continue
        lo = max(0, S - L + 1 - W) if W > 0 else 0
        kv += (S - lo) * wl.num_kv_heads * 2 * wl.head_dim * kv_elem
    qo = wl.num_tokens * wl.num_q_heads * wl.head_dim * (wl.q.element_size() + 2)
    return kv, qo


# --------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def _smi_id(self):
        """nvidia-smi id of this process's CUDA device (matched by UUID, since
        CUDA_VISIBLE_DEVICES may renumber devices)."""
        try:
            import torch
            want = str(torch.cuda.get_device_properties(self.index).uuid).lower()
            want = want.replace("gpu-", "").replace("-", "")
            out = subprocess.run(["nvidia-smi", "--query-gpu=index,uuid",
                                  "--format=csv,noheader"], capture_output=True,
                                 text=True, timeout=30).stdout
            for ln in out.splitlines():
                idx, uuid = [x.strip() for x in ln.split(",")]
                if uuid.lower().replace("gpu-", "").replace("-", "") == want:
                    return idx
        except Exception:
            pass
        return str(self.index)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self._smi_id()}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        note = "sampled every 100 ms over >= 1 s of the same calls just before and during the timed steps"
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": [], "samples": 0, "note": note}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "note": note}


# ------------------------------------------------------------ the GPU arm
def traffic_from_profiles(kernel_src_hash: str, workload: str):
    """DRAM bytes per launch of the partition kernel from the committed ncu
    summary, if it was taken on the current kernel source and this workload."""
    path = os.path.join(ROOT, "profiles", "partition_traffic.txt")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_source_sha256") == kernel_src_hash:
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_cache_474_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import paged_kv_cache_474_b200 as pa
    from paged_kv_cache_474_b200.workloads import CONFIG_TITLES, config_workload

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    wl = config_workload(args.config, device=device, kv_dtype=args.kv_dtype, rows=args.rows)
    kv_bytes, qo_bytes = algorithmic_bytes(wl)
    call_bytes = kv_bytes + qo_bytes

    p = pa.params_for(wl, force_variant=VARIANTS[args.variant])
    ws = pa.alloc_workspace(p, wl.block_size, device=device)
    if ws is not None:
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    rc, plan = pa.pa_plan(p, wl.block_size)
    out = torch.empty_like(wl.q)
    sh = pa._stream_handle(stream)
    args_c = (out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(), wl.v_cache.data_ptr(),
              wl.block_tables.data_ptr(), wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(),
              wl.scale, wl.window, wl.block_size)

    def step(events=None):
        import ctypes
        if events is not None:
            arr = (ctypes.c_void_p * 2)(events[0].cuda_event, events[1].cuda_event)
            p.profile_events = ctypes.addressof(arr)
            step._keep = arr
        else:
            p.profile_events = None
        rc = pa.pa_decode(*args_c, p, sh)
        if rc != pa.PA_OK:
            raise RuntimeError(pa.pa_last_error())

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # Clock sampling covers a pre-roll of the same calls (at least ~1 s of
    # load, so nvidia-smi sees the clocks under this work) and the timed steps.
    with ClockSampler(local_rank) as clocks:
        t_pre = time.perf_counter()
        while time.perf_counter() - t_pre < 1.0:
            for _ in range(20):
                step()
            torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    elapsed_ms = t0.elapsed_time(t1)
    # Partition-kernel duration: the same steps again, with the library
    # recording events just before and after the partition kernel (kept out
    # of the timed region above so the reduce's early launch is undisturbed).
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in kev:     # torch creates the CUDA event on its first record
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for k in range(args.steps):
        step(kev[k])
    torch.cuda.synchronize()
    kern_ms = [a.elapsed_time(b) for a, b in kev]
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    elapsed_max = float(t.item())
    status = pa.pa_device_status(clear=True)
    if status:
        raise RuntimeError(f"device status {status:#x}")

    ms_per_step = elapsed_max / args.steps
    value = call_bytes * args.steps * world / (elapsed_max * 1e-3) / 1e9
    kern_avg_ms = sum(kern_ms) / len(kern_ms)
    peak, peak_kind = measured_hbm_peak()
    achieved = call_bytes / (kern_avg_ms * 1e-3) / 1e9
    title = CONFIG_TITLES[args.config] + ("" if args.kv_dtype == "bf16" else ", FP8 e4m3 KV")
    if args.rows is not None:
        title += f", first {wl.batch} rows"
    if args.variant != "auto":
        title += f", {args.variant} variant forced"
    traffic = traffic_from_profiles(kernel_source_hash(), title)

    # end to end through the host-buffer entry point
    e2e = run_e2e(args, wl, pa, torch, device, world)

    launches = args.steps * (1 if plan.one_shot else 2)
    result = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "us_per_call": round(ms_per_step * 1e3, 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if args.kv_dtype == "bf16" else "fp8_e4m3 KV, bf16 q/dst",
        "data": "synthetic",
        "config": {"workload": title,
                   "kv_bytes_per_call": kv_bytes, "q_dst_bytes_per_call": qo_bytes,
                   "l2": "inputs larger than L2 (no flush between steps)",
                   "parallelism": f"replicas x{world} (rows shard, no collective)",
                   "plan": {k: v for k, v in plan.as_dict().items()
                            if k in ("variant", "partition_tokens", "max_partitions",
                                     "one_shot", "grid_x", "grid_y", "grid_z",
                                     "block_threads", "ctas_per_sm")}},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "peak_source": peak_kind,
                     "kernel": {pa.PA_VARIANT_MMA: "pa_partition_mma_kernel",
                                pa.PA_VARIANT_TC: "pa_partition_tc_kernel"}.get(
                                    plan.variant, "pa_partition_fma_kernel"),
                     "kernel_us": round(kern_avg_ms * 1e3, 2),
                     "kernel_timing": "CUDA events the library records around the partition "
                                      "kernel, averaged over the timed steps re-run",
                     "traffic": traffic},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks.summary(),
    }
    return result


def run_e2e(args, wl, pa, torch, device, world):
    """Same metric through pa_decode_host: per step, pinned host q, block
    tables and lengths are copied in and dst is copied back."""
    import numpy as np
    S = np.ascontiguousarray(wl.seq_lens.cpu().numpy())
    L = np.ascontiguousarray(wl.query_lens.cpu().numpy())
    W = None if wl.windows is None else np.ascontiguousarray(wl.windows.cpu().numpy())
    bt = wl.block_tables.cpu().contiguous().pin_memory()
    Sp = torch.from_numpy(S).pin_memory()
    Lp = torch.from_numpy(L).pin_memory()
    Wp = None if W is None else torch.from_numpy(W).pin_memory()
    q_host = wl.q.cpu().contiguous().pin_memory()
    out_host = torch.empty(wl.q.shape, dtype=torch.bfloat16).pin_memory()
    # the device call's parameters (operand types and scales), hints left to
    # pa_decode_host, which computes them from the host lengths
    p = pa.params_for(wl, hints=False)
    p.windows = None if Wp is None else Wp.data_ptr()
    n = pa.pa_host_workspace_size(p, wl.block_size, wl.window, Sp.data_ptr(), Lp.data_ptr())
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    p.workspace, p.workspace_bytes = ws.data_ptr(), n
    stream = torch.cuda.current_stream()
    sh = pa._stream_handle(stream)

    def call():
        rc = pa.pa_decode_host(out_host.data_ptr(), q_host.data_ptr(), wl.k_cache.data_ptr(),
                               wl.v_cache.data_ptr(), bt.data_ptr(), Sp.data_ptr(),
                               Lp.data_ptr(), wl.scale, wl.window, wl.block_size, p, sh)
        if rc != pa.PA_OK:
            raise RuntimeError(pa.pa_last_error())

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call()
    torch.cuda.synchronize()
    el = time.perf_counter() - t0
    if world > 1:
        import torch.distributed as dist
        t = torch.tensor([el], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        el = float(t.item())
    kv, qo = algorithmic_bytes(wl)
    h2d = (q_host.numel() * q_host.element_size() + bt.numel() * 4 + S.nbytes + L.nbytes +
           (0 if W is None else W.nbytes))
    d2h = out_host.numel() * 2
    return {"value": round((kv + qo) * args.steps * world / el / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "us_per_call": round(el / args.steps * 1e6, 2),
            "api": "pa_decode_host (pinned host q/tables/lengths in, dst out, stream sync)"}


def run_other_configs(args, local_rank):
    """µs/call and KV GB/s of the five named workloads, L2 flushed before each
    call, median of the timed calls."""
    import torch
    import paged_kv_cache_474_b200 as pa
    from paged_kv_cache_474_b200.workloads import CONFIG_NAMES, config_workload

    device = torch.device("cuda", local_rank)
    peak, _ = measured_hbm_peak()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nflush = max(4 * l2, 512 << 20)
    flush_w = torch.empty(nflush, dtype=torch.uint8, device=device)
    flush_r = torch.ones(nflush // 4, dtype=torch.float32, device=device)

    def flush_l2():
        # Write a buffer larger than L2 (evicts the workload), then read
        # another one so the lines left in L2 are clean: otherwise the timed
        # call would pay for writing the flush buffer's dirty lines back.
        flush_w.zero_()
        flush_r.sum()

    stream = torch.cuda.current_stream()
    sh = pa._stream_handle(stream)

    def measure(wl, steady_calls):
        kv, qo = algorithmic_bytes(wl)
        p = pa.params_for(wl)
        ws = pa.alloc_workspace(p, wl.block_size, device=device)
        if ws is not None:
            p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
        out = torch.empty(wl.q.shape, dtype=torch.bfloat16, device=device)
        c = (out.data_ptr(), wl.q.data_ptr(), wl.k_cache.data_ptr(), wl.v_cache.data_ptr(),
             wl.block_tables.data_ptr(), wl.seq_lens.data_ptr(), wl.query_lens.data_ptr(),
             wl.scale, wl.window, wl.block_size)
        for _ in range(3):
            pa.pa_decode(*c, p, sh)
        n = max(10, min(50, args.steps * 5))
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for a, b in ev:
            flush_l2()
            a.record(stream)
            rc = pa.pa_decode(*c, p, sh)
            b.record(stream)
            if rc != pa.PA_OK:
                raise RuntimeError(pa.pa_last_error())
        torch.cuda.synchronize()
        us = statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3
        gbs = (kv + qo) / (us * 1e-6) / 1e9
        _, info = pa.pa_plan(p, wl.block_size)
        r = {"us_per_call": round(us, 2), "kv_bytes": kv, "gbs": round(gbs, 1),
             "frac_of_peak": round(gbs / peak, 4),
             "l2": "flushed before each call (write then read 4x L2)",
             "partitions": info.max_partitions, "partition_tokens": info.partition_tokens}
        if steady_calls:
            # Steady state: back-to-back calls over several copies of the KV
            # pool (one per layer of a model, >= 4x L2 in total), so no call
            # finds its KV in L2 and each call's launch overlaps the previous
            # call's tail.
            pool = wl.k_cache.numel() * wl.k_cache.element_size() * 2
            nlay = max(1, min(64, -(-(4 * l2) // pool)))
            layers = [(wl.k_cache, wl.v_cache)] + [(wl.k_cache.clone(), wl.v_cache.clone())
                                                   for _ in range(nlay - 1)]

            def layer_call(i):
                k, v = layers[i % nlay]
                return pa.pa_decode(c[0], c[1], k.data_ptr(), v.data_ptr(), *c[4:], p, sh)
            for i in range(nlay):
                layer_call(i)
            m = max(nlay, steady_calls)
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            t0.record(stream)
            for i in range(m):
                layer_call(i)
            t1.record(stream)
            torch.cuda.synchronize()
            us_ss = t0.elapsed_time(t1) * 1e3 / m
            gbs_ss = (kv + qo) / (us_ss * 1e-6) / 1e9
            r.update({"steady_us_per_call": round(us_ss, 2), "steady_gbs": round(gbs_ss, 1),
                      "steady_frac_of_peak": round(gbs_ss / peak, 4),
                      "steady": f"{m} back-to-back calls over {nlay} KV pool copies"})
            del layers
        del ws, out
        return r

    res = {}
    for cfg in (1, 2, 3, 4, 5):
        wl = config_workload(cfg, device=device)
        res[CONFIG_NAMES[cfg]] = measure(wl, 20 if cfg == 5 else 200)
        del wl
        torch.cuda.empty_cache()
    # The same workloads with FP8 e4m3 KV caches (per-tensor scales): half
    # the KV bytes per token; GB/s counts the bytes actually moved.
    for cfg in (2, 3, 4, 5):
        wl = config_workload(cfg, device=device, kv_dtype="fp8_e4m3")
        res[CONFIG_NAMES[cfg] + "/fp8_kv"] = measure(wl, 20 if cfg == 5 else 200)
        del wl
        torch.cuda.empty_cache()
    # The ExecuTorch page's standalone kernel benchmark shape (B=1, H_q=16,
    # H_kv=2, D=256, one decode token) over a paged cache, per context length.
    from paged_kv_cache_474_b200.workloads import make_workload
    sweep = {}
    for lk in (64, 512, 4096, 8192, 16384):
        wl = make_workload(seq_lens=[lk], query_lens=[1], num_q_heads=16, num_kv_heads=2,
                           head_dim=256, block_size=16, seed=lk, device=device)
        r = measure(wl, 0)
        sweep[str(lk)] = {"us_per_call": r["us_per_call"], "gbs": r["gbs"]}
        del wl
    res["executorch_shape_B1_Hq16_Hkv2_D256"] = sweep
    if pa.pa_device_status(clear=True):
        raise RuntimeError("device status set during the per-config runs")
    return res


# ------------------------------------------------------- the oracle arm
def oracle_sample_run(wl, rows, nthreads=0):
    """Runs the float64 oracle on the given rows of a workload (all heads);
    returns (seconds, kv+q+dst bytes of the sample, threads used)."""
    import oracle
    sub, _ = wl.subset(rows)
    pr = oracle.problem_from_workload(sub)
    sub_l = pr.query_lens.tolist()
    kv = 0
    for j, b in enumerate(sorted(set(rows))):
        S = int(pr.seq_lens[j])
        Lb = sub_l[j]
        W = int(pr.windows[j]) if pr.windows is not None else pr.window
        lo = max(0, S - Lb + 1 - W) if W > 0 else 0
        kv += (S - lo) * pr.hkv * 2 * pr.d * 2
    qo = 2 * sum(sub_l) * pr.hq * pr.d * 2
    threads = oracle.max_threads(nthreads)
    t0 = time.perf_counter()
    oracle.decode(pr, nthreads=nthreads)
    return time.perf_counter() - t0, kv + qo, threads


def _rows_for_budget(wl, budget_s):
    """Rows of the workload whose oracle pass takes about budget_s seconds
    (every row when the whole workload fits)."""
    rows = list(range(wl.batch))
    t, _, _ = oracle_sample_run(wl, rows[:2])
    n = max(2, min(len(rows), int(budget_s / max(t / 2, 1e-6))))
    return rows[:n]


def cpu_baseline(args, target_s=12.0):
    """The oracle as it stands, timed on this host's cores on a bounded
    sample of the bench workload: whole passes over as many rows as fit a few
    seconds, repeated until about target_s seconds of CPU work."""
    from paged_kv_cache_474_b200.workloads import config_workload
    wl = config_workload(args.config, device="cpu")
    rows = _rows_for_budget(wl, 3.0)
    tot_t, tot_b, passes, thr = 0.0, 0, 0, 1
    while tot_t < target_s and passes < 1000:
        t, b, thr = oracle_sample_run(wl, rows)
        tot_t += t
        tot_b += b
        passes += 1
    return {"value": round(tot_b / tot_t / 1e9, 4), "unit": "GB/s", "cores": thr,
            "kind": "oracle",
            "sample": (f"rows 0..{len(rows) - 1} of {wl.batch} (all heads), {passes} passes, "
                       f"{tot_t:.1f} s"),
            "seconds": round(tot_t, 2)}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from paged_kv_cache_474_b200.workloads import CONFIG_TITLES, config_workload
    wl = config_workload(args.config, device="cpu")
    # per step: every row whose oracle pass fits ~2 s, so K+W steps end in minutes
    rows = _rows_for_budget(wl, 2.0)
    # Under torchrun every process starts with OMP_NUM_THREADS=1, but only this
    # rank works: give the oracle all of the host's cores, as at N=1.
    nthreads = len(os.sched_getaffinity(0)) if world > 1 else 0
    for _ in range(args.warmup):
        oracle_sample_run(wl, rows, nthreads)
    tot_t = 0.0
    tot_b = 0
    thr = 1
    for _ in range(args.steps):
        t, b, thr = oracle_sample_run(wl, rows, nthreads)
        tot_t += t
        tot_b += b
    value = tot_b / tot_t / 1e9
    sample = f"rows 0..{len(rows) - 1} of {wl.batch} (all heads) per step"
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(tot_t / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic",
        "config": {"workload": CONFIG_TITLES[args.config], "sample": sample},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": thr,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--kv-dtype", choices=["bf16", "fp8_e4m3"], default="bf16",
                    help="KV cache element type of the timed workload (FP8: per-tensor scaled e4m3)")
    ap.add_argument("--variant", choices=sorted(VARIANTS), default="auto",
                    help="kernel variant of the timed workload (profiling; auto = the dispatcher's)")
    ap.add_argument("--rows", type=int, default=None,
                    help="keep only the first rows of the workload (a reduced case for profiling)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the per-config table and the CPU baseline")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        result = run_ours(args, rank, world, local_rank)
        if rank == 0 and not args.no_extra:
            result["configs"] = run_other_configs(args, local_rank)
            if world == 1:
                result["cpu_baseline"] = cpu_baseline(args)
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
