#!/usr/bin/env python
"""Benchmark: prefix-aware batched decode attention on B200.

One step = the whole hot path over one decode batch: pack on the host
(pa_plan_create: tree block table, profit model, split, tile selection), the
async upload of the plan, forward and merge on the GPU (pa_decode_step).  The
headline workload is the largest one of the five (stateful sessions: 32
sessions of 32768-131072 context tokens, 16 single-token queries each, batch
512, 32/8 heads, head_dim 128); the four others are measured in the same run
and reported under "per_config".

Metric: decode-attention queries/s (B / time per step), with the unique-KV bytes
per second beside it as a fraction of the measured HBM bandwidth.  The roofline
object credits the algorithmic bytes of the forward + merge launches: unique
KV (each shared page once), q, out, lse, the fp32 partial rows that are
written and read back, and the plan image.

Timing: W warm-up steps, then K steps bracketed by a barrier and a device sync
on both sides, timed with CUDA events on the launching stream; max over ranks.
KV pools larger than L2 are used as they are; smaller ones rotate over device
copies whose total exceeds L2, so no step finds its KV in L2.

--gpus N: N ranks, one per GPU, each with its own batch (seed + rank): weak
scaling, no collective on the data path.  Under torchrun the ranks come from
the environment; without it bench.py starts them itself.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

_ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, _ROOT)

METRIC = "decode-attn queries/s; unique-KV HBM GB/s as % of B200 peak (1 GPU)"
UNIT = "queries/s"
L2_BYTES = 126 * 2 ** 20


def peaks():
    p = os.path.join(_ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during a timed region.

    Samples carry nvidia-smi's own timestamps; only those inside the timed
    regions (each marked by mark_start / mark_end, plus 100 ms for the lag of
    the driver's counters) are summarised, so idle samples taken before, after
    and between them do not enter the median."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []
        self.proc = None
        self.t0 = self.t1 = None
        self.windows = []  # [start, end] of each timed region

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def mark_start(self):
        self.windows.append([time.time(), None])

    def mark_end(self):
        self.windows[-1][1] = time.time()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append([x.strip() for x in line.split(",")])

    @staticmethod
    def _when(field: str):
        try:
            return datetime.datetime.strptime(field, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [s for s in self.samples if len(s) >= 10 and s[2].replace(".", "").isdigit()]
        wins = self.windows or ([[self.t0, self.t1]] if self.t0 is not None else [])
        wins = [(a, (b or time.time()) + 0.1) for a, b in wins]

        def within(s):
            t = self._when(s[0]) or 0.0
            return any(a <= t <= b for a, b in wins)

        inside = [s for s in rows if not wins or within(s)]
        for a, b in wins:
            if not any(a <= (self._when(s[0]) or 0.0) <= b for s in inside):
                # a region shorter than the sampling period: the next sample
                inside += [s for s in rows if (self._when(s[0]) or 0.0) >= a][:1]
        sm = [float(s[2]) for s in inside]
        smax = [float(s[3]) for s in rows if s[3].replace(".", "").isdigit()]
        power = [float(s[4]) for s in inside if s[4].replace(".", "").isdigit()]
        reasons = set()
        for s in inside:
            for n, v in zip(self.REASONS, s[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "power_w_max": max(power) if power else None,
                "reasons": sorted(reasons), "samples": len(inside),
                "note": "samples inside the timed regions only (nvidia-smi timestamps, 20 ms period)"}


def kernels_hash() -> str:
    """sha256 prefix of kernels.cu's code: its lines with // comments and
    surrounding blanks removed, so an edit of the comments alone keeps a
    capture of the same code valid."""
    import hashlib
    src = open(os.path.join(_ROOT, "prefix_aware_decode_b200", "csrc", "kernels.cu"), encoding="utf-8").read()
    code = []
    for line in src.splitlines():
        line = line.split("//", 1)[0].strip()
        if line:
            code.append(line)
    return hashlib.sha256("\n".join(code).encode()).hexdigest()[:16]


def measured_traffic(config: int):
    """DRAM bytes per step of the forward launches from the committed ncu capture,
    or None when the kernels have changed since it was taken."""
    try:
        t = json.load(open(os.path.join(_ROOT, "profiles", "traffic.json")))
        if kernels_hash() != t.get("kernels_cu_sha256_16"):
            return None
    except OSError:
        return None
    w = t.get("workloads", {}).get(str(config))
    return sum(w.values()) if w else None


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def spawn_ranks(n: int) -> int:
    """Runs this script as n ranks (one per GPU) under torch.distributed.run."""
    import socket

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = ["timeout", "-k", "60", "1800", sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def reference_arm(args, rank, world):
    """The fp64 CPU oracle timed on the host cores (bounded sample per step)."""
    if rank != 0:
        return
    import oracle
    from prefix_aware_decode_b200 import workload as wl

    w = wl.make_config(args.config, seed=1000 + args.config)
    cores = os.cpu_count() or 1
    n = min(w.B, args.ref_queries)
    qs = np.arange(n, dtype=np.int32)
    for _ in range(args.warmup):
        oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=qs[:1], nthreads=cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=qs, nthreads=cores)
    dt = (time.perf_counter() - t0) / args.steps
    value = n / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.CONFIG_NAMES[args.config], "queries_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"first {n} of {w.B} queries of the workload per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))


def merged_rows(plan) -> int:
    """Partial rows that go through the fp32 partial buffers (pairs with two or
    more partial rows; a pair with one row is written straight to the output)."""
    import ctypes

    import prefix_aware_decode_b200 as pad
    img = plan.host_image()
    h = pad.PaImageHeader.from_buffer_copy(img[:ctypes.sizeof(pad.PaImageHeader)].tobytes())
    n = h.batch * h.num_kv_heads
    off = np.frombuffer(img[h.off_prow_off:h.off_prow_off + 4 * (n + 1)].tobytes(), dtype=np.int32)
    cnt = np.diff(off)
    return int(cnt[cnt > 1].sum())


def algorithmic_bytes(w, st: dict, n_merged: int) -> dict:
    """Bytes the forward + merge launches must move for one batch: the unique
    KV, q, out and lse, the partial rows written and read back (G rows of D + 1
    floats each), and the plan image."""
    G = w.Hq // w.Hkv
    parts = {"unique_kv": int(w.unique_kv_bytes), "q": int(w.q.nbytes), "out": w.B * w.Hq * w.D * 2,
             "lse": w.B * w.Hq * 4, "partials": 2 * n_merged * G * (w.D + 1) * 4, "image": int(st["image_bytes"])}
    parts["total"] = sum(parts.values())
    return parts


class Bench:
    def __init__(self, args, rank, world, local):
        import torch

        self.torch = torch
        self.args, self.rank, self.world = args, rank, world
        torch.cuda.set_device(local)
        self.dist = None
        if world > 1:
            import datetime

            import torch.distributed as dist
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
            self.dist = dist
        self.hbm_peak, self.bf16_peak, self.peak_kind = peaks()
        self.stream = torch.cuda.current_stream()

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max_over_ranks(self, x: float) -> float:
        if self.dist is None:
            return x
        t = self.torch.tensor([x], device="cuda")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def dev(self, a):
        return self.torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(self.torch.bfloat16)

    def measure(self, config: int, headline: bool) -> dict:
        """Times K steps of pa_decode_step on one workload; returns its fields."""
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad
        from prefix_aware_decode_b200 import workload as wl

        w = wl.make_config(config, seed=1000 + config + 7919 * self.rank, scale=args.scale)
        pool_bytes = w.k_pool.nbytes + w.v_pool.nbytes
        copies = args.copies or (1 if pool_bytes > 3 * L2_BYTES else int(np.ceil(3 * L2_BYTES / pool_bytes)) + 1)
        q = self.dev(w.q)
        k0, v0 = self.dev(w.k_pool), self.dev(w.v_pool)
        pools = [(k0, v0)] + [(k0.clone(), v0.clone()) for _ in range(copies - 1)]
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        kv_lens, block_table = w.kv_lens, w.block_table

        probe = pad.Plan(kv_lens, block_table, w.num_pages, w.Hq, w.Hkv, w.D)
        pst = probe.stats()
        n_merged = merged_rows(probe)
        ws_bytes = probe.workspace_bytes
        probe.close()
        algo = algorithmic_bytes(w, pst, n_merged)
        ws = torch.empty((ws_bytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")

        def mk_events(n):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
            for e in evs:
                e.record(stream)
            return evs

        nsteps = args.warmup + args.steps
        prof_every = 4  # profiling events on every 4th step of the timed region
        step_events = [mk_events(4) if i % prof_every == 0 else None for i in range(nsteps)]
        host_us = []
        # one stepper per pool copy (their arguments are marshalled once), all
        # on the same image buffer
        stepper = pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, q, k0, v0, ws, out, lse, stream=stream)
        steppers = [stepper] + [pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, q, kc, vc, ws, out, lse, stream=stream,
                                               images=stepper.images) for kc, vc in pools[1:]]

        def step(i):
            t = time.perf_counter()
            steppers[i % copies](kv_lens, block_table, events=step_events[i])
            host_us.append((time.perf_counter() - t) * 1e6)

        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        chk = pad.Plan(kv_lens, block_table, w.num_pages, w.Hq, w.Hkv, w.D)
        chk.upload(ws, stream)
        chk.attend(q, k0, v0, ws, out, lse, stream)
        status = chk.device_status(ws, stream)
        chk.close()
        assert status == pad.PA_OK, status

        clocks = ClockSampler(torch.cuda.current_device())
        clocks.start()
        time.sleep(0.3)
        self.barrier()
        torch.cuda.synchronize()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        host_us.clear()
        clocks.mark_start()
        ev0.record(stream)
        for i in range(args.warmup, nsteps):
            step(i)
        ev1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
        # forward + merge on the device: the step's plan, uploaded once, attended
        # K times back to back over the rotated pools (the host stays ahead, so
        # nothing but the launches is timed)
        dplan = pad.Plan(kv_lens, block_table, w.num_pages, w.Hq, w.Hkv, w.D)
        dplan.upload(ws, stream)
        for i in range(args.warmup):
            dplan.attend(q, *pools[i % copies], ws, out, lse, stream)
        torch.cuda.synchronize()
        time.sleep(0.3)  # the same start as the decode loop's: clocks not yet held down by the power cap
        self.barrier()
        clocks.mark_start()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(2):  # queued ahead of the first event, so the device is busy when it fires
            dplan.attend(q, *pools[i % copies], ws, out, lse, stream)
        d0.record(stream)
        for i in range(args.steps):
            dplan.attend(q, *pools[(i + 2) % copies], ws, out, lse, stream)
        d1.record(stream)
        torch.cuda.synchronize()
        fwd_ms = self.max_over_ranks(d0.elapsed_time(d1)) / args.steps
        dstatus = dplan.device_status(ws, stream)
        dplan.close()
        assert dstatus == pad.PA_OK, dstatus
        clocks.mark_end()
        self.barrier()
        clk = clocks.stop()
        ms_step = self.max_over_ranks(ev0.elapsed_time(ev1)) / args.steps
        # forward + merge inside the decode steps: when the device has caught
        # up with the host, the first event also counts the host's submission
        # of the launches
        fwd_in_step_ms = statistics.mean(step_events[i][0].elapsed_time(step_events[i][1])
                                         for i in range(args.warmup, nsteps) if step_events[i] is not None)
        launches = (pst["mma_ctas"] > 0) + (pst["simt_warps"] > 0) + (pst["num_tail_pairs"] > 0)
        achieved = algo["total"] / (fwd_ms * 1e-3) / 1e9
        hbm = self.hbm_peak
        res = {
            "workload": wl.CONFIG_NAMES[config], "batch": w.B, "seed": w.seed,
            "unique_kv_bytes": int(w.unique_kv_bytes), "prefix_ratio": round(w.prefix_ratio, 4),
            "l2": (f"KV pools ({pool_bytes / 2**20:.0f} MiB) larger than L2" if copies == 1 else
                   f"KV pools rotated over {copies} device copies ({copies * pool_bytes / 2**20:.0f} MiB > L2)"),
            "ms_per_step": ms_step, "queries_per_s": w.B * self.world / (ms_step * 1e-3),
            "unique_kv_frac_of_hbm": w.unique_kv_bytes / (ms_step * 1e-3) / 1e9 / hbm,
            "forward_merge_us": fwd_ms * 1e3,
            "forward_merge_us_in_step": fwd_in_step_ms * 1e3,
            "forward_queries_per_s": w.B / (fwd_ms * 1e-3),
            "forward_unique_kv_frac_of_hbm": w.unique_kv_bytes / (fwd_ms * 1e-3) / 1e9 / hbm,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": measured_traffic(config),
                         "algorithmic_bytes": algo,
                         "kernel": "forward launches of both tile classes with the merge fused, plus the tail "
                                   "merge launch when the plan has one, timed together with CUDA events over "
                                   "K back-to-back calls of the step's plan",
                         "launches_per_step": launches,
                         "peak_kind": f"{self.peak_kind} hbm_gbs (copy, burst)"},
            "plan_us": pst["plan_us"], "host_us_per_step_median": statistics.median(host_us),
            "plan": {k: pst[k] for k in ("num_segments_simt", "num_segments_mma", "simt_warps", "mma_ctas",
                                         "num_tail_pairs", "num_partial_rows", "read_kv_bytes",
                                         "workspace_bytes", "image_bytes")},
            "clocks": clk, "gpu_launches": args.steps * launches,
            "gpu_launches_device_loop": args.steps * launches,
        }

        if config == 1 and args.amortise > 0:
            res["amortised"] = self.amortised(w)
        if config == 2 and args.layers > 0:
            res["multi_layer"] = self.multi_layer(w, q, k0, v0, ws, out, lse, pool_bytes)
        if config == 2 and args.decode_steps > 0 and args.layers > 0:
            res["decode_steps"] = self.decode_steps(w, q, k0, v0, out, lse)
        if config == 5 and args.session_steps > 0:
            del pools
            pools = None
            torch.cuda.empty_cache()
            res["sessions"] = self.sessions(w)
        if headline and not args.no_e2e:
            res.update(self.e2e(w, q, k0, v0, out, lse, ws_bytes))
        if headline and self.rank == 0 and not args.no_cpu_baseline:
            import oracle
            cores = os.cpu_count() or 1
            n = min(w.B, args.ref_queries)
            qs = np.arange(n, dtype=np.int32)
            t0 = time.perf_counter()
            oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=qs, nthreads=cores)
            dt = time.perf_counter() - t0
            res["cpu_baseline"] = {"value": n / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                                   "sample": f"first {n} of {w.B} queries of the same workload, one pass"}
        del pools, q, k0, v0, out, lse, ws, stepper, steppers
        torch.cuda.empty_cache()
        return res

    def sessions(self, w) -> dict:
        # registered queries against live sessions (config-5 shape: 32
        # sessions x 16 queries): each session's context grows by a quarter of
        # its final length per step through the session page allocator, and
        # every step's batch of registered queries is planned and run;
        # reported: forward + merge time against the mean context length
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad
        from prefix_aware_decode_b200.session import SessionPool

        n = args.session_steps
        final = [int(w.kv_lens[16 * s]) for s in range(w.B // 16)]
        n_pages = sum((L + 15) // 16 for L in final) + 64
        pool = SessionPool(n_pages, 16)
        # pool contents do not change the work: one bf16 N(0,1) fill on the device
        kp = torch.randn((n_pages, w.Hkv, 16, w.D), device="cuda", dtype=torch.float32).to(torch.bfloat16)
        vp = torch.randn_like(kp)
        q = torch.randn((w.B, w.Hq, w.D), device="cuda", dtype=torch.float32).to(torch.bfloat16)
        for sid in range(len(final)):
            pool.open(sid)
            for j in range(16):
                pool.register(sid, 16 * sid + j)
        out = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
        points = []
        grown = [0] * len(final)
        for step in range(n):
            for sid, L in enumerate(final):
                target = L * (step + 1) // n
                pool.append(sid, target - grown[sid])
                grown[sid] = target
            qids, _, bt, kv = pool.batch()
            plan = pad.Plan(kv, bt, n_pages, w.Hq, w.Hkv, w.D)
            st = plan.stats()
            ws = plan.alloc_workspace()
            plan.upload(ws, stream)
            for _ in range(3):
                plan.attend(q, kp, vp, ws, out, lse, stream)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(args.steps):
                plan.attend(q, kp, vp, ws, out, lse, stream)
            b.record(stream)
            torch.cuda.synchronize()
            assert plan.device_status(ws, stream) == pad.PA_OK
            us = a.elapsed_time(b) / args.steps * 1e3
            points.append({"mean_context_tokens": float(np.mean(kv)), "forward_merge_us": us,
                           "queries_per_s": len(qids) / (us * 1e-6),
                           "unique_kv_frac_of_hbm": st["unique_kv_bytes"] / (us * 1e-6) / 1e9 / self.hbm_peak,
                           "plan_us": st["plan_us"]})
            plan.close()
            del ws
        del kp, vp
        torch.cuda.empty_cache()
        return {"steps": points,
                "note": "32 sessions x 16 registered queries; contexts grow to the workload's lengths in equal "
                        "steps through session.SessionPool; each step plans the registered queries' batch and "
                        "times forward + merge on the device (KV resident); time per query grows with the "
                        "context's bytes, the unique-KV fraction of HBM is the per-step efficiency"}

    def amortised(self, w) -> dict:
        # config 1 is a few hundred KB, far below what one launch can stream:
        # n independent config-1 problems planned together, forward + merge
        # launches timed on the device (plan time beside it, outside the timing)
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad
        from prefix_aware_decode_b200 import workload as wl

        wa = wl.config1_stream(args.amortise, seed=w.seed)
        qa, ka, va = self.dev(wa.q), self.dev(wa.k_pool), self.dev(wa.v_pool)
        oa = torch.empty((wa.B, wa.Hq, wa.D), dtype=torch.bfloat16, device="cuda")
        la = torch.empty((wa.B, wa.Hq), dtype=torch.float32, device="cuda")
        pa_ = pad.Plan(wa.kv_lens, wa.block_table, wa.num_pages, wa.Hq, wa.Hkv, wa.D)
        wsa = pa_.alloc_workspace()
        pa_.upload(wsa, stream)
        for _ in range(3):
            pa_.attend(qa, ka, va, wsa, oa, la, stream)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.steps):
            pa_.attend(qa, ka, va, wsa, oa, la, stream)
        a1.record(stream)
        torch.cuda.synchronize()
        t_us = a0.elapsed_time(a1) / args.steps * 1e3
        assert pa_.device_status(wsa, stream) == pad.PA_OK
        algo = algorithmic_bytes(wa, pa_.stats(), merged_rows(pa_))
        r = {"problems": args.amortise, "batch": wa.B, "unique_kv_bytes": int(wa.unique_kv_bytes),
             "forward_merge_us": t_us, "queries_per_s": wa.B / (t_us * 1e-6),
             "unique_kv_frac_of_hbm": wa.unique_kv_bytes / (t_us * 1e-6) / 1e9 / self.hbm_peak,
             "roofline_frac": algo["total"] / (t_us * 1e-6) / 1e9 / self.hbm_peak,
             "plan_us": pa_.stats()["plan_us"],
             "note": "one plan and upload, then forward + merge launches timed back to back on the device "
                     f"(the KV of all problems stays resident; {wa.unique_kv_bytes / 1e6:.0f} MB, above L2)"}
        pa_.close()
        return r

    def multi_layer(self, w, q, k0, v0, ws, out, lse, pool_bytes) -> dict:
        # one decode step of a model: the plan is made and uploaded once and
        # read by every layer's attention (each layer has its own KV pools)
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad

        lay = [(k0.clone(), v0.clone()) for _ in range(args.layers)]

        def layer_step():
            p_ = pad.Plan(w.kv_lens, w.block_table, w.num_pages, w.Hq, w.Hkv, w.D)
            p_.upload(ws, stream)
            for kl_, vl_ in lay:
                p_.attend(q, kl_, vl_, ws, out, lse, stream)
            p_.close()

        for _ in range(3):
            layer_step()
        torch.cuda.synchronize()
        nst = max(3, args.steps // 10)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        th = time.perf_counter()
        b0.record(stream)
        for _ in range(nst):
            layer_step()
        b1.record(stream)
        th = (time.perf_counter() - th) / nst * 1e6
        torch.cuda.synchronize()
        t_us = b0.elapsed_time(b1) / nst * 1e3
        del lay
        return {"layers": args.layers, "us_per_step": t_us, "us_per_layer": t_us / args.layers,
                "queries_per_s_per_layer": w.B * args.layers / (t_us * 1e-6),
                "unique_kv_frac_of_hbm": w.unique_kv_bytes * args.layers / (t_us * 1e-6) / 1e9 / self.hbm_peak,
                "host_us_per_step": th,
                "note": "per step: pack + upload once, then one forward + merge per layer, each layer with its "
                        f"own KV pools ({args.layers} x {pool_bytes / 2**20:.0f} MiB)"}

    def decode_steps(self, w, q, k0, v0, out, lse) -> dict:
        # decode steps of a model: every request gains one token per step (a
        # page of its own when its last one is full); the plan of each step
        # comes from the previous one by pa_plan_advance and serves every
        # layer.  The host time of a plan made from scratch for the same
        # inputs is taken beside it.
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad

        n = args.decode_steps
        n_pages = w.num_pages + w.B * (n // w.P + 2)
        kv = w.kv_lens.astype(np.int32).copy()
        bt = np.full((w.B, w.block_table.shape[1] + n // w.P + 2), -1, np.int32)
        bt[:, :w.block_table.shape[1]] = w.block_table

        def grown(t):  # the pool with zeroed spare pages after the workload's
            g = torch.zeros((n_pages,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            g[:w.num_pages].copy_(t)
            return g

        lay2 = [(grown(k0), grown(v0)) for _ in range(args.layers)]
        free = [w.num_pages]

        def grow():
            for b in range(w.B):
                if kv[b] % w.P == 0:
                    bt[b, kv[b] // w.P] = free[0]
                    free[0] += 1
                kv[b] += 1

        plan = pad.Plan(kv, bt, n_pages, w.Hq, w.Hkv, w.D, flags=pad.PA_PLAN_KEEP_PACK)
        wsd = torch.empty((2 * plan.workspace_bytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
        adv_us, full_us = [], []

        def decode_step(timed: bool):
            nonlocal plan
            grow()
            t = time.perf_counter()
            nxt = plan.advance(kv, bt, n_pages)
            t = (time.perf_counter() - t) * 1e6
            plan.close()
            plan = nxt
            if plan.workspace_bytes > wsd.numel():
                raise RuntimeError("decode-steps workspace too small")
            plan.upload(wsd, stream)
            for kl_, vl_ in lay2:
                plan.attend(q, kl_, vl_, wsd, out, lse, stream)
            if timed:
                adv_us.append(t)
                fp = pad.Plan(kv, bt, n_pages, w.Hq, w.Hkv, w.D)
                full_us.append(fp.stats()["plan_us"])
                fp.close()

        for _ in range(3):
            decode_step(False)
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(n):
            decode_step(True)
        c1.record(stream)
        torch.cuda.synchronize()
        assert plan.device_status(wsd, stream) == pad.PA_OK
        t_us = c0.elapsed_time(c1) / n * 1e3
        plan.close()
        del lay2, wsd
        return {"steps": n, "layers": args.layers, "us_per_step": t_us, "us_per_layer": t_us / args.layers,
                "advance_us_median": statistics.median(adv_us), "create_us_median": statistics.median(full_us),
                "note": "each step: every request appends a token, pa_plan_advance, upload, then one forward + "
                        "merge per layer; create_us is pa_plan_create on the same inputs (host only)"}

    def e2e(self, w, q, k0, v0, out, lse, ws_bytes) -> dict:
        # end to end through the public API with host buffers: every input
        # copied from pinned host memory each step, the result read back
        torch, args, stream = self.torch, self.args, self.stream
        import prefix_aware_decode_b200 as pad

        hq = torch.from_numpy(np.ascontiguousarray(w.q).view(np.int16)).pin_memory()
        hk = torch.from_numpy(np.ascontiguousarray(w.k_pool).view(np.int16)).pin_memory()
        hv = torch.from_numpy(np.ascontiguousarray(w.v_pool).view(np.int16)).pin_memory()
        ho = torch.empty((w.B, w.Hq, w.D), dtype=torch.int16).pin_memory()
        hl = torch.empty((w.B, w.Hq), dtype=torch.float32).pin_memory()
        dq = torch.empty_like(q)
        dk, dv = k0, v0  # the device pools are overwritten by the copies
        ws = torch.empty((ws_bytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
        stepper = pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, dq, dk, dv, ws, out, lse, stream=stream)

        def e2e_step(copy_kv: bool):
            dq.view(torch.int16).copy_(hq, non_blocking=True)
            if copy_kv:
                dk.view(torch.int16).copy_(hk, non_blocking=True)
                dv.view(torch.int16).copy_(hv, non_blocking=True)
            stepper(w.kv_lens, w.block_table)
            ho.copy_(out.view(torch.int16), non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        # every input copied each step: bound by the host link, timed over
        # --e2e-steps steps
        for _ in range(2):
            e2e_step(True)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step(True)
        b.record(stream)
        torch.cuda.synchronize()
        res = {True: self.max_over_ranks(a.elapsed_time(b)) / args.e2e_steps}

        # the serving case, run as a serving loop runs it, over the same K steps
        # as the device figure: step k's q goes up on an upload stream and its
        # out and lse come back on a download stream, so those transfers overlap
        # the neighbouring steps' kernels; step k uses buffer set k % 2, which
        # its upload reuses once step k - 2's kernels have read it and its
        # kernels once step k - 2's results have been read back (events)
        up, down = torch.cuda.Stream(), torch.cuda.Stream()
        dqs = [torch.empty_like(q) for _ in range(2)]
        outs = [torch.empty_like(out) for _ in range(2)]
        lses = [torch.empty_like(lse) for _ in range(2)]
        hos = [torch.empty((w.B, w.Hq, w.D), dtype=torch.int16).pin_memory() for _ in range(2)]
        hls = [torch.empty((w.B, w.Hq), dtype=torch.float32).pin_memory() for _ in range(2)]
        steppers = [pad.DecodeStep(w.num_pages, w.Hq, w.Hkv, w.D, dqs[j], k0, v0, ws, outs[j], lses[j], stream=stream)
                    for j in range(2)]
        q_ready = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        fetched = [torch.cuda.Event() for _ in range(2)]
        for j in range(2):  # every event recorded once, so the first waits pass at once
            q_ready[j].record(up)
            computed[j].record(stream)
            fetched[j].record(down)

        def serving_step(k: int):
            j = k % 2
            up.wait_event(computed[j])
            with torch.cuda.stream(up):
                dqs[j].view(torch.int16).copy_(hq, non_blocking=True)
                q_ready[j].record(up)
            stream.wait_event(q_ready[j])
            stream.wait_event(fetched[j])
            steppers[j](w.kv_lens, w.block_table)
            computed[j].record(stream)
            down.wait_event(computed[j])
            with torch.cuda.stream(down):
                hos[j].copy_(outs[j].view(torch.int16), non_blocking=True)
                hls[j].copy_(lses[j], non_blocking=True)
                fetched[j].record(down)

        for k in range(4):
            serving_step(k)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start = torch.cuda.Event()
        a.record(stream)
        start.record(stream)
        up.wait_event(start)
        for k in range(args.steps):
            serving_step(k)
        stream.wait_event(fetched[(args.steps - 1) % 2])
        b.record(stream)
        torch.cuda.synchronize()
        res[False] = self.max_over_ranks(a.elapsed_time(b)) / args.steps
        # the loop's last result read back is the device figure's, bit for bit
        # (same inputs and plan), so its stream order is as intended
        last = (args.steps - 1) % 2
        if not (torch.equal(hos[last], out.view(torch.int16).cpu()) and torch.equal(hls[last], lse.cpu())):
            raise RuntimeError("end-to-end serving loop: the result read back differs from the device run's")
        h2d = w.q.nbytes + w.k_pool.nbytes + w.v_pool.nbytes
        d2h = out.numel() * 2 + lse.numel() * 4
        del hq, hk, hv, ho, hl
        return {"e2e": {"value": w.B * self.world / (res[True] * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h,
                        "note": "every input (q and both KV pools) copied from pinned host memory each step; "
                                "bound by the host link, not by the kernels"},
                "e2e_kv_resident": {"value": w.B * self.world / (res[False] * 1e-3), "unit": UNIT,
                                    "h2d_bytes_per_step": w.q.nbytes, "d2h_bytes_per_step": d2h,
                                    "note": "the serving case: q from pinned host memory, the KV cache resident "
                                            "on the device, out and lse read back each step; uploads and "
                                            "read-backs on their own streams, two buffer sets"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="pa", choices=["pa", "reference"])
    ap.add_argument("--config", type=int, default=5, help="headline workload (1-5)")
    ap.add_argument("--per-config", default="1,2,3,4",
                    help="other workloads measured in the same run (comma list; empty: none)")
    ap.add_argument("--copies", type=int, default=0, help="KV pool copies rotated between steps (0: enough to exceed L2)")
    ap.add_argument("--ref-queries", type=int, default=16)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=3,
                    help="steps of the end-to-end case that copies every input (the KV cache too) each step; "
                         "the KV-resident case times --steps steps")
    ap.add_argument("--layers", type=int, default=32,
                    help="layers of the multi-layer step measured beside config 2 (0: skip)")
    ap.add_argument("--decode-steps", type=int, default=16,
                    help="config 2: also time this many growing decode steps of --layers layers whose plans "
                         "come from pa_plan_advance (0: skip)")
    ap.add_argument("--scale", type=float, default=1.0,
                    help="shrink the workloads (batch and lengths) for small profiler captures; 1 = the named sizes")
    ap.add_argument("--session-steps", type=int, default=4,
                    help="config 5: growing-session steps of registered queries (0: skip)")
    ap.add_argument("--amortise", type=int, default=1024,
                    help="config-1 problems batched together for the amortised config-1 figure (0: skip)")
    args = ap.parse_args()
    rank, world, local = dist_env()
    if args.warmup < 3:
        args.warmup = 3
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        sys.exit(spawn_ranks(args.gpus))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
        sys.exit(2)

    if args.impl == "reference":
        reference_arm(args, rank, world)
        return

    bench = Bench(args, rank, world, local)
    head = bench.measure(args.config, headline=True)
    per = {}
    for c in [int(x) for x in args.per_config.split(",") if x.strip()]:
        if c != args.config:
            per[str(c)] = bench.measure(c, headline=False)

    line = {
        "metric": METRIC, "value": head["queries_per_s"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": head["workload"], "batch": head["batch"], "heads": "32/8" if args.config > 1 else "8/2",
                   "head_dim": 128 if args.config > 1 else 64, "page": 16, "seed": head["seed"],
                   "unique_kv_bytes": head["unique_kv_bytes"], "prefix_ratio": head["prefix_ratio"],
                   "l2": head["l2"], "step": "pack (host) + upload + forward + merge",
                   "parallelism": f"replicas x{world}"},
        "unique_kv_gbs": head["unique_kv_bytes"] / (head["ms_per_step"] * 1e-3) / 1e9,
        "unique_kv_frac_of_hbm": head["unique_kv_frac_of_hbm"],
        "device_ms": {"forward_merge": head["forward_merge_us"] * 1e-3},
        "forward_queries_per_s": head["forward_queries_per_s"],
        "forward_unique_kv_frac": head["forward_unique_kv_frac_of_hbm"],
        "plan_us": head["plan_us"], "host_us_per_step_median": head["host_us_per_step_median"],
        "plan": head["plan"], "roofline": head["roofline"], "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    for k in ("e2e", "e2e_kv_resident", "cpu_baseline", "sessions"):
        if k in head:
            line[k] = head[k]
    line["per_config"] = per
    if rank == 0:
        print(json.dumps(line))
    if bench.dist is not None:
        bench.dist.destroy_process_group()


if __name__ == "__main__":
    main()
