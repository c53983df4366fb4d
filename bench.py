"""Benchmark: paged decode KV-read GB/s and seq-steps/s on a continuous-batching trace.

Default workload: 64 sequences, lengths uniform in [1, 2048], 32 q heads / 8 kv
heads, head_dim 128, bf16 cache, sequences ending after Geometric(1/256)
decode steps and replaced from a queue (the scheduler of
paged_kv_cache_408_b200.runtime drives every step).  One step = copy_blocks
(copy-on-write pairs, if any) + write_kv (the step's new K/V: one token per
decoding sequence plus the prompts of admitted sequences) + decode (+ its
split-K merge) [+ chunked prefill in the mixed workload].

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank runs its own independent replica of the
trace (per-GPU work fixed: weak scaling, no collective on the data path);
value is the work of all ranks over the slowest rank's time.  Rank 0 prints
one JSON line.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_FLUSH_BYTES = 256 << 20  # > 126 MB L2
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0       # B200 HBM3e peak as specified (about 8 TB/s)

METRIC = "paged decode KV-read GB/s (% of B200 HBM peak); seq-steps/s at 64x2K GQA"


# ------------------------------------------------------------------ helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        return float(json.load(open(p))["bf16_tflops"]), "measured (cuBLAS bf16 GEMM, burst)"
    return 1590.0, "fallback"


def file_sha(path):
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def profiled_traffic(kernel_file, workload):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on
    the current source of the kernel."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(workload)
        if d and d.get("source_sha") == file_sha(os.path.join(ROOT, kernel_file)):
            return d.get("dram_bytes_per_launch")
    except (ValueError, OSError):
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x.strip() for x in vis.split(",")] if vis else []
        self.gpu = ids[gpu_index] if gpu_index < len(ids) else str(gpu_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        rows = []
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[0] > 0.5 * r[1]] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


class L2Flush:
    """Evict the L2 between timed steps: write a buffer larger than L2, then
    read another one, so the next step starts with no useful data cached and
    no dirty lines left to write back."""

    def __init__(self, torch, device):
        self.w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=device)

    def __call__(self):
        self.w.zero_()
        self.sink = self.r.sum()


def kv_bytes(lens, Hkv, D, eb):
    return int(np.asarray(lens, np.int64).sum()) * Hkv * D * 2 * eb


def decode_alg_flops(lens, Hq, D):
    """CUDA-core FLOPs of one decode launch: for every cached token and q
    head, q.k and p.v over D dims, 2 FLOP per multiply-add."""
    return 4 * D * Hq * int(np.asarray(lens, np.int64).sum())


def roof_time(nbytes, bytes_per_s, flops, flops_per_s):
    """Shortest time for work that moves nbytes and does flops: the slower of
    the memory roof and the arithmetic roof."""
    return max(nbytes / bytes_per_s, flops / flops_per_s)


def decode_math_on_cuda_cores(Hq, Hkv, fp8):
    """The decode kernel does q.k and p.v on the CUDA cores except for an fp8
    cache with GQA 8, where it uses the tensor cores (mma.sync, f16)."""
    return not (fp8 and Hq // Hkv == 8)


def alu_peak(sm_mhz):
    """fp32 FMA peak of the CUDA cores: 148 SMs x 128 lanes x 2 FLOP per
    clock, at the SM clock sampled during the timed region."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def decode_alg_bytes(lens, Hq, Hkv, D, eb):
    lens = np.asarray(lens, np.int64)
    B = len(lens)
    return (kv_bytes(lens, Hkv, D, eb) + 2 * B * Hq * D * 2 + int(((lens + 15) // 16).sum()) * 4 + B * 4)


# ----------------------------------------------------------------- workloads
def _traces():
    from paged_kv_cache_408_b200 import traces
    return {"batch64_2k": traces.batch64_2k, "prefix_share_fp8": traces.prefix_share_fp8, "mixed": traces.mixed,
            "long_context": traces.long_context}


class _Lazy(dict):
    def __missing__(self, k):
        self.update(_traces())
        return dict.__getitem__(self, k)


TRACES = _Lazy()


# ----------------------------------------------------------------- our arm
from paged_kv_cache_408_b200.executor import DeviceStep  # noqa: E402  (re-exported for the host tests)


def prefill_flops(cu_q, prefix_lens, Hq, D):
    """Algorithmic FLOPs of causal chunked prefill: per chunk of C queries over
    a prefix of P keys, C*P + C(C+1)/2 query-key pairs, 4*D flops per pair
    (q.k and p.v), for every query head."""
    C = np.diff(np.asarray(cu_q, np.int64))
    P = np.asarray(prefix_lens, np.int64)
    return int((Hq * 4 * D * (C * P + C * (C + 1) // 2)).sum())


def run_ours(args, rank, world, device, workload=None, legs_only=False):
    """Drive a synthetic trace through the scheduler and the kernels.

    Every step's plan is made on the host first (timed separately); then
    warm-up steps, then the timed steps, each one programmatic launch chain
    copy_blocks -> write_kv -> decode (+ merge) [-> prefill], bracketed by
    CUDA events with the L2 flushed in between (outside the events).  Then
    the same steps again with only the decode call timed (its roofline), the
    prefill call (where the trace attends prefill chunks) and, for cascade
    steps, the suffix stage alone.  legs_only: return only the prefill
    call's figures (the prefill leg of another workload's run)."""
    import torch

    from paged_kv_cache_408_b200 import ops
    from paged_kv_cache_408_b200.executor import StepExecutor

    workload = workload or args.workload
    torch.cuda.set_device(device)
    tr = TRACES[workload](args.seed + rank)
    Hq, Hkv, D, fp8 = tr.Hq, tr.Hkv, tr.D, tr.fp8
    eb = 1 if fp8 else 2
    pool = tr.sched.alloc.num_blocks
    t_plan = time.perf_counter()
    plans = tr.plans(args.warmup + args.steps)
    t_plan = (time.perf_counter() - t_plan) / len(plans)
    attend_prefill = workload == "mixed"  # elsewhere admitted prompts are written, not attended

    g = torch.Generator(device=device).manual_seed(1234 + rank)
    shape = (pool, Hkv, 16, D)
    if fp8:
        k_cache = torch.randint(0, 120, shape, dtype=torch.uint8, device=device, generator=g)
        v_cache = torch.randint(0, 120, shape, dtype=torch.uint8, device=device, generator=g)
        k_scale = torch.full((Hkv,), 0.01, device=device)
        v_scale = torch.full((Hkv,), 0.01, device=device)
    else:
        k_cache = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        v_cache = torch.randn(shape, generator=g, device=device).to(torch.bfloat16)
        k_scale = v_scale = None
    Tmax = max(p.slots.shape[0] for p in plans)
    Bmax = max(p.num_decode for p in plans)
    Pmax_tok = max(p.num_prefill_tokens for p in plans)
    new_k = torch.randn((max(Tmax, 1), Hkv, D), generator=g, device=device).to(torch.bfloat16)
    new_v = torch.randn((max(Tmax, 1), Hkv, D), generator=g, device=device).to(torch.bfloat16)
    q = torch.randn((max(Bmax, 1), Hq, D), generator=g, device=device).to(torch.bfloat16)
    out = torch.empty_like(q)
    pq = torch.randn((max(Pmax_tok, 1), Hq, D), generator=g, device=device).to(torch.bfloat16)
    pout = torch.empty_like(pq)
    scale = 1.0 / math.sqrt(D)
    ex = StepExecutor(k_cache, v_cache, Hq, scale, k_scale, v_scale, attend_prefill=attend_prefill,
                      cascade=not args.no_cascade, partition_tokens=args.partition)
    ex.reserve(plans)
    flush = L2Flush(torch, device)

    dsteps = [DeviceStep(p, torch, device, cascade=not args.no_cascade) for p in plans]
    for ds in dsteps:
        if ds.pb:
            st_ = np.full_like(ds.plan.decode_tables, -1)
            st_[:, :st_.shape[1] - ds.pb] = ds.plan.decode_tables[:, ds.pb:]
            ds.sfx_tables = torch.from_numpy(st_).to(device)
            ds.sfx_lens = torch.from_numpy(ds.plan.decode_lens - 16 * ds.pb).to(device)
    torch.cuda.synchronize()
    st = torch.cuda.current_stream()

    def suffix_decode(ds):
        # the suffix stage of a cascade step on its own: the same keys through
        # the decode kernel (suffix tables and lengths), for its roofline
        ops.decode(out[:ds.B], q[:ds.B], k_cache, v_cache, ds.sfx_tables, ds.sfx_lens, scale, k_scale, v_scale,
                   ex.ws, 0)

    def timed_pass(fn, steps):
        """fn(ds) for each step, each bracketed by events, L2 flushed in
        between; a GPU sleep holds the stream while the host enqueues, so the
        events see device time only."""
        ev = []
        torch.cuda._sleep(hold_cycles(len(steps)))
        for ds in steps:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush()
            e0.record(st)
            n = fn(ds)
            e1.record(st)
            ev.append((e0, e1, ds, n))
        torch.cuda.synchronize()
        return ev

    with ClockSampler(torch.cuda.current_device()) as clk:
        # ---- warm-up, with the clock sampler already running: its start-up pause
        # must not leave the GPU idle (clocks falling back) right before the
        # timed steps; the warm-up steps flush L2 like the timed ones
        for ds in dsteps[:args.warmup]:
            flush()
            ex.enqueue(ds, q, out, new_k, new_v, pq, pout)
        torch.cuda.synchronize()
        if ops.get_last_device_error() != 0:
            raise RuntimeError("device status word set during warm-up")
        timed = dsteps[args.warmup:]
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()
        # ---- timed: whole steps (one programmatic launch chain each; an event
        # inside a step would cut the chain)
        step_ev = timed_pass(lambda ds: ex.enqueue(ds, q, out, new_k, new_v, pq, pout), timed)
        # ---- each call alone, same steps and cache, for the kernels' rooflines
        dec_ev = timed_pass(lambda ds: ex.decode(ds, q, out), [d for d in timed if d.B])
        pre_ev = timed_pass(lambda ds: ex.prefill(ds, pq, pout), [d for d in timed if d.n_prefill]) \
            if attend_prefill else []
        sfx_ev = [] if legs_only else timed_pass(suffix_decode, [d for d in timed if d.B and d.pb])
    if world > 1:
        dist.barrier()

    def ms(e):
        return e[0].elapsed_time(e[1])

    step_ms = [ms(e) for e in step_ev]
    dec_ms = [ms(e) for e in dec_ev]
    cascade = None
    if sfx_ev:
        n = len(sfx_ev)
        lens_sfx = [e[2].plan.decode_lens - 16 * e[2].pb for e in sfx_ev]
        cascade = {
            "steps": n, "prefix_blocks": sorted({int(e[2].pb) for e in sfx_ev}),
            "call_ms": sum(ms(e) for e in dec_ev if e[2].pb) / n,
            "suffix_ms": sum(ms(e) for e in sfx_ev) / n,
            "prefix_flops": sum(4 * D * Hq * e[2].B * 16 * e[2].pb for e in sfx_ev) / n,
            "suffix_flops": sum(decode_alg_flops(x, Hq, D) for x in lens_sfx) / n,
            "suffix_bytes": sum(decode_alg_bytes(x, Hq, Hkv, D, eb) for x in lens_sfx) / n,
            "unique_bytes": sum(decode_alg_bytes(x, Hq, Hkv, D, eb) + 16 * e[2].pb * Hkv * D * 2 * eb
                                for x, e in zip(lens_sfx, sfx_ev)) / n,
        }
    prefill = None
    if pre_ev:
        pms = [ms(e) for e in pre_ev]
        pfl = [prefill_flops(e[2].plan.prefill_cu, e[2].plan.prefill_prefix, Hq, D) for e in pre_ev]
        prefill = {"ms": sum(pms) / len(pms), "flops": sum(pfl) / len(pfl), "steps": len(pms),
                   "tokens": sum(e[2].n_prefill for e in pre_ev) / len(pre_ev),
                   "chunks": sum(e[2].nchunks for e in pre_ev) / len(pre_ev), "workload": tr.name,
                   "clocks": clk.summary()}
    flags = ops.get_last_device_error()
    if flags:
        raise RuntimeError(f"device status word {flags:#x} after the timed steps")
    if legs_only:
        return {"prefill": prefill}

    tot_ms = sum(step_ms)
    kvb = sum(kv_bytes(ds.plan.decode_lens, Hkv, D, eb) for ds in timed)
    seqsteps = sum(ds.B for ds in timed)
    algb = [decode_alg_bytes(ds.plan.decode_lens, Hq, Hkv, D, eb) for ds in timed if ds.B]
    algf = [decode_alg_flops(ds.plan.decode_lens, Hq, D) for ds in timed if ds.B]
    launches = sum(e[3] for e in step_ev)

    # ---- end to end: per-step inputs from pinned host memory, results read back.
    # A serving loop's overlap: while step k runs, one copy stream brings step
    # k+1's inputs in and another reads step k-1's outputs back (double
    # buffers).  Step k's events end only once both have finished, so every
    # copy lies inside some step's events: step k's time = max(its kernels,
    # the copy of step k+1's inputs, the read of step k-1's outputs); step 0
    # also covers its own inputs' copy, the last step its own read-back.
    e2e = None
    if not args.no_e2e:
        hsteps = [DeviceStep(p, torch, device, pin=True, cascade=not args.no_cascade) for p in plans[args.warmup:]]
        hq, hk, hv = q.cpu().pin_memory(), new_k.cpu().pin_memory(), new_v.cpu().pin_memory()
        hpq = pq.cpu().pin_memory()
        hout, hpout = torch.empty_like(hq).pin_memory(), torch.empty_like(hpq).pin_memory()
        dbuf = [(torch.empty_like(q), torch.empty_like(new_k), torch.empty_like(new_v), torch.empty_like(pq),
                 torch.empty_like(out), torch.empty_like(pout)) for _ in range(2)]
        cs_in, cs_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
        n = len(hsteps)
        # device buffers allocated before timing (an allocation inside the
        # loop could synchronise the device)
        dmeta = [torch.empty(hs.nbytes(), dtype=torch.uint8, device=device) for hs in hsteps]
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in hsteps]
        landed, ran, read = ([torch.cuda.Event() for _ in hsteps] for _ in range(3))
        dsteps_e2e = [None] * n
        nbytes = {"h2d": 0, "d2h": 0}

        def n_pf(hs):
            return hs.n_prefill * Hq * D * 2 if attend_prefill else 0

        def bring_in(k, after):  # step k's inputs, on the input copy stream, once `after` is reached
            hs = hsteps[k]
            cs_in.wait_event(after)
            with torch.cuda.stream(cs_in):
                dsteps_e2e[k] = hs.to(device, out=dmeta[k])
                dq, dk, dv, dpq = dbuf[k % 2][:4]
                if hs.B:
                    dq[:hs.B].copy_(hq[:hs.B], non_blocking=True)
                if hs.T:
                    dk[:hs.T].copy_(hk[:hs.T], non_blocking=True)
                    dv[:hs.T].copy_(hv[:hs.T], non_blocking=True)
                if n_pf(hs):
                    dpq[:hs.n_prefill].copy_(hpq[:hs.n_prefill], non_blocking=True)
                landed[k].record(cs_in)
            nbytes["h2d"] += hs.nbytes() + hs.B * Hq * D * 2 + 2 * hs.T * Hkv * D * 2 + n_pf(hs)

        def read_back(k, stream, after):  # step k's outputs to pinned host memory
            hs = hsteps[k]
            stream.wait_event(after)
            with torch.cuda.stream(stream):
                dout, dpout = dbuf[k % 2][4:]
                if hs.B:
                    hout[:hs.B].copy_(dout[:hs.B], non_blocking=True)
                if n_pf(hs):
                    hpout[:hs.n_prefill].copy_(dpout[:hs.n_prefill], non_blocking=True)
                read[k].record(stream)
            nbytes["d2h"] += hs.B * Hq * D * 2 + n_pf(hs)

        def run(m):  # the first m steps, pipelined as described above
            for k in range(m):
                flush()
                e0, e1 = ee[k]
                e0.record(st)
                if k == 0:
                    bring_in(0, e0)
                if k + 1 < m:
                    bring_in(k + 1, e0)  # into the other buffer set, free since step k-1 ended
                if k > 0:
                    read_back(k - 1, cs_out, e0)  # step k-1's outputs, done before step k began
                st.wait_event(landed[k])
                dq, dk, dv, dpq, dout, dpout = dbuf[k % 2]
                ex.enqueue(dsteps_e2e[k], dq, dout, dk, dv, dpq, dpout)
                ran[k].record(st)
                if k + 1 == m:
                    read_back(k, st, ran[k])
                for ev in ([landed[k + 1]] if k + 1 < m else []) + ([read[k - 1]] if k > 0 else []):
                    st.wait_event(ev)
                e1.record(st)

        run(min(2, n))  # untimed: the host path's and the copy streams' first run (the same steps again below)
        torch.cuda.synchronize()
        nbytes["h2d"] = nbytes["d2h"] = 0
        # as in the device-timed legs, the stream is held while the host
        # enqueues every step (a serving loop runs its host work ahead of the GPU)
        torch.cuda._sleep(hold_cycles(n))
        run(n)
        torch.cuda.synchronize()
        e2e_steps = [a.elapsed_time(b) for a, b in ee]
        e2e = {"ms": sum(e2e_steps), "h2d": nbytes["h2d"] / n, "d2h": nbytes["d2h"] / n, "kvb": kvb,
               "step_ms": e2e_steps}

    return dict(tot_ms=tot_ms, step_ms=step_ms, dec_ms=dec_ms, kvb=kvb, seqsteps=seqsteps, algb=algb, algf=algf,
                launches=launches, clocks=clk.summary(), e2e=e2e, plan_ms=t_plan * 1e3, tr=tr, plans=plans,
                cascade=cascade, prefill=prefill, copies=sum(len(ds.plan.copies) for ds in timed),
                k_cache=k_cache, v_cache=v_cache, Hq=Hq, Hkv=Hkv, D=D, eb=eb, fp8=fp8, scale=scale,
                k_scale=k_scale, v_scale=v_scale, q=q, pool=pool)


# ------------------------------------------------------------ oracle timing
def oracle_sample(plans, kc, vc, qh, Hq, Hkv, D, eb, scale, ks, vs, per_step_s=2.0, budget_s=None, warmup=0):
    """Time the fp64 oracle, as it stands, on the decode of the trace's steps:
    a whole step where that takes at most about ``per_step_s`` on these
    cores, else the first n sequences of every step, n sized from a probe of
    the first step so that a step takes about ``per_step_s``.  ``warmup``
    steps run untimed first; timing stops after ``budget_s`` seconds if given.
    Both the CPU baseline of our arm and the reference arm use this sample."""
    import oracle
    nthreads = os.cpu_count() or 1

    def run(p, rows):
        t0 = time.perf_counter()
        oracle.decode(qh[rows], kc, vc, p.decode_tables[rows], p.decode_lens[rows], scale, ks, vs,
                      nthreads=nthreads)
        return time.perf_counter() - t0

    Bmax = max(p.num_decode for p in plans)
    probe = plans[0]
    n0 = max(1, min(8, probe.num_decode))
    per_row = run(probe, np.arange(n0)) / n0
    nrows = int(max(1, min(Bmax, per_step_s / max(per_row, 1e-6))))
    for p in plans[:warmup]:
        run(p, np.arange(min(nrows, p.num_decode)))
    secs, kvb, seqsteps, nsteps = 0.0, 0, 0, 0
    for p in plans[warmup:]:
        rows = np.arange(min(nrows, p.num_decode))
        secs += run(p, rows)
        kvb += kv_bytes(p.decode_lens[rows], Hkv, D, eb)
        seqsteps += len(rows)
        nsteps += 1
        if budget_s is not None and secs >= budget_s:
            break
    what = "whole steps" if nrows >= Bmax else f"the first {nrows} sequences of each step"
    return {"value": kvb / secs / 1e9, "unit": "GB/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"decode of {nsteps} steps of the same trace, {what} (fp64 C oracle, OpenMP over sequence "
                      f"x head), {secs:.1f} s", "seq_steps_per_s": seqsteps / secs, "secs": secs, "steps": nsteps}


def host_copy(t, torch):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


# ---------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The oracle timed as the reference arm on the host cores."""
    if rank != 0:
        return None
    from paged_kv_cache_408_b200 import traces, inputs as I
    import oracle
    tr = TRACES[args.workload](args.seed)
    plans = tr.plans(args.warmup + args.steps)
    rng = np.random.default_rng(7)
    shape = (tr.sched.alloc.num_blocks, tr.Hkv, 16, tr.D)
    if tr.fp8:
        kc = rng.integers(0, 120, shape).astype(np.uint8)
        vc = rng.integers(0, 120, shape).astype(np.uint8)
        ks = np.full(tr.Hkv, 0.01, np.float32)
        vs = ks.copy()
    else:
        kc, vc = I.normal_bf16(rng, shape), I.normal_bf16(rng, shape)
        ks = vs = None
    eb = 1 if tr.fp8 else 2
    Bmax = max(p.num_decode for p in plans)
    qh = I.normal_bf16(rng, (Bmax, tr.Hq, tr.D))
    scale = 1.0 / math.sqrt(tr.D)
    smp = oracle_sample(plans, kc, vc, qh, tr.Hq, tr.Hkv, tr.D, eb, scale, ks, vs, per_step_s=2.0,
                        warmup=args.warmup)
    value, secs = smp["value"], smp["secs"]
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "impl": "reference", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, tr),
            "seq_steps_per_s": smp["seq_steps_per_s"],
            "cpu_baseline": {"value": value, "unit": "GB/s", "kind": "oracle", "cores": smp["cores"],
                             "sample": smp["sample"]},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def workload_config(args, tr):
    return {"workload": tr.name, "trace": args.workload, "seqs": tr.sched.cfg.max_num_seqs, "q_heads": tr.Hq,
            "kv_heads": tr.Hkv, "head_dim": tr.D, "block_size": 16, "cache_dtype": "fp8_e4m3" if tr.fp8 else "bf16",
            "pool_blocks": tr.sched.alloc.num_blocks, "partition_tokens": args.partition or "balanced",
            "kv_bytes": "logical: every decoded sequence's cached K/V (a shared prefix counts once per sequence)",
            "l2": "flushed between steps outside the timed events (256 MiB written, then 256 MiB read)", "parallelism": "replicas"}


# ---------------------------------------------------------------- driver
def aggregate(tot_s, kv_bytes_done, seq_steps, world, device):
    """Whole-job figures over independent replicas: the slowest rank's device
    time and the work of all ranks (weak scaling: no data-path collective,
    only this reduction of the measurements)."""
    if world <= 1:
        return tot_s, kv_bytes_done, seq_steps
    import torch
    import torch.distributed as dist
    t = torch.tensor([tot_s], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([kv_bytes_done, seq_steps], device=device, dtype=torch.float64)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t.item()), float(w[0].item()), float(w[1].item())



def hold_cycles(n_steps):
    """GPU clock cycles of the sleep that holds the stream while the host
    enqueues n timed steps (outside the timed events): about 10 ms plus
    0.5 ms a step at 1.965 GHz, well above the enqueue time (tens of us a
    step)."""
    return int(2e7 + 1e6 * n_steps)


def cascade_roofline(c, hbm_peak, hbm_kind, apeak, sm_mhz, workload, cuda_core_math=True):
    """Roofline of a cascade decode call (fp8 widening, prefix attention on
    the tensor cores, suffix decode, merge).  The suffix stage is timed on
    its own (the decode kernel over the suffix tables); the prefix stage is
    the call minus that.  The line's roofline is the stage that takes
    longer; both stages and the call's combined roof are listed."""
    t_call, t_sfx = c["call_ms"] / 1e3, c["suffix_ms"] / 1e3
    t_pre = max(t_call - t_sfx, 1e-9)
    tpeak, tkind = tensor_peak()
    pre_tfl = c["prefix_flops"] / t_pre / 1e12
    prefix = {"bound": "tensor", "achieved": pre_tfl, "peak": tpeak, "unit": "TFLOP/s", "frac": pre_tfl / tpeak,
              "peak_kind": tkind, "kernel": "prefill_kernel (shared-prefix mode) + fp8 widening",
              "ms_per_launch": t_pre * 1e3, "alg_flops_per_launch": c["prefix_flops"],
              "timing": "cascade call minus the suffix stage timed alone", "traffic": None}
    sfx_flops_per_s = (apeak if cuda_core_math else tpeak) * 1e12
    if cuda_core_math and c["suffix_flops"] / sfx_flops_per_s > c["suffix_bytes"] / (hbm_peak * 1e9):
        tfl = c["suffix_flops"] / t_sfx / 1e12
        suffix = {"bound": "alu", "achieved": tfl, "peak": apeak, "unit": "TFLOP/s", "frac": tfl / apeak,
                  "peak_kind": f"derived: 148 SMs x 128 fp32 lanes x 2 FLOP x {sm_mhz:.0f} MHz"}
    else:
        gbs = c["suffix_bytes"] / t_sfx / 1e9
        suffix = {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s", "frac": gbs / hbm_peak,
                  "peak_kind": f"{hbm_kind} (copy bandwidth)"}
    suffix.update({"kernel": "decode_kernel + merge_kernel (suffix)", "ms_per_launch": t_sfx * 1e3,
                   "alg_flops_per_launch": c["suffix_flops"], "alg_bytes_per_launch": c["suffix_bytes"],
                   "timing": "decode call over the suffix tables, CUDA events",
                   "traffic": profiled_traffic("paged_kv_cache_408_b200/csrc/decode.cu", workload + ":suffix")})
    roof_s = (c["prefix_flops"] / (tpeak * 1e12) +
              roof_time(c["suffix_bytes"], hbm_peak * 1e9, c["suffix_flops"], sfx_flops_per_s))
    out = dict(suffix if t_sfx >= t_pre else prefix)
    out["stages"] = {"prefix": prefix, "suffix": suffix,
                     "call": {"ms_per_launch": t_call * 1e3, "roof_ms": roof_s * 1e3, "frac": roof_s / t_call,
                              "unique_kv_bytes": c["unique_bytes"], "prefix_blocks": c["prefix_blocks"]}}
    return out


def cascade_blocks(plan, args):
    """Shared prefix blocks a step's decode attends through cascade decode
    (0: plain decode); see executor.cascade_blocks."""
    from paged_kv_cache_408_b200.executor import cascade_blocks as cb
    return cb(plan, not args.no_cascade)


def static_prefill(args, device, fp8=False, n=30):
    """The mixed step's prefill as a fixed workload (8 chunks of 512 tokens
    over prefixes uniform in [0, 4096], 32/8 heads, d128; the chunks' K/V
    written first), the prefill call timed alone n times, L2 flushed before
    each: median device time and algorithmic FLOPs."""
    import torch

    from paged_kv_cache_408_b200 import inputs as I
    from paged_kv_cache_408_b200 import ops
    pc = I.mixed_step_prefill(args.seed, fp8=fp8)
    if fp8:
        kc, vc = torch.from_numpy(pc.k_cache).to(device), torch.from_numpy(pc.v_cache).to(device)
        ks, vs = torch.from_numpy(pc.k_scale).to(device), torch.from_numpy(pc.v_scale).to(device)
    else:
        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
        kc, vc = bf(pc.k_cache), bf(pc.v_cache)
        ks = vs = None

    def bfq(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.int32)).to(device)

    ops.write_kv(bfq(pc.new_k), bfq(pc.new_v), torch.from_numpy(pc.slot_mapping).to(device), kc, vc, ks, vs)
    q = bfq(pc.q)
    out = torch.empty_like(q)
    cu, pf, bt = i32(pc.cu_q), i32(pc.prefix_lens), i32(pc.block_tables)
    flush = L2Flush(torch, device)
    st = torch.cuda.current_stream()
    for _ in range(3):
        ops.prefill_chunk(out, q, cu, pf, bt, kc, vc, pc.scale, pc.max_q_len, ks, vs)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    torch.cuda._sleep(hold_cycles(n))
    for e0, e1 in ev:
        flush()
        e0.record(st)
        ops.prefill_chunk(out, q, cu, pf, bt, kc, vc, pc.scale, pc.max_q_len, ks, vs)
        e1.record(st)
    torch.cuda.synchronize()
    if ops.get_last_device_error():
        raise RuntimeError("device status word set during the static prefill step")
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    fl = prefill_flops(pc.cu_q, pc.prefix_lens, 32, 128)
    peak, kind = tensor_peak()
    tfl = fl / (ms / 1e3) / 1e12
    return {"workload": "8 chunks x 512 over prefixes U[0,4096] (static), 32/8 heads, d128, " +
                        ("fp8 E4M3 cache" if fp8 else "bf16"),
            "ms_per_launch": ms, "flops_per_launch": fl, "tflops": tfl, "frac": tfl / peak, "peak": peak,
            "peak_kind": kind, "launches": n, "timing": "median of n calls alone, CUDA events, L2 flushed before each"}


def prefill_block(pf):
    """The prefill call's figures: algorithmic FLOPs over its CUDA-event time,
    against the measured bf16 GEMM peak (the call is timed alone)."""
    tfl = pf["flops"] / (pf["ms"] / 1e3) / 1e12
    bf16_peak, kind = tensor_peak()
    return {"tflops": tfl, "ms_per_launch": pf["ms"], "flops_per_launch": pf["flops"],
            "tokens_per_launch": pf["tokens"], "chunks_per_launch": pf["chunks"], "steps": pf["steps"],
            "workload": pf["workload"], "clocks": pf.get("clocks"),
            "roofline": {"bound": "tensor", "achieved": tfl, "peak": bf16_peak, "unit": "TFLOP/s",
                         "frac": tfl / bf16_peak, "peak_kind": kind, "kernel": "pa_prefill_chunk (prefill_kernel)",
                         "timing": "the prefill call of every timed step of the mixed trace alone, CUDA events, "
                                   "L2 flushed before each"}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["batch64_2k", "prefix_share_fp8", "mixed", "long_context"],
                    default="batch64_2k")
    ap.add_argument("--partition", type=int, default=0)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-cascade", action="store_true", help="plain decode even where rows share prefix blocks")
    ap.add_argument("--no-prefill-leg", action="store_true",
                    help="skip timing the mixed trace's chunked prefill after a decode-only workload")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    import torch
    device = torch.device(f"cuda:{local}")
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(device)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)

    r = run_ours(args, rank, world, device)
    # a decode-only workload also times chunked prefill: the prefill call of
    # the mixed trace (the scheduler's chunks over their paged prefixes)
    leg = None
    if args.workload != "mixed" and not args.no_prefill_leg:
        import types
        largs = types.SimpleNamespace(**vars(args))
        largs.steps, largs.warmup = min(args.steps, 10), 3
        leg = run_ours(largs, rank, world, device, workload="mixed", legs_only=True)["prefill"]

    tot_s, kvb, seqsteps = aggregate(r["tot_ms"] / 1e3, r["kvb"], r["seqsteps"], world, device)
    e2e = r["e2e"]
    if e2e is not None:  # whole job too: the slowest rank's time, every rank's bytes
        e2e_s, e2e_kvb, e2e_h2d = aggregate(e2e["ms"] / 1e3, e2e["kvb"], e2e["h2d"], world, device)
        _, _, e2e_d2h = aggregate(0.0, 0.0, e2e["d2h"], world, device)
        e2e = dict(e2e, ms=e2e_s * 1e3, kvb=e2e_kvb, h2d=e2e_h2d, d2h=e2e_d2h)

    if rank == 0:
        peak, peak_kind = peaks()
        dec_ms = sum(r["dec_ms"]) / len(r["dec_ms"])
        alg = sum(r["algb"]) / len(r["algb"])
        flops = sum(r["algf"]) / len(r["algf"])
        achieved = alg / (dec_ms / 1e3) / 1e9
        # the binding roof: HBM bytes, or CUDA-core FLOPs where the decode
        # kernel does its products on the CUDA cores and they take longer
        sm_mhz = (r["clocks"] or {}).get("sm_mhz") or 1965.0
        apeak = alu_peak(sm_mhz)
        cuda_core_math = decode_math_on_cuda_cores(r.get("Hq", 32), r.get("Hkv", 8), r["fp8"])
        alu_bound = cuda_core_math and roof_time(alg, peak * 1e9, flops, apeak * 1e12) > alg / (peak * 1e9)
        if alu_bound:
            tfl = flops / (dec_ms / 1e3) / 1e12
            roof = {"bound": "alu", "achieved": tfl, "peak": apeak, "unit": "TFLOP/s", "frac": tfl / apeak,
                    "peak_kind": f"derived: 148 SMs x 128 fp32 lanes x 2 FLOP x {sm_mhz:.0f} MHz",
                    "hbm_achieved_gbs": achieved, "hbm_frac": achieved / peak}
        else:
            roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                    "peak_kind": f"{peak_kind} (copy bandwidth)"}
        roof["frac_of_spec"] = achieved / SPEC_HBM_GBS
        roof["spec_peak"] = SPEC_HBM_GBS
        roof.update({"kernel": "pa_decode (decode + merge)",
                     "traffic": profiled_traffic("paged_kv_cache_408_b200/csrc/decode.cu", args.workload),
                     "alg_bytes_per_launch": alg, "alg_flops_per_launch": flops, "ms_per_launch": dec_ms})
        if r.get("cascade"):
            roof = cascade_roofline(r["cascade"], peak, peak_kind, apeak, sm_mhz, args.workload, cuda_core_math)
        tr = r["tr"]
        line = {
            "metric": METRIC, "value": kvb / tot_s / 1e9, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["tot_ms"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if not r["fp8"] else "fp8_e4m3",
            "data": "synthetic", "config": workload_config(args, tr),
            "seq_steps_per_s": seqsteps / tot_s,
            "decode_path": "cascade" if r.get("cascade") else "decode",
            "pct_of_hbm_peak": 100.0 * (kvb / tot_s / 1e9) / peak,
            "pct_of_hbm_spec": 100.0 * (kvb / tot_s / 1e9) / SPEC_HBM_GBS,
            "hbm_denominators": {"measured_copy_gbs": peak, "measured_kind": peak_kind, "spec_gbs": SPEC_HBM_GBS},
            "roofline": roof,
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
            "host_plan_ms_per_step": r["plan_ms"],
            "kv_accounting": tr.sched.kv_accounting() if hasattr(tr.sched, "kv_accounting") else None,
            "blocks_copied_per_step": r.get("copies", 0) / args.steps,
            "preemptions": tr.sched.num_preemptions,
        }
        if e2e is not None:
            e = e2e
            line["e2e"] = {"value": e["kvb"] / (e["ms"] / 1e3) / 1e9, "unit": "GB/s",
                           "h2d_bytes_per_step": int(e["h2d"]), "d2h_bytes_per_step": int(e["d2h"]),
                           "ms_per_step": e["ms"] / args.steps,
                           "ms_per_step_min_median_max": [min(e["step_ms"]), statistics.median(e["step_ms"]),
                                                          max(e["step_ms"])],
                           "timing": "per step, inside its CUDA events: the step through the C ABI and, on "
                                     "two copy streams overlapping it, the pinned host->device copy of the next "
                                     "step's metadata, q and new K/V and the device->host read of the previous "
                                     "step's outputs (step 0 also copies its own inputs, the last step reads its "
                                     "own outputs); host enqueue runs ahead of the GPU; L2 flushed between steps "
                                     "outside the events"}
        pf = r.get("prefill") or leg
        if pf:
            line["prefill"] = prefill_block(pf)
            if not args.no_prefill_leg:
                line["prefill"]["static_step"] = static_prefill(args, device)
                line["prefill"]["static_step_fp8"] = static_prefill(args, device, fp8=True)
        if world == 1 and not args.no_cpu_baseline and r.get("plans"):
            import torch as _t
            kc, vc = host_copy(r["k_cache"], _t), host_copy(r["v_cache"], _t)
            qh = host_copy(r["q"], _t)
            ks = r["k_scale"].cpu().numpy() if r["k_scale"] is not None else None
            vs = r["v_scale"].cpu().numpy() if r["v_scale"] is not None else None
            cb = oracle_sample(r["plans"][args.warmup:], kc, vc, qh, r["Hq"], r["Hkv"], r["D"], r["eb"], r["scale"],
                               ks, vs, per_step_s=2.0, budget_s=15.0)
            cb.pop("secs")
            cb.pop("steps")
            line["cpu_baseline"] = cb
        print(json.dumps(line), flush=True)

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
