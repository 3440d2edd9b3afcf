#!/usr/bin/env python
"""Benchmark of the exact tiled attention path on B200: forward and forward+backward
TFLOP/s and fraction of the B200 dense BF16 tensor peak.

One step = one fa_fwd (O, LSE) and one fa_bwd (its three launches: preprocess,
main, dQ conversion) over one batch of the chosen workload, with inputs
resident in HBM.  FLOPs follow the metric's convention: 4*B*H*N^2*d for the
forward (halved for causal masks, scaled by the kept-tile density for block
masks and by sum(kv_len)/(B*N) for key padding), and 2.5 times that for the
backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the FP64 CPU oracle, timed

Multi-GPU: one process per GPU, either launched by torchrun or, when
``--gpus N`` is given to a plain command, started here under
torch.distributed.run.  Every rank runs its own copy of the workload on its
own GPU (independent problems, no data-path collective); the reported value
is the FLOPs of all ranks over the slowest rank's time ("weak" scaling).
Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import itertools
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "attention fwd and fwd+bwd TFLOP/s and % of B200 BF16 tensor peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DATASHEET_BF16_TFLOPS = 2250.0
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------
# workload arithmetic (metric convention)
# ----------------------------------------------------------------------------

def density(x):
    """Fraction of the N x N score matrix the metric counts (mask-dependent)."""
    B, H, N, d = x.q.shape
    f = 1.0
    if x.causal:
        f *= 0.5
    if x.block_mask is not None:
        f *= float(x.block_mask.double().mean())
    if x.kv_len is not None:
        f *= float(x.kv_len.double().sum()) / (B * N)
    return f


def flops_fwd(x):
    B, H, N, d = x.q.shape
    return 4.0 * B * H * N * N * d * density(x)


def packed_lengths(x):
    """--varlen: the workload's sequences without padding (key lengths, else N)."""
    B, H, N, d = x.q.shape
    return [int(l) for l in x.kv_len] if x.kv_len is not None else [N] * B


def flops_fwd_packed(x):
    """Forward FLOPs of the packed batch: each sequence its own L x L problem."""
    B, H, N, d = x.q.shape
    f = 0.5 if x.causal else 1.0
    return sum(4.0 * H * L * L * d * f for L in packed_lengths(x))


def ideal_bytes(x, rows=None):
    """Each input read once and each output written once (bytes); ``rows`` = the rows of
    every head together (default B*H*N; a packed batch has T*H)."""
    B, H, N, d = x.q.shape
    R = B * H * N if rows is None else rows
    E = R * d
    fwd = 3 * 2 * E + 2 * E + 4 * R                    # Q, K, V in; O, LSE out
    bwd_main = 4 * 2 * E + 2 * 4 * R + 2 * 2 * E + 2 * 4 * E   # Q K V dO, lse2 D in; dK dV out; dQ acc
    return fwd, bwd_main


def launches_per_step(d):
    """Kernels of one forward + backward: the forward, the preprocess, the main
    backward (d = 256: a dK and a dV pass) and one dQ kernel (the conversion of the
    accumulator, the ordered dQ kernel, or at d = 256 the dQ pass)."""
    return 5 if d == 256 else 4


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# the sources the benchmarked kernels and their launches are compiled from (fa_api.cu
# sets grid sizes and the unit order, which move DRAM traffic too)
BENCHED_KERNEL_SOURCES = ("fa_api.cu", "fa_bwd.cuh", "fa_d256.cuh", "fa_fwd.cuh", "sm100.cuh")


def kernel_source_hash():
    """Hash of the sources of the benchmarked kernels and of their launch code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_63_b200", "csrc")
    for name in BENCHED_KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    ent = rec.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (the slowest rank decides)."""
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_tflops(flops_per_rank, world, ms):
    """Throughput of the whole job: every rank's FLOPs over the slowest rank's time."""
    return flops_per_rank * world / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------
# clocks (nvidia-smi sampled during the load)
# ----------------------------------------------------------------------------

REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class ClockSampler:
    def __init__(self, index):
        self.proc = None
        self.index = index
        self.path = None

    def start(self):
        q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             + ",".join("clocks_event_reasons." + r for r in REASONS))
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index)], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self, t_begin, t_end):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except Exception:
                    continue
        os.unlink(self.path)
        window = [r for r in rows if t_begin - 0.05 <= r[0] <= t_end + 0.05]
        if not window:
            window = rows
        if not window:
            return None
        reasons = sorted({REASONS[i] for r in window for i, v in enumerate(r[3])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in window),
                "sm_max_mhz": max(r[2] for r in window), "reasons": reasons,
                "samples": len(window)}


def workload_or_shape(args):
    """The named workload, or (with --shape B,H,N,d) the same kind of inputs at another
    size (used for profiling captures on a smaller case)."""
    from exact_io_aware_63_b200 import inputs
    if not args.shape:
        return inputs.workload_inputs(args.workload)
    w = inputs.WORKLOADS[args.workload]
    B, H, N, d = (int(t) for t in args.shape.split(","))
    return inputs.make_inputs(B, H, N, d, scale=w.scale if d == w.d else None, causal=w.causal,
                              seed=w.seed, key_padding=(N // 2, N) if w.key_padding else None,
                              block_keep=(1.0 / 16.0) if w.block_sparse else None)


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args):
    import torch
    from exact_io_aware_63_b200 import binding, inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load(build_if_missing=False)

    w = inputs.WORKLOADS[args.workload]
    x = workload_or_shape(args)
    B, H, N, d = x.q.shape
    if args.varlen and x.block_mask is not None:
        raise SystemExit("--varlen: packed batches take no block mask")
    q, k, v, do = (t.to(dev) for t in (x.q, x.k, x.v, x.dout))
    if args.varlen:
        # the same tensors, each sequence's own rows packed token by token ([T, H, d])
        lens = packed_lengths(x)
        def pack(t):
            return torch.cat([t[b, :, :lens[b]].transpose(0, 1) for b in range(B)]).contiguous()

        pq, pkk, pv, pdo = (pack(t) for t in (q, k, v, do))
        T = pq.shape[0]
        cu = torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32, device=dev)
        po, pdq, pdk, pdv = (torch.empty_like(pq) for _ in range(4))
        plse = torch.empty((H, T), dtype=torch.float32, device=dev)
    bm = None if x.block_mask is None else x.block_mask.to(dev)
    kl = None if x.kv_len is None else x.kv_len.to(dev)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_bytes = binding.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    S = stream.cuda_stream
    scale, causal = x.scale, x.causal

    def check(rc, what):
        if rc != 0:
            raise RuntimeError(f"{what}: {binding.fa_status_string(rc)}")

    drop = args.dropout
    seed, offset = 0x5EED, 0

    def fwd_call():
        if args.varlen:
            return binding.fa_fwd_varlen(pq, pkk, pv, po, plse, cu, B, H, N, T, d, scale, causal,
                                         0.0, 0, 0, S)
        if drop > 0:
            return binding.fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, bm, kl, drop,
                                          seed, offset, S)
        return binding.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, bm, kl, S)

    def bwd_call():
        if args.varlen:
            return binding.fa_bwd_varlen(pq, pkk, pv, po, plse, pdo, pdq, pdk, pdv, cu, B, H, N, T,
                                         d, scale, causal, 0.0, 0, 0, ws, ws_bytes, S)
        if drop > 0:
            return binding.fa_bwd_dropout(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, scale,
                                          causal, bm, kl, drop, seed, offset, ws, ws_bytes, S)
        bwd = binding.fa_bwd_deterministic if args.deterministic else binding.fa_bwd
        return bwd(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, scale, causal, bm, kl, ws,
                   ws_bytes, S)

    def step(ev=None, inner=True):
        """One forward + backward.  ev[0] / ev[4] bracket the step; with ``inner`` the
        phases are bracketed as well (ev[1..3]), which serialises the kernels' launches."""
        if ev is not None:
            ev[0].record(stream)
        check(fwd_call(), "forward")
        if not inner:
            check(bwd_call(), "backward")
            if ev is not None:
                ev[4].record(stream)
            return
        if ev is not None:
            ev[1].record(stream)
        if drop > 0 or args.varlen:
            # one call, three kernels: timed together as the "main" interval
            if ev is not None:
                ev[2].record(stream)
            check(bwd_call(), "backward")
            if ev is not None:
                ev[3].record(stream)
                ev[4].record(stream)
            return
        # fa_bwd is phases 0, 1, 2; fa_bwd_deterministic is 0, 1, 3
        for i, ph in enumerate((0, 1, 3) if args.deterministic else (0, 1, 2)):
            check(binding.fa_bwd_phase(ph, q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, scale,
                                       causal, bm, kl, ws, ws_bytes, S), "fa_bwd_phase")
            if ev is not None:
                ev[2 + i].record(stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = binding.fa_get_device_status(S)
    if st != 0:
        raise RuntimeError("device status after warm-up: " + binding.fa_status_string(st))

    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_id = cvd.split(",")[local].strip() if cvd else str(local)
    sampler = ClockSampler(smi_id)
    sampler.start()
    time.sleep(0.3)
    t_load0 = time.time()
    # untimed sustained load so that clock samples see the kernels running
    t_end_sustain = time.time() + args.clock_window
    while time.time() < t_end_sustain:
        for _ in range(8):
            flush.zero_()
            step()
        torch.cuda.synchronize()

    n_ev = 5
    # timed steps: the whole step between two events (the library's kernels follow one
    # another with programmatic dependent launch); then as many steps with every phase
    # bracketed by events, for the per-kernel times and the roofline
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for kk in range(args.steps):
        flush.zero_()                      # L2 flushed between timed steps
        step(evs[kk], inner=False)
    torch.cuda.synchronize()
    barrier()
    for kk in range(args.steps):
        flush.zero_()
        step(evp[kk])
    torch.cuda.synchronize()
    barrier()
    t1 = time.time()
    clocks = sampler.stop(t_load0, t1)
    st = binding.fa_get_device_status(S)
    if st != 0:
        raise RuntimeError("device status after timing: " + binding.fa_status_string(st))

    step_ms = [e[0].elapsed_time(e[4]) for e in evs]
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evp]
    pre_ms = [e[1].elapsed_time(e[2]) for e in evp]
    main_ms = [e[2].elapsed_time(e[3]) for e in evp]
    post_ms = [e[3].elapsed_time(e[4]) for e in evp]
    mean = lambda a: sum(a) / len(a)
    step_t, fwd_t, pre_t, main_t, post_t = max_over_ranks(
        [mean(step_ms), mean(fwd_ms), mean(pre_ms), mean(main_ms), mean(post_ms)], dist, dev)

    # ---------------------------------------------------------------- e2e
    # Through the public calls with host buffers: every step copies its Q, K, V, dO in
    # from pinned host memory and its O, LSE, dQ, dK, dV out.  Steps are pipelined the
    # way a caller streaming batches would run them: two sets of device buffers, the
    # copies in of step k+1 and out of step k-1 on their own streams (the GPU's copy
    # engines) while step k computes.
    e2e = None
    if not args.no_e2e and not args.varlen:
        hin = [t.pin_memory() for t in (x.q, x.k, x.v, x.dout)]
        hout = [[torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(4)] +
                [torch.empty((B, H, N), dtype=torch.float32).pin_memory()] for _ in range(2)]
        dbuf = [[torch.empty_like(q) for _ in range(4)] +                     # q, k, v, dO
                [torch.empty_like(q) for _ in range(4)] +                     # o, dq, dk, dv
                [torch.empty((B, H, N), dtype=torch.float32, device=dev)]     # lse
                for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]
        for e in ev_comp + ev_out:
            e.record(stream)

        def e2e_step(it):
            b = it % 2
            qq, kk, vv, dd = dbuf[b][:4]
            oo, gq, gk, gv, ll = dbuf[b][4:]
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[b])          # step it-2 is done with these inputs
                for dst, src in zip((qq, kk, vv, dd), hin):
                    dst.copy_(src, non_blocking=True)
                ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])             # step it-2's outputs are copied out
            if drop > 0:
                rc_f = binding.fa_fwd_dropout(qq, kk, vv, oo, ll, B, H, N, d, scale, causal, bm,
                                              kl, drop, seed, offset, S)
                rc_b = binding.fa_bwd_dropout(qq, kk, vv, oo, ll, dd, gq, gk, gv, B, H, N, d,
                                              scale, causal, bm, kl, drop, seed, offset, ws,
                                              ws_bytes, S)
            else:
                rc_f = binding.fa_fwd(qq, kk, vv, oo, ll, B, H, N, d, scale, causal, bm, kl, S)
                bwd = binding.fa_bwd_deterministic if args.deterministic else binding.fa_bwd
                rc_b = bwd(qq, kk, vv, oo, ll, dd, gq, gk, gv, B, H, N, d, scale, causal, bm, kl,
                           ws, ws_bytes, S)
            check(rc_f, "forward")
            check(rc_b, "backward")
            ev_comp[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[b])
                for dst, src in zip(hout[b], (oo, gq, gk, gv, ll)):
                    dst.copy_(src, non_blocking=True)
                ev_out[b].record(s_out)

        e2e_steps = max(2, min(args.steps, 20))
        for it in range(2):
            e2e_step(it)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for it in range(2, 2 + e2e_steps):
            e2e_step(it)
        e1.record(s_out)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1) / e2e_steps], dist, dev)[0]
        E, R = B * H * N * d, B * H * N
        h2d = 4 * 2 * E
        d2h = 4 * 2 * E + 4 * R
        e2e = {"value": whole_job_tflops(3.5 * flops_fwd(x), world, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "pipelining": "copies in of step k+1 and out of step k-1 overlap step k"}

    # ---------------------------------------------------------------- report
    peaks, peak_kind = load_peaks()
    ff = flops_fwd_packed(x) if args.varlen else flops_fwd(x)
    fb = 2.5 * ff
    value = whole_job_tflops(3.5 * ff, world, step_t)
    fwd_tflops = ff / (fwd_t * 1e-3) / 1e12
    main_tflops = fb / (main_t * 1e-3) / 1e12
    bwd_tflops = fb / ((pre_t + main_t + post_t) * 1e-3) / 1e12
    per_gpu = value / world
    # dominant kernel by time: the backward main kernel or the forward kernel
    ib = ideal_bytes(x, T * H if args.varlen else None)
    if main_t >= fwd_t:
        dom, dom_t, dom_flops, dom_bytes = "fa_bwd_kernel", main_t, fb, ib[1]
    else:
        dom, dom_t, dom_flops, dom_bytes = "fa_fwd_kernel", fwd_t, ff, ib[0]
    # DRAM bytes were captured for the plain kernels on the [B][H][N][d] layout only
    plain = not args.varlen and drop == 0
    achieved = dom_flops / (dom_t * 1e-3) / 1e12
    roofline = {"kernel": dom, "bound": "tensor", "achieved": achieved,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"],
                "peak_source": f"{peak_kind} bf16_tflops (burst)",
                "traffic": (ncu_traffic(dom, args.workload + (f"@{args.shape}" if args.shape else ""))
                            if plain else None),
                "algorithmic_bytes": dom_bytes,
                "algorithmic_flops": dom_flops,
                "ms_per_launch": dom_t}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_t, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {**workload_config(args, w, x),
                   "l2": "flushed between timed steps (256 MiB write)",
                   "timing": ("value: K whole steps, CUDA events around each step; ms and "
                              "roofline: K further steps with an event between kernels"),
                   "parallelism": f"replica x{world}",
                   "backward": ("fa_bwd_dropout (its three kernels timed together as bwd_main)"
                                if drop > 0 else
                                "fa_bwd_varlen (its three kernels timed together as bwd_main)"
                                if args.varlen else "fa_bwd_deterministic" if args.deterministic
                                else "fa_bwd"),
                   "dropout": drop,
                   "packed": ({"total_tokens": int(T), "max_seqlen": N,
                               "flops": "4*H*d*sum(L_b^2) per forward, x1/2 causal"}
                              if args.varlen else None)},
        "fwd_tflops": fwd_tflops,
        "bwd_tflops": bwd_tflops,
        "fwd_bwd_pct_of_peak": per_gpu / peaks["bf16_tflops"],
        "fwd_pct_of_peak": fwd_tflops / peaks["bf16_tflops"],
        "peak_bf16_tflops": peaks["bf16_tflops"], "peak_source": peak_kind,
        "datasheet_bf16_tflops": DATASHEET_BF16_TFLOPS,
        "ms": {"fwd": fwd_t, "bwd_pre": pre_t, "bwd_main": main_t, "bwd_dq": post_t},
        "bwd_main_tflops": main_tflops,
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step(d) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and drop == 0 and not args.varlen:
        line["cpu_baseline"] = cpu_baseline(x, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# the FP64 CPU oracle, timed on a bounded sample
# ----------------------------------------------------------------------------

def allowed_entries(x, rows):
    """Allowed (row, key) entries of one head for the given query rows, per batch."""
    import numpy as np
    B, H, N, d = x.q.shape
    rows = np.asarray(rows)
    tot = np.zeros(B)
    c = np.arange(N)
    bm = None if x.block_mask is None else x.block_mask.numpy().astype(bool)
    for b in range(B):
        L = N if x.kv_len is None else int(x.kv_len[b])
        for r in rows:
            ok = c < L
            if x.causal:
                ok &= c <= r
            if bm is not None:
                ok &= np.repeat(bm[r // 128], 128)
            tot[b] += ok.sum()
    return tot


def oracle_sample(x, n_heads, n_rows):
    """The first n_heads heads (batch-major) and query rows [0, n_rows) of each."""
    import torch
    B, H, N, d = x.q.shape
    heads = [(b, h) for b in range(B) for h in range(H)][:n_heads]
    sel = lambda t: torch.stack([t[b, h] for b, h in heads])[:, None].to(torch.float64).numpy()
    kl = None if x.kv_len is None else [int(x.kv_len[b]) for b, _ in heads]
    return heads, sel(x.q), sel(x.k), sel(x.v), sel(x.dout), kl


def workload_config(args, w, x):
    """The keys that name the workload, the same in both arms' lines."""
    B, H, N, d = x.q.shape
    return {"workload": args.workload + (f" at shape {args.shape}" if args.shape else ""),
            "description": w.description, "B": B, "H": H, "N": N, "d": d,
            "causal": bool(x.causal), "key_padding": x.kv_len is not None,
            "block_sparse": x.block_mask is not None, "flop_density": density(x),
            "seed": w.seed}


def sample_band(N, n_rows):
    """Query rows [r0, r1) of a sample: the middle n_rows rows of N.  Under a causal mask a
    middle row has about N/2 keys, the mean over all rows; the first rows have almost none,
    and a sample of them would time mostly the oracle's fixed cost per head."""
    r0 = (N - n_rows) // 2
    return r0, r0 + n_rows


def time_oracle(x, n_heads, n_rows, threads):
    import numpy as np
    import oracle
    heads, q, k, v, do, kl = oracle_sample(x, n_heads, n_rows)
    bm = None if x.block_mask is None else x.block_mask.numpy()
    kl = None if kl is None else np.array(kl, np.int32)
    B, H, N, d = x.q.shape
    r0, r1 = sample_band(N, n_rows)
    t0 = time.perf_counter()
    oracle.attention_forward_band(q, k, v, x.scale, x.causal, bm, kl, r0, r1, threads)
    oracle.attention_backward_band(q, k, v, do, x.scale, x.causal, bm, kl, r0, r1, threads)
    dt = time.perf_counter() - t0
    # metric FLOPs of the sample: the workload's per-entry rate times the sample's entries
    per_b = allowed_entries(x, range(r0, r1))
    entries = sum(per_b[b] for b, _ in heads)
    all_entries = allowed_entries(x, range(N)).sum() * H
    flops = 3.5 * flops_fwd(x) * entries / all_entries
    return dt, flops, heads


def sample_plan(x, threads):
    B, H, N, d = x.q.shape
    n_rows = N if N <= 4096 else 256
    n_heads = min(B * H, max(1, threads))
    return n_heads, n_rows


def grow_sample(x, threads, budget_s):
    """Whole heads (or a band of rows for N > 4096), doubled until one timing of the sample
    takes about budget_s CPU-seconds (or the sample is the whole workload).  Returns
    (n_heads, n_rows, seconds, flops, heads) of the last timing."""
    B, H, N, d = x.q.shape
    n_heads, n_rows = sample_plan(x, threads)
    while True:
        dt, flops, heads = time_oracle(x, n_heads, n_rows, threads)
        used = min(threads, len(heads))
        if dt * used >= budget_s or (n_heads >= B * H and n_rows >= N) or dt > budget_s:
            return n_heads, n_rows, dt, flops, heads
        if n_heads < B * H:
            n_heads = min(B * H, n_heads * 2)
        else:
            n_rows = min(N, n_rows * 2)


def sample_text(x, n_heads, n_rows):
    B, H, N, d = x.q.shape
    r0, r1 = sample_band(N, n_rows)
    return (f"FP64 oracle fwd+bwd on {n_heads} of {B * H} heads, query rows {r0}..{r1 - 1} of "
            f"{N} (FLOPs counted as the metric counts them: the workload's rate per allowed "
            f"(query, key) entry times the sample's entries)")


def cpu_baseline(x, budget_s=20.0):
    """Oracle throughput on a bounded sample of about budget_s CPU-seconds."""
    threads = os.cpu_count() or 1
    n_heads, n_rows, dt, flops, heads = grow_sample(x, threads, budget_s)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": min(threads, len(heads)),
            "kind": "oracle", "host_cpus": threads, "seconds": dt,
            "sample": sample_text(x, len(heads), n_rows)}


def run_reference(args):
    """The reference arm: the FP64 CPU oracle (as it stands) on the same workload, metric
    and unit, one bounded sample per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from exact_io_aware_63_b200 import inputs
    w = inputs.WORKLOADS[args.workload]
    x = workload_or_shape(args)
    threads = os.cpu_count() or 1
    B, H, N, d = x.q.shape
    # the kind of sample the CPU baseline takes, sized so that the K + W steps take about
    # 120 CPU-seconds together (0.5 at least each): the same heads and rows in every step
    per_step = max(0.5, min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
    n_heads, n_rows, _, _, _ = grow_sample(x, threads, per_step)
    for _ in range(args.warmup):
        time_oracle(x, n_heads, n_rows, threads)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, flops, heads = time_oracle(x, n_heads, n_rows, threads)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    used = min(threads, n_heads)
    sample = sample_text(x, n_heads, n_rows)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {**workload_config(args, w, x), "parallelism": "cpu threads"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# comparison with standard attention (materialised score matrix)
# ----------------------------------------------------------------------------

def standard_allowed(x, dev):
    """Boolean [B or 1, 1, N, N] mask of allowed (query, key) pairs, the same
    definition the library and the oracle use."""
    import torch
    B, H, N, d = x.q.shape
    r = torch.arange(N, device=dev)
    allowed = torch.ones((1, 1, N, N), dtype=torch.bool, device=dev)
    if x.causal:
        allowed = allowed & (r[None, None, None, :] <= r[None, None, :, None])
    if x.block_mask is not None:
        bm = x.block_mask.to(dev).bool()
        allowed = allowed & bm.repeat_interleave(128, 0).repeat_interleave(128, 1)[None, None]
    if x.kv_len is not None:
        kl = x.kv_len.to(dev)
        allowed = allowed & (r[None, None, None, :] < kl[:, None, None, None])
    return allowed


def run_vs_standard(args):
    """Times fwd+bwd of standard attention written with plain PyTorch ops (S and P
    materialised in HBM, softmax in float32, autograd for the backward; "Standard
    Attention Algorithm" of the FlashAttention pages) against this library on the
    same inputs, and reports the ratio of step times and of the extra device memory
    each needs beyond inputs and outputs."""
    import torch
    from exact_io_aware_63_b200 import binding
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    binding.load(build_if_missing=False)
    x = workload_or_shape(args)
    B, H, N, d = x.q.shape
    # S (f32), P (bf16) and their gradients: skip sizes whose score matrices do not fit
    score_bytes = B * H * N * N * (4 + 2 + 4 + 2)
    line = {"metric": "fwd+bwd step time and extra device memory: standard attention vs this library",
            "workload": args.workload if not args.shape else args.shape,
            "config": {"B": B, "H": H, "N": N, "d": d, "causal": bool(x.causal),
                       "key_padding": x.kv_len is not None, "block_sparse": x.block_mask is not None},
            "pages_claim": "2-4x faster than standard attention; memory linear instead of quadratic in N"}
    if score_bytes > 100e9:
        line["standard"] = f"skipped: score matrices would need {score_bytes / 1e9:.0f} GB"
        print(json.dumps(line))
        return
    q, k, v, do = (t.to(dev) for t in (x.q, x.k, x.v, x.dout))
    bm = None if x.block_mask is None else x.block_mask.to(dev)
    kl = None if x.kv_len is None else x.kv_len.to(dev)
    allowed = standard_allowed(x, dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def std_step():
        qq, kk, vv = (t.detach().requires_grad_() for t in (q, k, v))
        s = torch.matmul(qq, kk.transpose(-1, -2)).float() * x.scale
        s = s.masked_fill(~allowed, float("-inf"))
        pm = torch.softmax(s, dim=-1).to(torch.bfloat16)
        out = torch.matmul(pm, vv)
        out.backward(do)
        return out, qq.grad, kk.grad, vv.grad

    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_bytes = binding.fa_bwd_workspace_size(B, H, N, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    def our_step():
        for rc in (binding.fa_fwd(q, k, v, o, lse, B, H, N, d, x.scale, x.causal, bm, kl,
                                  stream.cuda_stream),
                   binding.fa_bwd(q, k, v, o, lse, do, dq, dk, dv, B, H, N, d, x.scale, x.causal,
                                  bm, kl, ws, ws_bytes, stream.cuda_stream)):
            if rc != 0:
                raise RuntimeError(binding.fa_status_string(rc))

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        ts.sort()
        return ts[len(ts) // 2]

    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    sampler = ClockSampler(cvd.split(",")[0].strip() if cvd else "0")
    sampler.start()
    time.sleep(0.3)
    t_begin = time.time()
    ours_ms = timed(our_step)
    std_ms = timed(lambda: std_step())
    torch.cuda.synchronize()
    clocks = sampler.stop(t_begin, time.time())
    # extra memory beyond inputs and outputs: ours = LSE + backward workspace;
    # standard = peak of one step above what was allocated before it, minus its outputs
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)
    base = torch.cuda.memory_allocated(dev)
    res = std_step()
    torch.cuda.synchronize()
    out_bytes = sum(t.numel() * t.element_size() for t in res)
    std_extra = torch.cuda.max_memory_allocated(dev) - base - out_bytes
    our_extra = lse.numel() * 4 + ws_bytes
    o_std = res[0].detach().float()
    has_key = allowed.expand(B, H, N, N).any(-1)[..., None]  # rows with an allowed key
    o_diff = float((o.float() - o_std).abs().masked_fill(~has_key, 0.0).max())
    line.update({"ours_ms": ours_ms, "standard_ms": std_ms, "speedup": std_ms / ours_ms,
                 "ours_extra_bytes": our_extra, "standard_extra_bytes": int(std_extra),
                 "memory_ratio": std_extra / our_extra, "max_abs_diff_O": o_diff,
                 "l2": "flushed between timed steps", "timing": "median of steps, CUDA events",
                 "clocks": clocks,
                 "pages_framing": "2-4x faster and 5-20x less memory than PyTorch standard "
                                  "attention, on A100-class GPUs"})
    print(json.dumps(line))


def free_port():
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_ranks(n):
    """Runs this command again as n ranks under torch.distributed.run (one process per
    GPU, rendezvous on 127.0.0.1) and returns its exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr=127.0.0.1", f"--master-port={free_port()}",
           os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long16k_causal",
                    help="tiny | bert | gpt2 | long16k | long16k_causal (default: the 16K causal "
                         "long-context workload, the largest that fits one GPU) | sparse64k")
    ap.add_argument("--shape", default="",
                    help="B,H,N,d: the workload's kind of inputs at another size (profiling)")
    ap.add_argument("--clock-window", type=float, default=1.5,
                    help="seconds of untimed load before timing, sampled for clocks")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="CPU-seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--deterministic", action="store_true",
                    help="time fa_bwd_deterministic (ordered dQ kernel) instead of fa_bwd")
    ap.add_argument("--varlen", action="store_true",
                    help="time fa_fwd_varlen / fa_bwd_varlen on the workload's sequences packed "
                         "without padding")
    ap.add_argument("--dropout", type=float, default=0.0,
                    help="time fa_fwd_dropout / fa_bwd_dropout with this probability")
    ap.add_argument("--vs-standard", action="store_true",
                    help="instead of the benchmark line, compare one step with standard "
                         "attention (S and P materialised) on the same inputs")
    args = ap.parse_args()
    modes = [m for m, on in (("--deterministic", args.deterministic), ("--varlen", args.varlen),
                             ("--dropout", args.dropout > 0)) if on]
    if len(modes) > 1:
        ap.error(" and ".join(modes) + " select different backward paths: give one")
    if not 0.0 <= args.dropout < 1.0:
        ap.error("--dropout must lie in [0, 1)")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and not args.vs_standard:
        # one process per GPU: start them here under torch.distributed.run
        sys.exit(spawn_ranks(args.gpus))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "ours" and not args.vs_standard and args.gpus != world:
        ap.error(f"--gpus {args.gpus} with {world} process(es): launch one process per GPU, "
                 f"e.g. python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py "
                 f"--gpus {args.gpus}")
    if args.warmup < 3 and args.impl == "ours":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3
    if args.vs_standard:
        run_vs_standard(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
