"""Throughput of S²-Attn forward + backward on B200 (TFLOP/s, fraction of dense-BF16 peak).

One step = one pass of the whole hot path over one batch: forward (O, LSE), backward
preprocess (D), the dK/dV kernel (which also hands its bf16 dS tiles to the dQ pass) and the
dQ kernel (dQ = scale * dS K over those tiles), all through the C ABI. FLOPs are algorithmic:
7 * B * Hq * N * G * d per fwd+bwd (causal half of each G x G group; fwd 2, bwd 5).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
                  [--bwd-path handoff|recompute] [--workspace-cap BYTES]

--bwd-path recompute times the minimum-workspace backward (the dQ kernel recomputes S and dP);
--workspace-cap bounds the dS hand-off workspace, so long sequences run the dK/dV + dQ kernels
once per group of kv heads that fits (the whole backward is then timed as one span).

N > 1 runs under torchrun, one process per GPU, each on its own batch of the same workload
(weak scaling, no data-path collective); timing is the max over ranks of device time.
`--impl reference` times the fp64 CPU oracle (the reference arm) on a bounded sample.
Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shifted_sparse_attention_fwd_b200.inputs import METRIC_WORKLOAD, WORKLOADS, make_inputs  # noqa: E402

METRIC = "S²-Attn fwd+bwd TFLOP/s (N=8192,G=2048,bf16); % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def fwd_bwd_flops(w) -> float:
    return 7.0 * w.B * w.Hq * w.N * w.G * w.d


def max_over_ranks(values, dist=None, device=None):
    """Elementwise maximum over all ranks (identity on one process): multi-GPU times are the
    slowest rank's."""
    if dist is None:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def weak_scaling_value(world, flops_per_step, steps, total_ms):
    """Whole-job throughput in TFLOP/s: every rank ran `steps` steps of its own batch."""
    return world * flops_per_step * steps / (total_ms * 1e-3) / 1e12


def kernel_flops(w, G=None):
    """Algorithmic FLOPs per launch (causal half of each in-group G x G block)."""
    unit = float(w.B) * w.Hq * w.N * (w.G if G is None else G) * w.d
    return {"s2_fwd": 2 * unit, "s2_bwd_dkdv": 4 * unit, "s2_bwd_dq_ds": 1 * unit,
            "s2_bwd_dq": 1 * unit, "s2_bwd": 5 * unit}


def dq_ds_bytes(w, ds_tiles) -> float:
    # dS tiles read once (32 KB each), K read once, dQ written once (bf16)
    return ds_tiles * 32768.0 + 2.0 * w.B * w.N * w.Hkv * w.d + 2.0 * w.B * w.N * w.Hq * w.d


def pre_bytes(w) -> float:
    # O and dO read once (bf16), LSE read, D and LSE*log2(e) written (fp32)
    return 2.0 * (2 * w.B * w.N * w.Hq * w.d) + 3.0 * 4 * w.B * w.Hq * w.N


def bench_config(w, world=1):
    """The workload description both arms print (identical dicts, so the two lines compare)."""
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "G": w.G,
            "d": w.d, "shift_heads": f"{w.Hq // 2}-{w.Hq - 1}", "batch_per_gpu": w.B,
            "l2": f"flushed before every GPU step ({L2_FLUSH_BYTES >> 20} MiB write, untimed)",
            "parallelism": f"{world} independent replicas (weak scaling)"}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------------------------------
# Clock sampling during the timed region (NVML).
# ------------------------------------------------------------------------------------------
REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that, never guess
            self.nv, self.err = None, str(e)

    def sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            for bit, name in REASON_BITS.items():
                if mask & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def wait(self, event):
        """Sample from the calling thread until `event` has completed: the host enqueues the
        timed steps long before the GPU finishes them, so this covers the rest of the region."""
        while not event.query():
            if self.nv is not None:
                self.sample()              # paced by the NVML calls themselves
            else:
                time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            # the timed loop holds the interpreter lock between launches: switch threads often
            # enough that the sampler runs several times even in a ~15 ms timed region
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
            sys.setswitchinterval(self._switch)

    def summary(self):
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples),
                "sm_mhz_range": [min(self.samples), max(self.samples)] if self.samples else None}


# ------------------------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of the workload.
# ------------------------------------------------------------------------------------------
def oracle_sample(w, target_s: float = 12.0):
    """Time the fp64 oracle's fwd+bwd over whole heads of the workload (all groups of each),
    alternating unrolled and rolled heads, until about target_s seconds have passed."""
    import numpy as np
    from oracle import s2attn_oracle as orc
    from shifted_sparse_attention_fwd_b200.inputs import to_f64
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    q, k, v, do = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed)
    rep = w.Hq // w.Hkv
    order = []
    for i in range(w.Hq // 2):   # 0, Hq/2, 1, Hq/2+1, ...
        order += [i, w.Hq // 2 + i]
    done, elapsed = 0, 0.0
    for h in order:
        kvh = h // rep
        sl = lambda x, j: to_f64(x[:, :, j:j + 1])  # noqa: E731
        shb = 0 if h >= w.Hq // 2 else 1
        qh, kh, vh, doh = sl(q, h), sl(k, kvh), sl(v, kvh), sl(do, h)
        t0 = time.perf_counter()
        orc.s2attn_forward(qh, kh, vh, w.G, w.scale, shift_head_begin=shb)
        orc.s2attn_backward(qh, kh, vh, doh, w.G, w.scale, shift_head_begin=shb)
        elapsed += time.perf_counter() - t0
        done += 1
        if elapsed >= target_s:
            break
    flops = 7.0 * w.B * done * w.N * w.G * w.d
    return {"value": flops / elapsed / 1e12, "unit": UNIT, "cores": int(cores),
            "nproc": os.cpu_count(), "cores_note": "cores = BLAS threads numpy used; nproc = host CPUs",
            "kind": "oracle",
            "sample": f"{done} of {w.Hq} heads (all {w.N // w.G} groups, B={w.B}) fwd+bwd, "
                      f"{elapsed:.1f} s, numpy fp64", "seconds": round(elapsed, 2)}


# ------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------
def run_gpu(args, rank, world, local_rank):
    import shifted_sparse_attention_fwd_b200 as s2
    dist = torch.distributed if world > 1 else None
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    stream = torch.cuda.current_stream()

    # Each rank: its own batch of the workload (weak scaling).
    q, k, v, do = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed + 7919 * rank)
    qd, kd, vd, dod = (x.to(dev) for x in (q, k, v, do))
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    ws_min = s2.s2attn_bwd_workspace_size(w.B, w.Hq, w.N)
    ws_all = s2.s2attn_bwd_workspace_size_ex(w.B, w.Hq, w.Hkv, w.N, w.d, w.G)
    if args.bwd_path == "recompute":
        ws_bytes, passes = ws_min, 0
    else:
        ws_bytes = s2.s2attn_bwd_workspace_size_ex(w.B, w.Hq, w.Hkv, w.N, w.d, w.G,
                                                   cap_bytes=args.workspace_cap)
        per_head = (ws_all - ws_min) // w.Hkv
        passes = -(-w.Hkv // ((ws_bytes - ws_min) // per_head))
    ds_tiles = (ws_all - ws_min) // 32768
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    # One step = forward + the whole backward; events between the stages that are timed apart.
    if args.bwd_path == "recompute":
        names = ["s2_fwd", "s2_bwd_pre", "s2_bwd_dkdv", "s2_bwd_dq"]
    elif passes == 1:
        names = ["s2_fwd", "s2_bwd_pre", "s2_bwd_dkdv", "s2_bwd_dq_ds"]
    else:
        names = ["s2_fwd", "s2_bwd"]      # `passes` dK/dV + dQ passes inside one span

    def step(ev=None):
        if ev: ev[0].record(stream)
        s2.s2attn_fwd(qd, kd, vd, o, lse, w.G, w.scale)
        if ev: ev[1].record(stream)
        if len(names) == 2:
            s2.s2attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, w.G, w.scale, workspace=ws)
            if ev: ev[2].record(stream)
            return
        s2.s2attn_bwd_preprocess(o, lse, dod, ws)
        if ev: ev[2].record(stream)
        if args.bwd_path == "recompute":
            s2.s2attn_bwd_dkdv(qd, kd, vd, dod, dk, dv, w.G, ws, w.scale)
            if ev: ev[3].record(stream)
            s2.s2attn_bwd_dq(qd, kd, vd, dod, dq, w.G, ws, w.scale)
        else:
            s2.s2attn_bwd_dkdv_ds(qd, kd, vd, dod, dk, dv, w.G, ws, w.scale)
            if ev: ev[3].record(stream)
            s2.s2attn_bwd_dq_ds(kd, dq, w.G, ws, w.scale)
        if ev: ev[4].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    st, code = s2.s2attn_get_device_error()
    if st != s2.S2ATTN_OK:
        raise RuntimeError(f"device error {st} code {code:#x} during warm-up")

    # Timed region: K steps, L2 flushed (untimed) before each, per-stage CUDA events.
    nev = len(names) + 1
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    if dist: dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(dev.index)
    with sampler:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            step(evs[i])
        sampler.wait(evs[-1][nev - 1])
        torch.cuda.synchronize()
    if dist: dist.barrier()
    st, code = s2.s2attn_get_device_error()
    if st != s2.S2ATTN_OK:
        raise RuntimeError(f"device error {st} code {code:#x} in the timed region")
    per_k = {n: [e[j].elapsed_time(e[j + 1]) for e in evs] for j, n in enumerate(names)}
    step_ms = [e[0].elapsed_time(e[nev - 1]) for e in evs]
    total_ms = sum(step_ms)
    if args.bwd_path == "recompute":
        launches_per_step = 4
    elif passes == 1:
        launches_per_step = 4
    else:
        launches_per_step = 2 + 2 * passes

    # The next-row kernel measured beside the step (not part of it): RoPE with Position
    # Interpolation (4k -> 8k, scale 0.5) of this workload's Q and K, out of place, L2 flushed.
    rq, rk = torch.empty_like(qd), torch.empty_like(kd)
    rope_reps = 20
    rope_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(rope_reps)]
    for i in range(rope_reps + 2):
        flush.fill_(i & 0xFF)
        if i >= 2: rope_ev[i - 2][0].record(stream)
        s2.s2attn_rope_pi(qd, rq, pi_scale=0.5)
        s2.s2attn_rope_pi(kd, rk, pi_scale=0.5)
        if i >= 2: rope_ev[i - 2][1].record(stream)
    torch.cuda.synchronize()
    rope_ms = sum(e[0].elapsed_time(e[1]) for e in rope_ev) / rope_reps
    rope_bytes = 2 * (qd.numel() + kd.numel()) * 2

    # The preprocess alone, after an L2 flush whose dirty lines were then evicted by a read-only
    # pass (so the kernel pays no one else's write-backs): its own streaming rate.
    pre_alone = None
    if args.bwd_path == "handoff" and passes == 1:
        clean = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        pts = []
        for i in range(12):
            flush.fill_(i & 0xFF)
            clean.sum()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            s2.s2attn_bwd_preprocess(o, lse, dod, ws)
            b_.record(stream)
            torch.cuda.synchronize()
            if i >= 2:
                pts.append(a.elapsed_time(b_))
        pre_alone = statistics.median(pts)
        del clean

    # RoPE with PI of the queries fused into the forward's query-tile path (s2attn_fwd_rope_q)
    # against the separate passes, alternating on this GPU, L2 flushed before each:
    #   separate: rope(Q), rope(K), forward;   fused: rope(K), forward with Q rotated inside.
    rope_ab = None
    if args.workload == METRIC_WORKLOAD:
        qrot = torch.empty_like(qd)
        times = {"separate": [], "fused": [], "fwd": [], "fwd_rope_q": []}
        for i in range(12):
            for mode in ("separate", "fused"):
                flush.fill_(i & 0xFF)
                ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                ev[0].record(stream)
                if mode == "separate":
                    s2.s2attn_rope_pi(qd, rq, pi_scale=0.5)
                    s2.s2attn_rope_pi(kd, rk, pi_scale=0.5)
                    ev[1].record(stream)
                    s2.s2attn_fwd(rq, rk, vd, o, lse, w.G, w.scale)
                else:
                    s2.s2attn_rope_pi(kd, rk, pi_scale=0.5)
                    ev[1].record(stream)
                    s2.s2attn_fwd_rope_q(qd, rk, vd, o, lse, qrot, w.G, w.scale, pi_scale=0.5)
                ev[2].record(stream)
                torch.cuda.synchronize()
                if i >= 2:
                    times[mode].append(ev[0].elapsed_time(ev[2]))
                    times["fwd" if mode == "separate" else "fwd_rope_q"].append(ev[1].elapsed_time(ev[2]))
        # the two rotations differ slightly (angle addition vs per-row fp32 angles)
        rope_diff = float((qrot.float() - rq.float()).abs().max())
        rope_ab = {k_: round(statistics.median(v_), 4) for k_, v_ in times.items()}
        rope_ab["max_abs_q_rot_difference"] = round(rope_diff, 5)
        st, code = s2.s2attn_get_device_error()
        if st != s2.S2ATTN_OK:
            raise RuntimeError(f"device error {st} code {code:#x} in the RoPE comparison")

    # Full causal attention (the pages' Phase 2, standard attention after fine-tuning) through
    # the same kernels: one group of N rows and no roll (G = N, no rolled head), on the metric
    # workload's tensors, beside the step (not part of it), L2 flushed.
    full_causal = None
    if args.workload == METRIC_WORKLOAD:
        fc_ws = torch.empty(s2.s2attn_bwd_workspace_size_ex(w.B, w.Hq, w.Hkv, w.N, w.d, w.N, w.Hq, 0),
                            dtype=torch.uint8, device=dev)
        fc_reps = 10
        fc_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(fc_reps)]
        for i in range(fc_reps + 3):
            flush.fill_(i & 0xFF)
            if i >= 3: fc_ev[i - 3][0].record(stream)
            s2.s2attn_fwd(qd, kd, vd, o, lse, w.N, w.scale, shift_head_begin=w.Hq, shift=0)
            if i >= 3: fc_ev[i - 3][1].record(stream)
            s2.s2attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, w.N, w.scale, shift_head_begin=w.Hq,
                          shift=0, workspace=fc_ws)
            if i >= 3: fc_ev[i - 3][2].record(stream)
        torch.cuda.synchronize()
        st, code = s2.s2attn_get_device_error()
        if st != s2.S2ATTN_OK:
            raise RuntimeError(f"device error {st} code {code:#x} in the full-causal run")
        full_causal = {"fwd_ms": sum(e[0].elapsed_time(e[1]) for e in fc_ev) / fc_reps,
                       "bwd_ms": sum(e[1].elapsed_time(e[2]) for e in fc_ev) / fc_reps,
                       "workspace_bytes": fc_ws.numel()}
        del fc_ws

    # End to end through the public API with host buffers: every step copies its inputs from
    # pinned host memory, runs fwd + bwd and copies its results back, all inside the timed
    # region. Steps are pipelined the way a training loop with a prefetching loader would run
    # them: two sets of device buffers, host-to-device copies on one stream, kernels on another,
    # device-to-host copies on a third, so step i+1's inputs and step i-1's results move over
    # PCIe (both directions at once) while step i computes.
    hq_, hk_, hv_, hdo_ = (x.pin_memory() for x in (q, k, v, do))
    dbuf = [dict(q=qd, k=kd, v=vd, do=dod, o=o, lse=lse, dq=dq, dk=dk, dv=dv)]
    dbuf.append({n: torch.empty_like(t) for n, t in dbuf[0].items()})
    hout = [{n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in dbuf[0].items()
             if n in ("o", "lse", "dq", "dk", "dv")} for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_step(i):
        b = i % 2
        db, hb = dbuf[b], hout[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_comp[b])        # step i-2 no longer reads these inputs
            for n, src in (("q", hq_), ("k", hk_), ("v", hv_), ("do", hdo_)):
                db[n].copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if i >= 2:
            stream.wait_event(ev_out[b])           # step i-2's results have been copied out
        s2.s2attn_fwd(db["q"], db["k"], db["v"], db["o"], db["lse"], w.G, w.scale, stream=stream)
        s2.s2attn_bwd(db["q"], db["k"], db["v"], db["o"], db["lse"], db["do"], db["dq"], db["dk"],
                      db["dv"], w.G, w.scale, workspace=ws, stream=stream)
        ev_comp[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for n in ("o", "lse", "dq", "dk", "dv"):
                hb[n].copy_(db[n], non_blocking=True)
            ev_out[b].record(s_out)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    if dist: dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(2, 2 + e2e_steps):
        e2e_step(i)
    e1.record(s_out)                               # after the last step's results are out
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    # same inputs every step and deterministic kernels: both buffer sets must hold equal results
    for n in ("o", "dq", "dk"):
        if not torch.equal(hout[0][n], hout[1][n]):
            raise RuntimeError(f"pipelined end-to-end steps disagree on {n}")
    h2d = sum(x.numel() * x.element_size() for x in (hq_, hk_, hv_, hdo_))
    d2h = sum(x.numel() * x.element_size() for x in hout[0].values())

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], dist, dev)
    if rank != 0:
        return None

    flops_step = fwd_bwd_flops(w)
    value = weak_scaling_value(world, flops_step, args.steps, total_ms)
    peaks, peak_src = load_peaks()
    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    avg = {n: sum(v_) / len(v_) for n, v_ in per_k.items()}
    kflops = kernel_flops(w)
    dominant = max(avg, key=avg.get)
    traffic = load_traffic(dominant, args.workload)
    if dominant in kflops:
        achieved = kflops[dominant] / (avg[dominant] * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 1),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4),
                "traffic": traffic, "peak_source": f"{peak_src} (burst bf16)",
                "algorithmic_per_launch": kflops[dominant]}
    else:
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        achieved = pre_bytes(w) / (avg[dominant] * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": hbm,
                "unit": "GB/s", "frac": round(achieved / hbm, 4), "traffic": traffic,
                "peak_source": peak_src}
    kern = {}
    for n in names:
        entry = {"ms": round(avg[n], 4)}
        if n in kflops:
            tf = kflops[n] / (avg[n] * 1e-3) / 1e12
            entry.update(tflops_algorithmic=round(tf, 1), frac=round(tf / peak_tf, 4))
        if n == "s2_bwd_pre":
            entry.update(gbs=round(pre_bytes(w) / (avg[n] * 1e-3) / 1e9, 1))
            if pre_alone is not None:
                entry.update(alone_after_clean_l2_ms=round(pre_alone, 4),
                             alone_gbs=round(pre_bytes(w) / (pre_alone * 1e-3) / 1e9, 1))
        if n == "s2_bwd_dq_ds":
            entry.update(gbs=round(dq_ds_bytes(w, ds_tiles) / (avg[n] * 1e-3) / 1e9, 1),
                         ds_tiles=int(ds_tiles))
        if n == "s2_bwd_dq":
            entry.update(executed_units=3, note="recomputes S and dP: 3 GEMMs for 1 algorithmic")
        if n == "s2_bwd":
            entry.update(passes=passes, note="preprocess + one dK/dV and one dQ launch per pass")
        kern[n] = entry
    bwd_ms = sum(avg[n] for n in names if n != "s2_fwd")
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    next_rows = {"rope_pi": {
        "what": "s2attn_rope_pi on Q and K of the workload (PI scale 0.5), outside the step",
        "ms": round(rope_ms, 4), "bytes": rope_bytes,
        "gbs": round(rope_bytes / (rope_ms * 1e-3) / 1e9, 1),
        "frac_of_hbm": round(rope_bytes / (rope_ms * 1e-3) / 1e9 / hbm, 4)}}
    if rope_ab is not None:
        next_rows["rope_pi_fused_q"] = {
            "what": "RoPE-PI of Q fused into the forward (s2attn_fwd_rope_q) vs separate passes, "
                    "median ms, alternating, L2 flushed: separate = rope(Q) + rope(K) + forward, "
                    "fused = rope(K) + forward rotating Q itself",
            **rope_ab,
            "fused_minus_separate_ms": round(rope_ab["fused"] - rope_ab["separate"], 4)}
    if full_causal is not None:
        fc_flops = 7.0 * w.B * w.Hq * w.N * w.N * w.d
        fc_ms = full_causal["fwd_ms"] + full_causal["bwd_ms"]
        fc_tf = fc_flops / (fc_ms * 1e-3) / 1e12
        fwd_fc_tf = kernel_flops(w, G=w.N)["s2_fwd"] / (full_causal["fwd_ms"] * 1e-3) / 1e12
        next_rows["full_causal"] = {
            "what": f"full causal attention (G = N = {w.N}, no rolled head), fwd + bwd through "
                    "the same kernels, outside the step",
            "ms": round(fc_ms, 4), "fwd_ms": round(full_causal["fwd_ms"], 4),
            "bwd_ms": round(full_causal["bwd_ms"], 4), "flops": fc_flops,
            "tflops": round(fc_tf, 1), "workspace_bytes": full_causal["workspace_bytes"],
            "roofline": {"bound": "tensor", "achieved": round(fc_tf, 1), "peak": peak_tf,
                         "unit": "TFLOP/s", "frac": round(fc_tf / peak_tf, 4),
                         "fwd_frac": round(fwd_fc_tf / peak_tf, 4)}}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total_ms / args.steps, 4),
        "step_ms_spread": {
            "min": round(min(step_ms), 4), "median": round(sorted(step_ms)[len(step_ms) // 2], 4),
            "max": round(max(step_ms), 4),
            "first_half": round(sum(step_ms[:len(step_ms) // 2]) / max(1, len(step_ms) // 2), 4),
            "second_half": round(sum(step_ms[len(step_ms) // 2:]) /
                                 max(1, len(step_ms) - len(step_ms) // 2), 4)},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V/dO, Llama2 attention layer shape)",
        "config": bench_config(w, world),
        "pct_of_peak": round(100 * value / peak_tf, 2),
        "fwd": {"ms": round(avg["s2_fwd"], 4),
                "tflops": round(kflops["s2_fwd"] / (avg["s2_fwd"] * 1e-3) / 1e12, 1)},
        "bwd": {"ms": round(bwd_ms, 4),
                "tflops": round(kflops["s2_bwd"] / (bwd_ms * 1e-3) / 1e12, 1),
                "path": ("dQ recomputed (minimum workspace)" if args.bwd_path == "recompute"
                         else "dS hand-off"),
                "passes": passes, "workspace_bytes": int(ws_bytes),
                "workspace_bytes_one_pass": int(ws_all)},
        "peak": {"bf16_tflops": peak_tf, "source": peak_src},
        "kernels": kern,
        "roofline": roof,
        "e2e": {"value": round(weak_scaling_value(world, flops_step, e2e_steps, e2e_ms), 2),
                "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "ms_per_step": round(e2e_ms / e2e_steps, 4),
                "pipelining": "double-buffered: H2D, kernels and D2H on three streams"},
        "clocks": sampler.summary(),
        "gpu_launches": launches_per_step * args.steps,
        "next_rows": next_rows,
    }
    return line


KERNEL_SOURCES = {
    "s2_fwd": ["s2_fwd.cuh"],
    "s2_bwd_pre": ["s2_bwd_pre.cuh"],
    "s2_bwd_dkdv": ["s2_bwd_dkdv.cuh"],
    "s2_bwd_dq_ds": ["s2_bwd_dq_ds.cuh", "s2_bwd_dkdv.cuh"],
}
COMMON_SOURCES = ["s2_common.cuh", "s2_device.cuh", "s2_tiles.cuh", "s2_tmem_wide.cuh"]


def kernel_source_hash(kernel: str) -> str:
    """Hash of the sources a kernel is built from; DRAM counters recorded under another hash
    are stale."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, []) + COMMON_SOURCES:
        with open(os.path.join(ROOT, "shifted_sparse_attention_fwd_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """DRAM bytes per launch of `kernel` from the committed ncu summary (profiles/traffic.json),
    or None when there is none or the kernels changed since it was captured."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload, {}).get(kernel)
    if e is None or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ------------------------------------------------------------------------------------------
# Reference arm: the CPU oracle, as it stands.
# ------------------------------------------------------------------------------------------
def oracle_group_step(w, units, q, k, v, do):
    """One reference step: the oracle's row-restricted evaluation of whole (head, group)
    units (every row of the group, o/lse/dq and dk/dv), cycling over heads and groups."""
    from oracle import s2attn_oracle as orc
    from shifted_sparse_attention_fwd_b200.inputs import to_f64
    rep = w.Hq // w.Hkv
    t0 = time.perf_counter()
    for (b, h, g) in units:
        shift = w.G // 2 if h >= w.Hq // 2 else 0
        rows = list(range(w.G))
        orc.head_group_rows(to_f64(q[b, :, h]), to_f64(k[b, :, h // rep]), to_f64(v[b, :, h // rep]),
                            to_f64(do[b, :, h]), w.G, w.scale, shift, g, rows, kv_rows=rows)
    dt = time.perf_counter() - t0
    return 7.0 * len(units) * w.G * w.G * w.d / dt / 1e12, dt


def run_reference(args, rank):
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    q, k, v, do = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed)
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:
        cores = os.cpu_count() or 1
    ng = w.N // w.G
    seq = [(b, h, g) for b in range(w.B) for g in range(ng)
           for i in range(w.Hq // 2) for h in (i, w.Hq // 2 + i)]
    pos = 0

    def next_unit():
        nonlocal pos
        u = seq[pos % len(seq)]
        pos += 1
        return [u]

    for _ in range(args.warmup):
        oracle_group_step(w, next_unit(), q, k, v, do)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        tf, dt = oracle_group_step(w, next_unit(), q, k, v, do)
        vals.append(tf)
        secs += dt
    value = statistics.mean(vals)
    cb = {"value": round(value, 6), "unit": UNIT, "cores": int(cores), "nproc": os.cpu_count(),
          "cores_note": "cores = BLAS threads numpy used; nproc = host CPUs", "kind": "oracle",
          "sample": f"each step: one (batch, head, group) unit of G={w.G} rows, fwd+bwd, all "
                    f"rows; heads alternate unrolled/rolled; {secs:.1f} s over {args.steps} steps"}
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "ms_per_step": round(1e3 * secs / max(1, args.steps), 3),
            "config": bench_config(w, 1),
            "cpu_baseline": cb,
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="s2attn", choices=["s2attn", "reference"])
    ap.add_argument("--workload", default=METRIC_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--bwd-path", default="handoff", choices=["handoff", "recompute"])
    ap.add_argument("--workspace-cap", type=int, default=0,
                    help="bytes for the dS hand-off workspace (0: all kv heads in one pass)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)

    if args.impl == "reference":
        line = run_reference(args, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        line = run_gpu(args, rank, world, local_rank)
        if line is not None:
            if not args.no_cpu_baseline and world == 1:
                line["cpu_baseline"] = oracle_sample(WORKLOADS[args.workload])
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
