"""S2-Attn fwd+bwd throughput on B200 (TFLOP/s, counted FLOPs) through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-e2e] [--no-cpu-baseline]

A step = one forward (RoPE+PI stage, per-group attention) and one backward (RoPE+PI
stage, dO.O row sums, dK/dV pass, dQ pass) over one batch of the workload, inputs resident
in HBM. Counted FLOPs: forward 4*B*H*N*G*d/2 (causal), backward 2.5x forward.
With N > 1 (torchrun), every rank runs its own batch (independent problems: no data-path
collective); `value` is the sum over ranks of counted FLOPs / the slowest rank's time.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from workloads import HEADLINE, WORKLOADS  # noqa: E402
from longlora_shifted_sparse_b200 import flops  # noqa: E402

METRIC = "S2-Attn fwd+bwd TFLOP/s (bf16, 1 B200) and % of dense bf16 tensor-core peak"
UNIT = "TFLOP/s"


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own independent batch of the workload."""
    return seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(step_flops: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's counted FLOPs over the slowest rank's step time."""
    return step_flops * world / (ms_per_step * 1e-3) / 1e12


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16=p["bf16_tflops"],
                    bf16_sustained=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    sm_max_mhz=p.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, sm_max_mhz=1965.0,
                source="fallback")


def _counted_step_flops(w, ranks=1):
    f = flops.attention_fwd_flops(w.B, w.N, w.Hq, w.d, w.G, w.causal)
    if w.backward:
        f += flops.attention_bwd_flops(w.B, w.N, w.Hq, w.d, w.G, w.causal)
    return f * ranks


def _kernel_work(name, w, es):
    """(bound, algorithmic work per launch, unit) of one library kernel."""
    fwd = flops.attention_fwd_flops(w.B, w.N, w.Hq, w.d, w.G, w.causal)
    if name.startswith("fwd_"):
        work = fwd                      # S = QK^T and O = PV
    elif name.startswith("bwd_dkdv"):
        work = 2.0 * fwd                # S, dP = dO V^T, dV += P^T dO, dK += dS^T Q
    elif name.startswith("bwd_dq"):
        work = 1.5 * fwd                # S, dP, dQ += dS K
    elif name == "rope_pi":       # read q, k and the cos/sin table; write q~, k~
        return "hbm", 2.0 * w.B * w.N * (w.Hq + w.Hkv) * w.d * es + w.N * w.d * 4, "GB/s"
    elif name == "rope_table":    # write the cos/sin table
        return "hbm", w.N * w.d * 4.0, "GB/s"
    elif name == "bwd_rowsum":    # read dO, O, LSE; write D and the 32-byte row terms
        return "hbm", 2.0 * w.B * w.N * w.Hq * w.d * es + 40.0 * w.B * w.Hq * w.N, "GB/s"
    else:
        return None, 0.0, None
    return ("tensor" if name.endswith("_tc") else "alu"), work, "TFLOP/s"


class ClockSampler:
    """SM clock and throttle reasons while the timed region runs: `nvidia-smi` samples (100 ms
    period) plus NVML reads of the same counters every few milliseconds, so that a timed
    region shorter than the `nvidia-smi` period still has samples of its own."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    NVML_PERIOD_S = 0.005

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None
        self.first = 0   # index of the first sample taken after mark()
        self.nvml = None         # (module, device handle) when NVML answers
        self.nvml_samples = []   # (sm MHz, max MHz, reason bits) taken after mark()
        self.nvml_on = threading.Event()
        self.nvml_stop = threading.Event()
        self.nvml_thread = None

    def start(self):
        self._start_nvml()
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        # nvidia-smi takes a moment to start: wait for its first sample (bounded), so that a
        # short timed region still gets samples of its own
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)

    def _start_nvml(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return
        self.nvml = (pynvml, h)
        self.nvml_thread = threading.Thread(target=self._poll_nvml, daemon=True)
        self.nvml_thread.start()

    def _poll_nvml(self):
        nv, h = self.nvml
        smax = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.nvml_stop.is_set():
            if self.nvml_on.is_set():
                try:
                    sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    return
                self.nvml_samples.append((float(sm), float(smax), int(bits)))
            time.sleep(self.NVML_PERIOD_S)

    def mark(self):
        """The timed region starts: samples from here on describe it."""
        self.first = len(self.lines)
        self.nvml_on.set()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def _stop_nvml(self):
        if self.nvml is None:
            return []
        self.nvml_stop.set()
        self.nvml_thread.join(timeout=5)
        nv = self.nvml[0]
        bit = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
               "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
               "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
               "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
        try:
            nv.nvmlShutdown()
        except Exception:
            pass
        return [(sm, smax, {r for r in self.REASONS if bits & bit[r]})
                for sm, smax, bits in self.nvml_samples]

    def stop(self):
        nvml = self._stop_nvml()
        smi = []
        if self.proc is not None:
            # without NVML, a region shorter than the sampling period may end before its
            # first sample: take the next one (at most one period later, bounded wait)
            t0 = time.time()
            while (not nvml and len(self.lines) <= self.first and time.time() - t0 < 0.5
                   and self.proc.poll() is None):
                time.sleep(0.005)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=5)
            for ln in self.lines[self.first:]:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) != len(self.FIELDS):
                    continue
                try:
                    sm, smax = float(parts[0]), float(parts[1])
                except ValueError:
                    continue
                smi.append((sm, smax, {r for r, v in zip(self.REASONS, parts[3:])
                                       if v.lower() == "active"}))
        allx = smi + nvml
        reasons = set().union(*(r for _, _, r in allx)) if allx else set()
        return {"sm_mhz": statistics.median(x[0] for x in allx) if allx else None,
                "sm_max_mhz": max(x[1] for x in allx) if allx else None,
                "reasons": sorted(reasons), "samples": len(smi), "nvml_samples": len(nvml)}


def _traffic(kernel: str):
    """ncu DRAM bytes per launch of `kernel`, if recorded for the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    import hashlib
    src = os.path.join(ROOT, "longlora_shifted_sparse_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != rec["sha256_16"]:
            return None  # the kernel changed since the counters were taken
    return rec["bytes_per_launch"]


def _oracle_sample(w, inputs):
    """One (batch 0, head 0, group 0) unit of the workload through the oracle: forward at
    all G rows, then backward (dq at all rows, dk/dv at all rows); rows over host threads.
    Returns (seconds, counted FLOPs of the unit, threads)."""
    import oracle
    q, k, v, do = inputs
    rows = np.arange(w.G)
    t0 = time.perf_counter()
    oracle.fwd_rows(q, k, v, w.G, w.pi_scale, 0, 0, 0, rows, w.rope_base, w.causal,
                    shift=w.shift)
    if w.backward:
        oracle.bwd_rows(q, k, v, do, w.G, w.pi_scale, 0, 0, 0, rows, rows, w.rope_base,
                        w.causal, shift=w.shift)
    dt = time.perf_counter() - t0
    R = w.Hq // w.Hkv
    unit_fwd = flops.attention_fwd_flops(1, w.G, 1, w.d, w.G, w.causal)
    # head 0's forward, then the backward of all R query heads of kv head 0
    counted = unit_fwd * (1 + 2.5 * R) if w.backward else unit_fwd
    return dt, counted, oracle.max_threads()


SAMPLE_DESC = ("fp64 oracle on one (batch 0, head 0, group 0) unit of {name}: forward at all "
               "{G} rows + backward (dq, dk, dv) at all rows, rows spread over host threads; "
               "FLOPs counted as for the GPU (fwd 2*G*G*d, bwd 2.5x)")


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inputs = synth.s2attn_inputs(w.seed, w.B, w.N, w.Hq, w.Hkv, w.d, w.in_scale, w.dtype)
    steps = []
    for i in range(args.warmup + args.steps):
        dt, counted, cores = _oracle_sample(w, inputs)
        if i >= args.warmup:
            steps.append(dt)
    mean = sum(steps) / len(steps)
    value = counted / mean / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": mean * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.Hq, "H_kv": w.Hkv,
                   "d": w.d, "G": w.G, "pi_scale": w.pi_scale, "rope_base": w.rope_base,
                   "causal": w.causal, "shift": w.shift, "fwd_bwd": w.backward,
                   "parallelism": "host threads"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": SAMPLE_DESC.format(name=w.name, G=w.G)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist
    from longlora_shifted_sparse_b200 import s2attn as s2

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    es = 2 if w.dtype == "bf16" else 4

    # seeded host inputs, one independent batch per rank
    q, k, v, do = synth.s2attn_inputs(rank_seed(w.seed, rank), w.B, w.N, w.Hq, w.Hkv, w.d,
                                      w.in_scale, w.dtype)

    def host_pinned(x):
        t = torch.from_numpy(x.view(np.int16) if w.dtype == "bf16" else x)
        t = t.view(tdt) if w.dtype == "bf16" else t
        return t.pin_memory()

    hq, hk, hv, hdo = (host_pinned(x) for x in (q, k, v, do))
    dq_ = [hx.to(dev) for hx in (hq, hk, hv, hdo)]
    tq, tk, tv, tdo = dq_
    o = torch.empty_like(tq)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    gq, gk, gv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)
    code = s2.S2_BF16 if w.dtype == "bf16" else s2.S2_FP32
    ws = s2.workspace(w.B, w.N, w.Hq, w.Hkv, w.d, code, dev)

    def step():
        s2.forward(tq, tk, tv, w.G, w.pi_scale, w.rope_base, w.causal, ws=ws, out=o, lse=lse,
                   shift=w.shift)
        if w.backward:
            # the training-step order: the backward reuses the rotation the forward left in
            # the workspace (s2attn_bwd_after_fwd), as the autograd wrapper does
            s2.backward(tq, tk, tv, o, lse, tdo, w.G, w.pi_scale, w.rope_base, w.causal, ws=ws,
                        grads=(gq, gk, gv), after_forward=True, shift=w.shift)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    if s2.device_status(ws) != s2.S2_OK:
        raise RuntimeError("device status reports an expired wait during warm-up")

    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    gpu_uuid = str(getattr(props, "uuid", "")) or str(local)
    if gpu_uuid and not gpu_uuid.startswith("GPU-") and len(gpu_uuid) > 8:
        gpu_uuid = "GPU-" + gpu_uuid
    sampler = ClockSampler(gpu_uuid)
    sampler.start()
    s2.check(s2.s2attn_profile_enable(1))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    sampler.mark()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    prof = s2.profile_summary()
    s2.check(s2.s2attn_profile_enable(0))
    clocks = sampler.stop()
    elapsed_ms = e0.elapsed_time(e1)
    if s2.device_status(ws) != s2.S2_OK:
        raise RuntimeError("device status reports an expired wait in the timed region")
    elapsed_ms = max_over_ranks(elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps
    step_flops = _counted_step_flops(w)
    value = aggregate_tflops(step_flops, world, ms_per_step)

    # End to end: every step copies its inputs from pinned host memory to the device, runs
    # forward + backward through the C ABI, and copies all of its outputs back to pinned host
    # memory. As a training input pipeline does, the three stages run on separate streams
    # (two copy streams per direction) with two device buffer sets: the copy-in of step i+1
    # and the copy-out of step i-1 overlap step i's kernels (the copy engines and the SMs
    # work at the same time).
    e2e = None
    if not args.no_e2e:
        outs0 = [o, lse] + ([gq, gk, gv] if w.backward else [])
        ins0 = [tq, tk, tv] + ([tdo] if w.backward else [])
        hins = [hq, hk, hv] + ([hdo] if w.backward else [])
        houts = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in outs0]
        h2d = sum(x.numel() * x.element_size() for x in hins)
        d2h = sum(x.numel() * x.element_size() for x in outs0)
        sets = [(ins0, outs0, ws),
                ([torch.empty_like(x) for x in ins0], [torch.empty_like(x) for x in outs0],
                 torch.empty_like(ws))]
        NS = 2   # copy streams per direction: concurrent copies keep more copy engines busy
        s_ins = [torch.cuda.Stream(dev) for _ in range(NS)]
        s_outs = [torch.cuda.Stream(dev) for _ in range(NS)]
        s_in, s_out = s_ins[0], s_outs[-1]
        ev = {key: [[torch.cuda.Event() for _ in range(NS)] for _ in range(2)]
              for key in ("in", "out")}
        ev["comp"] = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]

        def e2e_step(i):
            k_ = i % 2
            ins, outs, ws_ = sets[k_]
            for si, st in enumerate(s_ins):
                with torch.cuda.stream(st):
                    if used[k_]:
                        st.wait_event(ev["comp"][k_])
                    for j, (d, hsrc) in enumerate(zip(ins, hins)):
                        if j % NS == si:
                            d.copy_(hsrc, non_blocking=True)
                    ev["in"][k_][si].record(st)
            for si in range(NS):
                stream.wait_event(ev["in"][k_][si])
            if used[k_]:
                for si in range(NS):
                    stream.wait_event(ev["out"][k_][si])
            s2.forward(ins[0], ins[1], ins[2], w.G, w.pi_scale, w.rope_base, w.causal, ws=ws_,
                       out=outs[0], lse=outs[1], shift=w.shift)
            if w.backward:
                s2.backward(ins[0], ins[1], ins[2], outs[0], outs[1], ins[3], w.G, w.pi_scale,
                            w.rope_base, w.causal, ws=ws_, grads=tuple(outs[2:]),
                            after_forward=True, shift=w.shift)
            ev["comp"][k_].record(stream)
            for si, st in enumerate(s_outs):
                with torch.cuda.stream(st):
                    st.wait_event(ev["comp"][k_])
                    for j, (hx, x) in enumerate(zip(houts, outs)):
                        if j % NS == si:
                            hx.copy_(x, non_blocking=True)
                    ev["out"][k_][si].record(st)
            used[k_] = True

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        barrier()
        e0.record(s_in)
        for st in s_ins[1:]:
            st.wait_stream(s_in)
        for i in range(args.steps):
            e2e_step(i)
        for st in s_outs[:-1]:
            s_out.wait_stream(st)
        e1.record(s_out)   # after the last copy-out, which follows every earlier stage
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        for ws_ in (sets[0][2], sets[1][2]):
            if s2.device_status(ws_) != s2.S2_OK:
                raise RuntimeError("device status reports an expired wait in the e2e loop")
        e2e = {"value": aggregate_tflops(step_flops, world, e2e_ms / args.steps), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e2e_ms / args.steps,
               "pipeline": "copy-in (two streams), kernels and copy-out (two streams) of "
                           "consecutive steps overlapped, two device buffer sets"}

    peaks = _peaks()
    roofline = None
    if prof:
        name, (n, ms) = max(prof.items(), key=lambda kv: kv[1][1])
        bound, work, unit = _kernel_work(name, w, es)
        avg_s = ms / n * 1e-3
        if bound == "tensor":
            # burst: the larger (stricter) measured figure; the step is far shorter than the
            # seconds-long loop the sustained figure comes from (reported beside it)
            peak = peaks["bf16"]
            achieved = work / avg_s / 1e12
        elif bound == "alu":
            # fp32 FMA pipes: 148 SMs x 128 lanes x 2 FLOP x max SM clock
            peak = 148 * 128 * 2 * peaks["sm_max_mhz"] * 1e6 / 1e12
            achieved = work / avg_s / 1e12
        else:
            peak = peaks["hbm_gbs"]
            achieved = work / avg_s / 1e9
        roofline = {"kernel": name, "bound": bound, "achieved": achieved, "peak": peak,
                    "unit": unit, "frac": achieved / peak, "traffic": _traffic(name),
                    "peak_source": peaks["source"] + (" burst bf16 (cuBLAS 8192^3)"
                                                      if bound == "tensor" else ""),
                    "frac_of_sustained": (achieved / peaks["bf16_sustained"]
                                          if bound == "tensor" else None),
                    "launches": n, "avg_ms": ms / n,
                    "kernels": {k_: {"launches": n_, "total_ms": t_} for k_, (n_, t_) in
                                prof.items()}}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, counted, cores = _oracle_sample(w, (q, k, v, do))
        cpu_baseline = {"value": counted / dt / 1e12, "unit": UNIT, "cores": cores,
                        "kind": "oracle", "sample": SAMPLE_DESC.format(name=w.name, G=w.G)}

    paths = {s2.s2attn_kernel_path(w.B, w.N, w.Hq, w.Hkv, w.d, w.G, s2.mode(w.causal, w.shift),
                                   code)}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "H_q": w.Hq, "H_kv": w.Hkv,
                   "d": w.d, "G": w.G, "pi_scale": w.pi_scale, "rope_base": w.rope_base,
                   "causal": w.causal, "shift": w.shift, "fwd_bwd": w.backward, "parallelism": "independent batch per GPU",
                   "l2": "inputs exceed L2 (q, k, v, dO are %.0f MB each)" %
                         (tq.numel() * es / 1e6),
                   "kernel_path": "tcgen05" if paths == {1} else "cuda-core"},
        "tflops_frac_of_peak": {"measured_burst": value / world / peaks["bf16"],
                                "measured_sustained": value / world / peaks["bf16_sustained"],
                                "spec_2250": value / world / 2250.0},
        "clocks": clocks,
        "gpu_launches": int(sum(n_ for n_, _ in prof.values())) if prof else 0,
        "e2e": e2e,
        "roofline": roofline,
        "cpu_baseline": cpu_baseline,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=HEADLINE)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
