"""Benchmark: banded log-domain Sinkhorn attention, forward + R=2 one-reference
backward, tokens*heads per second on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long32k] [--schedule one_reference|direct]

One step = one forward (T stopped-base iterations, R tail iterations, O = P V)
and one backward (dQ, dK, dV for a fixed cotangent dO) over one batch of the
workload, inputs already resident in HBM.  L2 is flushed (a 256 MiB write)
between timed steps, outside the timed events.  Each step is timed with CUDA
events on the launching stream; with N ranks (torchrun, NCCL) every rank runs
its own copy of the workload (weak scaling: the (batch, head) problems are
independent, so there is no data-path collective) and the step time is the
maximum over ranks.

Extra keys: ``roofline`` for the dominant kernel (per-launch CUDA events
recorded by the library around each launch, see sa_params.trace_*, in up to 10
traced replicas of the step run after the timed ones, which carry no such
events),
``cpu_baseline`` (the CPU oracle on a bounded sample, rank 0 at N=1), ``e2e``
(the same step through the library's host-buffer call
``sinkhorn_attn_step_host``: pinned-host inputs copied in and the results copied
out inside the timed region, pipelined by the library over ``--e2e-groups``
groups of problems), ``gpu_launches`` and ``clocks`` (nvidia-smi sampled every
50 ms during the timed region).

``--impl reference`` times the CPU oracle (the only reference implementation
of this method) on a bounded sample of the same workload.
``--bias-certificate`` prints the bias certificate of the workload's solve
instead of timing steps.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "Sinkhorn-attn fwd+R=2 bwd tokens·heads/s at 1 B200; % of roofline"
UNIT = "tokens*heads/s"


def support_size(L, W, n_valid=None):
    n = L if n_valid is None else n_valid
    return n * (2 * W + 1) - W * (W + 1) if n > W else n * n


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        j = json.load(open(p))
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                    sm_max_mhz=j.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


# FP32 FFMA peak of the SIMT path: 148 SMs x 128 FP32 lanes x 2 FLOP x max SM clock.
def fp32_alu_peak_tflops(sm_max_mhz):
    return 148 * 128 * 2 * sm_max_mhz * 1e6 / 1e12


# algorithmic band contractions (2 d |Omega| FLOPs each) per launch of each kernel kind
CONTRACTIONS = {"lse_sweep": 1, "pv": 2, "wsum": 1, "ds": 3}

# DRAM bytes (read + write) per launch from one ncu capture (profiles/), keyed by
# (workload, kernel kind), with the SHA-256 of the kernel source the capture was
# taken from: a changed source reports traffic as null until it is captured again.
MEASURED_TRAFFIC = {
    # profiles/tc_rowsum_sweep_long32k.md: 164.78 MB read + 12.45 MB written (the
    # source hashed here differs from the captured one in a comment only)
    ("long32k", "lse_sweep"): (177.23e6, "banded_log_domain_b200/csrc/tc_rowsum.cuh",
                               "d11722421a5b8399ea46d399a2d667d90ddda52ce494b1c84dec9191a87ba0fb"),
}


def measured_traffic(workload, kind):
    e = MEASURED_TRAFFIC.get((workload, kind))
    if e is None:
        return None
    nbytes, src, digest = e
    import hashlib
    try:
        with open(os.path.join(ROOT, src), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest() != digest:
                return None
    except OSError:
        return None
    return nbytes


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = os.path.join("/tmp", f"sa_clocks_{os.getpid()}.csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        busy = [r for r in rows if r["power"] > 200.0] or rows
        return {"sm_mhz": statistics.median(r["sm"] for r in busy),
                "sm_max_mhz": max(r["smax"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows), "samples_under_load": len(busy),
                "power_w_max": max(r["power"] for r in rows)}


def dist_setup(backend=None, timeout_s=120):
    """One process per GPU (torchrun's RANK / LOCAL_RANK / WORLD_SIZE).  NCCL on
    GPUs; the same code path runs on CPU with gloo (the multi-process tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return ws, rank, local


def _coll_device():
    import torch.distributed as dist

    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def allreduce_max(x: float, ws: int) -> float:
    """The largest value over the ranks (per-step device time: the job ends with
    its slowest rank)."""
    if ws == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=_coll_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist

        dist.barrier()


def whole_job_value(ws: int, units_per_rank: float, ms_per_step: float) -> float:
    """Weak scaling: every rank processes its own copy of the workload, so the
    job's throughput is all ranks' units over the slowest rank's step time."""
    return ws * units_per_rank / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_sample_rate(w, L_s, schedule, heads=1):
    """tokens*heads/s of the oracle's forward + backward on ``heads`` heads of
    the workload truncated to their first L_s tokens."""
    import oracle

    x = workloads.draw(1, heads, L_s, w.d, dtype=w.dtype, seed=0)
    t0 = time.perf_counter()
    o, st = oracle.forward(x["q"], x["k"], x["v"], W=w.W, eps=w.eps, T=w.T, R=w.R)
    oracle.backward(x["q"], x["k"], x["v"], st, x["dO"], W=w.W, eps=w.eps, R=w.R,
                    schedule=schedule)
    dt = time.perf_counter() - t0
    return heads * L_s / dt, dt


def size_sample(w, schedule, target_s):
    """(heads, tokens) of a sample of about target_s seconds of oracle work."""
    L1 = min(w.L, max(2 * w.W + 2, 2048))
    _, dt1 = oracle_sample_rate(w, L1, schedule)
    per_tok = max(dt1, 1e-4) / L1
    L_s = int(min(w.L, max(L1, target_s / per_tok)))
    heads = int(min(w.B * w.H, max(1, round(target_s / (per_tok * L_s)))))
    return heads, L_s


def oracle_cores():
    n = os.environ.get("OMP_NUM_THREADS")
    if n:
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, schedule, target_s=20.0):
    heads, L_s = size_sample(w, schedule, target_s)
    rate, dt = oracle_sample_rate(w, L_s, schedule, heads)
    return {"value": rate, "unit": UNIT, "cores": oracle_cores(), "kind": "oracle",
            "sample": f"{heads} head(s) x first {L_s} tokens of {w.name} (W={w.W}, T={w.T}, "
                      f"R={w.R}, d={w.d}), forward + {schedule} backward, float64, {dt:.1f} s"}


def run_reference(args, w):
    ws, rank, _ = int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0
    if rank != 0:
        return
    # size each step's sample so that the whole run stays near two minutes
    # (at most 3 s of oracle work per step)
    heads, L_s = size_sample(w, args.schedule, min(3.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_rate(w, L_s, args.schedule, heads)
    times = []
    for _ in range(args.steps):
        _, dt = oracle_sample_rate(w, L_s, args.schedule, heads)
        times.append(dt)
    total = sum(times)
    value = args.steps * heads * L_s / total
    sample = (f"{heads} head(s) x first {L_s} tokens of {w.name} per step, forward + "
              f"{args.schedule} backward, float64")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_certificate(args, w):
    """One JSON line: eta_R for the workload's N = T + R iteration solve (full
    backpropagation as the reference), R*, and the device time it took."""
    if w.dustbin:
        raise SystemExit("the bias certificate is defined here without a dustbin")
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--bias-certificate runs on one GPU")
    import banded_log_domain_b200 as sa

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sa.load()
    _, x = workloads.make(w)
    dt = torch.float32 if args.cert_dtype == "f32" else torch.bfloat16
    d = {k: (None if v is None else (v.to(dev) if k == "mask" else v.to(dev).to(dt)))
         for k, v in x.items() if k in ("q", "k", "v", "dO", "mask")}
    N = w.T + w.R
    Rs = tuple(sorted({int(r) for r in args.cert_rs.split(",") if int(r) <= N}))
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    eta, sel = sa.bias_certificate(d["q"], d["k"], d["v"], d["dO"], N=N, Rs=Rs, tau=args.cert_tau,
                                   W=w.W, eps=w.eps, mask=d["mask"], schedule=args.schedule)
    e1.record(stream)
    torch.cuda.synchronize()
    print(json.dumps({
        "mode": "bias_certificate", "workload": w.name, "N": N, "storage": args.cert_dtype,
        "schedule": args.schedule, "eta": {str(r): eta[r] for r in Rs}, "tau": args.cert_tau,
        "R_star": sel, "seconds": round(e0.elapsed_time(e1) / 1e3, 3),
        "solves": len(Rs) + (0 if N in Rs else 1)}))


def config_of(w, args):
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "W": w.W, "eps": w.eps,
            "T": w.T, "R": w.R, "storage": w.dtype, "dustbin": w.dustbin,
            "schedule": args.schedule,
            "l2": "flushed between timed steps (256 MiB write); inputs 256 MiB > L2"}


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long32k", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--schedule", default="one_reference", choices=["one_reference", "direct"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=5,
                    help="problem groups the host-buffer call pipelines its copies over")
    ap.add_argument("--bias-certificate", action="store_true",
                    help="instead of timing steps, print the bias certificate eta_R of the "
                         "workload's solve (N = T + R iterations) on one GPU")
    ap.add_argument("--cert-dtype", default="f32", choices=["f32", "bf16"],
                    help="storage type for the certificate (f32: the inputs upcast exactly)")
    ap.add_argument("--cert-rs", default="0,1,2,4,8")
    ap.add_argument("--cert-tau", type=float, default=1e-5)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
        return
    if args.bias_certificate:
        run_certificate(args, w)
        return

    ws, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import banded_log_domain_b200 as sa

    sa.load()
    _, x = workloads.make(w)
    mask = x["mask"]
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    kw = dict(W=w.W, eps=w.eps, R=w.R, mask=d["mask"], dustbin=w.dustbin,
              dustbin_score=w.dustbin_score, v_dust=d["v_dust"])
    q, k, v, dO = d["q"], d["k"], d["v"], d["dO"]
    o = torch.empty_like(q)
    p = sa.make_params(w.B, w.H, w.L, w.d, W=w.W, eps=w.eps, T=w.T, R=w.R, dtype=q.dtype,
                       dustbin=w.dustbin)
    state = torch.empty(sa.sinkhorn_attn_state_size(p), dtype=torch.float32, device=dev)
    fws, bws = sa.sinkhorn_attn_workspace_size(p)
    ws_f = torch.zeros(fws, dtype=torch.uint8, device=dev)
    ws_b = torch.zeros(bws, dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    tr_f, tr_b = sa.LaunchTrace(256), sa.LaunchTrace(256)

    def step(trace=True):
        o_, st_ = sa.sinkhorn_attn_fwd(q, k, v, T=w.T, o=o, state=state, ws=ws_f,
                                       trace=tr_f if trace else None, **kw)
        sa.sinkhorn_attn_bwd(q, k, v, o_, dO, st_, schedule=args.schedule, dq=dq, dk=dk, dv=dv,
                             ws=ws_b, trace=tr_b if trace else None, **kw)

    for _ in range(args.warmup):
        step(trace=False)
    torch.cuda.synchronize()
    barrier(ws)

    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    step_ms = []
    kern = {}          # kind -> [total ms, launches]
    launches = 0
    torch.cuda.synchronize()
    barrier(ws)
    # the timed steps run without the library's per-launch trace events (which
    # sit between the kernels); the per-kernel breakdown and the launch count
    # come from traced replicas of the same step right after them
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step(trace=False)
        e1.record(stream)
        torch.cuda.synchronize()
        step_ms.append(e0.elapsed_time(e1))
    torch.cuda.synchronize()
    barrier(ws)
    clk = clocks.stop()
    n_traced = min(args.steps, 10)
    for _ in range(n_traced):
        flush.zero_()
        step()
        torch.cuda.synchronize()
        for tr in (tr_f, tr_b):
            launches += tr.count.value
            for kind, ms in tr.durations():
                a = kern.setdefault(kind, [0.0, 0])
                a[0] += ms
                a[1] += 1
    launches = launches * args.steps // max(n_traced, 1)
    torch.cuda.synchronize()
    barrier(ws)
    total_ms = allreduce_max(sum(step_ms), ws)
    ms_per_step = total_ms / args.steps
    units = w.B * w.H * w.L
    value = whole_job_value(ws, units, ms_per_step)

    peaks = load_peaks()
    # per-problem support size (valid tokens; workloads with masks use their mean)
    if mask is None:
        omega = support_size(w.L, w.W) * w.B * w.H
    else:
        omega = sum(support_size(w.L, w.W, int(n)) for n in mask.sum(1).tolist()) * w.H
    if w.dustbin:
        omega += (2 * w.L + 1) * w.B * w.H
    unit_flops = 2.0 * w.d * omega
    dom = max(kern.items(), key=lambda kv: kv[1][0])
    dom_kind, (dom_ms, dom_n) = dom[0], dom[1]
    avg_ms = dom_ms / dom_n
    # bf16 storage without a dustbin runs on the tensor cores; the rest on FP32 SIMT
    simt = not (w.dtype == "bf16" and not w.dustbin)
    achieved = CONTRACTIONS.get(dom_kind, 1) * unit_flops / (avg_ms * 1e-3) / 1e12
    # exponentials: one per support entry per launch of a sweep (diagnostic ceiling)
    mufu_peak = 148 * 16 * peaks["sm_max_mhz"] * 1e6
    exp_rate = (omega / (avg_ms * 1e-3)) if dom_kind in ("lse_sweep", "wsum", "pv") else None
    if simt:
        peak = fp32_alu_peak_tflops(peaks["sm_max_mhz"])
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": None, "kernel": dom_kind,
                "peak_source": "FP32 FFMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock",
                "launches_per_step": dom_n / n_traced, "avg_launch_ms": avg_ms}
    else:
        # the burst peak: each launch is well under a millisecond, inside a step of a
        # few milliseconds, not a seconds-long loop under the power cap
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": measured_traffic(w.name, dom_kind),
                "kernel": dom_kind,
                "peak_source": f"{peaks['source']} bf16 dense (burst)",
                "launches_per_step": dom_n / n_traced, "avg_launch_ms": avg_ms,
                "exp_per_s": exp_rate, "exp_frac_of_mufu": (exp_rate / mufu_peak) if exp_rate else None,
                "mufu_peak_per_s": mufu_peak}
    # the whole step against the method's roofline: (T + R + 9) band contractions at the
    # bf16 tensor peak vs the algorithmic bytes at the HBM peak, whichever is slower
    elt = 2 if w.dtype == "bf16" else 4
    step_flops = (w.T + w.R + 9) * unit_flops
    step_bytes = w.B * w.H * w.L * w.d * elt * 12 + 12 * 4 * w.B * w.H * (w.L + w.dustbin)
    t_roof = max(step_flops / (peaks["bf16_tflops"] * 1e12), step_bytes / (peaks["hbm_gbs"] * 1e9))
    kernels = {kd: {"ms_per_step": a[0] / n_traced, "launches_per_step": a[1] / n_traced,
                    "share": a[0] / max(sum(b[0] for b in kern.values()), 1e-9)}
               for kd, a in kern.items()}

    # e2e: pinned host inputs in, results out, inside the timed region
    e2e = None
    if not args.no_e2e:
        # the library's host-buffer call: it copies groups of problems in and results
        # out on its own copy streams while other groups compute
        hq, hk, hv, hdO = (t.to("cpu").pin_memory() for t in (q, k, v, dO))
        hmask = None if mask is None else mask.to("cpu").contiguous().pin_memory()
        hvd = None if d["v_dust"] is None else d["v_dust"].to("cpu").contiguous().pin_memory()
        ho, hdq, hdk, hdv = (torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(4))
        h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdO, hmask, hvd)
                  if t is not None)
        d2h = sum(t.numel() * t.element_size() for t in (ho, hdq, hdk, hdv))
        ph = sa.make_params(w.B, w.H, w.L, w.d, W=w.W, eps=w.eps, T=w.T, R=w.R, dtype=q.dtype,
                            dustbin=w.dustbin, schedule=args.schedule)
        ws_h = torch.empty(sa.sinkhorn_attn_step_host_workspace_size(ph, args.e2e_groups),
                           dtype=torch.uint8, device=dev)
        kwh = dict(W=w.W, eps=w.eps, R=w.R, mask=hmask, dustbin=w.dustbin,
                   dustbin_score=w.dustbin_score, v_dust=hvd)

        def e2e_step():
            sa.sinkhorn_attn_step_host(hq, hk, hv, hdO, T=w.T, schedule=args.schedule,
                                       groups=args.e2e_groups, o=ho, dq=hdq, dk=hdk, dv=hdv,
                                       ws=ws_h, **kwh)

        e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        ems = []
        for _ in range(args.steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            torch.cuda.synchronize()
            ems.append(e0.elapsed_time(e1))
        etot = allreduce_max(sum(ems), ws)
        e2e = {"value": ws * units / (etot / args.steps * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": etot / args.steps, "api": "sinkhorn_attn_step_host",
               "groups": args.e2e_groups}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, args.schedule)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32" if simt else "bf16", "data": "synthetic",
                "config": config_of(w, args), "roofline": roof,
                "roofline_step": {"ms": 1e3 * t_roof, "frac": 1e3 * t_roof / ms_per_step,
                                  "flops": step_flops, "bytes": step_bytes,
                                  "peaks": peaks["source"]},
                "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches, "clocks": clk}
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
