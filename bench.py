"""Benchmark of gla_forward on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 720p] [--impl ours|reference]

One step = one gla_forward call (state reduction, combine, read-out) over one
batch of the workload's synthetic, seeded inputs already resident in HBM.
Under torchrun each rank runs its own copy of the workload on its own GPU
(independent layers, no collective on the data path: weak scaling); the timed
region is bracketed by a barrier and a device synchronisation on both sides
and the reported time is the maximum over ranks.  Rank 0 prints one JSON line.

The inputs of one 720p step are 755 MB (q, k, v, g, beta read + out written),
six times the 126 MB L2, so no step can hit in L2 from the previous one; no
extra flush is done.

--impl reference times the fp64 CPU oracle (oracle/gla_oracle.py) as it
stands, on the host cores, on a bounded sample of the same workload per step.

--variant causal | mx | layer | anchor times the other entry points on the
workload's shape (token-level causal read-out from a zero state, FP8 inputs,
projection + operator + W_o, the gated softmax anchor), each with its own
metric and roofline kernel; --workload blk runs the block-causal sequence.
--profile runs warm-up + steps only (for ncu); --ingest-ncu turns an ncu raw
export into profiles/traffic.json entries.
"""
import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from gated_bidirectional_linear_b200 import replicas, workloads  # noqa: E402

METRIC = "gla_forward tokens/s (20x128 heads, 14720 tok) and HBM GB/s vs B200 peak"
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CSRC = os.path.join(ROOT, "gated_bidirectional_linear_b200", "csrc")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="720p", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--variant", default="bidirectional",
                    choices=["bidirectional", "causal", "mx", "layer", "anchor"],
                    help="causal: the token-level causal read-out (gla_causal_step) of the "
                         "workload, one step = one call from a zero state; mx: gla_forward on "
                         "FP8 (OCP MX) inputs; layer: input projection, gla_forward and W_o "
                         "(gla_layer_forward) at the workload's width; anchor: the gated softmax "
                         "anchor layer (gla_softmax_anchor) on the workload's q, k, v, g")
    ap.add_argument("--cpu-sample-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="only run warmup + steps of gla_forward (for ncu captures)")
    ap.add_argument("--repeats", type=int, default=5,
                    help="timed regions of --steps steps each; the median is reported")
    ap.add_argument("--ingest-ncu", metavar="CSV",
                    help="write profiles/traffic.json entries for --workload from an "
                         "`ncu -i <report> --page raw --csv` export, then exit")
    return ap.parse_args()


def workload_config(wl):
    return {
        "workload": (f"{wl.name}: batch {wl.batch}, {wl.heads} heads x {wl.head_dim}, grid "
                     f"{wl.T}x{wl.H}x{wl.W} ({wl.tokens} tokens), {wl.dtype}, "
                     f"q/k/v/g ~ N(0,1), beta = sigmoid(N(0,1)), theta {wl.rope_theta:g}, "
                     f"eps {wl.eps:g}, seed {wl.seed}"),
        "batch": wl.batch, "heads": wl.heads, "head_dim": wl.head_dim,
        "grid": [wl.T, wl.H, wl.W], "tokens_per_step": wl.batch * wl.tokens,
        "l2": (f"no flush: {wl.alg_bytes_per_call() / 1e6:.0f} MB moved per step vs "
               "126 MB L2"),
    }


def host_info():
    """The host the CPU baseline ran on: logical CPUs, those this process may
    use, and the CPU model."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        usable = os.cpu_count()
    return {"nproc": os.cpu_count(), "usable_cpus": usable, "cpu_model": model}


def timed_repeats(run, stream, dist, sync, dev, repeats):
    """`repeats` timed regions of the same K steps (each bracketed by a
    barrier and a device synchronisation, max over ranks); returns the median
    region time and all of them, in ms."""
    reps = [replicas.timed(run, replicas.CudaTimer(stream), dist, sync, dev)
            for _ in range(max(1, repeats))]
    return float(np.median(reps)), reps


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, "fallback"


def source_sha():
    """Hash of every kernel source file: a traffic record is valid only for
    the code it was captured on."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


_BYTE_UNITS = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
_TIME_UNITS = {"ns": 1e-3, "us": 1.0, "usecond": 1.0, "msecond": 1e3, "ms": 1e3, "nsecond": 1e-3}


def kernel_base_name(full):
    """'void gla::tc_apply_kernel<0>(CUtensorMap_st, ...)' -> 'tc_apply_kernel'."""
    import re
    head = re.sub(r"<.*>", "", full.split("(")[0])
    return head.split()[-1].split("::")[-1]


def ingest_ncu(csv_path, workload):
    """Per kernel of an ncu raw-page CSV export: the mean over its captured
    launches of dram__bytes_read.sum + dram__bytes_write.sum (bytes per
    launch) and of gpu__time_duration.sum, written to profiles/traffic.json
    under (kernel, workload) with the hash of the current kernel sources."""
    import csv
    with open(csv_path, newline="") as f:
        rows = [r for r in csv.reader(f)]
    head = next(i for i, r in enumerate(rows) if "Kernel Name" in r)
    cols, units, data = rows[head], rows[head + 1], rows[head + 2:]
    ix = {name: cols.index(name) for name in
          ("Kernel Name", "dram__bytes_read.sum", "dram__bytes_write.sum",
           "gpu__time_duration.sum")}
    per = {}
    for r in data:
        if len(r) != len(cols):
            continue
        name = kernel_base_name(r[ix["Kernel Name"]])
        byt = sum(float(r[ix[m]]) * _BYTE_UNITS[units[ix[m]]]
                  for m in ("dram__bytes_read.sum", "dram__bytes_write.sum"))
        dur = float(r[ix["gpu__time_duration.sum"]]) * _TIME_UNITS[units[ix["gpu__time_duration.sum"]]]
        per.setdefault(name, []).append((byt, dur))
    try:
        with open(TRAFFIC_FILE) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        doc = {}
    doc["_note"] = ("ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, mean over the "
                    "captured launches, written by `python bench.py --ingest-ncu <csv> "
                    "--workload <w>` from an `ncu -i <report> --page raw --csv` export; valid "
                    "only while the kernel sources hash to source_sha")
    sha = source_sha()
    for name, v in sorted(per.items()):
        doc.setdefault(name, {})[workload] = {
            "bytes_per_launch": int(round(float(np.mean([b for b, _ in v])))),
            "duration_us_under_ncu": round(float(np.mean([t for _, t in v])), 2),
            "launches": len(v), "source_sha": sha, "capture": os.path.basename(csv_path)}
        print(f"{name} [{workload}]: {doc[name][workload]}")
    with open(TRAFFIC_FILE, "w") as f:
        json.dump(doc, f, indent=1, sort_keys=True)
        f.write("\n")


def traffic_for(kernel, workload):
    """ncu DRAM bytes per launch from profiles/traffic.json, if it was taken on
    the current kernel sources; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            doc = json.load(f)
    except (OSError, ValueError):
        return None
    ent = doc.get(kernel, {}).get(workload)
    if not ent or ent.get("source_sha") != source_sha():
        return None
    return ent.get("bytes_per_launch")


class ClockMonitor:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sms.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sms)) if sms else None,
                "sm_max_mhz": max(maxes) if maxes else None,
                "reasons": sorted(reasons), "samples": len(sms)}


def cpu_oracle_rate(wl, seconds, threads=None):
    """The oracle, as it stands, on whole heads of the workload until
    `seconds` have passed: returns (tokens/s of the full layer, heads, s,
    threads).  threads=None: the BLAS threads as configured; else that many."""
    if threads is not None:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=threads, user_api="blas"):
            return cpu_oracle_rate(wl, seconds)
    import oracle.gla_oracle as O
    from threadpoolctl import threadpool_info
    t_used, th = 0.0, 0
    heads = 0
    for idx in range(wl.batch * wl.heads):
        x = workloads.as_f64(workloads.draw(1, wl.tokens, 1, wl.head_dim, wl.dtype, 1000 + idx))
        t0 = time.perf_counter()
        O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.T, wl.H, wl.W,
                  wl.rope_theta, wl.eps)
        t_used += time.perf_counter() - t0
        th += wl.tokens
        heads += 1
        if t_used >= seconds:
            break
    blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
    cores = blas[0] if blas else 1
    return th / t_used / wl.heads, heads, t_used, cores


def run_reference(args, wl, rank):
    if rank != 0:
        return
    import oracle.gla_oracle as O
    from threadpoolctl import threadpool_info
    # One step = the oracle on one head over the first two latent frames.
    T_s = min(2, wl.T)
    n_s = T_s * wl.H * wl.W
    x = workloads.as_f64(workloads.draw(1, n_s, 1, wl.head_dim, wl.dtype, 77))
    for _ in range(args.warmup):
        O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T_s, wl.H, wl.W, wl.rope_theta, wl.eps)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T_s, wl.H, wl.W, wl.rope_theta, wl.eps)
    dt = time.perf_counter() - t0
    value = n_s * args.steps / dt / wl.heads
    blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
    cores = blas[0] if blas else 1
    sample = (f"per step: oracle.forward on 1 of {wl.batch * wl.heads} heads, first {T_s} "
              f"frames ({n_s} tokens); tokens/s of the full layer = token-heads/s / {wl.heads}")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample, "host": host_info()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    wl = workloads.WORKLOADS[args.workload]
    if args.ingest_ncu:
        ingest_ncu(args.ingest_ncu, wl.name)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, wl, rank)
        return

    from gated_bidirectional_linear_b200 import gla
    gla.lib()  # fail loudly if the library is missing
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if wl.n_blocks > 1:
        run_block_causal(args, wl, gla, dev, dist, world, rank, local)
        return
    if args.variant == "causal":
        run_causal(args, wl, gla, dev, dist, world, rank, local)
        return
    if args.variant == "mx":
        run_mx(args, wl, gla, dev, dist, world, rank, local)
        return
    if args.variant == "layer":
        run_layer(args, wl, gla, dev, dist, world, rank, local)
        return
    if args.variant == "anchor":
        run_anchor(args, wl, gla, dev, dist, world, rank, local)
        return

    inp = workloads.make_inputs(wl, seed=replicas.replica_seed(wl.seed, rank))
    d = {k: v.to(dev) for k, v in inp.items()}
    B, N, Hh, hd = d["q"].shape
    code = gla.GLA_DTYPE_BF16 if d["q"].dtype == torch.bfloat16 else gla.GLA_DTYPE_F32
    out = torch.empty_like(d["q"])
    ws = gla.alloc_workspace(gla.gla_forward_workspace_size(B, Hh, hd, wl.T, wl.H, wl.W, code), dev)
    stream = torch.cuda.current_stream(dev)

    def step(events):
        gla.gla_forward_timed(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W,
                              events, wl.rope_theta, wl.eps, out=out, workspace=ws,
                              stream=stream)

    none4 = [None] * 4
    if args.profile:
        for _ in range(args.warmup + args.steps):
            step(none4)
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "steps": args.warmup + args.steps,
                          "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        step(none4)
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK

    def plain_step():
        gla.gla_forward(d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W,
                        wl.rope_theta, wl.eps, out=out, workspace=ws, stream=stream)

    # Timed region: K plain steps (the kernels chain by programmatic dependent
    # launch, so nothing is recorded between them); max over ranks.
    def sync():
        torch.cuda.synchronize(dev)

    def timed_steps():
        for _ in range(args.steps):
            plain_step()

    with ClockMonitor(local) as mon:
        elapsed_ms, reps = timed_repeats(timed_steps, stream, dist, sync, dev, args.repeats)
    status = gla.gla_get_device_status(stream)
    if status != gla.GLA_OK:
        raise RuntimeError(f"device status after the timed region: {gla.status_string(status)}")

    # Per-kernel durations for the roofline: a second timed pass of K steps
    # with CUDA events recorded on the launching stream around each kernel
    # (events between kernels stop them overlapping, so the pass is timed
    # apart from the headline region).
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e4 in evs:          # torch creates its events lazily, at the first record
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    k_state = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    k_comb = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    k_apply = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))
    step_ev = np.array([e[0].elapsed_time(e[3]) for e in evs])
    k_step_events = float(np.mean(step_ev))

    # ---- end to end: host buffers through gla_forward_host, copies timed.
    pinned = {k: v.pin_memory() for k, v in inp.items()}
    out_h = torch.empty_like(pinned["q"]).pin_memory()
    arena = gla.alloc_workspace(gla.gla_forward_host_arena_size(B, Hh, hd, wl.T, wl.H, wl.W, code), dev)
    e2e_steps = max(3, min(args.steps, 200))
    for _ in range(3):
        gla.gla_forward_host(pinned["q"], pinned["k"], pinned["v"], pinned["beta"], pinned["g"],
                             wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, out=out_h, arena=arena,
                             stream=stream)

    def host_steps():
        for _ in range(e2e_steps):
            gla.gla_forward_host(pinned["q"], pinned["k"], pinned["v"], pinned["beta"],
                                 pinned["g"], wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, out=out_h,
                                 arena=arena, stream=stream)

    e2e_ms = replicas.timed(host_steps, replicas.CudaTimer(stream), dist, sync, dev)

    th = B * N * Hh
    esz = 2 if code == gla.GLA_DTYPE_BF16 else 4
    tokens_per_step = B * N
    ms_per_step = elapsed_ms / args.steps
    value = replicas.aggregate_rate(world, tokens_per_step, args.steps, elapsed_ms)
    e2e_value = replicas.aggregate_rate(world, tokens_per_step, e2e_steps, e2e_ms)
    peak, peak_kind = measured_peaks()
    apply_bytes = th * hd * esz * 3                # q, g read + out written
    state_bytes = th * hd * esz * 2 + th * esz     # k, v, beta read
    apply_gbs = apply_bytes / (k_apply * 1e-3) / 1e9
    state_gbs = state_bytes / (k_state * 1e-3) / 1e9
    step_gbs = wl.alg_bytes_per_call() / (ms_per_step * 1e-3) / 1e9

    line = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            rate, heads, secs, cores = cpu_oracle_rate(wl, args.cpu_sample_seconds)
            rate1, heads1, secs1, _ = cpu_oracle_rate(wl, args.cpu_sample_seconds / 3, threads=1)
            cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                   "sample": (f"oracle.forward on {heads} whole heads ({wl.tokens} tokens each) "
                              f"of the {wl.name} workload, {secs:.1f} s; tokens/s of the full "
                              f"layer = token-heads/s / {wl.heads}; cores = BLAS threads"),
                   "host": host_info(),
                   "single_core": {"value": rate1, "unit": "tokens/s", "cores": 1,
                                   "sample": f"{heads1} whole heads, {secs1:.1f} s, one BLAS thread"}}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "repeats": len(reps),
            "repeat_ms_per_step": [round(r / args.steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl), parallelism=f"replicas x{world}"),
            "hbm_gbs_per_gpu": step_gbs,
            "roofline": {"bound": "hbm", "kernel": "tc_apply_kernel", "achieved": apply_gbs,
                         "peak": peak, "unit": "GB/s", "frac": apply_gbs / peak,
                         "peak_kind": peak_kind,
                         "traffic": traffic_for("tc_apply_kernel", wl.name),
                         "alg_bytes_per_launch": apply_bytes, "ms_per_launch": k_apply},
            "kernels_ms": {"tc_state_kernel": k_state, "combine_kernel": k_comb,
                           "tc_apply_kernel": k_apply, "step_with_events": k_step_events,
                           "how": "second timed pass of the same K steps, events around each kernel"},
            "kernels_gbs": {"tc_state_kernel": state_gbs, "tc_apply_kernel": apply_gbs},
            "step_ms_events": {"p10": float(np.percentile(step_ev, 10)),
                               "p50": float(np.percentile(step_ev, 50)),
                               "p90": float(np.percentile(step_ev, 90)),
                               "how": "per step of the events pass (events between kernels)"},
            "step_frac_of_peak": step_gbs / peak,
            "step_frac_of_nominal_8tbs": step_gbs / 8000.0,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": th * hd * esz * 4 + th * esz,
                    "d2h_bytes_per_step": th * hd * esz, "steps": e2e_steps},
            "gpu_launches": 3 * args.steps,
            "clocks": mon.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_causal(args, wl, gla, dev, dist, world, rank, local):
    """One step = one gla_causal_step over the whole workload from a zero
    state (a new sequence): the token-level causal variant's own measurement."""
    inp = workloads.make_inputs(wl, seed=replicas.replica_seed(wl.seed, rank))
    d = {k: v.to(dev) for k, v in inp.items()}
    B, N, Hh, hd = d["q"].shape
    code = gla.GLA_DTYPE_BF16 if d["q"].dtype == torch.bfloat16 else gla.GLA_DTYPE_F32
    S = torch.zeros(B, Hh, hd, hd, dtype=torch.float32, device=dev)
    z = torch.zeros(B, Hh, hd, dtype=torch.float32, device=dev)
    out = torch.empty_like(d["q"])
    ws = gla.alloc_workspace(gla.gla_causal_workspace_size(B, Hh, hd, wl.T, wl.H, wl.W, code), dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        S.zero_()
        z.zero_()
        if events is None:
            gla.gla_causal_step(S, z, d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T, wl.H, wl.W,
                                0, wl.rope_theta, wl.eps, out=out, workspace=ws, stream=stream)
        else:
            gla.gla_causal_step_timed(S, z, d["q"], d["k"], d["v"], d["beta"], d["g"], wl.T,
                                      wl.H, wl.W, events, 0, wl.rope_theta, wl.eps, out=out,
                                      workspace=ws, stream=stream)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "variant": "causal",
                          "steps": args.warmup + args.steps, "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK

    def sync():
        torch.cuda.synchronize(dev)

    def timed_steps():
        for _ in range(args.steps):
            step()

    with ClockMonitor(local) as mon:
        elapsed_ms, reps = timed_repeats(timed_steps, stream, dist, sync, dev, args.repeats)
    if gla.gla_get_device_status(stream) != gla.GLA_OK:
        raise RuntimeError("device status after the timed region")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e4 in evs:
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    k_state = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    k_prefix = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    k_read = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))

    # End to end through the host entry: inputs from pinned host memory, the
    # call, the output back; the state stays on the device.
    pinned = {k: v.pin_memory() for k, v in inp.items()}
    out_h = torch.empty_like(pinned["q"]).pin_memory()
    arena = gla.alloc_workspace(gla.gla_causal_host_arena_size(B, Hh, hd, wl.T, wl.H, wl.W, code),
                                dev)

    def host_step():
        S.zero_()
        z.zero_()
        gla.gla_causal_step_host(S, z, pinned["q"], pinned["k"], pinned["v"], pinned["beta"],
                                 pinned["g"], wl.T, wl.H, wl.W, 0, wl.rope_theta, wl.eps,
                                 out=out_h, arena=arena, stream=stream)

    e2e_steps = max(3, min(args.steps, 100))
    for _ in range(2):
        host_step()

    def host_steps():
        for _ in range(e2e_steps):
            host_step()

    e2e_ms = replicas.timed(host_steps, replicas.CudaTimer(stream), dist, sync, dev)

    th = B * N * Hh
    esz = 2 if code == gla.GLA_DTYPE_BF16 else 4
    ms_per_step = elapsed_ms / args.steps
    peak, peak_kind = measured_peaks()
    alg = wl.alg_bytes_per_call()                  # q, k, v, g, beta read + out written
    read_gbs = alg / (k_read * 1e-3) / 1e9
    step_gbs = alg / (ms_per_step * 1e-3) / 1e9
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            import oracle.gla_oracle as O
            from threadpoolctl import threadpool_info
            # The oracle's running-sum form on whole heads of the first two
            # frames (its memory grows as N d^2), scaled to the layer.
            T_s = min(2, wl.T)
            n_s = T_s * wl.H * wl.W
            secs, heads = 0.0, 0
            while secs < args.cpu_sample_seconds:
                x = workloads.as_f64(workloads.draw(1, n_s, 1, hd, wl.dtype, 3000 + heads))
                c0 = time.perf_counter()
                O.causal_forward(x["q"], x["k"], x["v"], x["beta"], x["g"], T_s, wl.H, wl.W,
                                 wl.rope_theta, wl.eps)
                secs += time.perf_counter() - c0
                heads += 1
            blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
            cpu = {"value": heads * n_s / secs / wl.heads, "unit": "tokens/s",
                   "cores": blas[0] if blas else 1, "kind": "oracle",
                   "sample": (f"oracle.causal_forward on {heads} heads of the first {T_s} frames "
                              f"({n_s} tokens each) of the {wl.name} grid, {secs:.1f} s; tokens/s "
                              f"of the full layer = token-heads/s / {wl.heads}; cores = BLAS "
                              f"threads"),
                   "host": host_info()}
        line = {
            "metric": (f"gla_causal_step tokens/s ({wl.heads}x{hd} heads, {wl.tokens} tok, "
                       "token-level causal)"),
            "value": replicas.aggregate_rate(world, B * N, args.steps, elapsed_ms),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "repeats": len(reps),
            "repeat_ms_per_step": [round(r / args.steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if code == gla.GLA_DTYPE_BF16 else "f32", "data": "synthetic",
            "config": dict(workload_config(wl), variant="token-level causal from a zero state",
                           parallelism=f"replicas x{world}"),
            "roofline": {"bound": "hbm", "kernel": "tc_causal_kernel", "achieved": read_gbs,
                         "peak": peak, "unit": "GB/s", "frac": read_gbs / peak,
                         "peak_kind": peak_kind,
                         "traffic": traffic_for("tc_causal_kernel", wl.name),
                         "alg_bytes_per_launch": alg, "ms_per_launch": k_read},
            "kernels_ms": {"tc_state_kernel": k_state, "combine_prefix_kernel": k_prefix,
                           "tc_causal_kernel": k_read,
                           "how": "second timed pass of the same K steps, events around each kernel"},
            "step_gbs_at_min_bytes": step_gbs, "step_frac_of_peak": step_gbs / peak,
            "e2e": {"value": replicas.aggregate_rate(world, B * N, e2e_steps, e2e_ms),
                    "unit": "tokens/s", "h2d_bytes_per_step": th * hd * esz * 4 + th * esz,
                    "d2h_bytes_per_step": th * hd * esz, "steps": e2e_steps},
            "gpu_launches": 3 * args.steps,
            "clocks": mon.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_mx(args, wl, gla, dev, dist, world, rank, local):
    """One step = one gla_forward_mx call on the workload with q, k, v, g in
    FP8 (E4M3 codes, one E8M0 scale per 32 channels) and beta in bf16."""
    xh = workloads.draw_mx(wl.batch, wl.tokens, wl.heads, wl.head_dim,
                           replicas.replica_seed(wl.seed, rank))
    x = {k: v.to(dev) for k, v in xh.items()}
    B, N, Hh, hd = x["q"].shape
    out = torch.empty(B, N, Hh, hd, dtype=torch.bfloat16, device=dev)
    ws = gla.alloc_workspace(gla.lib().gla_forward_mx_workspace_size(B, Hh, hd, wl.T, wl.H, wl.W,
                                                                     gla.GLA_PATH_AUTO), dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        gla.gla_forward_mx(x, wl.T, wl.H, wl.W, wl.rope_theta, wl.eps, out=out, workspace=ws,
                           stream=stream, events=events)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "variant": "mx",
                          "steps": args.warmup + args.steps, "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK

    def sync():
        torch.cuda.synchronize(dev)

    def timed_steps():
        for _ in range(args.steps):
            step()

    with ClockMonitor(local) as mon:
        elapsed_ms, reps = timed_repeats(timed_steps, stream, dist, sync, dev, args.repeats)
    if gla.gla_get_device_status(stream) != gla.GLA_OK:
        raise RuntimeError("device status after the timed region")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e4 in evs:
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        step(evs[i])
    torch.cuda.synchronize(dev)
    k_state = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    k_comb = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    k_apply = float(np.mean([e[2].elapsed_time(e[3]) for e in evs]))

    # End to end: the inputs from pinned host memory (one copy per tensor),
    # the call, the output back, every step.
    pinned = {k: v.pin_memory() for k, v in xh.items()}
    out_h = torch.empty(B, N, Hh, hd, dtype=torch.bfloat16).pin_memory()

    def host_step():
        for k in x:
            x[k].copy_(pinned[k], non_blocking=True)
        step()
        out_h.copy_(out, non_blocking=True)

    e2e_steps = max(3, min(args.steps, 100))
    host_step()

    def host_steps():
        for _ in range(e2e_steps):
            host_step()

    e2e_ms = replicas.timed(host_steps, replicas.CudaTimer(stream), dist, sync, dev)

    th = B * N * Hh
    ms_per_step = elapsed_ms / args.steps
    peak, peak_kind = measured_peaks()
    apply_bytes = th * (hd + 4) * 2 + th * hd * 2      # q, g codes + scales read, out written
    state_bytes = th * (hd + 4) * 2 + th * 2           # k, v codes + scales, beta
    alg = apply_bytes + state_bytes                     # 786 B per token-head at d = 128
    apply_gbs = apply_bytes / (k_apply * 1e-3) / 1e9
    step_gbs = alg / (ms_per_step * 1e-3) / 1e9
    if rank == 0:
        line = {
            "metric": (f"gla_forward_mx tokens/s ({wl.heads}x{hd} heads, {wl.tokens} tok, "
                       "FP8 MX inputs)"),
            "value": replicas.aggregate_rate(world, B * N, args.steps, elapsed_ms),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "repeats": len(reps),
            "repeat_ms_per_step": [round(r / args.steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3+bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl), inputs="q, k, v, g E4M3 + E8M0 per 32 channels, "
                           "beta bf16, out bf16", parallelism=f"replicas x{world}"),
            "roofline": {"bound": "hbm", "kernel": "tc_apply_mx_kernel", "achieved": apply_gbs,
                         "peak": peak, "unit": "GB/s", "frac": apply_gbs / peak,
                         "peak_kind": peak_kind,
                         "traffic": traffic_for("tc_apply_mx_kernel", wl.name),
                         "alg_bytes_per_launch": apply_bytes, "ms_per_launch": k_apply},
            "kernels_ms": {"tc_state_mx_kernel": k_state, "combine_kernel": k_comb,
                           "tc_apply_mx_kernel": k_apply,
                           "how": "second timed pass of the same K steps, events around each kernel"},
            "kernels_gbs": {"tc_state_mx_kernel": state_bytes / (k_state * 1e-3) / 1e9,
                            "tc_apply_mx_kernel": apply_gbs},
            "hbm_gbs_per_gpu": step_gbs, "step_frac_of_peak": step_gbs / peak,
            "alg_bytes_per_step": alg,
            "e2e": {"value": replicas.aggregate_rate(world, B * N, e2e_steps, e2e_ms),
                    "unit": "tokens/s", "h2d_bytes_per_step": state_bytes + th * (hd + 4) * 2,
                    "d2h_bytes_per_step": th * hd * 2, "steps": e2e_steps,
                    "via": "one torch copy per input tensor from pinned memory, gla_forward_mx, "
                           "one copy of the output back"},
            "gpu_launches": 3 * args.steps,
            "clocks": mon.summary(),
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def measured_tflops(sustained=True):
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["bf16_tflops_sustained" if sustained else "bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return (1400.0 if sustained else 1590.0), "fallback"


def run_layer(args, wl, gla, dev, dist, world, rank, local):
    """One step = gla_layer_forward on the workload: x [tokens, C] (C = heads *
    head_dim, the model width) -> q, k, v, g, beta by one projection GEMM whose
    epilogue writes the operator's inputs -> gla_forward -> W_o.  Synthetic
    bf16 x ~ N(0, 1) and weights ~ N(0, 1/fan_in)."""
    Hh, d = wl.heads, wl.head_dim
    C = Hh * d
    tokens = wl.batch * wl.tokens
    rng = np.random.Generator(np.random.PCG64(replicas.replica_seed(wl.seed, rank) + 100))
    mk = lambda shape, sc: torch.from_numpy(rng.standard_normal(shape, dtype=np.float32) * sc).to(
        torch.bfloat16).to(dev)
    x = mk((tokens, C), 1.0)
    W_in = mk((4 * C + Hh, C), C ** -0.5)
    W_o = mk((C, C), C ** -0.5)
    y = torch.empty(tokens, C, dtype=torch.bfloat16, device=dev)
    ws = gla.alloc_workspace(gla.lib().gla_layer_workspace_size(wl.batch, Hh, d, wl.T, wl.H, wl.W),
                             dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        gla.gla_layer_forward(x, W_in, W_o, wl.batch, Hh, d, wl.T, wl.H, wl.W, wl.rope_theta,
                              wl.eps, out=y, workspace=ws, stream=stream)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "variant": "layer",
                          "steps": args.warmup + args.steps, "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK

    def sync():
        torch.cuda.synchronize(dev)

    steps = max(1, args.steps // 10)

    def timed_steps():
        for _ in range(steps):
            step()

    with ClockMonitor(local) as mon:
        elapsed_ms, reps = timed_repeats(timed_steps, stream, dist, sync, dev, args.repeats)
    if gla.gla_get_device_status(stream) != gla.GLA_OK:
        raise RuntimeError("device status after the timed region")

    # Per stage, events around the three calls (the stages then do not
    # overlap), one set per step, the steps back to back with one
    # synchronisation at the end.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for ev in evs:
        ev[0].record(stream)
        p = gla.gla_project_in(x, W_in, wl.batch, wl.tokens, Hh, d, stream=stream)
        ev[1].record(stream)
        o = gla.gla_forward(p["q"], p["k"], p["v"], p["beta"], p["g"], wl.T, wl.H, wl.W,
                            wl.rope_theta, wl.eps, stream=stream)
        ev[2].record(stream)
        gla.gla_gemm_bf16(o.view(tokens, C), W_o, out=y, stream=stream)
        ev[3].record(stream)
    torch.cuda.synchronize(dev)
    t_in = [ev[0].elapsed_time(ev[1]) for ev in evs]
    t_op = [ev[1].elapsed_time(ev[2]) for ev in evs]
    t_out = [ev[2].elapsed_time(ev[3]) for ev in evs]
    k_in, k_op, k_out = (float(np.median(t)) for t in (t_in, t_op, t_out))

    ms_per_step = elapsed_ms / steps
    flops_in = 2.0 * tokens * (4 * C + Hh) * C
    flops_out = 2.0 * tokens * C * C
    peak, peak_kind = measured_tflops(sustained=True)
    in_tf = flops_in / (k_in * 1e-3) / 1e12
    if rank == 0:
        line = {
            "metric": (f"gla_layer_forward tokens/s (width {C}, {Hh}x{d} heads, {wl.tokens} tok: "
                       "projection, operator, W_o)"),
            "value": replicas.aggregate_rate(world, tokens, steps, elapsed_ms), "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "repeats": len(reps), "repeat_ms_per_step": [round(r / steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl), layer=(f"x [{tokens}, {C}], W_in [{4 * C + Hh}, "
                                                       f"{C}], W_o [{C}, {C}], N(0, 1/fan_in)"),
                           parallelism=f"replicas x{world}"),
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel (input projection)",
                         "achieved": in_tf, "peak": peak, "unit": "TFLOP/s", "frac": in_tf / peak,
                         "peak_kind": peak_kind + " sustained bf16",
                         "traffic": None, "alg_flops_per_launch": flops_in, "ms_per_launch": k_in},
            "stages_ms": {"project_in": k_in, "gla_forward": k_op, "project_out": k_out,
                          "how": "events around each of the three calls, steps back to back, "
                                 "median"},
            "stages_tflops": {"project_in": in_tf,
                              "project_out": flops_out / (k_out * 1e-3) / 1e12},
            "e2e": None,
            "gpu_launches": 5 * steps,
            "clocks": mon.summary(),
            "cpu_baseline": None,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def anchor_cpu_rate(wl, seconds, rows=256):
    """The oracle's softmax_anchor, as it stands, on `rows` query rows of one
    head at a time (all N keys) until `seconds` have passed: returns (tokens/s
    of the full layer, query rows done, s, BLAS threads)."""
    import oracle.gla_oracle as O
    from threadpoolctl import threadpool_info
    t_used, done, idx = 0.0, 0, 0
    while t_used < seconds:
        x = workloads.as_f64(workloads.draw(1, wl.tokens, 1, wl.head_dim, wl.dtype, 2000 + idx))
        sel = np.linspace(0, wl.tokens - 1, rows).astype(np.int64)
        t0 = time.perf_counter()
        O.softmax_anchor(x["q"], x["k"], x["v"], x["g"], wl.T, wl.H, wl.W, wl.rope_theta,
                         queries=sel)
        t_used += time.perf_counter() - t0
        done += rows
        idx += 1
    blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
    return done / t_used / wl.heads, done, t_used, (blas[0] if blas else 1)


def run_anchor(args, wl, gla, dev, dist, world, rank, local):
    """One step = gla_softmax_anchor on the workload's q, k, v, g (bf16, the
    operator's draw): q/k RMSNorm + 3D RoPE, then bidirectional softmax
    attention over all N tokens with the sigmoid output gate."""
    x = workloads.draw(wl.batch, wl.tokens, wl.heads, wl.head_dim, wl.dtype,
                       replicas.replica_seed(wl.seed, rank))
    d = {n: x[n].to(dev) for n in "qkvg"}
    out = torch.empty_like(d["q"])
    ws = gla.alloc_workspace(gla.gla_softmax_anchor_workspace_size(
        wl.batch, wl.heads, wl.head_dim, wl.T, wl.H, wl.W), dev)
    stream = torch.cuda.current_stream(dev)

    def step(events=None):
        gla.gla_softmax_anchor(d["q"], d["k"], d["v"], d["g"], wl.T, wl.H, wl.W, wl.rope_theta,
                               out=out, workspace=ws, stream=stream, events=events)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            step()
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "variant": "anchor",
                          "steps": args.warmup + args.steps, "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK

    def sync():
        torch.cuda.synchronize(dev)

    steps = max(5, args.steps // 100)
    # Per-kernel times come from the timed region itself: every call records
    # events before the prep, between the kernels and after the attention
    # (the events cost the programmatic overlap of the two kernels, a few µs
    # of a multi-millisecond call).  Created up front, one set per call.
    ev_sets = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
               for _ in range(max(1, args.repeats))]
    rep_i = [0]

    def timed_steps():
        for ev in ev_sets[rep_i[0]]:
            step(ev)
        rep_i[0] += 1

    with ClockMonitor(local) as mon:
        elapsed_ms, reps = timed_repeats(timed_steps, stream, dist, sync, dev, args.repeats)
    t_prep = [ev[0].elapsed_time(ev[1]) for evs in ev_sets for ev in evs]
    t_attn = [ev[1].elapsed_time(ev[2]) for evs in ev_sets for ev in evs]
    if gla.gla_get_device_status(stream) != gla.GLA_OK:
        raise RuntimeError("device status after the timed region")
    k_prep, k_attn = float(np.median(t_prep)), float(np.median(t_attn))

    # End to end: pinned host q, k, v, g in, the output back to pinned host memory.
    host = {n: x[n].pin_memory() for n in "qkvg"}
    out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()

    def e2e_steps():
        for _ in range(steps):
            for n in "qkvg":
                d[n].copy_(host[n], non_blocking=True)
            step()
            out_h.copy_(out, non_blocking=True)

    e2e_ms, _ = timed_repeats(e2e_steps, stream, dist, sync, dev, 1)

    tokens = wl.batch * wl.tokens
    flops = 4.0 * wl.batch * wl.heads * float(wl.tokens) ** 2 * wl.head_dim
    peak, peak_kind = measured_tflops(sustained=True)
    tf = flops / (k_attn * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, rows, t_used, cores = anchor_cpu_rate(wl, args.cpu_sample_seconds)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": (f"oracle.softmax_anchor on {rows} query rows (256 per call, all "
                          f"{wl.tokens} keys, one head per call) in {t_used:.1f} s; tokens/s of "
                          f"the full layer = query-head rows/s / {wl.heads}"),
               "host": host_info()}
    if rank == 0:
        line = {
            "metric": (f"gla_softmax_anchor tokens/s ({wl.heads}x{wl.head_dim} heads, "
                       f"{wl.tokens} tok, bidirectional softmax) and TFLOP/s vs B200 peak"),
            "value": replicas.aggregate_rate(world, tokens, steps, elapsed_ms), "unit": "tokens/s",
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / steps,
            "repeats": len(reps), "repeat_ms_per_step": [round(r / steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl), variant="gated softmax anchor",
                           l2="no flush: K/V of a head are re-read from L2 by design",
                           parallelism=f"replicas x{world}"),
            "roofline": {"bound": "tensor", "kernel": "anchor_attn_kernel",
                         "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "peak_kind": peak_kind + " sustained bf16",
                         "traffic": traffic_for("anchor_attn_kernel", wl.name),
                         "alg_flops_per_launch": flops, "ms_per_launch": k_attn},
            "stages_ms": {"anchor_prep_kernel": k_prep, "anchor_attn_kernel": k_attn,
                          "how": "events around each kernel of every call of the timed "
                                 "region, median"},
            "e2e": {"value": replicas.aggregate_rate(world, tokens, steps, e2e_ms),
                    "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 2 * steps,
            "clocks": mon.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def run_block_causal(args, wl, gla, dev, dist, world, rank, local):
    """One step = a whole sequence of wl.n_blocks blocks through
    gla_block_causal_step, from a zero state (a new sequence).  Not the
    headline metric: the block-causal row's own measurement."""
    inp = workloads.make_inputs(wl, seed=replicas.replica_seed(wl.seed, rank))
    L = wl.tokens
    blocks = [{k: v[:, i * L:(i + 1) * L].contiguous().to(dev) for k, v in inp.items()}
              for i in range(wl.n_blocks)]
    B, _, Hh, hd = blocks[0]["q"].shape
    code = gla.GLA_DTYPE_BF16
    S = torch.zeros(B, Hh, hd, hd, dtype=torch.float32, device=dev)
    z = torch.zeros(B, Hh, hd, dtype=torch.float32, device=dev)
    outs = [torch.empty_like(b["q"]) for b in blocks]
    ws = gla.alloc_workspace(gla.gla_block_causal_workspace_size(B, Hh, hd, wl.T, wl.H, wl.W, code), dev)
    stream = torch.cuda.current_stream(dev)

    def sequence():
        S.zero_()
        z.zero_()
        for i, b in enumerate(blocks):
            gla.gla_block_causal_step(S, z, b["q"], b["k"], b["v"], b["beta"], b["g"], wl.T, wl.H,
                                      wl.W, i * wl.T, wl.rope_theta, wl.eps, out=outs[i],
                                      workspace=ws, stream=stream)

    if args.profile:
        for _ in range(args.warmup + args.steps):
            sequence()
        torch.cuda.synchronize(dev)
        status = gla.gla_get_device_status(stream)
        print(json.dumps({"profile_run": wl.name, "sequences": args.warmup + args.steps,
                          "status": gla.status_string(status)}))
        if status != gla.GLA_OK:
            sys.exit(1)
        return
    for _ in range(max(args.warmup, 3)):
        sequence()
    torch.cuda.synchronize(dev)
    assert gla.gla_get_device_status(stream) == gla.GLA_OK
    steps = max(1, args.steps // wl.n_blocks)
    def sync():
        torch.cuda.synchronize(dev)

    def timed_sequences():
        for _ in range(steps):
            sequence()

    with ClockMonitor(local) as mon:
        ms, reps = timed_repeats(timed_sequences, stream, dist, sync, dev, args.repeats)
    if gla.gla_get_device_status(stream) != gla.GLA_OK:
        raise RuntimeError("device status after the timed region")

    # End to end through the library's host entry: every block's inputs from
    # pinned host memory into the device arena, the step on the device-resident
    # state, and the block's output back to pinned host memory.
    pinned = [{k: v.cpu().pin_memory() for k, v in b.items()} for b in blocks]
    outs_h = [torch.empty_like(o, device="cpu").pin_memory() for o in outs]
    arena = gla.alloc_workspace(
        gla.gla_block_causal_host_arena_size(B, Hh, hd, wl.T, wl.H, wl.W, code), dev)

    def sequence_host():
        S.zero_()
        z.zero_()
        for i, bp in enumerate(pinned):
            gla.gla_block_causal_step_host(S, z, bp["q"], bp["k"], bp["v"], bp["beta"], bp["g"],
                                           wl.T, wl.H, wl.W, i * wl.T, wl.rope_theta, wl.eps,
                                           out=outs_h[i], arena=arena, stream=stream)

    e2e_steps = max(3, min(steps, 50))
    sequence_host()
    def host_sequences():
        for _ in range(e2e_steps):
            sequence_host()

    e2e_ms = replicas.timed(host_sequences, replicas.CudaTimer(stream), dist, sync, dev)

    tokens = B * wl.total_tokens
    th = tokens * Hh
    alg = wl.alg_bytes_per_call() * wl.n_blocks
    state_io = 2 * (B * Hh * hd * hd * 4 + B * Hh * hd * 4) * wl.n_blocks
    ms_step = ms / steps
    peak, peak_kind = measured_peaks()
    gbs = alg / (ms_step * 1e-3) / 1e9
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            import oracle.gla_oracle as O
            from threadpoolctl import threadpool_info
            # Whole heads of the sequence until the sample time has passed
            # (all B x heads of them is the whole job).
            secs, heads = 0.0, 0
            for idx in range(B * Hh):
                x = workloads.as_f64(workloads.draw(1, wl.total_tokens, 1, hd, wl.dtype, 2000 + idx))
                c0 = time.perf_counter()
                O.block_causal_forward(x["q"], x["k"], x["v"], x["beta"], x["g"], wl.n_blocks,
                                       wl.T, wl.H, wl.W, wl.rope_theta, wl.eps)
                secs += time.perf_counter() - c0
                heads += 1
                if secs >= args.cpu_sample_seconds:
                    break
            blas = [p["num_threads"] for p in threadpool_info() if p.get("user_api") == "blas"]
            cpu = {"value": heads * wl.total_tokens / secs / wl.heads, "unit": "tokens/s",
                   "cores": blas[0] if blas else 1, "kind": "oracle",
                   "sample": (f"oracle.block_causal_forward on {heads} of the {B * Hh} heads of "
                              f"the {wl.name} sequence ({wl.n_blocks} blocks each), {secs:.1f} s; "
                              f"tokens/s of the full layer = token-heads/s / {wl.heads}; "
                              f"cores = BLAS threads"),
                   "host": host_info()}
        line = {
            "metric": "gla_block_causal_step tokens/s (20x128 heads, 20 blocks of 3x23x40)",
            "value": replicas.aggregate_rate(world, tokens, steps, ms), "unit": "tokens/s",
            "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "repeats": len(reps), "repeat_ms_per_step": [round(r / steps, 5) for r in reps],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": dict(workload_config(wl), blocks=wl.n_blocks,
                           step=f"{wl.n_blocks} gla_block_causal_step calls from a zero state",
                           parallelism=f"replicas x{world}"),
            "roofline": {"bound": "hbm", "kernel": "whole step", "achieved": gbs, "peak": peak,
                         "unit": "GB/s", "frac": gbs / peak, "peak_kind": peak_kind,
                         "traffic": None, "alg_bytes_per_step": alg,
                         "state_bytes_per_step": state_io},
            "e2e": {"value": replicas.aggregate_rate(world, tokens, e2e_steps, e2e_ms),
                    "unit": "tokens/s",
                    "h2d_bytes_per_step": th * hd * 2 * 4 + th * 2,
                    "d2h_bytes_per_step": th * hd * 2, "steps": e2e_steps},
            "gpu_launches": 3 * wl.n_blocks * steps,
            "clocks": mon.summary(),
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
