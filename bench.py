#!/usr/bin/env python
"""SSM-layer decode throughput of the replay scheme on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload: the small-model-like decode layer (batch 256, 64 heads, head_dim
64, d_state 128, 8 groups, fp32 checkpoint 2 MiB per request, bf16 x/B/C,
interval 16), synthetic inputs from hybrid_model_ssm_replay_b200.inputs.
One step = one interval of the replay scheme (ReplaySSM article s1): 16
rssm_decode_step calls plus one rssm_flush, so every step moves the same
bytes and the checkpoint-update cost is inside the number (s2). The value is
whole-job tokens/s (requests x tokens, all ranks) over K timed steps; the
state read per token (512 MiB) is larger than L2, so no flush of L2 is
needed between steps. Under torchrun each rank runs its own replica of the
layer (requests are independent: weak scaling, no collective on the data
path); the barrier and the max-over-ranks time use torch.distributed.

Also reported in the same JSON line: the conventional per-token
read+write kernel on the same layer (the in-run comparison), the
large-model-like layer (batch 512, 128 heads), the decode kernel's HBM
roofline, an end-to-end number with host buffers, and the fp64 CPU oracle's
throughput on a bounded sample (cpu_baseline).

--impl reference times the fp64 CPU oracle (the checker; there is no
installable reference implementation of this method) on the same workload
and metric, on rank 0 only.
"""
import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSM decode tokens/s at batch 256/512; achieved HBM GB/s vs B200 peak"
WORKLOAD = ("small_b256: replay decode, batch 256, 64 heads, head_dim 64, d_state 128, 8 groups, fp32 checkpoint, "
            "bf16 x/B/C, interval 16")
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=512)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--fused", action="store_true", help="fold the buffer inside the 16th decode (no flush call)")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the comparison, large-layer, e2e and CPU-baseline legs")
    p.add_argument("--profile", nargs="?", const="all", default=None,
                   help="untimed: run hot kernels a few times on the bench workloads (for ncu); "
                        "a comma-separated list of sections, or all")
    return p.parse_args()


# --------------------------------------------------------------- helpers

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s"


def kernel_source_hash():
    h = hashlib.sha1()
    for name in ("rssm_kernels.cu", "rssm_device.cuh"):
        with open(os.path.join(ROOT, "hybrid_model_ssm_replay_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def ncu_traffic(kernel_tag):
    """DRAM bytes per launch from a committed ncu summary, if it was taken
    on the current kernel source (else None)."""
    sha = kernel_source_hash()
    for path in glob.glob(os.path.join(ROOT, "profiles", "*.md")):
        for line in open(path):
            m = re.search(r"bench-traffic:\s*kernel=(\S+)\s+sha=(\w+)\s+bytes_per_launch=(\d+)", line)
            if m and m.group(1) == kernel_tag and m.group(2) == sha:
                return int(m.group(3))
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.sw_power_cap,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 6:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0, t1):
        sel = [p for (t, p) in self.samples if t0 - 0.05 <= t <= t1 + 0.05]
        if not sel:
            sel = [p for (_, p) in self.samples]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[0]) for p in sel if num(p[0]) is not None]
        mx = [num(p[1]) for p in sel if num(p[1]) is not None]
        names = ["sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
        reasons = sorted({names[i] for p in sel for i in range(4) if p[2 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(sel)}


def smi_gpu_id(torch, dev):
    try:
        pr = torch.cuda.get_device_properties(dev)
        return "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[dev]
        return dev


# ---------------------------------------------------- multi-rank plumbing

def reduce_max(value, dist=None, device=None):
    """Max of a per-rank float over all ranks (the job's time is the slowest
    rank's); identity on one rank."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, max_ms):
    """Whole-job units/s: every rank processed units_per_rank in at most max_ms."""
    return world * units_per_rank / (max_ms / 1e3)


# ------------------------------------------------------ analytic bytes

def shape_bytes(shape, in_bytes=2):
    H, P, N, G = shape.nheads, shape.head_dim, shape.d_state, shape.ngroups
    return dict(state=4 * H * P * N, entry=H * P * in_bytes + G * N * in_bytes + 4 * H,
                inputs=H * P * in_bytes + 2 * G * N * in_bytes + 4 * H, y=4 * H * P)


def decode_bytes_per_request(shape, pos):
    """Algorithmic HBM bytes of one replay-decode token of one request at
    buffer position pos: checkpoint read, pos buffered entries read, the
    new entry written, the token's inputs read, y written."""
    b = shape_bytes(shape)
    return b["state"] + pos * b["entry"] + b["entry"] + b["inputs"] + b["y"]


def flush_bytes_per_request(shape, T):
    b = shape_bytes(shape)
    return 2 * b["state"] + T * b["entry"]


def conv_bytes_per_request(shape):
    b = shape_bytes(shape)
    return 2 * b["state"] + b["inputs"] + b["y"]


# --------------------------------------------------------- our arm (GPU)

def run_ours(args):
    import torch
    import torch.distributed as dist

    from hybrid_model_ssm_replay_b200 import rssm
    from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    rssm.lib()

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v):
        return reduce_max(v, dist, dev)

    K, W = args.steps, args.warmup
    wl = WORKLOADS["small_b256"]
    shape = wl["shape"]
    L = shape.interval
    peak, peak_src = measured_peaks()
    main = replay_loop(rssm, torch, shape, wl, K, W, dev, rank, barrier, max_over_ranks, world, args.fused,
                       repeats=0 if args.no_extra else 5)
    ms = main["ms"]
    value = job_throughput(shape.batch * L * K, world, ms)
    dec_avg_ms = main["decode_us"] / 1e3
    dec_bytes = sum(decode_bytes_per_request(shape, i) for i in range(L)) / L * shape.batch
    achieved = dec_bytes / (dec_avg_ms / 1e3) / 1e9
    traffic = ncu_traffic("replay_decode_small_b256")
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "batch_per_gpu": shape.batch, "tokens_per_step": shape.batch * L * world,
                   "step": ("16 x rssm_decode_step with the fused fold on the 16th" if args.fused else
                            "16 x rssm_decode_step + 1 x rssm_flush") +
                           ", replayed as CUDA graphs of the same launches (the 16 decodes, then the flush), "
                           "with CUDA events between the graphs",
                   "l2": "no flush: the 512 MiB fp32 state read each token exceeds the 126 MB L2",
                   "parallelism": f"replicas x{world} (independent requests)"},
        "roofline": {"kernel": "k_replay_pipe (rssm_decode_step)", "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_source": peak_src, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic,
                     "traffic_source": None if traffic is None else
                     "ncu dram__bytes_read.sum + dram__bytes_write.sum per launch, from the summary under "
                     "profiles/ taken on this kernel source (matched by source hash), not measured in this run",
                     "algorithmic_bytes_per_launch": dec_bytes,
                     "avg_launch_us": main["decode_us"],
                     "launch_time_source": "CUDA events on the launching stream around each replay of the "
                                           "16-decode graph inside the timed region, / 16",
                     "achieved_dram": None if traffic is None else traffic / (dec_avg_ms / 1e3) / 1e9,
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "nominal_peak": NOMINAL_HBM_GBS},
        "gpu_launches": K * (L + (0 if args.fused else 1)),
        "clocks": main["clocks"],
    }
    if main.get("repeats"):
        out["repeats"] = main["repeats"]
    if not args.fused:
        fl_us = main["flush_us"]
        fl_bytes = flush_bytes_per_request(shape, L) * shape.batch
        out["flush_kernel"] = {"kernel": "k_fold_pipe (rssm_flush)", "avg_launch_us": fl_us,
                               "achieved_gbs": fl_bytes / (fl_us / 1e6) / 1e9,
                               "frac": fl_bytes / (fl_us / 1e6) / 1e9 / peak,
                               "launch_time_source": "CUDA events around each replay of the flush graph inside the "
                                                     "timed region"}
        out["roofline"]["reconcile_us"] = {"16_decode_plus_flush": 16 * main["decode_us"] + fl_us,
                                           "step": ms / K * 1e3}
    inp, st = main["inp"], main["state"]
    rp = read_peak(torch, dev)
    out["roofline"]["read_peak_gbs"] = rp
    out["roofline"]["frac_of_read_peak"] = achieved / rp
    out["roofline"]["read_peak_source"] = "in-run: torch.sum over 4 GiB of fp32 (a library read-only kernel), best of 5"
    if not args.no_extra:
        out["conventional"] = conv_leg(rssm, torch, shape, inp, K, W, dev, barrier, max_over_ranks, world, peak)
        out["speedup_vs_conventional"] = value / out["conventional"]["value"]
        out["bytes_saved_ratio"] = bytes_saved_ratio(shape, fused=args.fused)
        out["e2e"] = e2e_leg(rssm, torch, st, shape, inp, max(2, min(K, 20)), W, dev, barrier, max_over_ranks,
                             world, args.fused)
        del st, inp, main
        torch.cuda.empty_cache()
        if not args.fused:
            fz = replay_loop(rssm, torch, shape, wl, K, W, dev, rank, barrier, max_over_ranks, world, True)
            fz_value = job_throughput(shape.batch * L * K, world, fz["ms"])
            out["fused_b256"] = {"step": "16 x rssm_decode_step with RSSM_FLAG_FUSED_FLUSH (the 16th decode folds "
                                         "the buffer; no flush call)", "value": fz_value, "unit": UNIT,
                                 "ms_per_step": fz["ms"] / K, "decode_avg_launch_us": fz["decode_us"],
                                 "speedup_vs_conventional": fz_value / out["conventional"]["value"],
                                 "bytes_saved_ratio": bytes_saved_ratio(shape, fused=True),
                                 "vs_separate_flush": fz_value / value}
            del fz
            torch.cuda.empty_cache()
        gpu_id = smi_gpu_id(torch, dev.index if dev.index is not None else 0)

        def clocked(fn, *fargs):
            # the leg's result with the SM clock and throttle reasons sampled while it ran
            sampler = ClockSampler(gpu_id)
            sampler.start()
            t0 = time.time()
            res = fn(*fargs)
            t1 = time.time()
            time.sleep(0.06)
            sampler.stop()
            res["clocks"] = sampler.summary(t0, t1)
            torch.cuda.empty_cache()
            return res

        out["large_b512"] = clocked(large_leg, rssm, torch, WORKLOADS["large_b512"], max(2, min(K, 50)), W, dev,
                                    barrier, max_over_ranks, world, peak, args.fused)
        out["spec_b512_k4"] = clocked(spec_leg, rssm, torch, WORKLOADS["spec_b512_k4"], max(2, min(K, 32)), W, dev,
                                      barrier, max_over_ranks, world, peak)
        out["split_b256"] = clocked(split_leg, rssm, torch, WORKLOADS["split_b256"], max(2, min(K, 50)), W, dev,
                                    barrier, max_over_ranks, world, peak)
        out["prefill_b256"] = clocked(prefill_leg, rssm, torch, WORKLOADS["small_b256"], dev, barrier,
                                      max_over_ranks, world)
        out["batch_sweep_large"] = clocked(sweep_leg, rssm, torch, WORKLOADS["large_b512"], max(2, min(K, 20)), W,
                                           dev, barrier, max_over_ranks, world, peak)
        out["stage_b256"] = clocked(stage_leg, rssm, torch, max(2, min(K, 10)), W, dev, barrier, max_over_ranks,
                                    world)
    if rank == 0 and world == 1 and not args.no_extra:
        out["cpu_baseline"] = cpu_baseline()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))


def replay_loop(rssm, torch, shape, wl, K, W, dev, rank, barrier, max_over_ranks, world, fused, repeats=0):
    """The headline loop: K steps of one interval each (16 decodes + the
    flush, or 16 decodes with the fused fold), replayed as CUDA graphs -- one
    graph of the 16 decodes per input window and one graph of the flush --
    with CUDA events between the graph launches on the launching stream.
    The events give the per-kernel averages inside the timed region; the
    first and last give the time of the K steps. repeats > 0 re-runs the
    timed region that many more times (the median-of-runs protocol)."""
    from hybrid_model_ssm_replay_b200.inputs import make_inputs
    L = shape.interval
    WIN = 2 * L  # distinct tokens of inputs, cycled
    inp = make_inputs(shape, WIN, wl["seed"] + rank, wl["in_dtype"], device=dev)
    flags = rssm.RSSM_FLAG_FUSED_FLUSH if fused else 0
    desc = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups,
                          interval=L, flags=flags)
    st = rssm.RssmState(desc, dev)
    st.ckpt.copy_(inp["ckpt"])
    y = torch.empty((L, shape.batch, shape.nheads, shape.head_dim), device=dev)
    stream = torch.cuda.current_stream()

    def decodes(w):
        for i in range(L):
            t = w * L + i
            rssm.rssm_decode_step(st, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y[i])

    def flush():
        rssm.rssm_flush(st, inp["A"])

    # eager warm-up (loads the kernels, sets their attributes), then capture
    for k in range(W):
        decodes(k % (WIN // L))
        if not fused:
            flush()
    torch.cuda.synchronize()
    g_dec = []
    for w in range(WIN // L):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            decodes(w)
        g_dec.append(g)
    g_fl = None
    if not fused:
        g_fl = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_fl):
            flush()
    st.pos.zero_()
    st.ckpt.copy_(inp["ckpt"])

    def run(k):
        g_dec[k % len(g_dec)].replay()
        if g_fl is not None:
            g_fl.replay()

    for k in range(W):
        run(k)
    torch.cuda.synchronize()
    sampler = ClockSampler(smi_gpu_id(torch, dev.index if dev.index is not None else 0))
    sampler.start()
    time.sleep(0.15)

    def timed_region(K):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K + 1)]
        barrier()
        torch.cuda.synchronize()
        for k in range(K):
            ev[2 * k].record(stream)
            g_dec[k % len(g_dec)].replay()
            ev[2 * k + 1].record(stream)
            if g_fl is not None:
                g_fl.replay()
        ev[2 * K].record(stream)
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ms = ev[0].elapsed_time(ev[2 * K])
        dec = sum(ev[2 * k].elapsed_time(ev[2 * k + 1]) for k in range(K)) / (K * L)
        fl = sum(ev[2 * k + 1].elapsed_time(ev[2 * k + 2]) for k in range(K)) / K
        return ms, dec, fl

    t0 = time.time()
    ms_local, dec_ms, fl_ms = timed_region(K)
    t1 = time.time()
    ms = max_over_ranks(ms_local)
    if rssm.rssm_get_error(st) != 0:
        raise RuntimeError("device error during the timed run")
    res = {"ms": ms, "decode_us": dec_ms * 1e3, "flush_us": fl_ms * 1e3 if not fused else None,
           "inp": inp, "state": st}
    if repeats:
        # each run: two untimed intervals, then at least 512 decode tokens
        KR = max(K, -(-512 // L))
        runs = []
        for _ in range(repeats):
            run(0)
            run(1)
            m, d, f = timed_region(KR)
            runs.append((max_over_ranks(m), d, f))
        vals = sorted(world * shape.batch * L * KR / (m / 1e3) for m, _, _ in runs)
        res["repeats"] = {"runs": repeats, "steps_each": KR, "decode_tokens_each": KR * L,
                          "warmup_intervals_each": 2, "unit": UNIT,
                          "median": statistics.median(vals), "min": vals[0], "max": vals[-1],
                          "decode_us_median": statistics.median(d * 1e3 for _, d, _ in runs),
                          "flush_us_median": None if fused else statistics.median(f * 1e3 for _, _, f in runs),
                          "note": "the timed region run again after the contract run, each run at least 512 decode tokens after two untimed intervals"}
    time.sleep(0.06)
    sampler.stop()
    res["clocks"] = sampler.summary(t0, t1)
    del g_dec, g_fl
    return res


def bytes_saved_ratio(shape, fused=False):
    """Conventional bytes per token / replay bytes per token (an interval of
    16 decodes plus the flush, or the fused fold), algorithmic."""
    L = shape.interval
    b = shape_bytes(shape)
    rep = sum(decode_bytes_per_request(shape, i) for i in range(L))
    if fused:
        rep += b["state"] - b["entry"]  # the filling token writes the folded state instead of its entry
    else:
        rep += flush_bytes_per_request(shape, L)
    return conv_bytes_per_request(shape) * L / rep


def sweep_leg(rssm, torch, wl, K, W, dev, barrier, max_over_ranks, world, peak, batches=(1, 32, 128, 512)):
    """The large layer (128 heads, 64 x 128, 8 groups) at batch 1, 32, 128
    and 512: replay (16 decodes + flush per step) against the conventional
    step, each step a CUDA graph. "hot" replays the steps back to back (at
    batch 1 and 32 the state, 4 and 128 MiB, stays in the 126 MB L2 or
    nearly); "l2_flushed" writes a 256 MiB buffer before each step, outside
    the events that time the step."""
    from hybrid_model_ssm_replay_b200.inputs import LayerShape, make_inputs
    base = wl["shape"]
    L = base.interval
    res = {"workload": "large layer shapes (128 heads, head_dim 64, d_state 128, 8 groups, interval 16)",
           "steps": K, "points": []}
    scrub = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for bsz in batches:
        shape = LayerShape(bsz, base.nheads, base.head_dim, base.d_state, base.ngroups, L)
        inp = make_inputs(shape, L, wl["seed"], wl["in_dtype"], device=dev)
        desc = rssm.make_desc(bsz, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups, interval=L)
        st = rssm.RssmState(desc, dev)
        st.ckpt.copy_(inp["ckpt"])
        h = inp["ckpt"].clone()
        y = torch.empty((bsz, shape.nheads, shape.head_dim), device=dev)

        def rstep():
            for i in range(L):
                rssm.rssm_decode_step(st, inp["x"][i], inp["B"][i], inp["C"][i], inp["dt"][i], inp["A"], inp["D"], y)
            rssm.rssm_flush(st, inp["A"])

        def cstep():
            for i in range(L):
                rssm.rssm_conv_step(desc, h, inp["x"][i], inp["B"][i], inp["C"][i], inp["dt"][i], inp["A"],
                                    inp["D"], y)

        point = {"batch": bsz, "state_mib": 4 * shape.nheads * shape.head_dim * shape.d_state * bsz / 2 ** 20}
        for name, fn in (("replay", rstep), ("conventional", cstep)):
            for _ in range(W):
                fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            for _ in range(W):
                g.replay()
            torch.cuda.synchronize()
            barrier()
            a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(K):
                g.replay()
            e.record()
            torch.cuda.synchronize()
            hot = max_over_ranks(a.elapsed_time(e)) / K
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
            for i in range(K):
                scrub.fill_(i & 0xFF)
                evs[i][0].record()
                g.replay()
                evs[i][1].record()
            torch.cuda.synchronize()
            barrier()
            cold = max_over_ranks(statistics.median(x.elapsed_time(z) for x, z in evs))
            point[name] = {"hot_tokens_per_s": world * bsz * L / (hot / 1e3), "hot_ms_per_step": hot,
                           "l2_flushed_tokens_per_s": world * bsz * L / (cold / 1e3), "l2_flushed_ms_per_step": cold}
            del g
        rb = (sum(decode_bytes_per_request(shape, i) for i in range(L)) + flush_bytes_per_request(shape, L)) * bsz
        point["replay"]["l2_flushed_frac"] = rb / (point["replay"]["l2_flushed_ms_per_step"] / 1e3) / 1e9 / peak
        cb = conv_bytes_per_request(shape) * L * bsz
        point["conventional"]["l2_flushed_frac"] = cb / (point["conventional"]["l2_flushed_ms_per_step"] / 1e3) / 1e9 / peak
        point["speedup_hot"] = point["conventional"]["hot_ms_per_step"] / point["replay"]["hot_ms_per_step"]
        point["speedup_l2_flushed"] = (point["conventional"]["l2_flushed_ms_per_step"] /
                                       point["replay"]["l2_flushed_ms_per_step"])
        res["points"].append(point)
        if rssm.rssm_get_error(st) != 0:
            raise RuntimeError("device error in the batch sweep")
        del st, h, inp, y
        torch.cuda.empty_cache()
    del scrub
    return res


def stage_leg(rssm, torch, K, W, dev, barrier, max_over_ranks, world):
    """A synthetic hybrid decode stage (hybrid_model_ssm_replay_b200.stage)
    at the small layer's shapes, batch 256: 6 Mamba-2 blocks (in_proj GEMM,
    conv1d + SiLU, SSM step, gated norm, out_proj GEMM; d_model 2048) and one
    attention block (16 query / 4 KV heads of 128, a 2048-token KV cache),
    random weights. Replay SSM step (with the flush every 16 tokens) against
    the conventional step on the same weights and inputs; one interval of 16
    tokens per CUDA graph, K graph replays timed."""
    from hybrid_model_ssm_replay_b200.stage import HybridStage, StageShape, make_weights
    shape = StageShape(batch=256, d_model=2048, nheads=64, head_dim=64, d_state=128, ngroups=8, interval=16,
                       n_ssm=6, n_attn=1, attn_heads=16, kv_heads=4, attn_head_dim=128, ctx=2048)
    weights = make_weights(shape, 21, device=dev)
    L = shape.interval
    res = {"workload": "synthetic hybrid stage: batch 256, d_model 2048, 6 Mamba-2 blocks (64 heads x 64 x 128, "
                       "8 groups) + 1 attention block (16/4 heads x 128, 2048-token KV cache)",
           "steps": K, "tokens_per_step": shape.batch * L * world,
           "library_calls": "GEMMs (torch.matmul, cuBLAS), pre-norms and attention (torch SDPA)"}
    ms = {}
    for scheme in ("replay", "conventional"):
        stg = HybridStage(shape, weights, scheme=scheme, seed=22, device=dev)
        u = (torch.randn(shape.batch, shape.d_model, device=dev) * 0.5).to(torch.bfloat16)
        for _ in range(L):
            u = stg.step(u)
        torch.cuda.synchronize()
        u_in = u.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            o = u_in
            for _ in range(L):
                o = stg.step(o)
        for _ in range(W):
            g.replay()
        torch.cuda.synchronize()
        barrier()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(K):
            g.replay()
        e.record()
        torch.cuda.synchronize()
        barrier()
        ms[scheme] = max_over_ranks(a.elapsed_time(e))
        if scheme == "replay":
            for st in stg.ssm:
                if rssm.rssm_get_error(st["state"]) != 0:
                    raise RuntimeError("device error in the stage leg")
        del g, stg, o, u, u_in
        torch.cuda.empty_cache()
    for scheme, m in ms.items():
        res[scheme] = {"tokens_per_s": world * shape.batch * L * K / (m / 1e3), "us_per_token_step": m / (K * L) * 1e3}
    res["stage_speedup"] = ms["conventional"] / ms["replay"]
    res["context_pages"] = "decode-stage speed-up 1.20-1.47x at batch 256 (other models and hardware; context only)"
    return res


def read_peak(torch, dev, nbytes=4 << 30, reps=5):
    """Read-only HBM bandwidth of this GPU, measured in the run: a library
    reduction (torch.sum) over a buffer far larger than L2."""
    x = torch.ones(nbytes // 4, dtype=torch.float32, device=dev)
    x.sum()
    torch.cuda.synchronize()
    best = None
    for _ in range(reps):
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        x.sum()
        e.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(e)
        best = ms if best is None else min(best, ms)
    del x
    torch.cuda.empty_cache()
    return nbytes / (best / 1e3) / 1e9


def conv_leg(rssm, torch, shape, inp, K, W, dev, barrier, max_over_ranks, world, peak):
    desc = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups)
    h = inp["ckpt"].clone()
    L = shape.interval
    y = torch.empty((shape.batch, shape.nheads, shape.head_dim), device=dev)
    n_win = inp["x"].shape[0]

    def step(k):
        for i in range(L):
            t = (k * L + i) % n_win
            rssm.rssm_conv_step(desc, h, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y)

    for k in range(W):
        step(k)
    torch.cuda.synchronize()
    barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for k in range(K):
        step(k)
    e.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(s.elapsed_time(e))
    per_launch = ms / (K * L)
    gbs = conv_bytes_per_request(shape) * shape.batch / (per_launch / 1e3) / 1e9
    return {"kernel": "k_conv (rssm_conv_step)", "value": world * shape.batch * L * K / (ms / 1e3), "unit": UNIT,
            "avg_launch_us": per_launch * 1e3, "achieved_gbs": gbs, "frac": gbs / peak}


def e2e_leg(rssm, torch, st, shape, inp, K, W, dev, barrier, max_over_ranks, world, fused):
    """Same metric through the public API with host buffers: every step
    copies its 16 tokens of inputs from pinned host memory and reads its 16
    outputs back to pinned host memory, inside the timed region. The steps
    are pipelined over three streams, as a serving loop would run them: step
    k's inputs go up while step k-1 computes and step k-2's outputs come
    down (two device buffers each for inputs and outputs; events order every
    reuse)."""
    L = shape.interval
    keys = ("x", "B", "C", "dt")
    hin = [inp[k][:L].cpu().pin_memory() for k in keys]
    NB = 2
    din = [[torch.empty_like(inp[k][:L]) for k in keys] for _ in range(NB)]
    dy = [torch.empty((L, shape.batch, shape.nheads, shape.head_dim), device=dev) for _ in range(NB)]
    hy = [torch.empty(dy[0].shape, dtype=torch.float32).pin_memory() for _ in range(NB)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]
    ev_cmp = [torch.cuda.Event() for _ in range(NB)]
    ev_out = [torch.cuda.Event() for _ in range(NB)]
    st.pos.zero_()
    torch.cuda.synchronize()

    def step(k):
        i = k % NB
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_cmp[i])  # step k-2 has finished reading din[i]
            for d, hsrc in zip(din[i], hin):
                d.copy_(hsrc, non_blocking=True)
            ev_in[i].record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[i])
            s_cmp.wait_event(ev_out[i])  # step k-2's outputs have left dy[i]
            dx, dB, dC, ddt = din[i]
            for t in range(L):
                rssm.rssm_decode_step(st, dx[t], dB[t], dC[t], ddt[t], inp["A"], inp["D"], dy[i][t])
            if not fused:
                rssm.rssm_flush(st, inp["A"])
            ev_cmp[i].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[i])
            hy[i].copy_(dy[i], non_blocking=True)
            ev_out[i].record(s_out)

    for k in range(W):
        step(k)
    torch.cuda.synchronize()
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for k in range(K):
        step(W + k)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_cmp)
    t1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(t0.elapsed_time(t1))
    h2d = sum(t.numel() * t.element_size() for t in hin)
    return {"value": world * shape.batch * L * K / (ms / 1e3), "unit": UNIT, "steps": K,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hy[0].numel() * 4,
            "path": "pinned host -> cudaMemcpyAsync -> rssm_decode_step x16 + rssm_flush -> pinned host, "
                    "steps pipelined over three streams"}


def large_leg(rssm, torch, wl, K, W, dev, barrier, max_over_ranks, world, peak, fused):
    from hybrid_model_ssm_replay_b200.inputs import make_inputs
    shape = wl["shape"]
    L = shape.interval
    inp = make_inputs(shape, L, wl["seed"], wl["in_dtype"], device=dev)
    desc = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups, interval=L,
                          flags=rssm.RSSM_FLAG_FUSED_FLUSH if fused else 0)
    st = rssm.RssmState(desc, dev)
    st.ckpt.copy_(inp["ckpt"])
    y = torch.empty((shape.batch, shape.nheads, shape.head_dim), device=dev)

    def rstep():
        for i in range(L):
            rssm.rssm_decode_step(st, inp["x"][i], inp["B"][i], inp["C"][i], inp["dt"][i], inp["A"], inp["D"], y)
        if not fused:
            rssm.rssm_flush(st, inp["A"])

    def cstep(h):
        for i in range(L):
            rssm.rssm_conv_step(desc, h, inp["x"][i], inp["B"][i], inp["C"][i], inp["dt"][i], inp["A"], inp["D"], y)

    def timed(fn, *a):
        for _ in range(W):
            fn(*a)
        torch.cuda.synchronize()
        barrier()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(K):
            fn(*a)
        e.record()
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(s.elapsed_time(e))

    ms_r = timed(rstep)
    del st
    h = inp["ckpt"].clone()
    ms_c = timed(cstep, h)
    tok = world * shape.batch * L * K
    rep_bytes = (sum(decode_bytes_per_request(shape, i) for i in range(L)) +
                 (0 if fused else flush_bytes_per_request(shape, L))) * shape.batch
    return {"workload": "large_b512: batch 512, 128 heads, 64 x 128, 8 groups, interval 16", "steps": K,
            "replay_tokens_per_s": tok / (ms_r / 1e3), "conventional_tokens_per_s": tok / (ms_c / 1e3),
            "speedup": ms_c / ms_r, "replay_step_gbs": rep_bytes / (ms_r / K / 1e3) / 1e9,
            "replay_step_frac": rep_bytes / (ms_r / K / 1e3) / 1e9 / peak,
            "conventional_gbs": conv_bytes_per_request(shape) * shape.batch * L / (ms_c / K / 1e3) / 1e9}


def spec_leg(rssm, torch, wl, K, W, dev, barrier, max_over_ranks, world, peak):
    """Speculative decoding (s3) on the large layer with K = 4 drafts: per
    step, replay verify of the pending token and 4 drafts + accept(n) + the
    masked flush, against the conventional verify that writes one state copy
    per token + accept (copy index). n ~ U{0..4} per request and step, the
    same table for both. Metric: accepted tokens/s = sum(n + 1) / time."""
    from hybrid_model_ssm_replay_b200.inputs import accept_lengths, make_inputs
    shape = wl["shape"]
    L, Kd = shape.interval, shape.max_draft
    WIN = 8
    inp = make_inputs(shape, WIN, wl["seed"], wl["in_dtype"], device=dev, ntok=Kd + 1)
    n_tab = accept_lengths(W + K, shape.batch, Kd, wl["seed"], device=dev)
    n_host = n_tab.cpu()
    desc = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups, interval=L,
                          max_draft=Kd)
    ys = torch.empty((shape.batch, Kd + 1, shape.nheads, shape.head_dim), device=dev)
    st = rssm.RssmState(desc, dev)
    st.ckpt.copy_(inp["ckpt"])
    ev_v = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    def rstep(s, ev=None):
        w = s % WIN
        if ev is not None:
            ev[0].record()
        rssm.rssm_verify(st, Kd, inp["x"][w], inp["B"][w], inp["C"][w], inp["dt"][w], inp["A"], inp["D"], ys)
        if ev is not None:
            ev[1].record()
        rssm.rssm_accept(st, n_tab[s])
        rssm.rssm_flush(st, inp["A"])

    def timed(fn, evs=None):
        for s in range(W):
            fn(s)
        torch.cuda.synchronize()
        barrier()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for i in range(K):
            if evs is not None:
                fn(W + i, evs[i])
            else:
                fn(W + i)
        e.record()
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(a.elapsed_time(e))

    ms_r = timed(rstep, ev_v)
    if rssm.rssm_get_error(st) != 0:
        raise RuntimeError("device error in the speculative leg")
    # verify bytes from the positions the accept table implies (pos += n + 1, folded at >= L)
    b = shape_bytes(shape)
    pos = torch.zeros(shape.batch, dtype=torch.int64)
    vbytes = []
    for s in range(W + K):
        if s >= W:
            vbytes.append(int((b["state"] + pos * b["entry"] + (Kd + 1) * (b["entry"] + b["inputs"] + b["y"])).sum()))
        pos += n_host[s].long() + 1
        pos = torch.where(pos >= L, torch.zeros_like(pos), pos)
    v_ms = [x.elapsed_time(y) for x, y in ev_v]
    v_gbs = [vb / (m / 1e3) / 1e9 for vb, m in zip(vbytes, v_ms)]
    del st
    torch.cuda.empty_cache()
    # the same speculative run on a split-precision state: verify reads the
    # FP4 output copy, the refresh after accept updates the bf16 copy with SR
    dsp = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups, interval=L,
                         max_draft=Kd, update_dtype=rssm.RSSM_BF16, out_copy=rssm.RSSM_OUTCOPY_FP4, seed=wl["seed"])
    st = rssm.RssmState(dsp, dev)
    st.ckpt.copy_(inp["ckpt"].to(torch.bfloat16))
    rssm.rssm_lowprec_refresh(st, inp["A"], force=True)
    ev_s = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]

    def sstep(s, ev=None):
        w = s % WIN
        if ev is not None:
            ev[0].record()
        rssm.rssm_verify(st, Kd, inp["x"][w], inp["B"][w], inp["C"][w], inp["dt"][w], inp["A"], inp["D"], ys)
        if ev is not None:
            ev[1].record()
        rssm.rssm_accept(st, n_tab[s])
        rssm.rssm_lowprec_refresh(st, inp["A"])

    ms_s = timed(sstep, ev_s)
    if rssm.rssm_get_error(st) != 0:
        raise RuntimeError("device error in the split-precision speculative leg")
    s_ms = [x.elapsed_time(y) for x, y in ev_s]
    del st
    torch.cuda.empty_cache()
    copies = torch.empty((Kd + 1,) + tuple(inp["ckpt"].shape), device=dev)
    copies[0].copy_(inp["ckpt"])
    cur = torch.zeros(shape.batch, dtype=torch.int32, device=dev)

    def cstep(s):
        w = s % WIN
        rssm.rssm_conv_verify(desc, copies, cur, Kd, inp["x"][w], inp["B"][w], inp["C"][w], inp["dt"][w], inp["A"],
                              inp["D"], ys)
        rssm.rssm_conv_accept(desc, n_tab[s], cur, Kd)

    ms_c = timed(cstep)
    del copies
    acc = world * int((n_host[W:W + K].long() + 1).sum())
    return {"workload": "spec_b512_k4: batch 512, 128 heads, 64 x 128, 8 groups, interval 16, K = 4 drafts, "
                        "accepted n ~ U{0..4}", "steps": K,
            "replay_accepted_tokens_per_s": acc / (ms_r / 1e3),
            "conventional_accepted_tokens_per_s": acc / (ms_c / 1e3), "speedup": ms_c / ms_r,
            "replay_step_us": ms_r / K * 1e3, "conventional_step_us": ms_c / K * 1e3,
            "verify_avg_launch_us": sum(v_ms) / len(v_ms) * 1e3,
            "verify_gbs": statistics.mean(v_gbs), "verify_frac": statistics.mean(v_gbs) / peak,
            "split_bf16_fp4": {"replay_accepted_tokens_per_s": acc / (ms_s / 1e3),
                               "speedup_vs_conventional": ms_c / ms_s, "step_us": ms_s / K * 1e3,
                               "verify_avg_launch_us": sum(s_ms) / len(s_ms) * 1e3}}


def split_leg(rssm, torch, wl, K, W, dev, barrier, max_over_ranks, world, peak):
    """Precision split (s4) on the small layer: 16 decodes reading the FP4
    output copy + one refresh of the bf16 (or e4m3) update copy with Philox
    SR, and the shared-copy controls (one FP4 copy, or one bf16 copy with SR,
    read and updated). Timed like the headline loop: CUDA graphs of the 16
    decodes and of the refresh, CUDA events between them."""
    from hybrid_model_ssm_replay_b200.inputs import make_inputs
    shape = wl["shape"]
    L = shape.interval
    H, P, N = shape.nheads, shape.head_dim, shape.d_state
    inp = make_inputs(shape, L, wl["seed"], wl["in_dtype"], device=dev)
    y = torch.empty((shape.batch, H, P), device=dev)
    b = shape_bytes(shape)
    fp4 = H * P * N // 2 + H * P * N // 16
    tok_other = sum(i * b["entry"] for i in range(L)) / L + b["entry"] + b["inputs"] + b["y"]
    out = {"workload": "split_b256: batch 256, 64 heads, 64 x 128, 8 groups, interval 16; decode reads the FP4 "
                       "copy, refresh every 16 tokens", "steps": K,
           "refresh_kernel": "k_fold_umma (the fold of two heads of a group as one tcgen05.mma M128 N128 K16 "
                             "per 16 buffered tokens into tensor memory, x_w split bf16 hi + mid + lo; epilogue "
                             "one accumulator row per thread: Philox SR and FP4 blocks in registers)"}
    hpn = H * P * N
    # (name, update dtype, output copy, bytes of the copy decode reads, of the update copy, of the output copy)
    modes = [("bf16_fp4", rssm.RSSM_BF16, rssm.RSSM_OUTCOPY_FP4, fp4, 2 * hpn, fp4),
             ("e4m3_fp4", rssm.RSSM_E4M3, rssm.RSSM_OUTCOPY_FP4, fp4, hpn, fp4),
             ("shared_fp4", rssm.RSSM_FP4, rssm.RSSM_OUTCOPY_NONE, fp4, fp4, 0),
             ("shared_bf16", rssm.RSSM_BF16, rssm.RSSM_OUTCOPY_NONE, 2 * hpn, 2 * hpn, 0)]
    for name, upd, oc, rd_bytes, upd_bytes, out_bytes in modes:
        desc = rssm.make_desc(shape.batch, H, P, N, shape.ngroups, interval=L, update_dtype=upd, out_copy=oc,
                              seed=wl["seed"])
        st = rssm.RssmState(desc, dev)
        if upd == rssm.RSSM_FP4:
            d0 = rssm.make_desc(shape.batch, H, P, N, shape.ngroups, interval=L, out_copy=rssm.RSSM_OUTCOPY_FP4)
            s0 = rssm.RssmState(d0, dev)
            s0.ckpt.copy_(inp["ckpt"])
            rssm.rssm_lowprec_refresh(s0, inp["A"], force=True)
            st.ckpt.copy_(s0.out_codes)
            st.ckpt_scales.copy_(s0.out_scales)
            del s0
        else:
            st.ckpt.copy_(inp["ckpt"].to(torch.bfloat16 if upd == rssm.RSSM_BF16 else torch.float8_e4m3fn)
                          .view(st.ckpt.dtype))
            rssm.rssm_lowprec_refresh(st, inp["A"], force=True)
        def decodes():
            for i in range(L):
                rssm.rssm_decode_step(st, inp["x"][i], inp["B"][i], inp["C"][i], inp["dt"][i], inp["A"], inp["D"], y)

        def refresh():
            rssm.rssm_lowprec_refresh(st, inp["A"])

        # eager warm-up, then the interval as two CUDA graphs (the 16 decodes,
        # the refresh) replayed with events between them, as the headline loop
        for k in range(W):
            decodes()
            refresh()
        torch.cuda.synchronize()
        g_dec, g_ref = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_dec):
            decodes()
        with torch.cuda.graph(g_ref):
            refresh()
        for k in range(W):
            g_dec.replay()
            g_ref.replay()
        torch.cuda.synchronize()
        barrier()
        stream = torch.cuda.current_stream()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K + 1)]
        for k in range(K):
            ev[2 * k].record(stream)
            g_dec.replay()
            ev[2 * k + 1].record(stream)
            g_ref.replay()
        ev[2 * K].record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = max_over_ranks(ev[0].elapsed_time(ev[2 * K]))
        if rssm.rssm_get_error(st) != 0:
            raise RuntimeError("device error in the precision-split leg")
        del g_dec, g_ref
        d_us = sum(ev[2 * k].elapsed_time(ev[2 * k + 1]) for k in range(K)) / (K * L) * 1e3
        r_us = sum(ev[2 * k + 1].elapsed_time(ev[2 * k + 2]) for k in range(K)) / K * 1e3
        dec_bytes = (rd_bytes + tok_other) * shape.batch
        ref_bytes = (2 * upd_bytes + out_bytes + L * b["entry"]) * shape.batch
        out[name] = {"tokens_per_s": world * shape.batch * L * K / (ms / 1e3), "decode_avg_launch_us": d_us,
                     "decode_gbs": dec_bytes / (d_us / 1e6) / 1e9, "decode_frac": dec_bytes / (d_us / 1e6) / 1e9 / peak,
                     "refresh_avg_launch_us": r_us, "refresh_gbs": ref_bytes / (r_us / 1e6) / 1e9,
                     "refresh_frac": ref_bytes / (r_us / 1e6) / 1e9 / peak,
                     "step_bytes_per_token": (dec_bytes * L + ref_bytes) / (shape.batch * L)}
        del st
        torch.cuda.empty_cache()
    return out


def prefill_leg(rssm, torch, wl, dev, barrier, max_over_ranks, world, T0=512, reps=5):
    """Prefill of a 512-token prompt into the fp32 checkpoint of the small
    layer (rssm_prefill): prompt tokens/s. At these shapes (bf16, d_state 128,
    head_dim 64) the fold is one tensor-core contraction per (request, head),
    X_w^T B with K = T0, and the kernel is bound by HBM: algorithmic bytes per
    request = the prompt's x (H P T0 2) + B (G N T0 2) + dt (4 H T0) + one
    read and one write of the fp32 state (2 x 4 H P N)."""
    from hybrid_model_ssm_replay_b200.inputs import make_inputs
    shape = wl["shape"]
    inp = make_inputs(shape, T0, wl["seed"] + 11, wl["in_dtype"], device=dev)
    desc = rssm.make_desc(shape.batch, shape.nheads, shape.head_dim, shape.d_state, shape.ngroups,
                          interval=shape.interval)
    st = rssm.RssmState(desc, dev)
    st.ckpt.copy_(inp["ckpt"])
    rssm.rssm_prefill(st, inp["x"], inp["B"], inp["dt"], inp["A"])
    torch.cuda.synchronize()
    barrier()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        rssm.rssm_prefill(st, inp["x"], inp["B"], inp["dt"], inp["A"])
    e.record()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(a.elapsed_time(e)) / reps
    if rssm.rssm_get_error(st) != 0:
        raise RuntimeError("device error in the prefill leg")
    H, P, N, G = shape.nheads, shape.head_dim, shape.d_state, shape.ngroups
    req_bytes = H * P * T0 * 2 + G * N * T0 * 2 + 4 * H * T0 + 2 * 4 * H * P * N
    gbs = req_bytes * shape.batch / (ms / 1e3) / 1e9
    peak, peak_src = measured_peaks()
    flops = 2.0 * H * P * N * T0 * shape.batch
    return {"workload": f"small_b256 shapes, prompt of {T0} tokens per request", "prompt_tokens_per_s":
            world * shape.batch * T0 / (ms / 1e3), "ms_per_prefill": ms,
            "kernel": "k_prefill_umma (tcgen05.mma M128 N128 K16 bf16 -> fp32 in tensor memory, two heads per CTA, "
                      "x_w split hi + mid + lo)",
            "bound": "hbm", "algorithmic_bytes_per_request": req_bytes, "achieved_gbs": gbs, "peak": peak,
            "peak_source": peak_src, "frac": gbs / peak,
            "contraction_tflops": flops / (ms / 1e3) / 1e12,
            "note": "fold flops = 2 H P N T0 per request; the hi + mid + lo split issues three times that on the tensor cores"}


# ---------------------------------------------------- the CPU oracle arm

def oracle_interval_sample(n_requests, seed=5):
    """Inputs of n_requests requests of the small layer, one interval, in
    fp64 numpy (same recipe as the GPU run, drawn on the CPU)."""
    import torch
    from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, LayerShape, make_inputs
    s = WORKLOADS["small_b256"]["shape"]
    shape = LayerShape(n_requests, s.nheads, s.head_dim, s.d_state, s.ngroups, s.interval)
    inp = make_inputs(shape, s.interval, seed, torch.bfloat16, device="cpu")
    return {k: v.double().numpy() for k, v in inp.items()}, shape


def oracle_interval(orc, f, b, L):
    req = orc.ReplayRequest(f["ckpt"][b], f["B"].shape[2], L, f["A"], f["D"])
    for t in range(L):
        req.decode(f["x"][t, b], f["B"][t, b], f["C"][t, b], f["dt"][t, b])
    req.flush()
    return L


def _oracle_worker(job):
    """One host core's share of the sharded oracle run (spawned process)."""
    f, L, target_s = job
    from oracle import oracle as orc
    nb = f["ckpt"].shape[0]
    oracle_interval(orc, f, 0, L)  # warm (loads the library)
    tok, b, t0 = 0, 0, time.perf_counter()
    while time.perf_counter() - t0 < target_s:
        tok += oracle_interval(orc, f, b % nb, L)
        b += 1
    return tok, time.perf_counter() - t0, b


def request_slice(f, reqs):
    """The sampled inputs of some requests: ckpt [b], per-token arrays [t][b]."""
    return {k: (v[reqs] if k == "ckpt" else (v[:, reqs] if v.ndim >= 2 else v)) for k, v in f.items()}


def cpu_baseline(target_s=10.0):
    """The fp64 oracle on the host: single thread, then sharded by request
    over the host's cores (one spawned process per core, each on its own
    requests). Reported: the sharded run, with the single-thread figure."""
    import multiprocessing as mp
    from oracle import oracle as orc
    f, shape = oracle_interval_sample(8)
    L = shape.interval
    oracle_interval(orc, f, 0, L)  # warm (loads the library)
    tok, t0 = 0, time.perf_counter()
    b = 0
    while time.perf_counter() - t0 < target_s:
        tok += oracle_interval(orc, f, b % shape.batch, L)
        b += 1
    dt = time.perf_counter() - t0
    single = tok / dt
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    cores = max(1, min(cores, 64))
    jobs = [(request_slice(f, [(2 * i) % 8, (2 * i + 1) % 8]), L, target_s) for i in range(cores)]
    try:
        # spawned workers (no CUDA state is inherited); a worker that fails to
        # start breaks the executor instead of hanging it
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=cores, mp_context=mp.get_context("spawn")) as ex:
            res = list(ex.map(_oracle_worker, jobs, timeout=target_s + 120))
        s_tok = sum(r[0] for r in res)
        s_dt = max(r[1] for r in res)
        s_int = sum(r[2] for r in res)
        return {"value": s_tok / s_dt, "unit": UNIT, "cores": cores, "kind": "oracle",
                "sample": f"{s_int} request-intervals of the small_b256 layer (16 replay decodes + 1 flush each, "
                          f"fp64), sharded by request over {cores} processes, {s_dt:.1f} s",
                "single_thread": {"value": single, "cores": 1,
                                  "sample": f"{b} request-intervals, one thread, {dt:.1f} s"}}
    except Exception as e:  # a host that cannot spawn: the single-thread figure
        return {"value": single, "unit": UNIT, "cores": 1, "kind": "oracle",
                "sample": f"{b} request-intervals of the small_b256 layer (16 replay decodes + 1 flush each, "
                          f"fp64, single thread), {dt:.1f} s; sharded run failed: {type(e).__name__}"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as orc
    f, shape = oracle_interval_sample(8)
    L = shape.interval
    oracle_interval(orc, f, 0, L)
    for k in range(args.warmup):
        oracle_interval(orc, f, k % shape.batch, L)
    t0 = time.perf_counter()
    for k in range(args.steps):
        oracle_interval(orc, f, k % shape.batch, L)
    dt = time.perf_counter() - t0
    value = args.steps * L / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "step": "one request-interval (16 replay decodes + 1 flush) of the fp64 CPU oracle, "
                           "on requests of the same layer"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{args.steps} request-intervals, single thread"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


PROFILE_SECTIONS = ("decode", "fused", "conv", "spec", "conv_verify", "split_bf16", "split_e4m3", "shared_fp4",
                    "prefill")


def run_profile(sections):
    """Hot kernels on the bench workloads, untimed, for ncu. Sections (run in
    this order, each on the small_b256 layer unless noted):
      decode       2 intervals of 16 rssm_decode_step + rssm_flush
      fused        2 intervals with RSSM_FLAG_FUSED_FLUSH
      conv         32 rssm_conv_step
      spec         4 steps of rssm_verify (K = 4) + accept + flush (the last forced)
      conv_verify  4 steps of rssm_conv_verify (K = 4) + rssm_conv_accept
      split_bf16   bf16 + FP4 split: refresh(force), 16 decodes, refresh
      split_e4m3   the same with an e4m3 update copy
      shared_fp4   the shared FP4 control: refresh(force) of an fp32 + FP4
                   state to build the copy, 16 decodes, refresh
      prefill      rssm_prefill of a 512-token prompt"""
    import torch

    from hybrid_model_ssm_replay_b200 import rssm
    from hybrid_model_ssm_replay_b200.inputs import WORKLOADS, LayerShape, accept_lengths, make_inputs
    torch.cuda.set_device(0)
    wl = WORKLOADS["small_b256"]
    sh = wl["shape"]
    L = sh.interval
    inp = make_inputs(sh, L, wl["seed"], wl["in_dtype"], device="cuda")
    y = torch.empty((sh.batch, sh.nheads, sh.head_dim), device="cuda")
    mk = lambda **kw: rssm.make_desc(sh.batch, sh.nheads, sh.head_dim, sh.d_state, sh.ngroups, interval=L, **kw)

    def decodes(st):
        for t in range(L):
            rssm.rssm_decode_step(st, inp["x"][t], inp["B"][t], inp["C"][t], inp["dt"][t], inp["A"], inp["D"], y)

    def check(st):
        torch.cuda.synchronize()
        if rssm.rssm_get_error(st) != 0:
            raise RuntimeError("device error")

    for sec in sections:
        if sec in ("decode", "fused"):
            st = rssm.RssmState(mk(flags=rssm.RSSM_FLAG_FUSED_FLUSH if sec == "fused" else 0))
            st.ckpt.copy_(inp["ckpt"])
            for _ in range(2):
                decodes(st)
                if sec == "decode":
                    rssm.rssm_flush(st, inp["A"])
            check(st)
        elif sec == "conv":
            d = mk()
            h = inp["ckpt"].clone()
            for t in range(2 * L):
                rssm.rssm_conv_step(d, h, inp["x"][t % L], inp["B"][t % L], inp["C"][t % L], inp["dt"][t % L],
                                    inp["A"], inp["D"], y)
            torch.cuda.synchronize()
            del h
        elif sec in ("spec", "conv_verify"):
            K = 4
            ssh = LayerShape(sh.batch, sh.nheads, sh.head_dim, sh.d_state, sh.ngroups, L, K)
            si = make_inputs(ssh, 4, 3, wl["in_dtype"], device="cuda", ntok=K + 1)
            n = accept_lengths(4, sh.batch, K, 3, device="cuda")
            ds = mk(max_draft=K)
            ys = torch.empty((sh.batch, K + 1, sh.nheads, sh.head_dim), device="cuda")
            if sec == "spec":
                st = rssm.RssmState(ds)
                st.ckpt.copy_(si["ckpt"])
                for s_ in range(4):
                    rssm.rssm_verify(st, K, si["x"][s_], si["B"][s_], si["C"][s_], si["dt"][s_], si["A"], si["D"], ys)
                    rssm.rssm_accept(st, n[s_])
                    rssm.rssm_flush(st, si["A"], force=(s_ == 3))
                check(st)
            else:
                copies = torch.zeros((K + 1,) + tuple(si["ckpt"].shape), device="cuda")
                copies[0].copy_(si["ckpt"])
                cur = torch.zeros(sh.batch, dtype=torch.int32, device="cuda")
                for s_ in range(4):
                    rssm.rssm_conv_verify(ds, copies, cur, K, si["x"][s_], si["B"][s_], si["C"][s_], si["dt"][s_],
                                          si["A"], si["D"], ys)
                    rssm.rssm_conv_accept(ds, n[s_], cur, K)
                torch.cuda.synchronize()
                del copies
        elif sec in ("split_bf16", "split_e4m3"):
            upd = rssm.RSSM_BF16 if sec == "split_bf16" else rssm.RSSM_E4M3
            st = rssm.RssmState(mk(update_dtype=upd, out_copy=rssm.RSSM_OUTCOPY_FP4, seed=4))
            st.ckpt.copy_(inp["ckpt"].to(torch.bfloat16 if upd == rssm.RSSM_BF16 else torch.float8_e4m3fn)
                          .view(st.ckpt.dtype))
            rssm.rssm_lowprec_refresh(st, inp["A"], force=True)
            decodes(st)
            rssm.rssm_lowprec_refresh(st, inp["A"])
            check(st)
        elif sec == "shared_fp4":
            s0 = rssm.RssmState(mk(out_copy=rssm.RSSM_OUTCOPY_FP4))
            s0.ckpt.copy_(inp["ckpt"])
            rssm.rssm_lowprec_refresh(s0, inp["A"], force=True)
            st = rssm.RssmState(mk(update_dtype=rssm.RSSM_FP4, seed=4))
            st.ckpt.copy_(s0.out_codes)
            st.ckpt_scales.copy_(s0.out_scales)
            del s0
            decodes(st)
            rssm.rssm_lowprec_refresh(st, inp["A"])
            check(st)
        elif sec == "prefill":
            T0 = 512
            pi = make_inputs(sh, T0, wl["seed"] + 11, wl["in_dtype"], device="cuda")
            st = rssm.RssmState(mk())
            st.ckpt.copy_(pi["ckpt"])
            rssm.rssm_prefill(st, pi["x"], pi["B"], pi["dt"], pi["A"])
            check(st)
        else:
            raise ValueError(f"unknown profile section {sec!r}; choose from {PROFILE_SECTIONS}")
        st = None
        torch.cuda.empty_cache()
    print("profile run done:", ",".join(sections))


def main():
    args = parse_args()
    if args.profile:
        run_profile(PROFILE_SECTIONS if args.profile == "all" else args.profile.split(","))
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
