"""Benchmark of the LoReS decode step on B200.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
    (N > 1: launch with torch.distributed.run, one rank per GPU)

Workload (default): the 48-layer throughput sweep point at batch 256 per GPU, 32 heads,
d_k = d_v = 128, delta rule, scalar per-head decay, int8 state with one fp32 scale per
value row, stochastic rounding.  Each layer is its own handle with its own state and
inputs.  One step = one decode token through all 48 layers = 48 kernel launches.
Inputs are synthetic (seeded), resident in HBM; each layer's state (294 MB) exceeds the
126 MB L2, so no flush is needed between steps.

Metric: state updates per second, one update = one (sequence, head, layer, token).
Every rank runs its own batch (sequences are independent: weak scaling, no collective
on the data path); time is the max over ranks.

The JSON line also carries: roofline of the decode kernel against the measured HBM
copy bandwidth, an end-to-end number through the host-buffer C-ABI call, the clocks
seen during the timed region, and the CPU oracle's rate on a bounded sample.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "state-update steps/s (seq x head x token) and achieved HBM GB/s as % of B200 peak"
UNIT = "state-updates/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=256, help="sequences per GPU")
    ap.add_argument("--layers", type=int, default=48)
    ap.add_argument("--variant", default="int8", choices=["int8", "mixed", "fp32"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--e2e-streams", type=int, default=4,
                    help="streams the layers of the end-to-end run rotate over")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--formats", action="store_true",
                    help="launch time of one layer's step for every state format and mode "
                         "(batch --batch, 32 heads, 128 x 128), one JSON line")
    ap.add_argument("--sweep", action="store_true",
                    help="time every batch x state-format point of the 48-layer sweep (one GPU)")
    ap.add_argument("--sweep-variants", default="int8,mixed,fp32",
                    help="state formats of the sweep (comma list of int8, mixed, fp32)")
    ap.add_argument("--sweep-batches", default="1,16,64,256,1024",
                    help="batches of the sweep (comma list)")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------
# workload description and algorithmic bytes
# ---------------------------------------------------------------------------------------

def workload(args):
    from bit_recurrent_state_lores_b200 import synth
    return synth.workload("sweep", B=args.batch, layers=args.layers)


def layer_bits(args, wl, layer, policy=None):
    """Head bits of one layer.  Mixed precision: the 25 % slowest-decaying heads at 8 bits,
    by `policy` (the library's lores_assign_bits_by_decay on the GPU arm; the oracle's own
    copy of the rule on the CPU arm, which must not load the GPU library)."""
    from bit_recurrent_state_lores_b200 import synth
    if args.variant == "int8":
        return [8] * wl.H
    if args.variant == "fp32":
        return [32] * wl.H
    if policy is None:
        from bit_recurrent_state_lores_b200 import lores as L
        policy = L.lores_assign_bits_by_decay
    hp = synth.head_params(layer_workload(wl, layer))
    return [int(b) for b in policy(hp["mean_decay"], 0.25, 8, 4)]


def layer_workload(wl, layer):
    from bit_recurrent_state_lores_b200 import synth
    return synth.replace(wl, seed=wl.seed * 1000 + layer)


def tile_bytes(wl, bits):
    """Algorithmic bytes of one (sequence, head) update: codes + scales + q, k, v, alpha,
    beta read; codes + scales + o written (fp32 heads: the fp32 state, no scales)."""
    code = wl.d_v * wl.d_k * bits // 8
    scales = 0 if bits == 32 else wl.d_v * (wl.d_k // wl.G) * 4
    alpha = wl.d_k * 4 if wl.diag else 4
    read = code + scales + 2 * wl.d_k * 4 + wl.d_v * 4 + alpha + 4
    write = code + scales + wl.d_v * 4
    return read + write


def launch_bytes(wl, bits):
    return wl.B * sum(tile_bytes(wl, b) for b in bits)


def kernel_source_hash():
    """Hash of the decode-step kernels' source (csrc/lores_mma.cuh, csrc/lores_pair.cuh,
    csrc/lores_step.cuh, csrc/lores_device.cuh) with comments and blank space removed, so a
    change of wording leaves it unchanged."""
    import re
    h = hashlib.sha256()
    for f in ("lores_mma.cuh", "lores_pair.cuh", "lores_step.cuh", "lores_device.cuh"):
        src = open(os.path.join(ROOT, "bit_recurrent_state_lores_b200", "csrc", f)).read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def measured_peak():
    try:
        d = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(variant, batch):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    except Exception:
        return None
    e = d.get(f"{variant}-b{batch}")
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0, t1):
        rows = [r for (ts, r) in self.rows if t0 - 0.15 <= ts <= t1 + 0.15 and len(r) >= 10]
        note = "samples inside the timed region"
        if not rows:
            rows = [r for (ts, r) in self.rows if len(r) >= 10][-5:]
            note = "timed region shorter than the sampling period: nearest samples"
        if not rows:
            return None
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "power_w_max": max((num(r[4]) or 0) for r in rows),
                "note": note}


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline key)
# ---------------------------------------------------------------------------------------

def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def time_oracle_all_cores(wl, variant_bits, seconds, steps=None):
    """The oracle's decode step on every host core: the same C step (lo_tile_step) over the
    (sequence, head) tiles of the sample in an OpenMP loop (oracle/lores_oracle_omp.c).
    Sample: layer 0, enough sequences for at least four tiles per core, all heads, for
    successive steps until `seconds` elapse (or `steps` steps).  Returns (rate in
    state-updates/s, tiles done, elapsed s, threads used, description)."""
    import numpy as np
    from bit_recurrent_state_lores_b200 import synth
    from oracle import oracle as O

    cores = len(os.sched_getaffinity(0))
    nb = max(1, (4 * cores + wl.H - 1) // wl.H)
    wl0 = synth.replace(layer_workload(wl, 0), B=nb)
    hp = synth.head_params(wl0)
    cfgs = [O.TileCfg(wl0.d_k, wl0.d_v, group=wl0.G, bits=b, delta=wl0.delta, diag=wl0.diag)
            for b in variant_bits]
    n = nb * wl0.H
    cfg_of = [i % wl0.H for i in range(n)]
    states = [cfgs[c].zero_state() for c in cfg_of]
    done, elapsed, t, used = 0, 0.0, 0, 1
    while (steps is None and elapsed < seconds) or (steps is not None and t < steps):
        q, k, v, a, b = [x.numpy() for x in synth.step_inputs(wl0, t, hp, device="cpu")]
        sk = O.step_key(wl0.seed, t)
        keys = [O.tile_key(sk, i) for i in range(n)]
        t0 = time.perf_counter()
        _, _, used = O.batch_step(cfgs, cfg_of, [st[0] for st in states], [st[1] for st in states],
                                  q.reshape(n, -1), k.reshape(n, -1), v.reshape(n, -1),
                                  a.reshape(n, -1), b.reshape(n), keys)
        elapsed += time.perf_counter() - t0
        done += n
        t += 1
    desc = (f"oracle decode step on {used} threads (OpenMP over tiles): layer 0, batch {nb}, "
            f"{wl0.H} heads {wl0.d_v}x{wl0.d_k}, {t} steps ({done} (seq,head) updates, "
            f"{elapsed:.1f} s)")
    return done / elapsed, done, elapsed, used, desc


def time_oracle(wl, variant_bits, seconds, steps=None):
    """Run the oracle's decode step on a bounded sample of the workload: tiles of layer 0,
    batch 1, all heads, for successive steps until `seconds` elapse (or `steps` steps).
    Returns (rate in state-updates/s, tiles done, elapsed s, description)."""
    import numpy as np
    from bit_recurrent_state_lores_b200 import synth
    from oracle import oracle as O

    wl0 = synth.replace(layer_workload(wl, 0), B=1)
    hp = synth.head_params(wl0)
    cfgs = [O.TileCfg(wl0.d_k, wl0.d_v, group=wl0.G, bits=b, delta=wl0.delta, diag=wl0.diag)
            for b in variant_bits]
    states = [c.zero_state() for c in cfgs]
    done, elapsed, t = 0, 0.0, 0
    while (steps is None and elapsed < seconds) or (steps is not None and t < steps):
        q, k, v, a, b = [x.numpy() for x in synth.step_inputs(wl0, t, hp, device="cpu")]
        sk = O.step_key(wl0.seed, t)
        t0 = time.perf_counter()
        for hh, cfg in enumerate(cfgs):
            st, sc = states[hh]
            O.tile_step(cfg, st, sc, q[0, hh], k[0, hh], v[0, hh], a[0, hh], b[0, hh],
                        O.tile_key(sk, hh))
        elapsed += time.perf_counter() - t0
        done += len(cfgs)
        t += 1
    desc = (f"oracle decode step, single thread: layer 0, batch 1, {wl0.H} heads "
            f"{wl0.d_v}x{wl0.d_k}, {t} steps ({done} (seq,head) updates, {elapsed:.1f} s)")
    return done / elapsed, done, elapsed, desc


# ---------------------------------------------------------------------------------------
# ranks (one process per GPU; sequences are independent, so ranks share nothing)
# ---------------------------------------------------------------------------------------

def rank_seed(layer_seed, rank):
    """Rounding-dither seed of one layer on one rank: every rank decodes its own batch."""
    return (layer_seed << 8) + rank


def rank_input_step(rank, p):
    """Generator step index of input set p on `rank` (distinct inputs per rank)."""
    return 10_000 * rank + p


def reduce_max(x, device):
    """Max of a float over ranks (the job time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, batch, heads, layers, steps, max_ms):
    """Whole-job state updates per second: every rank's units over the slowest rank's time."""
    return world * batch * heads * layers * steps / (max_ms / 1e3)


# ---------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from bit_recurrent_state_lores_b200 import lores as L
    from bit_recurrent_state_lores_b200 import synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = workload(args)
    layers = []
    for layer in range(wl.layers):
        wll = layer_workload(wl, layer)
        bits = layer_bits(args, wl, layer)
        hp = synth.head_params(wll)
        h = L.lores_create(wl.B, wl.H, wl.d_k, wl.d_v, group_size=0, delta=wl.delta,
                           decay_diag=wl.diag, head_bits=bits, stochastic=1,
                           seed=rank_seed(wll.seed, rank), device=local_rank)
        inputs = [synth.step_inputs(wll, rank_input_step(rank, p), hp, device=dev)
                  for p in range(2)]
        o = torch.empty(wl.B, wl.H, wl.d_v, device=dev)
        layers.append((h, bits, inputs, o))
    bytes_per_launch = [launch_bytes(wl, bits) for (_, bits, _, _) in layers]
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream

    def one_step(step, ev=None):
        for li, (h, bits, inp, o) in enumerate(layers):
            q, k, v, a, b = inp[step & 1]
            if ev is not None:
                ev[li][0].record(stream)
            L.lores_decode_step(h, q, k, v, a, b, o, step, sptr)
            if ev is not None:
                ev[li][1].record(stream)

    for s in range(args.warmup):
        one_step(s)
    torch.cuda.synchronize(dev)
    for (h, _, _, _) in layers:
        st = L.lores_check_errors(h, sptr)
        assert st == L.LORES_OK, L.lores_status_string(st)

    clocks = None if args.no_clocks else ClockSampler(local_rank)
    if clocks:
        time.sleep(0.3)
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)]
            for _ in layers] for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    start.record(stream)
    for n in range(K):
        one_step(args.warmup + n, evs[n])
    end.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end)
    launch_ms = [evs[n][li][0].elapsed_time(evs[n][li][1]) for n in range(K)
                 for li in range(len(layers))]
    ms = reduce_max(ms, dev)
    clock_summary = None
    if clocks:
        time.sleep(0.2)
        clocks.stop()
        clock_summary = clocks.summary(t_wall0, t_wall1)
    for (h, _, _, _) in layers:
        st = L.lores_check_errors(h, sptr)
        assert st == L.LORES_OK, L.lores_status_string(st)

    value = job_rate(world, wl.B, wl.H, wl.layers, K, ms)
    kernel_label = {3: "decode_mma_kernel<128, scalar decay, delta, stochastic rounding> "
                       "(tensor-core contractions, one scale per row)",
                    1: "decode_pair_kernel<128, scalar decay, delta, stochastic rounding, "
                       "several scales per row> (two rows per lane)",
                    0: "decode_step_kernel<128, scalar decay, delta, stochastic rounding, "
                       "single token, plain>"}[L.lores_get_layout(layers[0][0], wl.H)[0].step_kernel]
    avg_launch_s = statistics.mean(launch_ms) / 1e3
    avg_bytes = statistics.mean(bytes_per_launch)
    peak, peak_kind = measured_peak()
    achieved = avg_bytes / avg_launch_s / 1e9
    traffic = profiled_traffic(args.variant, wl.B)

    # ---- end to end through the host-buffer C-ABI call --------------------------------
    e2e = None
    if not args.no_e2e:
        hin = []
        for (h, bits, inp, o) in layers:
            hin.append([x.cpu().pin_memory() for x in inp[0]] +
                       [torch.empty(wl.B, wl.H, wl.d_v).pin_memory()])
        Ke = max(1, args.e2e_steps)
        h2d = sum(sum(x.numel() * 4 for x in hi[:5]) for hi in hin)
        d2h = sum(hi[5].numel() * 4 for hi in hin)
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        # layers rotate over the streams, so the host<->device copies of the next layers
        # overlap the current layer's step; every copy and step is inside the timed region
        lanes = [torch.cuda.Stream(dev) for _ in range(max(1, args.e2e_streams))]

        def e2e_steps(n0, n):
            for ls in lanes:
                ls.wait_stream(stream)
            for t in range(n0, n0 + n):
                for li, (h, _, _, _) in enumerate(layers):
                    q, k, v, a, b, o = hin[li]
                    L.lores_decode_step_host_async(h, q, k, v, a, b, o, 1_000_000 + t,
                                                   lanes[li % len(lanes)].cuda_stream)
            for ls in lanes:
                stream.wait_stream(ls)

        # one untimed step first: the call allocates its device staging on first use
        e2e_steps(0, 1)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        s0.record(stream)
        e2e_steps(1, Ke)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        ems = reduce_max(s0.elapsed_time(s1), dev)

        # the same host<->device copies with no step between them: the bound the
        # end-to-end number works against (the PCIe link)
        dbuf = [[torch.empty_like(x, device=dev) for x in hi] for hi in hin]
        torch.cuda.synchronize(dev)
        s0.record(stream)
        for ls in lanes:
            ls.wait_stream(stream)
        for t in range(Ke):
            for li in range(len(layers)):
                with torch.cuda.stream(lanes[li % len(lanes)]):
                    for x, dx in zip(hin[li][:5], dbuf[li][:5]):
                        dx.copy_(x, non_blocking=True)
                    hin[li][5].copy_(dbuf[li][5], non_blocking=True)
        for ls in lanes:
            stream.wait_stream(ls)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        cms = reduce_max(s0.elapsed_time(s1), dev)
        del dbuf
        e2e = {"value": job_rate(world, wl.B, wl.H, wl.layers, Ke, ems), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": Ke,
               "ms_per_step": ems / Ke, "copies_only_ms_per_step": cms / Ke,
               "frac_of_copy_bound": cms / ems,
               "api": f"lores_decode_step_host_async (pinned host buffers; layers on "
                      f"{len(lanes)} streams, copies overlap steps)"}

    for (h, _, _, _) in layers:
        L.lores_destroy(h)

    result = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline(wl, layers[0][1], args.cpu_seconds)
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32+s8" if args.variant == "int8"
            else ("f32+s8/s4" if args.variant == "mixed" else "f32"),
            "data": "synthetic (seeded generators shaped like the 48-layer GDN-style sweep)",
            "config": {"workload": f"sweep-{args.variant}-b{wl.B}-L{wl.layers}",
                       "batch_per_gpu": wl.B, "heads": wl.H, "d_k": wl.d_k, "d_v": wl.d_v,
                       "layers": wl.layers, "delta": wl.delta, "decay": "scalar per head",
                       "group_size": wl.G, "rounding": "stochastic",
                       "parallelism": f"dp{world} (sequences; no collective)",
                       "l2": "state per layer > 126 MB L2 (inputs larger than L2; no flush)"},
            "gpu_launches": wl.layers * K,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_kind": f"{peak_kind} HBM copy bandwidth",
                         "kernel": kernel_label,
                         "bytes_per_launch": avg_bytes, "avg_launch_us": avg_launch_s * 1e6,
                         "frac_of_8TBps": achieved / 8000.0},
            "e2e": e2e, "cpu_baseline": cpu, "clocks": clock_summary,
        }
    return result


def cpu_baseline(wl, bits, seconds):
    """The oracle on the host: all cores (the reported value) and one core, half of
    `seconds` each."""
    rate, _, _, used, desc = time_oracle_all_cores(wl, bits, seconds / 2)
    rate1, _, _, desc1 = time_oracle(wl, bits, seconds / 2)
    return {"value": rate, "unit": UNIT, "cores": used, "kind": "oracle", "sample": desc,
            "cpu_model": cpu_model(), "affinity_cores": len(os.sched_getaffinity(0)),
            "one_core": {"value": rate1, "unit": UNIT, "cores": 1, "sample": desc1}}


def run_sweep(args):
    """Every point of the 48-layer throughput sweep on one GPU: batch in {1, 16, 64, 256,
    1024} x {int8, mixed int8/int4 (25% of heads at 8 bits by decay), fp32 state}.  Each
    point: `warmup` untimed steps, then `steps` timed steps (CUDA events around the whole
    step loop).  Points whose 48-layer state fits in the 126 MB L2 are flagged."""
    import torch
    from bit_recurrent_state_lores_b200 import lores as L
    from bit_recurrent_state_lores_b200 import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = measured_peak()
    points = []
    for variant in args.sweep_variants.split(","):
        for B in [int(x) for x in args.sweep_batches.split(",")]:
            a = argparse.Namespace(**vars(args))
            a.batch, a.variant = B, variant
            wl = workload(a)
            layers = []
            for layer in range(wl.layers):
                wll = layer_workload(wl, layer)
                bits = layer_bits(a, wl, layer)
                hp = synth.head_params(wll)
                h = L.lores_create(B, wl.H, wl.d_k, wl.d_v, delta=wl.delta, head_bits=bits,
                                   seed=wll.seed << 8, device=0)
                inp = synth.step_inputs(wll, 0, hp, device=dev)
                layers.append((h, bits, inp, torch.empty(B, wl.H, wl.d_v, device=dev)))
            sptr = torch.cuda.current_stream(dev).cuda_stream

            def step(t):
                for (h, _, (q, k, v, al, be), o) in layers:
                    L.lores_decode_step(h, q, k, v, al, be, o, t, sptr)

            for t in range(args.warmup):
                step(t)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(dev)
            e0.record()
            for t in range(args.steps):
                step(args.warmup + t)
            e1.record()
            torch.cuda.synchronize(dev)
            ms = e0.elapsed_time(e1)
            # the same steps replayed from one CUDA graph (the 48 launches and the device
            # step counter's advance captured once)
            dstep = torch.tensor([args.warmup + args.steps], dtype=torch.int64, device=dev)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                cs = torch.cuda.current_stream(dev).cuda_stream
                for (h, _, (q, k, v, al, be), o) in layers:
                    L.lores_decode_step_dev(h, q, k, v, al, be, o, dstep, cs)
                L.lores_advance_step(dstep, 1, cs)
            graph.replay()
            torch.cuda.synchronize(dev)
            e0.record()
            for t in range(args.steps):
                graph.replay()
            e1.record()
            torch.cuda.synchronize(dev)
            gms = e0.elapsed_time(e1)
            del graph
            for (h, _, _, _) in layers:
                assert L.lores_check_errors(h, sptr) == L.LORES_OK
            step_bytes = sum(launch_bytes(wl, bits) for (_, bits, _, _) in layers)
            state_bytes = sum(wl.B * sum(wl.d_v * wl.d_k * b // 8 for b in bits)
                              for (_, bits, _, _) in layers)
            gbs = step_bytes * args.steps / (ms / 1e3) / 1e9
            points.append({"variant": variant, "batch": B,
                           "value": wl.B * wl.H * wl.layers * args.steps / (ms / 1e3),
                           "unit": UNIT, "ms_per_step": ms / args.steps,
                           "algorithmic_GBps": gbs, "frac_of_peak": gbs / peak,
                           "graph_ms_per_step": gms / args.steps,
                           "graph_value": wl.B * wl.H * wl.layers * args.steps / (gms / 1e3),
                           "l2_resident": state_bytes < 126e6})
            for (h, _, _, _) in layers:
                L.lores_destroy(h)
            del layers
            torch.cuda.empty_cache()
    return {"metric": METRIC, "sweep": points, "peak_GBps": peak, "peak_kind": peak_kind,
            "steps": args.steps, "warmup": args.warmup,
            "config": {"workload": "sweep-48-layers", "heads": 32, "d_k": 128, "d_v": 128,
                       "delta": 1, "decay": "scalar per head", "group_size": 128,
                       "rounding": "stochastic"}}


def oracle_rate(c, wl, hp, seconds):
    """The oracle (one host core) on the same format: sequence 0's 32 tiles, step after
    step until `seconds` elapse; (seq, head) updates per second."""
    import numpy as np
    from bit_recurrent_state_lores_b200 import synth
    from oracle import oracle as O
    H = wl.H
    gb = c.get("group_bits")
    cfgs = [O.TileCfg(wl.d_k, wl.d_v, group=wl.d_k if c.get("axis") else c.get("G", wl.d_k),
                      bits=8 if gb else c["bits"][h], delta=c.get("delta", 1), diag=wl.diag,
                      stochastic=c.get("sr", 1), axis=c.get("axis", 0),
                      group_bits=gb[h] if gb else None, dense=c.get("dense", 0))
            for h in range(H)]
    states = [cf.zero_state() for cf in cfgs]
    done, elapsed, t = 0, 0.0, 0
    while elapsed < seconds or done == 0:
        q, k, v, a, b = [x.numpy() for x in synth.step_inputs(synth.replace(wl, B=1), t, hp)]
        sk = O.step_key(1, t)
        t0 = time.perf_counter()
        for h, cf in enumerate(cfgs):
            st, sc = states[h]
            O.tile_step(cf, st, sc, q[0, h], k[0, h], v[0, h], a[0, h], b[0, h], O.tile_key(sk, h))
        elapsed += time.perf_counter() - t0
        done += H
        t += 1
    return done / elapsed


def run_formats(args):
    """One layer (batch args.batch, 32 heads, 128 x 128, GDN-style inputs of step 0): the mean
    launch time of the decode step over `steps` launches after `warmup`, for every state
    format and mode the library has, with the algorithmic bytes of one launch.  Per-channel
    rows use 32-column groups with 8 bits on a quarter of the (head, group) pairs."""
    import torch
    from bit_recurrent_state_lores_b200 import lores as L
    from bit_recurrent_state_lores_b200 import synth

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = measured_peak()
    B, H, dk, dv = args.batch, 32, 128, 128
    mix = [8 if h % 4 == 0 else 4 for h in range(H)]
    chan = [[8 if (h + g) % 4 == 0 else 4 for g in range(4)] for h in range(H)]
    cases = [
        ("int8", dict(bits=[8] * H)), ("int8 round-to-nearest", dict(bits=[8] * H, sr=0)),
        ("int8 delta=0", dict(bits=[8] * H, delta=0)), ("int4", dict(bits=[4] * H)),
        ("mixed 25% int8 / int4 heads", dict(bits=mix)), ("fp32 reference state", dict(bits=[32] * H)),
        ("int6 one byte per code", dict(bits=[6] * H)), ("int6 dense planes", dict(bits=[6] * H, dense=1)),
        ("int5 dense planes", dict(bits=[5] * H, dense=1)), ("int7 dense planes", dict(bits=[7] * H, dense=1)),
        ("per-channel 8/4 bits, G = 32", dict(group_bits=chan, G=32)),
        ("key-axis scales, int8", dict(bits=[8] * H, axis=1)),
        ("key-axis scales, int4", dict(bits=[4] * H, axis=1)),
        ("int8, 8 tokens per call (per token)", dict(bits=[8] * H, tokens=8)),
    ]
    wl = synth.workload("sweep", B=B)
    hp = synth.head_params(wl)
    inp = synth.step_inputs(wl, 0, hp, device=dev)
    o = torch.empty(B, H, dv, device=dev)
    out = []
    for name, c in cases:
        gb = c.get("group_bits")
        h = L.lores_create(B, H, dk, dv, group_size=c.get("G", 0), delta=c.get("delta", 1),
                           head_bits=None if gb else c["bits"], stochastic=c.get("sr", 1),
                           seed=1, scale_axis=c.get("axis", 0), group_bits=gb,
                           dense_codes=c.get("dense", 0))
        lay, _ = L.lores_get_layout(h, H)
        T = c.get("tokens", 1)
        if T > 1:
            st = [torch.stack([x] * T).contiguous() for x in inp]
            oo = torch.empty(T, B, H, dv, device=dev)
            call = lambda t: L.lores_decode_steps(h, T, *st, oo, t * T)
        else:
            call = lambda t: L.lores_decode_step(h, *inp, o, t)
        for t in range(args.warmup):
            call(t)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for t in range(args.steps):
            call(args.warmup + t)
        e1.record()
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / args.steps / T
        assert L.lores_check_errors(h) == L.LORES_OK
        # algorithmic bytes per token: state read + written once per call, inputs per token
        vec = B * H * (2 * dk * 4 + 2 * dv * 4 + 8)  # q, k, v, alpha, beta read; o written
        state = 2 * (lay.code_bytes + lay.scale_count * 4)
        nbytes = state / T + vec
        orate = oracle_rate(c, wl, hp, args.cpu_seconds / len(cases))
        out.append({"format": name, "us_per_token": us, "state_bytes": lay.code_bytes + lay.scale_count * 4,
                    "algorithmic_GBps": nbytes / us / 1e3, "frac_of_peak": nbytes / us / 1e3 / peak,
                    "state_updates_per_s": B * H / (us * 1e-6),
                    "oracle_state_updates_per_s": orate})
        L.lores_destroy(h)
    return {"metric": "decode-step launch time per token by state format", "batch": B,
            "oracle": "one host core, sequence 0's 32 tiles, %.1f s per format" % (args.cpu_seconds / len(cases)),
            "heads": H, "d_k": dk, "d_v": dv, "steps": args.steps, "warmup": args.warmup,
            "peak_GBps": peak, "peak_kind": peak_kind, "formats": out}


def run_reference(args, rank, world):
    """The oracle as the reference arm: same metric, timed on every host core (the oracle's
    OpenMP tile loop); `warmup` untimed steps, then `steps` timed steps of the sample."""
    if rank != 0:
        return None
    from oracle import oracle as O
    wl = workload(args)
    bits = layer_bits(args, wl, 0, policy=O.assign_bits_by_decay)
    K = args.steps
    if args.warmup:
        time_oracle_all_cores(wl, bits, 0.0, steps=args.warmup)
    rate, done, el, used, desc = time_oracle_all_cores(wl, bits, 0.0, steps=K)
    return {
        "impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": None, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32+s8", "data": "synthetic",
        "config": {"workload": f"sweep-{args.variant}-b{wl.B}-L{wl.layers}",
                   "batch_per_gpu": wl.B, "heads": wl.H, "d_k": wl.d_k, "d_v": wl.d_v,
                   "layers": wl.layers},
        "cpu_baseline": {"value": rate, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": desc, "cpu_model": cpu_model(),
                         "affinity_cores": len(os.sched_getaffinity(0))},
        "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.sweep:
        print(json.dumps(run_sweep(args)), flush=True)
        return
    if args.formats:
        print(json.dumps(run_formats(args)), flush=True)
        return
    import torch
    import torch.distributed as dist
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
