#!/usr/bin/env python
"""Benchmark of the mHC Birkhoff projection (and, as extras, the residual mix).

Default workload: 131072 fp32 4x4 logit matrices per GPU -- the first half
N(0,1), the second half N(0,10^2) -- with an N(0,1) upstream gradient.  One
step is the method's hot path on that batch: the Newton forward (exact
projection) followed by the implicit backward.  ``value`` is matrices/s for
that fwd+bwd step, summed over all ranks (weak scaling: every rank owns its own
shard of matrices; the projection is independent per matrix, so no collective
runs on the data path).

Timing: W untimed warm-up steps; then, between a barrier and a device
synchronisation on both sides, exactly K steps run back to back -- captured
once in a CUDA graph and replayed between two CUDA events recorded on the
launching stream -- so that no host launch gap, event or cache flush sits
between the steps.  The inputs are larger than L2: the steps rotate over 16
replicas of the batch's inputs and outputs (512 MiB in all, four times the
126 MB L2), so every step reads inputs last touched 15 steps earlier and
evicted since.  The reported time is the K-step interval, maximised over
ranks.

Also reported: the end-to-end figure through the C ABI with pinned host buffers
(mhc_birkhoff_fwd_bwd_host: host -> device copies, kernels, device -> host
copies, pipelined, inside the timed region), the roofline of the dominant kernel
against the measured HBM copy bandwidth and the FP32 and MUFU issue peaks, the
fp64 CPU oracle timed on the host cores, SM clocks through NVML, and (unless
--no-extras) the 1M/4M/16M sweep, 20-iteration Sinkhorn, the layouts of the
Newton forward, and the residual-mix workloads.  The last key of the JSON line
is a compact ``targets`` summary of the fractions the extras measured.

``--impl reference`` times the fp64 CPU oracle (the reference implementation
of what the kernels compute) on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "4x4 projections/s (fwd, fwd+bwd) at 128K-16M; mix GB/s vs HBM peak"
UNIT = "matrices/s"
WORKLOAD = "birkhoff_fwd_bwd_131072"
N_MATS = 131072
BYTES_FWD = 128   # logits in, P out
BYTES_BWD = 192   # P and dP in, dlogits out
REPLICAS = 16     # rotating copies of the step's working set (16 x 32 MiB)
L2_FLUSH_BYTES = 512 << 20
FALLBACK_HBM_GBS = 6650.0
SM_COUNT = 148
FP32_LANES_PER_SM = 128   # FP32 lane operations per SM per clock
MUFU_LANES_PER_SM = 16    # SFU (MUFU) lane operations per SM per clock

# Algorithmic work of the Newton forward per matrix, counted from its
# arithmetic (FP32 add / multiply / fma lane operations, and MUFU operations:
# reciprocals and base-2 exponentials).  Start-up: two max shifts, 16
# compensated exponentials, one Sinkhorn round.  One iteration: column sums
# and error, the six Laplacian weights, damping, the grounded-Laplacian
# solve, three column factors, four row sums and the multiplicative update.
# The near-permutation step repeats an iteration's work on a cancellation-free
# gradient.  Line-search trials are not counted.
NEWTON_OPS = {"fp32_start": 168, "mufu_start": 24, "fp32_iter": 120, "mufu_iter": 10,
              "fp32_polish": 136, "mufu_polish": 10}


def parse():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--no-extras", action="store_true", help="skip the sweep and mix extras")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-oracle sample budget (Newton leg)")
    ap.add_argument("--e2e-pieces", type=int, default=4, help="pieces of the end-to-end host pipeline")
    ap.add_argument("--profile", default=None,
                    choices=["newton_fwd", "sinkhorn_fwd", "sinkhorn_bwd", "implicit_bwd", "mix_fwd", "mix_bwd",
                             "proj_mix_fwd", "proj_mix_bwd", "premap_fwd", "mix_post_bwd", "mix_premap_bwd",
                             "newton_fwd_n", "implicit_bwd_n", "composite_gain", "fwd_bwd_mapped"],
                    help="run one kernel --reps times on one case (for ncu) and exit")
    ap.add_argument("--method", default="newton", help="--profile newton_fwd: projection method")
    ap.add_argument("--layout", default="auto", choices=["auto", "thread", "lane_pair", "row_group"],
                    help="--profile newton_fwd: thread layout of the Newton forward")
    ap.add_argument("--size", type=int, default=1 << 22, help="--profile: matrices, or tokens T for the mix")
    ap.add_argument("--channels", type=int, default=4096, help="--profile: mix channels C")
    ap.add_argument("--dist", default="normal1", help="--profile: logit distribution")
    ap.add_argument("--n", type=int, default=8, help="--profile newton_fwd_n / implicit_bwd_n: matrix size")
    ap.add_argument("--reps", type=int, default=3)
    return ap.parse_args()


def headline_config(world):
    """The workload description both arms print."""
    return {"workload": WORKLOAD, "n_mats_per_gpu": N_MATS,
            "logits": "first half N(0,1), second half N(0,10^2), seed 2 (+7919*rank)",
            "step": "Newton fwd (to max|colsum-1|<1e-6, near-permutation relative-accuracy step) + implicit bwd",
            "l2": "inputs larger than L2: the steps rotate over %d replicas of the batch's inputs and outputs "
                  "(%d MiB, 4x the L2)" % (REPLICAS, REPLICAS * 32),
            "parallelism": "token-sharded replicas, no collective" if world > 1 else "single GPU"}


# ----------------------------------------------------------------- helpers


def measured_peaks(path=None):
    """HBM copy bandwidth (GB/s) from MEASURED_PEAKS.json and its source, or
    the fallback figure.  The entry may be a number or an object holding one
    (under "value", "gbs" or "burst")."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = json.load(f)["hbm_gbs"]
        if isinstance(v, dict):
            v = next(v[k] for k in ("value", "gbs", "burst") if k in v)
        v = float(v)
        if v > 0:
            return v, "measured"
    except Exception:
        pass
    return FALLBACK_HBM_GBS, "fallback"


# The sources the benchmark's two kernels (newton_fwd_kernel, implicit_bwd_kernel)
# are compiled from; the committed DRAM-traffic capture is used only while
# these are unchanged.
TRAFFIC_SOURCES = ("birkhoff_math.cuh", "launch.h", "mhc_birkhoff.cu", "pdl.cuh")


def csrc_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "doubly_stochastic_projection_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if the kernel
    sources have not changed since it was captured; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("csrc_hash") != csrc_hash():
        return None
    k = d.get("kernels", {}).get(kernel)
    return None if k is None else k.get("dram_bytes_per_launch_full_size")


class ClockSampler:
    """Polls SM clock and throttle reasons through NVML in a background thread."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index, period=0.002):
        self.samples = []
        self.period = period
        self._stop = threading.Event()
        self._on = threading.Event()
        self.max_mhz = None
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: clocks are reported as unknown
            self.err = repr(e)
        self.t = threading.Thread(target=self._run, daemon=True)
        if self.ok:
            self.t.start()

    def _run(self):
        while not self._stop.is_set():
            if self._on.is_set():
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
            time.sleep(self.period)

    def start(self):
        self._on.set()

    def pause(self):
        self._on.clear()

    def stop(self):
        self._stop.set()

    def summary(self, samples=None):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "unavailable"}
        s = list(self.samples if samples is None else samples)
        mhz = [m for m, _ in s]
        mask = 0
        for _, r in s:
            mask |= r
        reasons = [n for b, n in self.REASONS.items() if mask & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(s), "source": "nvml"}


# ----------------------------------------------------------------- distributed


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(x, pg, device):
    if pg is None:
        return x
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def barrier(pg, device):
    if pg is None:
        return
    import torch

    t = torch.zeros(1, device=device)
    pg.all_reduce(t)


# ----------------------------------------------------------------- CPU oracle


def _timed_loop(fn, seconds):
    done, t0 = 0, time.perf_counter()
    while True:
        done += fn()
        el = time.perf_counter() - t0
        if el >= seconds:
            return done, el


def cpu_oracle_rate(seconds, n_sample=16384):
    """The fp64 oracle, as it stands, on bounded samples of the benchmark's
    workloads: the headline Newton fwd + implicit bwd (matrices/s), the
    20-round Sinkhorn forward (matrices/s) and the residual mix forward and
    backward of both mix workloads (tokens/s); all host cores, and one core."""
    import numpy as np

    import oracle
    from doubly_stochastic_projection_b200 import inputs

    A, G = inputs.birkhoff_workload(WORKLOAD)
    half = n_sample // 2
    idx = np.concatenate([np.arange(half), N_MATS // 2 + np.arange(half)])
    A = A[idx].astype(np.float64)
    G = G[idx].astype(np.float64)
    oracle.newton(A[:64])
    cores = oracle.get_threads()

    def newton_step(a, g):
        P = oracle.newton(a, tol=1e-10, max_iter=200)
        oracle.implicit_bwd(P, g)
        return len(a)

    done, el = _timed_loop(lambda: newton_step(A, G), seconds)
    quarter = len(A) // 4
    A1 = np.concatenate([A[: quarter // 2], A[half: half + quarter // 2]])
    G1 = np.concatenate([G[: quarter // 2], G[half: half + quarter // 2]])
    sk_done, sk_el = _timed_loop(lambda: (oracle.sinkhorn(A, 20), len(A))[1], seconds / 4)
    mix = {}
    for name, T in (("mix_T16384_C4096", 256), ("mix_T65536_C7168", 128)):
        m = inputs.mix_workload(name, device="cpu", T=T)
        bits = lambda t: t.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
        X, F, dY = bits(m["X"]), bits(m["F"]), bits(m["dY"])
        H = oracle.newton(m["logits"].astype(np.float64))
        hp = m["h_post"].astype(np.float64)
        f_done, f_el = _timed_loop(lambda: (oracle.mix_fwd(X, H, hp, F), T)[1], seconds / 8)
        b_done, b_el = _timed_loop(lambda: (oracle.mix_bwd(X, H, hp, F, dY), T)[1], seconds / 8)
        mix[name] = {"fwd_tokens_per_s": f_done / f_el, "bwd_tokens_per_s": b_done / b_el,
                     "sample": "%d tokens (C = %d), fp64 over bf16-decoded inputs" % (T, m["C"])}
    oracle.set_threads(1)
    try:
        done1, el1 = _timed_loop(lambda: newton_step(A1, G1), seconds / 4)
        sk1, skel1 = _timed_loop(lambda: (oracle.sinkhorn(A1, 20), len(A1))[1], seconds / 8)
    finally:
        oracle.set_threads(cores)
    return {"value": done / el, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d matrices (%d of each half of the workload), Newton fwd to ||grad||<1e-10 + "
                      "implicit bwd in fp64, repeated for %.1f s" % (len(A), half, el),
            "single_core": {"value": done1 / el1, "unit": UNIT, "cores": 1,
                            "sample": "%d matrices (%d of each half), the same work, repeated for %.1f s"
                                      % (len(A1), len(A1) // 2, el1)},
            "sinkhorn20_fwd": {"value": sk_done / sk_el, "unit": UNIT, "cores": cores,
                               "single_core": sk1 / skel1,
                               "sample": "the same %d matrices, 20 Sinkhorn-Knopp rounds in fp64" % len(A)},
            "mix": {"unit": "tokens/s", "cores": cores, **mix}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    from doubly_stochastic_projection_b200 import inputs

    A, G = inputs.birkhoff_workload(WORKLOAD)
    A = A.astype(np.float64)
    G = G.astype(np.float64)
    # each step: a bounded sample of the workload, sized so that W + K steps
    # take about a minute at most
    total_budget = 60.0
    per_step = max(64, min(N_MATS, int(2.0e6 * total_budget / max(1, args.steps + args.warmup))))

    def step(i):
        s = (i * per_step) % (N_MATS - per_step + 1)
        P = oracle.newton(A[s:s + per_step], tol=1e-10, max_iter=200)
        oracle.implicit_bwd(P, G[s:s + per_step])

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = per_step * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(world),
        "cpu_baseline": {"kind": "oracle", "cores": oracle.get_threads(), "value": value, "unit": UNIT,
                         "sample": "%d consecutive matrices of the %d-matrix workload per step (the first rank's "
                                   "shard), fp64 Newton fwd to ||grad||<1e-10 + implicit bwd, on the host cores"
                                   % (per_step, N_MATS)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU timing


def event_time(fn, reps, stream, flush=None):
    """Mean device time (s) of fn() over reps, events on `stream`, flush outside."""
    import torch

    fn()  # warm-up: allocator and first-launch costs stay outside the events
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(reps):
        if flush is not None:
            flush()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1) * 1e-3
    return tot / reps


def capture(launches):
    """A CUDA graph of the given callables, launched in order (each enqueues
    work on the current stream)."""
    import torch

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in launches:
            f()
    return g


def upload(g, stream):
    """Uploads an instantiated graph to the device ahead of its first launch
    (cuGraphUpload), so that the first replay does not pay for it."""
    import ctypes

    import torch

    try:
        cu = ctypes.CDLL("libcuda.so.1")
        cu.cuGraphUpload.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        rc = cu.cuGraphUpload(ctypes.c_void_p(int(g.raw_cuda_graph_exec())), ctypes.c_void_p(stream.cuda_stream))
        torch.cuda.synchronize()
        return rc == 0
    except Exception:
        return False


def graph_time(g, stream, count):
    """Device time (s) of one replay of graph g, per unit of `count`."""
    import torch

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    e1.synchronize()
    return e0.elapsed_time(e1) * 1e-3 / count


def backtoback_time(make, n_rep, launches, stream):
    """Per-launch device time (s) of `launches` back-to-back launches, launch i
    working on replica i % n_rep (make(r) returns replica r's launcher), as
    one CUDA graph replayed once untimed and once timed."""
    reps = [make(r) for r in range(n_rep)]
    g = capture([reps[i % n_rep] for i in range(launches)])
    graph_time(g, stream, launches)
    t = graph_time(g, stream, launches)
    del g
    return t


# ----------------------------------------------------------------- rooflines


def projection_roofline(kname, n, t, hbm, mhz, its_mean=None, polished=None):
    """The three roofs of a projection launch of n matrices taking t seconds:
    HBM (algorithmic bytes), FP32 lane operations and MUFU operations (the
    method's executed work at the measured mean iteration count).  The bound
    is the roof with the longest minimum time."""
    f = (mhz or 1965) * 1e6
    fp32_peak = SM_COUNT * FP32_LANES_PER_SM * f
    mufu_peak = SM_COUNT * MUFU_LANES_PER_SM * f
    roofs = {}
    nbytes = (BYTES_FWD if "fwd" in kname else BYTES_BWD) * n
    roofs["hbm"] = {"min_us": nbytes / (hbm * 1e9) * 1e6, "achieved": nbytes / t / 1e9, "peak": hbm,
                    "unit": "GB/s", "work_per_launch": nbytes}
    if its_mean is not None:
        o = NEWTON_OPS
        fp = n * (o["fp32_start"] + o["fp32_iter"] * its_mean + o["fp32_polish"] * polished)
        mu = n * (o["mufu_start"] + o["mufu_iter"] * its_mean + o["mufu_polish"] * polished)
        roofs["fp32"] = {"min_us": fp / fp32_peak * 1e6, "achieved": fp / t / 1e12, "peak": fp32_peak / 1e12,
                         "unit": "T lane-ops/s", "work_per_launch": fp}
        roofs["mufu"] = {"min_us": mu / mufu_peak * 1e6, "achieved": mu / t / 1e12, "peak": mufu_peak / 1e12,
                         "unit": "T ops/s", "work_per_launch": mu}
    for r in roofs.values():
        r["frac"] = r["achieved"] / r["peak"]
    bound = max(roofs, key=lambda k: roofs[k]["min_us"])
    return bound, roofs


# ----------------------------------------------------------------- extras


def extras(dev, stream, flush, hbm, mhz, api, inputs):
    import torch

    out = {"sweep": [], "sinkhorn20": [], "mix": []}
    reps = 5
    for si, n in enumerate(inputs.SWEEP_SIZES):
        # back to back over replicas whose inputs and outputs together exceed
        # the L2 several times (as the headline step)
        R, L = (4, 16) if n <= (1 << 20) else (2, 8)
        for di, dist in enumerate(inputs.SWEEP_DISTS):
            A = torch.from_numpy(inputs.birkhoff_logits(n, dist, inputs.sweep_seed(si, di))).to(dev)
            G = torch.from_numpy(inputs.upstream_grad(n, inputs.sweep_seed(si, di) + 1000)).to(dev)
            As, Gs = [A] + [A.clone() for _ in range(R - 1)], [G] + [G.clone() for _ in range(R - 1)]
            Ps, Ds = [torch.empty_like(A) for _ in range(R)], [torch.empty_like(A) for _ in range(R)]
            for r in range(R):
                api.birkhoff_fwd(As[r], "newton", out=Ps[r])
            P, dl = Ps[0], Ds[0]
            _, its = api.birkhoff_fwd_diag(A)
            pol = near_permutation_fraction(P)
            tf = backtoback_time(lambda r: (lambda: api.birkhoff_fwd(As[r], "newton", out=Ds[r])), R, L, stream)
            ta = backtoback_time(lambda r: (lambda: api.birkhoff_fwd(As[r], "newton_absolute", out=Ds[r])), R, L,
                                 stream)
            tb = backtoback_time(lambda r: (lambda: api.birkhoff_bwd(Gs[r], P=Ps[r], out=Ds[r])), R, L, stream)
            itn = its.float()
            its_mean = float(itn.mean())
            bound, roofs = projection_roofline("newton_fwd", n, tf, hbm, mhz, its_mean, pol)
            out["sweep"].append({
                "n_mats": n, "dist": dist,
                "fwd_matrices_per_s": n / tf, "bwd_matrices_per_s": n / tb, "fwd_bwd_matrices_per_s": n / (tf + tb),
                "fwd_gbs": BYTES_FWD * n / tf / 1e9, "bwd_gbs": BYTES_BWD * n / tb / 1e9,
                "fwd_frac_hbm": BYTES_FWD * n / tf / 1e9 / hbm, "bwd_frac_hbm": BYTES_BWD * n / tb / 1e9 / hbm,
                "fwd_bwd_frac_hbm": (BYTES_FWD + BYTES_BWD) * n / (tf + tb) / 1e9 / hbm,
                "fwd_frac_fp32": roofs["fp32"]["frac"], "fwd_bound": bound,
                "fwd_frac_of_bound": roofs[bound]["frac"],
                "fwd_absolute_matrices_per_s": n / ta, "fwd_absolute_frac_hbm": BYTES_FWD * n / ta / 1e9 / hbm,
                "near_permutation_step_fraction": pol,
                "newton_iters_mean": its_mean, "newton_iters_max": int(its.max()),
                "newton_iters_warp_max_mean": float(itn.reshape(-1, 32).max(1).values.mean()),
            })
            if dist in ("normal1", "normal10"):
                ts = backtoback_time(lambda r: (lambda: api.birkhoff_fwd(As[r], "sinkhorn", 20, out=Ds[r])), R, L,
                                     stream)
                out["sinkhorn20"].append({"n_mats": n, "dist": dist, "fwd_matrices_per_s": n / ts,
                                          "fwd_gbs": BYTES_FWD * n / ts / 1e9,
                                          "fwd_frac_hbm": BYTES_FWD * n / ts / 1e9 / hbm})
            del A, G, As, Gs, Ps, Ds, P, dl, its
            torch.cuda.empty_cache()
    # Thread layouts of the Newton forward (thread per matrix, lane pair, row
    # group), back to back over rotating replicas
    out["layouts"] = []
    for n, dist, seed, R, L in ((131072, "halves_1_10", 2, 16, 32), (1 << 20, "normal1", 300, 4, 8),
                                (1 << 20, "normal10", 302, 4, 8)):
        A = torch.from_numpy(inputs.birkhoff_logits(n, dist, seed)).to(dev)
        As = [A.clone() for _ in range(R)]
        Ps = [torch.empty_like(A) for _ in range(R)]
        row = {"n_mats": n, "dist": dist}
        for lay in ("thread", "lane_pair", "row_group"):
            t = backtoback_time(lambda r, lay=lay: (lambda: api.birkhoff_fwd_layout(As[r], lay, "newton", out=Ps[r])),
                                R, L, stream)
            row[lay + "_us"] = t * 1e6
        out["layouts"].append(row)
        del A, As, Ps
        torch.cuda.empty_cache()
    # The pages' comparison (Birkhoff-acceleration summary, section 4): forward +
    # backward of the Newton projection with the implicit backward, against
    # 20-round Sinkhorn with the backward through the unrolled iteration.
    out["newton_vs_sinkhorn20_fwd_bwd"] = []
    for n, dist, seed in ((131072, "halves_1_10", 2), (1 << 20, "normal1", 300), (1 << 24, "normal1", 320),
                          (1 << 24, "normal10", 322)):
        A = torch.from_numpy(inputs.birkhoff_logits(n, dist, seed)).to(dev)
        G = torch.from_numpy(inputs.upstream_grad(n, seed + 1000)).to(dev)
        P = torch.empty_like(A)
        dl = torch.empty_like(A)
        t_nt = event_time(lambda: (api.birkhoff_fwd(A, "newton", out=P), api.birkhoff_bwd(G, P=P, out=dl)),
                          reps, stream, flush)
        t_sk = event_time(lambda: (api.birkhoff_fwd(A, "sinkhorn", 20, out=P), api.sinkhorn_bwd(G, A, 20, out=dl)),
                          reps, stream, flush)
        out["newton_vs_sinkhorn20_fwd_bwd"].append({
            "n_mats": n, "dist": dist, "newton_implicit_matrices_per_s": n / t_nt,
            "sinkhorn20_unrolled_matrices_per_s": n / t_sk, "speedup": t_sk / t_nt})
        del A, G, P, dl
        torch.cuda.empty_cache()
    for name in ("mix_T16384_C4096", "mix_T65536_C7168"):
        m = inputs.mix_workload(name, device=dev)
        T, C = m["T"], m["C"]
        X, F, dY = m["X"], m["F"], m["dY"]
        lg = torch.from_numpy(m["logits"]).to(dev)
        h = torch.from_numpy(m["h_post"]).to(dev)
        Y = torch.empty_like(X)
        H = api.birkhoff_fwd(lg, "newton")
        tf = event_time(lambda: api.residual_mix_fwd(X, H, h, F, out=Y), reps, stream, flush)
        tb = event_time(lambda: api.residual_mix_bwd(X, H, h, F, dY, need_dlogits=True), reps, stream, flush)
        tff = event_time(lambda: api.proj_mix_fwd(lg, h, X, F, out=Y, H_out=H), reps, stream, flush)
        tfb = event_time(lambda: api.proj_mix_bwd(H, h, X, F, dY), reps, stream, flush)
        bf = (18 * C + 80) * T
        bb = (28 * C + 160) * T
        bff = (18 * C + 128) * T          # + logits in, H out instead of H in
        bfb = (28 * C + 160) * T          # dH not written, dlogits written
        out["mix"].append({
            "workload": name, "T": T, "C": C,
            "fwd_gbs": bf / tf / 1e9, "fwd_frac_hbm": bf / tf / 1e9 / hbm, "fwd_tokens_per_s": T / tf,
            "bwd_gbs": bb / tb / 1e9, "bwd_frac_hbm": bb / tb / 1e9 / hbm, "bwd_tokens_per_s": T / tb,
            "fused_fwd_gbs": bff / tff / 1e9, "fused_fwd_frac_hbm": bff / tff / 1e9 / hbm,
            "fused_bwd_gbs": bfb / tfb / 1e9, "fused_bwd_frac_hbm": bfb / tfb / 1e9 / hbm,
            "fused_fwd_bwd_tokens_per_s": T / (tff + tfb),
        })
        # read map and the split backward (dF, dh_post first; then dX with the
        # pre-map's contribution, dH, dh_pre and dlogits in one pass over X)
        hpre = torch.from_numpy(inputs.birkhoff_logits(T, "normal1", 14)[:, 0, :].copy()).to(dev)
        dx_in = inputs.bf16_normal((T, C), 15, dev)
        x_in = torch.empty_like(F)
        tp = event_time(lambda: api.premap_fwd(X, hpre, out=x_in), reps, stream, flush)
        t_split = event_time(lambda: (api.mix_post_bwd(dY, F, h),
                                      api.mix_premap_bwd(X, H, hpre, dY, dx_in, need_dlogits=True)), reps, stream, flush)

        def unsplit():
            o = api.residual_mix_bwd(X, H, h, F, dY, need_dlogits=True)
            api.premap_bwd(X, hpre, dx_in, dX=o["dX"], accumulate=True)
        t_unsplit = event_time(unsplit, reps, stream, flush)
        bp = (10 * C + 16) * T
        out["mix"][-1].update({
            "premap_fwd_gbs": bp / tp / 1e9, "premap_fwd_frac_hbm": bp / tp / 1e9 / hbm,
            "split_bwd_with_premap_us": t_split * 1e6, "unsplit_bwd_then_premap_bwd_us": t_unsplit * 1e6,
            "split_bwd_gbs": (38 * C + 240) * T / t_split / 1e9,
            "split_bwd_frac_hbm": (38 * C + 240) * T / t_split / 1e9 / hbm})
        del m, X, F, dY, Y, H, lg, h, hpre, dx_in, x_in
        torch.cuda.empty_cache()
    # composite gain across 60 layers (the amax-gain drift of finite Sinkhorn)
    out["composite_gain"] = []
    Lg, Tg = 60, 65536
    for dist in ("normal1", "normal3", "normal10"):
        A = torch.from_numpy(inputs.birkhoff_logits(Lg * Tg, dist, 16)).to(dev)
        row = {"layers": Lg, "tokens": Tg, "dist": dist}
        for method, iters in (("newton", 0), ("sinkhorn", 20)):
            P = api.birkhoff_fwd(A, method, iters).reshape(Lg, Tg, 4, 4)
            _, gr, gc = api.composite_gain(P, need_M=False)
            tg = event_time(lambda: api.composite_gain(P, need_M=False), reps, stream, flush)
            row[method] = {"row_gain_max": float(gr.max()), "row_gain_p99": float(torch.quantile(gr, 0.99)),
                           "col_gain_max": float(gc.max())}
            row["kernel_gbs"] = Lg * Tg * 64 / tg / 1e9
            del P
        out["composite_gain"].append(row)
        del A
        torch.cuda.empty_cache()
    # general n (other expansion rates): Newton forward and implicit backward,
    # each n on about 256 MB of logits so that launch overhead does not dominate
    out["general_n"] = []
    for n in (2, 3, 6, 8):
        cnt = (1 << 26) // (n * n)
        A = torch.from_numpy(inputs.birkhoff_logits_n(cnt, n, 1.0, 20 + n)).to(dev)
        G = torch.from_numpy(inputs.birkhoff_logits_n(cnt, n, 1.0, 120 + n)).to(dev)
        P = torch.empty_like(A)
        dl = torch.empty_like(A)
        tf = event_time(lambda: api.birkhoff_fwd_n(A, "newton", out=P), reps, stream, flush)
        api.birkhoff_fwd_n(A, "newton", out=P)
        tb = event_time(lambda: api.birkhoff_bwd_n(G, P, out=dl), reps, stream, flush)
        fb, bb = 8 * n * n * cnt, 12 * n * n * cnt
        out["general_n"].append({
            "n": n, "n_mats": cnt, "dist": "normal1",
            "fwd_matrices_per_s": cnt / tf, "fwd_gbs": fb / tf / 1e9, "fwd_frac_hbm": fb / tf / 1e9 / hbm,
            "bwd_matrices_per_s": cnt / tb, "bwd_gbs": bb / tb / 1e9, "bwd_frac_hbm": bb / tb / 1e9 / hbm})
        del A, G, P, dl
        torch.cuda.empty_cache()
    return out


def near_permutation_fraction(P):
    """Fraction of matrices that take the near-permutation step (every row
    maximum above 0.6 and some row maximum above 0.995), from the output."""
    m = P.max(-1).values
    return float(((m.min(-1).values > 0.6) & (m.max(-1).values > 0.995)).float().mean())


def targets_summary(line, hbm):
    """The fractions the benchmark spec's targets are stated in, compactly, for the
    tail of the JSON line."""
    ex = line.get("extras") or {}
    t = {"hbm_peak_gbs": hbm}
    size_name = {1 << 20: "1M", 1 << 22: "4M", 1 << 24: "16M"}
    short = {"normal1": "n1", "normal3": "n3", "normal10": "n10", "near_identity": "nid", "near_permutation": "nperm"}
    fwd, fb, bound = {}, {}, {}
    for r in ex.get("sweep", []):
        k = "%s_%s" % (size_name.get(r["n_mats"], r["n_mats"]), short.get(r["dist"], r["dist"]))
        fwd[k] = round(r["fwd_frac_hbm"], 3)
        fb[k] = round(r["fwd_bwd_frac_hbm"], 3)
        bound[k] = "%s %.3f" % (r["fwd_bound"], r["fwd_frac_of_bound"])
    if fwd:
        t["newton_fwd_frac_hbm"] = fwd
        t["newton_fwd_frac_of_its_bound"] = bound
        t["newton_fwd_bwd_frac_hbm"] = fb
    sk = {"%s_%s" % (size_name.get(r["n_mats"], r["n_mats"]), short[r["dist"]]): round(r["fwd_frac_hbm"], 3)
          for r in ex.get("sinkhorn20", [])}
    if sk:
        t["sinkhorn20_fwd_frac_hbm"] = sk
    for r in ex.get("mix", []):
        t[r["workload"]] = {"fwd": round(r["fwd_frac_hbm"], 3), "bwd": round(r["bwd_frac_hbm"], 3),
                            "fused_fwd": round(r["fused_fwd_frac_hbm"], 3),
                            "fused_bwd": round(r["fused_bwd_frac_hbm"], 3),
                            "fused_fwd_bwd_tokens_per_s": round(r["fused_fwd_bwd_tokens_per_s"])}
    if ex.get("layouts"):
        t["newton_fwd_layout_us"] = {"%s_%s" % (size_name.get(r["n_mats"], r["n_mats"]), short.get(r["dist"], "halves")):
                                     [round(r["thread_us"], 1), round(r["lane_pair_us"], 1), round(r["row_group_us"], 1)]
                                     for r in ex["layouts"]}
        t["newton_fwd_layout_order"] = "thread, lane_pair, row_group"
    rl = line.get("roofline", {})
    t["headline"] = {"matrices_per_s": round(line["value"]), "e2e_matrices_per_s": round(line["e2e"]["value"]),
                     "dominant_kernel": rl.get("kernel"), "bound": rl.get("bound"),
                     "frac": round(rl.get("frac", 0.0), 3)}
    return t


# ----------------------------------------------------------------- GPU arm


def run_b200(args):
    import torch

    from doubly_stochastic_projection_b200 import api, inputs

    world, rank, local, pg = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    api.lib()
    stream = torch.cuda.current_stream(dev)
    hbm, hbm_src = measured_peaks()

    # this rank's shard: same distributions, its own seeds
    A_np, G_np = inputs.birkhoff_workload(WORKLOAD)
    if rank:
        A_np = inputs.birkhoff_logits(N_MATS, "halves_1_10", 2 + 7919 * rank)
        G_np = inputs.upstream_grad(N_MATS, 102 + 7919 * rank)
    A = torch.from_numpy(A_np).to(dev)
    G = torch.from_numpy(G_np).to(dev)
    # R replicas of inputs and outputs; step i works on replica i % R
    As = [A.clone() for _ in range(REPLICAS)]
    Gs = [G.clone() for _ in range(REPLICAS)]
    Ps = [torch.empty_like(A) for _ in range(REPLICAS)]
    dls = [torch.empty_like(A) for _ in range(REPLICAS)]
    P, dl = Ps[0], dls[0]

    def step_on(r):
        def f():
            api.birkhoff_fwd(As[r], "newton", out=Ps[r])
            api.birkhoff_bwd(Gs[r], P=Ps[r], out=dls[r])
        return f

    steps = [step_on(r) for r in range(REPLICAS)]
    K, W = args.steps, max(3, args.warmup)
    for i in range(W):
        steps[i % REPLICAS]()
    torch.cuda.synchronize()
    timed = capture([steps[(W + i) % REPLICAS] for i in range(K)])
    uploaded = upload(timed, stream)

    clocks = ClockSampler(local)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    barrier(pg, dev)
    torch.cuda.synchronize()
    clocks.start()
    e0.record(stream)
    timed.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks.pause()
    barrier(pg, dev)
    t_step = e0.elapsed_time(e1) * 1e-3
    t_max = max_over_ranks(t_step, pg, dev)
    value = world * N_MATS * K / t_max
    gpu_launches = 2 * K
    in_region = list(clocks.samples)
    clocks.samples = []
    # clocks: the timed region is usually shorter than NVML's update period, so
    # the same graph is replayed for about 0.3 s right after it while the
    # sampler runs; both sets of samples are reported
    window = []
    if clocks.ok:
        clocks.start()
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 0.3:
            timed.replay()
            torch.cuda.synchronize()
        clocks.pause()
        window = list(clocks.samples)
        clocks.samples = []
    del timed

    # per-kernel launch times, back to back over the replicas (the same
    # conditions as inside the step), and for comparison a launch isolated by
    # an L2 flush and its own events
    flush_buf = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.sum()

    nk = max(K, 64)
    t_fwd = backtoback_time(lambda r: (lambda: api.birkhoff_fwd(As[r], "newton", out=Ps[r])), REPLICAS, nk, stream)
    t_bwd = backtoback_time(lambda r: (lambda: api.birkhoff_bwd(Gs[r], P=Ps[r], out=dls[r])), REPLICAS, nk, stream)
    t_fwd_iso = event_time(lambda: api.birkhoff_fwd(A, "newton", out=P), 50, stream, flush)
    t_bwd_iso = event_time(lambda: api.birkhoff_bwd(G, P=P, out=dl), 50, stream, flush)
    t_step_iso = event_time(lambda: (api.birkhoff_fwd(A, "newton", out=P), api.birkhoff_bwd(G, P=P, out=dl)),
                            50, stream, flush)

    _, its = api.birkhoff_fwd_diag(A)
    itf = its.float()
    newton_iters = {"mean": float(itf.mean()), "max": int(its.max()),
                    "warp_max_mean": float(itf.reshape(-1, 32).max(1).values.mean())}
    api.birkhoff_fwd(A, "newton", out=P)
    polished = near_permutation_fraction(P)

    # end to end through the C ABI with pinned host buffers, copies or PCIe
    # traffic inside the timed region, two ways: the kernels reading and
    # writing the pinned buffers directly (zero-copy), and the copy pipeline
    # (pieces uploaded, computed and downloaded on overlapping streams)
    A_h = A.cpu().pin_memory()
    G_h = G.cpu().pin_memory()
    P_h = torch.empty_like(A_h).pin_memory()
    dl_h = torch.empty_like(A_h).pin_memory()
    work = [torch.empty_like(A) for _ in range(4)]
    pieces = args.e2e_pieces
    e2e_paths = {
        "mapped": lambda: api.birkhoff_fwd_bwd_mapped(A_h, G_h, P_h, dl_h, work[2]),
        "pipelined": lambda: api.birkhoff_fwd_bwd_host(A_h, G_h, P_h, dl_h, work, pieces),
    }
    e2e_steps = max(3, min(K, 50))
    e2e_t = {}
    for name, fn in e2e_paths.items():
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        tot = 0.0
        for i in range(e2e_steps):
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            fn()
            f1.record(stream)
            f1.synchronize()
            tot += f0.elapsed_time(f1) * 1e-3
        e2e_t[name] = max_over_ranks(tot / e2e_steps, pg, dev)
    # one more step of each with the device buffers poisoned first and the host
    # outputs zeroed: a kernel that read its inputs before they arrived would
    # leave NaN in the host results
    api.birkhoff_fwd(A, "newton", out=P)
    api.birkhoff_bwd(G, P=P, out=dl)
    matches = {}
    for name, fn in e2e_paths.items():
        for w in work:
            w.fill_(float("nan"))
        P_h.zero_()
        dl_h.zero_()
        fn()
        torch.cuda.synchronize()
        # (the zero-copy kernels inline the same solver into other kernels:
        # equal up to rounding)
        matches[name] = bool((P_h - P.cpu()).abs().max().item() <= 2e-6 and
                             (dl_h - dl.cpu()).abs().max().item() <= 1e-5 * dl.abs().max().item())
    nbytes = 2 * A.numel() * 4
    t_e2e = e2e_t["mapped"]
    e2e = {"value": world * N_MATS / t_e2e, "unit": UNIT, "h2d_bytes_per_step": nbytes,
           "d2h_bytes_per_step": nbytes, "ms_per_step": t_e2e * 1e3,
           "h2d_gbs": nbytes / t_e2e / 1e9, "d2h_gbs": nbytes / t_e2e / 1e9,
           "path": "mhc_birkhoff_fwd_bwd_mapped (C ABI): the Newton forward reads the logits from pinned host "
                   "memory and writes P to it (and to device memory), the implicit backward reads dP from and "
                   "writes dlogits to pinned host memory, over PCIe, inside the timed region",
           "matches_device_run": matches["mapped"],
           "pipelined": {"value": world * N_MATS / e2e_t["pipelined"], "ms_per_step": e2e_t["pipelined"] * 1e3,
                         "path": "mhc_birkhoff_fwd_bwd_host: copies in %d pieces on two copy streams, kernels on "
                                 "the launching stream" % pieces,
                         "matches_device_run": matches["pipelined"]}}

    # dominant kernel and its roofline
    mhz = clocks.max_mhz or 1965
    if t_fwd >= t_bwd:
        kname, kt = "newton_fwd_kernel", t_fwd
        bound, roofs = projection_roofline("newton_fwd", N_MATS, kt, hbm, mhz, newton_iters["mean"], polished)
        kt_iso = t_fwd_iso
    else:
        kname, kt = "implicit_bwd_kernel", t_bwd
        bound, roofs = projection_roofline("implicit_bwd", N_MATS, kt, hbm, mhz)
        kt_iso = t_bwd_iso
    top = roofs[bound]
    traffic = profiled_traffic(kname)
    roofline = {"bound": "hbm" if bound == "hbm" else "alu", "achieved": top["achieved"], "peak": top["peak"],
                "unit": top["unit"], "frac": top["frac"], "traffic": traffic, "kernel": kname,
                "peak_source": {"hbm": hbm_src, "fp32": "148 SMs x 128 lanes x %d MHz" % mhz,
                                "mufu": "148 SMs x 16 lanes x %d MHz" % mhz}[bound],
                "launch_us": kt * 1e6, "launch_us_isolated": kt_iso * 1e6,
                "roofs": {k: {"frac": v["frac"], "min_us": v["min_us"], "achieved": v["achieved"],
                              "peak": v["peak"], "unit": v["unit"], "work_per_launch": v["work_per_launch"]}
                          for k, v in roofs.items()},
                "note": "launch_us is the mean of back-to-back launches over the rotating replicas (a CUDA graph, "
                        "the conditions inside the step); launch_us_isolated is one launch between an L2 flush "
                        "and its own events, which adds the launch latency. hbm peak: the %s copy bandwidth; "
                        "fp32/mufu: the method's executed work at the measured mean of %.2f Newton iterations "
                        "(per-warp maximum %.2f, %.1f%% of matrices taking the near-permutation step)"
                        % (hbm_src, newton_iters["mean"], newton_iters["warp_max_mean"], 100 * polished)}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic", "config": headline_config(world),
        "fwd_matrices_per_s": world * N_MATS / max_over_ranks(t_fwd, pg, dev),
        "bwd_matrices_per_s": world * N_MATS / max_over_ranks(t_bwd, pg, dev),
        "step_us_isolated": t_step_iso * 1e6,
        "newton_iters": newton_iters, "near_permutation_step_fraction": polished,
        "e2e": e2e, "gpu_launches": gpu_launches, "roofline": roofline,
    }
    cl = clocks.summary(window + in_region)
    cl["samples_in_timed_region"] = len(in_region)
    cl["window"] = ("NVML every 2 ms during the timed region (%.2f ms) and over a 0.3 s replay of the same K-step "
                    "graph right after it" % (t_step * 1e3))
    line["config"]["graph_uploaded_before_timing"] = uploaded
    line["clocks"] = cl
    # the extras characterise one GPU; under torchrun the other ranks would sit in
    # the closing barrier meanwhile, so they run only when there is one rank
    if world == 1 and not args.no_extras:
        clocks.samples = []
        clocks.start()
        try:
            line["extras"] = extras(dev, stream, flush, hbm, mhz, api, inputs)
            tsk = event_time(lambda: api.birkhoff_fwd(A, "sinkhorn", 20, out=P), 20, stream, flush)
            line["extras"]["sinkhorn20_default_workload_matrices_per_s"] = N_MATS / tsk
        finally:
            clocks.pause()
        line["extras"]["clocks"] = clocks.summary()
    clocks.stop()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_rate(args.cpu_seconds)
    elif rank == 0:
        line["cpu_baseline"] = None
    line["targets"] = targets_summary(line, hbm)

    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        barrier(pg, dev)
        pg.destroy_process_group()
    return 0


def run_profile_case(args):
    """Run one kernel a few times on one case (for ncu captures)."""
    import torch

    from doubly_stochastic_projection_b200 import api, inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    k = args.profile
    if k == "composite_gain":
        L = 60
        A = torch.from_numpy(inputs.birkhoff_logits(L * args.size, args.dist, 16)).to(dev)
        P = api.birkhoff_fwd(A, "newton").reshape(L, args.size, 4, 4)
        fn = lambda: api.composite_gain(P, need_M=False)
        desc = {"layers": L, "tokens": args.size}
    elif k == "fwd_bwd_mapped":
        # the zero-copy host path: both kernels read and write pinned host buffers
        n = args.size
        if args.dist == "halves_1_10" and n == N_MATS:
            A_np, G_np = inputs.birkhoff_workload(WORKLOAD)
        else:
            A_np, G_np = inputs.birkhoff_logits(n, args.dist, 5), inputs.upstream_grad(n, 6)
        A_h = torch.from_numpy(A_np).pin_memory()
        G_h = torch.from_numpy(G_np).pin_memory()
        P_h = torch.empty_like(A_h).pin_memory()
        D_h = torch.empty_like(A_h).pin_memory()
        P_d = torch.empty(A_h.shape, device=dev)
        fn = lambda: api.birkhoff_fwd_bwd_mapped(A_h, G_h, P_h, D_h, P_d)
        desc = {"n_mats": n, "dist": args.dist, "path": "mhc_birkhoff_fwd_bwd_mapped"}
    elif k in ("newton_fwd_n", "implicit_bwd_n"):
        cnt = args.size
        A = torch.from_numpy(inputs.birkhoff_logits_n(cnt, args.n, 1.0, 20 + args.n)).to(dev)
        G = torch.from_numpy(inputs.birkhoff_logits_n(cnt, args.n, 1.0, 120 + args.n)).to(dev)
        P = api.birkhoff_fwd_n(A, "newton")
        out = torch.empty_like(A)
        fn = {"newton_fwd_n": lambda: api.birkhoff_fwd_n(A, "newton", out=out),
              "implicit_bwd_n": lambda: api.birkhoff_bwd_n(G, P, out=out)}[k]
        desc = {"n_mats": cnt, "n": args.n}
    elif k in ("newton_fwd", "sinkhorn_fwd", "sinkhorn_bwd", "implicit_bwd"):
        n = args.size
        if args.dist == "halves_1_10" and n == N_MATS:
            A_np, G_np = inputs.birkhoff_workload(WORKLOAD)
        else:
            A_np, G_np = inputs.birkhoff_logits(n, args.dist, 5), inputs.upstream_grad(n, 6)
        A = torch.from_numpy(A_np).to(dev)
        G = torch.from_numpy(G_np).to(dev)
        P = api.birkhoff_fwd(A, "newton")
        out = torch.empty_like(A)
        fn = {"newton_fwd": lambda: api.birkhoff_fwd_layout(A, args.layout, args.method, out=out),
              "sinkhorn_fwd": lambda: api.birkhoff_fwd(A, "sinkhorn", 20, out=out),
              "sinkhorn_bwd": lambda: api.sinkhorn_bwd(G, A, 20),
              "implicit_bwd": lambda: api.birkhoff_bwd(G, P=P, out=out)}[k]
        desc = {"n_mats": n, "dist": args.dist, "method": args.method, "layout": args.layout}
    else:
        m = inputs.mix_workload("mix_T16384_C4096", device=dev, T=args.size, C=args.channels)
        X, F, dY = m["X"], m["F"], m["dY"]
        lg = torch.from_numpy(m["logits"]).to(dev)
        h = torch.from_numpy(m["h_post"]).to(dev)
        H = api.birkhoff_fwd(lg, "newton")
        Y = torch.empty_like(X)
        hpre = torch.from_numpy(inputs.h_post(args.size, 17)).to(dev) - 1.0
        dx_in = dY[:, 0, :].contiguous()
        fn = {"mix_fwd": lambda: api.residual_mix_fwd(X, H, h, F, out=Y),
              "mix_bwd": lambda: api.residual_mix_bwd(X, H, h, F, dY, need_dlogits=True),
              "proj_mix_fwd": lambda: api.proj_mix_fwd(lg, h, X, F, out=Y, H_out=H),
              "proj_mix_bwd": lambda: api.proj_mix_bwd(H, h, X, F, dY),
              "premap_fwd": lambda: api.premap_fwd(X, hpre),
              "mix_post_bwd": lambda: api.mix_post_bwd(dY, F, h),
              "mix_premap_bwd": lambda: api.mix_premap_bwd(X, H, hpre, dY, dx_in)}[k]
        desc = {"T": args.size, "C": args.channels}
    for _ in range(args.reps):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"profile": k, "reps": args.reps, **desc}), flush=True)
    return 0


def main():
    args = parse()
    if args.profile:
        return run_profile_case(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_b200(args)


if __name__ == "__main__":
    sys.exit(main())
