"""Benchmark of the MoE-layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = one whole-layer forward (route -> permute -> gather -> expert FFN
up/down -> combine) over one batch of T tokens, through moe_forward with the
inputs resident in HBM. The default workload is the Mixtral-shaped layer
(T=4096, d=4096, E=8 experts, top-2, SwiGLU F=14336, bf16, dropless), synthetic
and seeded. Prints one JSON line (rank 0).

Timing: W untimed warm-up steps; then K steps bracketed by a barrier and a
device synchronize; between steps a 256 MB buffer is read to evict L2
(outside the timed events; a read, so the next step does not pay for writing
back the flush's own dirty lines), and each step streams ~2.8 GB of expert
weights, far more than the 126 MB L2; every step is timed with CUDA events recorded on
the launching stream by the library between its stages; the value is the
whole-job token rate, max over ranks of the summed step time. N > 1 runs N
independent replicas (one per GPU, each its own T tokens): the layer has no
cross-GPU exchange step, so there is no data-path collective (weak scaling).

--impl reference runs the CPU oracle (numpy float64) on the host cores as the
reference arm, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workloads import CONFIGS, make_inputs  # noqa: E402

METRIC = "MoE-layer fwd tokens/s on 1 B200 (Mixtral 8e top-2 bf16)"
UNIT = "tokens/s"
STAGES = ["route", "permute", "gather", "ffn_up", "ffn_down", "combine"]
FLUSH_BYTES = 256 << 20
SPEC_HBM_GBS = 8000.0       # nominal B200 HBM3e, for the spec-relative fractions
SPEC_BF16_TFLOPS = 2250.0   # nominal dense bf16
GEMM_SRC = os.path.join(ROOT, "mixture_experts_routing_route_b200", "csrc", "gemm_sm100.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--config", default="mixtral", choices=sorted(CONFIGS))
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-per-config", action="store_true",
                   help="skip the bounded runs of the other workloads (the per_config key)")
    p.add_argument("--binned", action="store_true",
                   help="padded-binned [E, C, hs] layout (capacity_factor 0: C = the largest count)")
    p.add_argument("--gather-in-gemm", action="store_true",
                   help="bf16: gather x rows inside the up projection (tile::gather4) instead of "
                        "the gather kernel")
    p.add_argument("--combine-in-gemm", action="store_true",
                   help="bf16, k = 1: the combine in the down projection's epilogue (no combine "
                        "kernel, no y_perm)")
    p.add_argument("--k", type=int, default=None, help="override top-k (e.g. 1 for --combine-in-gemm)")
    p.add_argument("--router-backward", action="store_true",
                   help="time the router backward (moe_route_backward: d_logits, dx, dWg) on the "
                        "workload's router instead of the layer forward; one GPU")
    p.add_argument("--T", type=int, default=None, help="override T (reduced case for profiling)")
    p.add_argument("--E", type=int, default=None, help="override E (reduced case for profiling)")
    p.add_argument("--F", type=int, default=None, help="override F (reduced case for profiling)")
    return p.parse_args()


def shape_of(args):
    sh = CONFIGS[args.config]
    if args.T is not None or args.E is not None or args.F is not None:
        sh = sh.with_(T=args.T or sh.T, E=args.E or sh.E, F=args.F or sh.F,
                      name=f"{sh.name}_T{args.T or sh.T}_E{args.E or sh.E}_F{args.F or sh.F}")
    if args.k is not None and args.k != sh.k:
        sh = sh.with_(k=args.k, name=f"{sh.name}_k{args.k}")
    return sh


def arm_config(sh, args, world):
    """The JSON line's config, the same in both arms for the same flags."""
    return dict(workload_config(sh), parallelism=f"replicas x{world}" if world > 1 else "1 GPU",
                **({"gather": "in the up projection (tile::gather4)"} if args.gather_in_gemm else {}),
                **({"layout": "binned [E, C, d]"} if args.binned else {}),
                **({"combine": "in the down projection's epilogue"} if args.combine_in_gemm else {}))


def workload_config(sh):
    return {"workload": f"{sh.name}: T={sh.T} d={sh.d} E={sh.E} top-{sh.k} {sh.act} F={sh.F} "
                        f"{sh.dtype}" + (f" cf={sh.cf}" if sh.cf > 0 else " dropless")
                        + ("" if sh.bias == "none" else f" bias={sh.bias}"),
            "T": sh.T, "d": sh.d, "E": sh.E, "k": sh.k, "F": sh.F, "act": sh.act,
            "capacity_factor": sh.cf, "global_batch_tokens": sh.T,
            "l2": "256 MB buffer read between timed steps (outside the events); per-step working set > L2"}


# ------------------------------------------------------------------ roofline
def algorithmic(sh, counts_kept, bucket_rows=None, combine_in_gemm=False):
    """Algorithmic flops and bytes per stage for one forward (no re-reads).

    R = kept rows, E_act = experts with R_e > 0, b = element bytes.
      route    bytes T*d*b + d*E*b + T*k*8 (x once, Wg once, idx + w out)
      permute  bytes S*4 + S*(4+4+4+1) (idx in; sorted_slot, slot_to_row,
               row_slot, drop out)
      gather   bytes T_used*d*b + R*d*b (each token read once, rows written);
               binned: + the bucket's padding rows written as zeros (E*C rows
               in all); with --gather-in-gemm no separate stage
      ffn_up   flops 2*R*d*F*(2 SwiGLU | 1 GELU); bytes weights of active
               experts + R*d*b (A rows: x_perm, or x gathered) + R*F*b
      ffn_down flops 2*R*F*d; bytes E_act*F*d*b + R*F*b + R*d*b
      combine  bytes R*d*b + S*8 + T*d*b; with --combine-in-gemm no separate
               stage (the down projection writes its R rows to out; the
               gather kernel also zeroes the T - R rows of dropped tokens, k = 1)
    """
    b = 2 if sh.dtype == "bf16" else 4
    T, d, E, k, F = sh.T, sh.d, sh.E, sh.k, sh.F
    S = T * k
    R = int(sum(counts_kept))
    e_act = int(sum(1 for c in counts_kept if c > 0))
    nup = 2 if sh.act == "swiglu" else 1
    zeroed = (T - R) if combine_in_gemm else 0
    return {
        "route": {"bytes": T * d * b + d * E * b + S * 8},
        "permute": {"bytes": S * 4 + S * 13},
        "gather": {"bytes": min(T, R) * d * b + (bucket_rows if bucket_rows is not None else R) * d * b
                   + zeroed * d * b},
        "ffn_up": {"flops": 2 * R * d * F * nup,
                   "bytes": e_act * d * F * b * nup + R * d * b + R * F * b},
        "ffn_down": {"flops": 2 * R * F * d, "bytes": e_act * F * d * b + R * F * b + R * d * b},
        "combine": {"bytes": R * d * b + S * 8 + T * d * b},
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def file_hash(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, or None when the
    kernel source changed since that capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    cur = file_hash(GEMM_SRC)
    with open(TRAFFIC_FILE) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel \
                    and parts[1] == workload and parts[3] == cur:
                return float(parts[2])
    return None


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpus):
        self.gpus = gpus
        self.proc = None
        self.path = os.path.join("/tmp", f"moe_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", ",".join(str(g) for g in self.gpus)],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        # nvidia-smi takes a moment to start: wait (bounded) for its first
        # sample so that the samples cover the timed region.
        t0 = time.time()
        while time.time() - t0 < 5.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                c = [x.strip() for x in line.split(",")]
                if len(c) < 9:
                    continue
                try:
                    sm.append(float(c[1]))
                    smax.append(float(c[2]))
                    power.append(float(c[3]))
                except ValueError:
                    continue
                for n, v in zip(names, c[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        hi = max(sm)
        load = [s for s, p in zip(sm, power) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(load), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "sm_mhz_peak_seen": hi}

    @staticmethod
    def rejected(c):
        bad = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
        if any(r in bad for r in c.get("reasons", [])):
            return True
        if c.get("sm_mhz") and c.get("sm_max_mhz") and not c["reasons"] and \
                c["sm_mhz"] < 0.6 * c["sm_max_mhz"]:
            return True
        return False


# ------------------------------------------------------------------ distributed
def dist_setup(n):
    if n <= 1:
        return 0, 1, 0
    import torch.distributed as dist
    from datetime import timedelta
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", n))
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def reduce_max(v, world):
    """Max over ranks of a per-rank time (the job's time is the slowest rank's)."""
    if world <= 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(sh, rank):
    """Token seed of replica `rank`: rank 0 uses the workload's own seed, the
    others draw their own tokens (the weights are the same on every rank)."""
    return sh.seed if rank == 0 else sh.seed + 7919 * rank


def job_value(tokens_per_rank, steps, world, total_ms_max):
    """Whole-job token rate: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank * steps / (total_ms_max * 1e-3)


# ------------------------------------------------------------------ end to end
def measure_e2e(layer, inp, sh, args, world, elem):
    """Tokens/s through the host-buffer entry point, as a serving loop runs
    it: each step copies its x from pinned host memory, runs the layer and
    copies out and aux back; two streams and two buffer sets alternate, so
    step i+1's copies and launches overlap step i's compute, and the host
    reads step i's result (aux) before it reuses that step's buffers. The
    timed region (CUDA events) runs from the first step's input copy to the
    last step's result copy. No L2 flush is needed: every step streams the
    experts' weights (several GB) through the 126 MB L2."""
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    xs = [inp.x.pin_memory(), inp.x.clone().pin_memory()]
    outs = [torch.empty(sh.T, sh.d, dtype=inp.x.dtype).pin_memory() for _ in range(2)]
    auxs = [torch.empty(1, dtype=torch.float32).pin_memory() for _ in range(2)]
    done = [None, None]

    def step(i):
        j = i % 2
        if done[j] is not None:
            done[j].synchronize()
            if not (auxs[j].item() >= 0.0):  # the host reads the step's result
                raise RuntimeError("aux loss not produced")
        layer.forward_host(xs[j], outs[j], auxs[j], stream=streams[j], slot=j)
        ev = torch.cuda.Event()
        ev.record(streams[j])
        done[j] = ev

    for i in range(max(2, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    done[:] = [None, None]
    barrier(world)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(streams[0])
    streams[1].wait_event(start)
    for i in range(args.steps):
        step(i)
    for j in range(2):
        if done[j] is not None:
            streams[0].wait_event(done[j])
    end.record(streams[0])
    end.synchronize()
    from mixture_experts_routing_route_b200 import _abi as abi
    for j in range(2):
        if abi.moe_get_device_error(layer.workspace(sh.T, host_io=True, slot=j)) != 0:
            raise RuntimeError("device error word set during the end-to-end steps")
    e_total = reduce_max(start.elapsed_time(end), world)
    return {"value": job_value(sh.T, args.steps, world, e_total), "unit": UNIT,
            "h2d_bytes_per_step": sh.T * sh.d * elem,
            "d2h_bytes_per_step": sh.T * sh.d * elem + 4,
            "api": "MoeLayer.forward_host -> moe_forward_host (pinned host x/out/aux; two "
                   "streams alternate, copies of one step overlap the compute of the next)"}


# ------------------------------------------------------------------ CPU oracle
def oracle_sample_run(inp, tokens, w64):
    """One oracle forward over a sample of the workload's tokens."""
    from oracle import moe_oracle as O
    sh = inp.shape
    x = inp.x[:tokens].float().numpy()
    bias = None if inp.bias is None else inp.bias.numpy()
    t0 = time.perf_counter()
    O.forward(x, inp.wg.float().numpy(), bias, w64["w1"], w64["w3"], w64["w2"], sh.k, sh.act, sh.cf)
    return time.perf_counter() - t0


def weights_f64(inp):
    cvt = lambda w: None if w is None else [w[e].to(torch.float64).numpy() for e in range(w.shape[0])]  # noqa: E731
    return {"w1": cvt(inp.w1), "w3": cvt(inp.w3), "w2": cvt(inp.w2)}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=None)
        if n:
            return int(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args):
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return 0
    sh = shape_of(args)
    inp = make_inputs(sh)
    w64 = weights_f64(inp)
    tokens = min(64, sh.T)
    for _ in range(args.warmup):
        oracle_sample_run(inp, tokens, w64)
    tot = 0.0
    for _ in range(args.steps):
        tot += oracle_sample_run(inp, tokens, w64)
    value = tokens * args.steps / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)", "config": arm_config(sh, args, max(1, args.gpus)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "cpu_model": cpu_model(),
                         "kind": "oracle",
                         "sample": f"{tokens} of the workload's {sh.T} tokens per step, whole "
                                   f"layer (route, permute, gather, expert FFN, combine) in "
                                   f"numpy float64"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline(sh, inp):
    """The oracle's whole layer over up to 4096 of the workload's tokens (all
    of the Mixtral workload's), repeated until at least 10 s of CPU work
    (at most 8 passes)."""
    w64 = weights_f64(inp)
    tokens = min(4096, sh.T)
    oracle_sample_run(inp, min(16, sh.T), w64)  # first touch of the converted weights
    t, reps = 0.0, 0
    while reps < 8 and (reps == 0 or t < 10.0):
        t += oracle_sample_run(inp, tokens, w64)
        reps += 1
    return {"value": tokens * reps / t, "unit": UNIT, "cores": cpu_threads(), "cpu_model": cpu_model(),
            "kind": "oracle",
            "sample": f"{reps} oracle forward(s) (numpy float64) of the first {tokens} of {sh.T} "
                      f"tokens of the same workload, {t:.1f} s in all"}


# ------------------------------------------------------------------ main
def run_router_backward(args):
    """The router backward on the workload's router (x [T, d], Wg [d, E]):
    inputs from one forward (moe_route_train), upstream gradients drawn from
    a seed (d_w ~ N(0, 1), d_aux = 0.01, d_z = 0.001), L2 evicted between
    steps. Algorithmic bytes per step: probs, logits, picks, weights and d_w
    read, d_logits written; x read once for dWg, dx written once, Wg read and
    dWg written (T*E*4*3 + T*k*12 + 2*T*d*b + d*E*(b+4))."""
    from mixture_experts_routing_route_b200 import _abi as abi
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    sh = shape_of(args)
    inp = make_inputs(sh)
    T, d, E, k = sh.T, sh.d, sh.E, sh.k
    x, wg = inp.x.to(dev), inp.wg.to(dev)
    bias = None if inp.bias is None else inp.bias.to(dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    aux = torch.empty(1, dtype=torch.float32, device=dev)
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    probs = torch.empty(T, E, dtype=torch.float32, device=dev)
    ws = torch.empty(max(abi.moe_route_workspace_size(T, d, E), 256), dtype=torch.uint8, device=dev)
    abi.moe_workspace_init(ws)
    abi.moe_route_train(x, wg, bias, None, T, d, E, k, idx, w, aux, None, logits, probs, ws)
    g = torch.from_numpy(np.random.default_rng(7).standard_normal((T, k)).astype(np.float32)).to(dev)
    d_logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    dx = torch.empty(T, d, dtype=x.dtype, device=dev)
    d_wg = torch.empty(d, E, dtype=torch.float32, device=dev)
    bws = torch.empty(max(abi.moe_route_backward_workspace_size(T, d, E), 256), dtype=torch.uint8,
                      device=dev)
    abi.moe_workspace_init(bws)
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    sink = torch.zeros(1, dtype=torch.int64, device=dev)
    step = lambda: abi.moe_route_backward(x, wg, T, d, E, k, probs, logits, idx, w, g, 0.01, 0.001, 1.0,
                                          d_logits, dx, d_wg, bws)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if abi.moe_get_device_error(bws) != 0:
        raise RuntimeError("device error word set during warm-up")
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    n0 = abi.moe_kernel_launches()
    # a spin on the GPU first, so that the host enqueues every step before the
    # GPU reaches it: the events then bracket device time only
    torch.cuda._sleep(int(2e5) * args.steps)
    for a, b in evs:
        torch.sum(flush, dim=0, dtype=torch.int64, out=sink[0])
        a.record()
        step()
        b.record()
    n1 = abi.moe_kernel_launches()
    torch.cuda.synchronize()
    if abi.moe_get_device_error(bws) != 0:
        raise RuntimeError("device error word set during the timed calls")
    times = sorted(a.elapsed_time(b) for a, b in evs)
    ms = statistics.median(times)
    eb = x.element_size()
    byts = T * E * 4 * 3 + T * k * 12 + 2 * T * d * eb + d * E * (eb + 4)
    peaks = load_peaks()
    gbs = byts / (ms * 1e-3) / 1e9
    line = {"metric": "router backward tokens/s (d_logits, dx, dWg)", "value": T / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "dtype": sh.dtype,
            "data": "synthetic (seeded)", "config": workload_config(sh),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_per_step": byts,
                         "timing": "median of CUDA events around each call (all calls enqueued "
                                   "behind a GPU spin), L2 evicted between"},
            "gpu_launches": n1 - n0}
    print(json.dumps(line), flush=True)
    return 0


PER_CONFIG = ("tiny_fp32", "fine_grained", "capacity_skew", "long_skewed", "long_skewed_cf")
PER_CONFIG_STEPS = 20


def stage_roofline(sh, stage_ms, alg, peaks, tc_peak, args):
    """Per-stage time, achieved GB/s and TFLOP/s and their fractions of the
    measured peaks (and of the spec figures)."""
    roof = {}
    for s_ in STAGES:
        t = stage_ms[s_] * 1e-3
        a = alg[s_]
        if s_ == "gather" and args.gather_in_gemm and sh.dtype == "bf16" and not args.combine_in_gemm:
            roof[s_] = {"us": stage_ms[s_] * 1e3, "fused_into": "ffn_up (tile::gather4 A loads)"}
            continue
        if s_ == "combine" and args.combine_in_gemm:
            roof[s_] = {"us": stage_ms[s_] * 1e3, "fused_into": "ffn_down (epilogue)"}
            continue
        r = {"us": stage_ms[s_] * 1e3, "GB_s": a["bytes"] / t / 1e9 if t > 0 else None}
        r["hbm_frac"] = r["GB_s"] / peaks["hbm_gbs"] if r["GB_s"] else None
        r["hbm_frac_spec"] = r["GB_s"] / SPEC_HBM_GBS if r["GB_s"] else None
        if "flops" in a:
            r["TFLOP_s"] = a["flops"] / t / 1e12 if t > 0 else None
            r["tensor_frac"] = r["TFLOP_s"] / tc_peak if r["TFLOP_s"] and sh.dtype == "bf16" else None
            r["tensor_frac_spec"] = r["TFLOP_s"] / SPEC_BF16_TFLOPS if r["TFLOP_s"] else None
        roof[s_] = r
    return roof


def dispatch_span_of(stage_ms, alg, peaks):
    """Route + permute + gather judged as one span against its bytes (the
    permute alone moves < 1 MB and is latency-bound)."""
    span_us = sum(stage_ms[s_] for s_ in ("route", "permute", "gather")) * 1e3
    span_bytes = sum(alg[s_]["bytes"] for s_ in ("route", "permute", "gather"))
    gbs = span_bytes / (span_us * 1e-6) / 1e9 if span_us > 0 else None
    return {"us": span_us, "bytes": span_bytes,
            "hbm_frac": gbs / peaks["hbm_gbs"] if gbs else None,
            "hbm_frac_spec": gbs / SPEC_HBM_GBS if gbs else None}


class LayerRun:
    """One workload's layer on the device with its input, output and the L2
    eviction buffer; timed_steps() runs the timed loop, stage_times() the
    separate per-stage pass."""

    def __init__(self, sh, inp, dev, args, flush):
        from mixture_experts_routing_route_b200 import MoeLayer
        self.sh, self.args = sh, args
        self.x = inp.x.to(dev)
        self.layer = MoeLayer(inp.wg.to(dev), inp.w1.to(dev), inp.w2.to(dev),
                              w3=None if inp.w3 is None else inp.w3.to(dev),
                              bias=None if inp.bias is None else inp.bias.to(dev),
                              k=sh.k, act=sh.act, capacity_factor=sh.cf,
                              gather_in_gemm=args.gather_in_gemm, binned=args.binned,
                              combine_in_gemm=args.combine_in_gemm)
        self.out = torch.empty(sh.T, sh.d, dtype=self.x.dtype, device=dev)
        self.aux = torch.empty(1, dtype=torch.float32, device=dev)
        self.flush = flush
        self.sink = torch.zeros(1, dtype=torch.int64, device=dev)

    def evict_l2(self):
        torch.sum(self.flush, dim=0, dtype=torch.int64, out=self.sink[0])

    def warm(self, n):
        for _ in range(n):
            self.layer.forward(self.x, self.out, self.aux)
        torch.cuda.synchronize()
        if self.layer.device_error(self.sh.T) != 0:
            raise RuntimeError(f"device error word set during warm-up ({self.sh.name})")
        v = self.layer.views(self.sh.T)
        self.kept = v["kept_counts"].cpu().tolist()
        self.bucket_rows = int(v["seg_offsets"][-1].item()) if self.args.binned else None

    def timed_steps(self, steps, world=1):
        """Timed steps record 4 events: before route, around the up projection
        (the roofline's kernel) and after combine; the other stage boundaries
        carry no event, so consecutive kernels overlap their launches as in
        use. Returns [(step ms, up-projection ms)] and the launches counted."""
        from mixture_experts_routing_route_b200 import _abi as abi
        evs = [[torch.cuda.Event(enable_timing=True) if j in (0, 3, 4, 6) else None for j in range(7)]
               for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        n0 = abi.moe_kernel_launches()
        for i in range(steps):
            self.evict_l2()
            self.layer.forward(self.x, self.out, self.aux, events=evs[i])
        n1 = abi.moe_kernel_launches()
        torch.cuda.synchronize()
        barrier(world)
        per = [(evs[i][0].elapsed_time(evs[i][6]), evs[i][3].elapsed_time(evs[i][4]))
               for i in range(steps)]
        return per, n1 - n0

    def stage_times(self, nb):
        """Median over nb steps of each stage's time, with an event at every
        stage boundary (the events serialise the stages). The first step
        starts on an idle GPU, so its events also span the host's enqueue of
        each launch: hence the median."""
        bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(nb)]
        for i in range(nb):
            self.evict_l2()
            self.layer.forward(self.x, self.out, self.aux, events=bevs[i])
        torch.cuda.synchronize()
        if self.layer.device_error(self.sh.T) != 0:
            raise RuntimeError(f"device error word set during the stage pass ({self.sh.name})")
        return {s_: statistics.median(bevs[i][j].elapsed_time(bevs[i][j + 1]) for i in range(nb))
                for j, s_ in enumerate(STAGES)}


def per_config_runs(dev, args, flush, peaks):
    """Every other workload of the layer on this GPU, with a bounded step
    count: tokens/s, ms per forward, the stages' times and fractions of the
    measured peaks (burst GEMM figure), and the dispatch span."""
    out = {}
    for name in PER_CONFIG:
        sh = CONFIGS[name]
        if args.k is not None and args.k != sh.k:
            continue
        inp = make_inputs(sh)
        run = LayerRun(sh, inp, dev, args, flush)
        del inp
        run.warm(3)
        per, launches = run.timed_steps(PER_CONFIG_STEPS)
        step_ms = [p[0] for p in per]
        up_ms = statistics.mean(p[1] for p in per)
        stage_ms = run.stage_times(PER_CONFIG_STEPS)
        alg = algorithmic(sh, run.kept, run.bucket_rows, combine_in_gemm=args.combine_in_gemm)
        ms = sum(step_ms) / len(step_ms)
        roof = stage_roofline(sh, stage_ms, alg, peaks, peaks["bf16_tflops"], args)
        out[name] = {
            "workload": workload_config(sh)["workload"],
            "tokens_per_s": sh.T / (ms * 1e-3), "ms_per_forward": ms, "steps": PER_CONFIG_STEPS,
            "gpu_launches_per_step": launches / PER_CONFIG_STEPS,
            "ffn_up_event_us": up_ms * 1e3,
            "stages": roof, "dispatch_span": dispatch_span_of(stage_ms, alg, peaks),
            "aux_loss": float(run.aux.item()), "rows": int(sum(run.kept)),
            "imbalance_max_over_mean": (max(run.kept) / (sum(run.kept) / sh.E)) if sum(run.kept) else None,
        }
        del run
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.router_backward:
        return run_router_backward(args)

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    sh = shape_of(args)
    # each replica draws its own tokens; the weights are the same everywhere
    inp = make_inputs(sh)
    if rank != 0:
        from workloads import make_x
        inp.x = make_x(sh.with_(seed=replica_seed(sh, rank)))
    flush = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    run = LayerRun(sh, inp, dev, args, flush)
    run.warm(max(3, args.warmup))
    kept, bucket_rows = run.kept, run.bucket_rows

    sampler = ClockSampler(list(range(world)) if rank == 0 else [])
    if rank == 0:
        sampler.start()
    per, launches = run.timed_steps(args.steps, world)
    clocks = sampler.stop() if rank == 0 else {}
    remeasure = int(rank == 0 and ClockSampler.rejected(clocks))
    if world > 1:
        # every rank takes the same collective steps: agree on a re-measurement
        import torch.distributed as dist
        t = torch.tensor([remeasure], dtype=torch.int32, device=dev)
        dist.broadcast(t, 0)
        remeasure = int(t.item())
    if remeasure:
        sampler = ClockSampler(list(range(world)) if rank == 0 else [])
        if rank == 0:
            sampler.start()
        per, launches = run.timed_steps(args.steps, world)
        if rank == 0:
            clocks = sampler.stop()
            clocks["remeasured"] = True
    step_ms = [p[0] for p in per]
    total_ms = reduce_max(sum(step_ms), world)
    up_ms = statistics.mean(p[1] for p in per)
    if run.layer.device_error(sh.T) != 0:
        raise RuntimeError("device error word set during the timed steps")

    # Stage breakdown: a separate, untimed pass with an event at every stage
    # boundary (the events serialise the stages).
    nb = min(args.steps, 20)
    stage_ms = run.stage_times(nb)
    alg = algorithmic(sh, kept, bucket_rows, combine_in_gemm=args.combine_in_gemm)
    peaks = load_peaks()
    # A timed region long enough to hit the 1 kW power cap is compared with the
    # sustained (power-capped) GEMM figure, a short one with the burst figure.
    capped = rank == 0 and "sw_power_cap" in (clocks or {}).get("reasons", [])
    if capped and peaks.get("bf16_tflops_sustained"):
        tc_peak, tc_kind = peaks["bf16_tflops_sustained"], "sustained (sw_power_cap active while timed)"
    else:
        tc_peak, tc_kind = peaks["bf16_tflops"], "burst"
    roof = stage_roofline(sh, stage_ms, alg, peaks, tc_peak, args)

    dom = "ffn_up"
    tf = alg[dom]["flops"] / (up_ms * 1e-3) / 1e12 if up_ms > 0 else None
    traffic = measured_traffic("grouped_gemm_up_swiglu", sh.name)
    roofline = {"kernel": "grouped GEMM, SwiGLU up/gate projection (CTA pairs for experts of >= 768 rows)",
                "bound": "tensor", "achieved": tf, "peak": tc_peak,
                "unit": "TFLOP/s", "frac": tf / tc_peak if tf else None,
                "traffic": traffic,
                "peak_source": f"{peaks['source']} bf16 dense {tc_kind}",
                "algorithmic_per_launch": f"2*R*d*2F = {alg[dom]['flops']:.4e} flop (R={sum(kept)} rows)",
                "launch_us": up_ms * 1e3,
                "timing": "CUDA events on the launch stream around the up projection, every timed step",
                "peak_spec": SPEC_BF16_TFLOPS, "frac_spec": tf / SPEC_BF16_TFLOPS if tf else None}
    dispatch_span = dispatch_span_of(stage_ms, alg, peaks)

    e2e = None
    if not args.no_e2e:
        e2e = measure_e2e(run.layer, inp, sh, args, world, run.x.element_size())

    if rank != 0:
        _finish(world)
        return 0
    aux_value = float(run.aux.item())
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(sh, inp)
    per_config = None
    if world == 1 and not args.no_per_config and sh.name == "mixtral" and not args.router_backward:
        del run
        torch.cuda.empty_cache()
        per_config = per_config_runs(dev, args, flush, peaks)
    value = job_value(sh.T, args.steps, world, total_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": sh.dtype,
        "data": "synthetic (seeded; random-init weights of the layer's shape)",
        "config": arm_config(sh, args, world),
        **({"bin_rows_C": bucket_rows // sh.E} if args.binned and sh.E else {}),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
        "stages": roof,
        "dispatch_span": dispatch_span,
        "stages_note": f"per-stage times: median over a separate pass of {nb} steps with an "
                       f"event at every stage boundary (events serialise the stages)",
        "aux_loss": aux_value,
        "rows": int(sum(kept)), "experts_active": int(sum(1 for c in kept if c > 0)),
        "imbalance_max_over_mean": (max(kept) / (sum(kept) / sh.E)) if sum(kept) else None,
        "per_config": per_config,
        "per_config_note": (f"each other workload of the layer on the same GPU after the headline: "
                            f"3 warm-up and {PER_CONFIG_STEPS} timed steps (L2 evicted between), "
                            f"stage times from a separate {PER_CONFIG_STEPS}-step pass; GEMM "
                            f"fractions of the burst bf16 peak") if per_config else None,
    }
    print(json.dumps(line), flush=True)
    _finish(world)
    return 0


def _finish(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
