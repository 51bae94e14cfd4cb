#!/usr/bin/env python
"""Benchmark of the VDA linear branch (prepare -> bidirectional scan -> readout).

One step = one pass of the whole path over one synthetic batch of the chosen
workload (default: the H3-like clip, B=1 H=24 d=128 T=40 U=1560 c=5 L=512, bf16
storage, fp32 state), with inputs resident in HBM. Prints one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config h3] [--impl reference]

N > 1 runs one process per GPU under torch.distributed.run (bench.py starts
it itself when launched without RANK in the environment). `--shard batch`
(default): every rank processes its own batch (independent problems, weak
scaling). `--shard heads`: the ranks share one batch and each serves a slice of
its heads in place (vda_config.H_total, h0; strong scaling). Neither form has a
data-path collective; the timed region is bracketed by barriers and the time is
the max over ranks.
`--impl reference` times the float64 CPU oracle on the host cores instead (rank
0 only), one (batch, head) pair of the workload per step.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from frame_level_delta_b200.inputs import CONFIGS, make_inputs  # noqa: E402

METRIC = "VDA bidir scan+readout tokens/s per head-layer; % of B200 bf16 tensor/HBM peak"
UNIT = "head-tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def workload_desc(cfg) -> str:
    extra = ", conv prep + RMSNorm/gate" if cfg.prep_conv else ""
    return (f"{cfg.name}: B={cfg.B} H={cfg.H} d={cfg.d} T={cfg.T} U={cfg.U} ({cfg.grid_h}x{cfg.grid_w}) "
            f"c={cfg.chunk} L={cfg.L} {cfg.dtype} storage, fp32 state{extra}")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------
# Ranks: one process per GPU, each rank its own batch (weak scaling). The only
# collectives are the barriers around the timed regions and the max-over-ranks
# reduction of the measured times; the data path has none.
# ----------------------------------------------------------------------------
def rank_env():
    """(rank, world size, local rank) as torch.distributed.run exports them."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(cfg, rank: int, shard: str = "batch") -> int:
    """Seed of the batch a rank draws: independent problems per rank, or the one
    shared batch when the ranks split its heads."""
    return cfg.seed + (rank if shard == "batch" else 0)


def relaunch_under_torchrun(argv, gpus: int) -> int:
    """Run this script again as `gpus` ranks under torch.distributed.run (one
    process per GPU of this node, rendezvous on 127.0.0.1) and return its exit
    code."""
    import socket
    import subprocess
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def init_ranks(world: int, device, timeout_s: float = 120.0):
    """Process group for the barriers and the time reduction (NCCL between CUDA
    ranks, gloo between CPU ranks); None for a single rank."""
    if world <= 1:
        return None
    import torch.distributed as dist
    timeout = datetime.timedelta(seconds=timeout_s)
    if device.type == "cuda":
        dist.init_process_group("nccl", timeout=timeout, device_id=device)
    else:
        dist.init_process_group("gloo", timeout=timeout)
    return dist


def barrier(dist) -> None:
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, ms: float, device) -> float:
    """The slowest rank's time: every rank takes part, every rank gets the max."""
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, cfg, steps: int, ms_max: float, shard: str = "batch") -> float:
    """Head-tokens all ranks processed divided by the slowest rank's time (each
    rank a batch; or, with the heads split, one batch among them all)."""
    batches = world if shard == "batch" else 1
    return batches * cfg.head_tokens * steps / (ms_max / 1e3)


# ----------------------------------------------------------------------------
# Algorithmic bytes / flops per launch of each kernel (each input byte read
# once, each output byte written once).
# ----------------------------------------------------------------------------
# Whether the tensor-core scan runs over composed chunk maps (VDA_SCAN_CHUNKED)
# or frame by frame (the default); set from --scan.
SCAN_CHUNKED = False
# Whether the Cholesky solve is selected (VDA_SOLVE_CHOLESKY); set from --solve.
SOLVE_CHOLESKY = False
# Whether the path runs from e4m3 keys, values and queries (--fp8).
FP8 = False
FP8_KEYS = ("Q8", "q_scale", "K8", "V8", "kv_scale", "Kt8", "Vt8", "kvt_scale", "alpha", "beta", "beta_txt")


def inject_in_scan(cfg) -> bool:
    """Whether the frame scan forms the injections itself, (S Diag(alpha_t) + B_t) P_t,
    so that the sweep solve writes P_t's images and no C_t for frames."""
    from frame_level_delta_b200 import vda as V
    return "inject=scan" in V.describe(V.make_config(cfg, cholesky=SOLVE_CHOLESKY, chunked=SCAN_CHUNKED))


def composed_chunks(cfg):
    """Frame counts of the chunk maps the tensor-core scan composes (forward
    chunks 0..J-3 over frames max(1, c m)..c(m+1)-1, reverse chunks 2..J-1 over
    c m..min(c(m+1)-1, T-2)); empty when the scan steps over frames directly."""
    c, T, J = cfg.chunk, cfg.T, cfg.J
    if not SCAN_CHUNKED or c <= 1 or J < 3:
        return []
    fwd = [max(0, c * (m + 1) - 1 - max(1, c * m) + 1) for m in range(0, J - 2)]
    rev = [max(0, min(c * (m + 1) - 1, T - 2) - c * m + 1) for m in range(2, J)]
    return fwd + rev


def kernel_bytes(name: str, cfg) -> float:
    B, H, d, T, U, L, c = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L, cfg.chunk
    esz = 4 if cfg.dtype == "f32" else 2
    F, NS, J = T - 2, T - 1, cfg.J
    BH = B * H
    dd4 = d * d * 4
    if name in ("gram_tc", "gram_simt"):
        return BH * ((F * U + L) * (2 * d * esz + 4) + 2 * NS * dd4)
    if name == "gram_fp8_tc":  # e4m3 K, V (one byte per channel), beta, the shared scale; A, B out
        return BH * ((F * U + L) * (2 * d + 4 + 4) + 2 * NS * dd4)
    if name == "readout_fp8_tc":  # e4m3 Q and its scale in, bf16 O out, the states, anchor zeros
        return BH * (F * U * (d + 4 + 2 * d) + 2 * J * dd4 + 2 * U * d * 2)
    if name == "solve_simt":
        return BH * (4 * NS * dd4 + F * d * 4)
    if name == "solve_tc" and inject_in_scan(cfg):  # the text grid: A and B read, C = S_T written
        return BH * 3 * dd4
    if name == "solve_tc_frames":  # the frame grid: A read, P's hi/lo images written
        return BH * F * 2 * dd4
    if name in ("solve_tc", "solve_chol_tc"):  # A, B, alpha read; C (fp32) and M's hi/lo operand images written
        return BH * (3 * NS * dd4 + F * dd4 + F * d * 4)
    if name in ("scan_tc", "scan_split_tc"):  # per step: a (chunk) map's hi/lo images + its C; S_T; readout states
        if composed_chunks(cfg):
            steps = 2 * (J - 2)
        else:
            steps = max(0, c * (J - 2) - 1) + max(0, (T - 2) - 2 * c + 1)
        alpha = steps * d * 4 if inject_in_scan(cfg) else 0  # per step: P images + B rows + alpha
        return BH * (steps * 2 * dd4 + alpha + 2 * dd4 + 2 * J * dd4)
    if name == "compose_tc":  # per frame of a composed chunk: M images + C; per chunk: map + C out
        ch = composed_chunks(cfg)
        return BH * (sum(ch) * 2 * dd4 + len(ch) * 2 * dd4)
    if name == "scan_simt":
        fwd = max(0, c * (J - 2) - 1)
        rev = max(0, (T - 2) - 2 * c + 1)
        return BH * ((fwd + rev) * 2 * dd4 + 2 * dd4 + 2 * J * dd4)
    if name in ("readout_tc", "readout_simt"):
        gate = 1 if cfg.norm_gate else 0
        zeros = 2 * U * d * esz if name == "readout_tc" else 0  # the tensor-core readout zeroes the anchors
        return BH * (F * U * d * esz * (2 + gate) + 2 * J * dd4 + zeros)
    if name == "zero_anchors":
        return BH * 2 * U * d * esz
    if name == "prep_video":
        return BH * (2 * T * U * d * esz + 2 * F * U * d * esz)
    if name == "prep_text":
        return BH * 4 * L * d * esz
    return 0.0


def kernel_flops(name: str, cfg) -> float:
    """Algorithmic flops per launch (the method's arithmetic, not the hi/lo split's)."""
    B, H, d, T, U, L, c = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L, cfg.chunk
    F, NS, J = T - 2, T - 1, cfg.J
    if name.startswith("gram"):
        return B * H * (F * U + L) * 4 * d * d
    if name == "readout_fp8_tc":
        return B * H * F * U * 2 * d * d
    if name == "solve_tc" and inject_in_scan(cfg):  # text grid: the inverse d^3 and C = B P (2 d^3)
        return B * H * 3 * d ** 3
    if name == "solve_tc_frames":  # frame grid: the inverse, d^3 per slot
        return B * H * F * d ** 3
    if name.startswith("solve"):  # Cholesky d^3/3, L^-1 d^3/3, P d^3/3, C = B P 2 d^3
        return B * H * NS * 3 * d ** 3
    if name == "compose_tc":  # two d x d x d products per absorbed frame
        return B * H * sum(max(0, n - 1) for n in composed_chunks(cfg)) * 2 * 2 * d ** 3
    if name == "scan_tc" and composed_chunks(cfg):
        return B * H * 2 * (J - 2) * 2 * d ** 3
    if name.startswith("scan"):
        fwd = max(0, c * (J - 2) - 1)
        rev = max(0, (T - 2) - 2 * c + 1)
        return B * H * (fwd + rev) * 2 * d ** 3
    if name.startswith("readout"):
        return B * H * F * U * 2 * d * d
    return 0.0


# Kernels whose time is set by dense contractions and their serial dependencies
# rather than by HBM streaming: their roofline is the bf16 tensor peak.
TENSOR_BOUND = ("solve_chol_tc", "solve_simt")

# Kernels whose time is set by fp32 FMAs on the CUDA cores. The sweep of a
# d x d matrix applies every pivot's rank-1 update to the whole matrix: d^3 FMAs
# per slot (the kernel exploits symmetry and executes about half of them). The
# separable conv prep takes a 5x5 spatial sum of every input frame and a 5-tap
# temporal sum per output: (25 T / (T-2) + 5) FMAs per prepared K or V value.
# Peak: 148 SMs x 128 fp32 lanes x 2 flop per FMA x the SM clock.
ALU_BOUND = ("solve_tc", "solve_tc_frames", "prep_video")


def kernel_alu_flops(name: str, cfg) -> float:
    if name == "solve_tc":
        slots = 1 if inject_in_scan(cfg) else cfg.T - 1  # the text grid alone in the P form
        return cfg.B * cfg.H * slots * 2 * cfg.d ** 3
    if name == "solve_tc_frames":
        return cfg.B * cfg.H * (cfg.T - 2) * 2 * cfg.d ** 3
    if name == "prep_video":
        F = cfg.T - 2
        return cfg.B * cfg.H * 2 * F * cfg.U * cfg.d * 2 * (25 * cfg.T / F + 5)
    return 0.0


def alu_peak_tflops(sm_mhz: float) -> float:
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def path_bytes(cfg) -> float:
    """Algorithmic bytes of one whole step: Q, K, V, beta read and O written once on
    non-anchor frames, plus text, alpha, anchor zero-fill (and, with conv prep,
    K and V of every frame plus the gate)."""
    B, H, d, T, U, L = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L
    esz = 4 if cfg.dtype == "f32" else 2
    F = T - 2
    per_head = F * U * (4 * d * esz + 4) + L * (2 * d * esz + 4) + F * d * 4 + 2 * U * d * esz
    if FP8:  # Q8, K8, V8 at one byte per channel with their scales; O in bf16
        per_head = F * U * (3 * d + 2 * d + 4 + 4 + 4) + L * (2 * d + 4 + 4) + F * d * 4 + 2 * U * d * 2
    if cfg.prep_conv:
        per_head += 2 * 2 * U * d * esz + F * U * d * esz  # anchor-frame K, V for the conv; gate
    return B * H * per_head


def path_flops(cfg) -> float:
    B, H, d, T, U, L, c = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L, cfg.chunk
    F, NS, J = T - 2, T - 1, cfg.J
    gram = (F * U + L) * 4 * d * d
    solve = NS * (d ** 3 + 2 * d ** 3)  # Cholesky + L^-1 + L^-T L^-1 (~d^3) and C = B P (2 d^3)
    fwd = max(0, c * (J - 2) - 1)
    rev = max(0, (T - 2) - 2 * c + 1)
    scan = (fwd + rev) * 2 * d ** 3
    readout = F * U * 2 * d * d
    return B * H * (gram + solve + scan + readout)


def source_digest(kernel: str):
    files = {"gram_tc": "gram_tc.cu", "readout_tc": "readout_tc.cu", "solve_tc": "solve_tc.cu",
             "gram_fp8_tc": "gram_fp8_tc.cu", "readout_fp8_tc": "readout_fp8_tc.cu",
             "solve_tc_frames": "solve_tc.cu", "window_attn_tc": "window_attn_tc.cu", "merge_tc": "merge_tc.cu",
             "scan_tc": "scan_tc.cu", "scan_split_tc": "scan_split_tc.cu", "compose_tc": "compose_tc.cu", "solve_chol_tc": "solve_chol_tc.cu",
             "prep_video": "prep_video.cu"}
    fn = files.get(kernel, "kernels_simt.cu")
    p = os.path.join(ROOT, "frame_level_delta_b200", "csrc", fn)
    with open(p, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, only if the kernel's
    source is unchanged since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        tab = json.load(f)
    e = tab.get(workload, {}).get(kernel)
    if not e or e.get("source_sha") != source_digest(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# Clock sampling during the timed region (NVML, the library nvidia-smi uses).
# ----------------------------------------------------------------------------
REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}


class ClockSampler:
    def __init__(self, device_index: int, period_s: float = 0.01):
        self.ok = False
        self.samples = []
        self.reasons = 0
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            props = torch.cuda.get_device_properties(device_index)
            h = None
            uuid = getattr(props, "uuid", None)
            if uuid is not None:
                s = str(uuid)
                for cand in (s if s.startswith("GPU-") else "GPU-" + s,):
                    try:
                        h = pynvml.nvmlDeviceGetHandleByUUID(cand)
                    except Exception:
                        h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = device_index
                parts = [x for x in vis.split(",") if x.strip()]
                if parts and parts[min(device_index, len(parts) - 1)].strip().isdigit():
                    idx = int(parts[device_index].strip())
                h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.h = h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that, do not guess
            self.err = repr(e)

    def _sample(self):
        nv = self.nv
        sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.samples.append(sm)
        self.reasons |= r

    def _loop(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(self.period)

    def start(self):
        if not self.ok:
            return
        self._stop = threading.Event()
        self._t = threading.Thread(target=self._loop, daemon=True)
        self._t.start()

    def stop(self):
        if not self.ok:
            return
        self._stop.set()
        self._t.join()
        try:
            self._sample()
        except Exception:
            pass

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": getattr(self, "err", "no samples")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in REASON_BITS.items() if self.reasons & b],
                "samples": len(self.samples), "source": "nvml"}


# ----------------------------------------------------------------------------
# CPU oracle timing (test infrastructure; bench.py's CPU-baseline leg)
# ----------------------------------------------------------------------------
def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        for d in info:
            if d.get("user_api") == "blas":
                return int(d.get("num_threads"))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def blas_library() -> str:
    """The BLAS numpy calls into, as threadpoolctl reports it (library and version)."""
    try:
        import threadpoolctl
        for d in threadpoolctl.threadpool_info():
            if d.get("user_api") == "blas":
                return f"{d.get('internal_api')} {d.get('version')} ({os.path.basename(str(d.get('filepath')))})"
    except Exception:
        pass
    return "unknown"


def one_blas_thread():
    """Context manager limiting numpy's BLAS to one thread."""
    import threadpoolctl
    return threadpoolctl.threadpool_limits(limits=1, user_api="blas")


def time_oracle(cfg, inp, heads, budget_s=None):
    from oracle.vda_oracle import vda_reference
    done = 0
    t0 = time.perf_counter()
    for bh in heads:
        vda_reference(inp, cfg, heads=[bh], keep=False)
        done += 1
        if budget_s is not None and time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return done, dt


def cpu_baseline(cfg, inp, budget_s=10.0):
    """The float64 oracle on the host cores: all the BLAS threads the process may
    use for ~budget_s, then one BLAS thread for ~budget_s / 2."""
    heads = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    threads = blas_threads()
    done, dt = time_oracle(cfg, inp, heads, budget_s=budget_s)
    value = done * cfg.T * cfg.U / dt
    with one_blas_thread():
        done1, dt1 = time_oracle(cfg, inp, heads, budget_s=budget_s / 2)
    value1 = done1 * cfg.T * cfg.U / dt1
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
            "blas": blas_library(), "host_cpus": len(os.sched_getaffinity(0)),
            "one_thread": {"value": value1, "unit": UNIT, "cores": 1,
                           "sample": f"{done1} (batch, head) pairs, {dt1:.2f} s"},
            "sample": f"float64 numpy oracle over {done} of {len(heads)} (batch, head) pairs of the "
                      f"workload ({cfg.T * cfg.U} tokens each), {dt:.2f} s, BLAS threads={threads} "
                      f"({blas_library()})"}


def run_reference(args, cfg, rank, world):
    if rank != 0:
        return 0
    inp = make_inputs(cfg)
    heads = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
    for i in range(args.warmup):
        time_oracle(cfg, inp, [heads[i % len(heads)]])
    t0 = time.perf_counter()
    for i in range(args.steps):
        time_oracle(cfg, inp, [heads[i % len(heads)]])
    dt = time.perf_counter() - t0
    value = args.steps * cfg.T * cfg.U / dt
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": workload_desc(cfg), "step": "one (batch, head) pair of the workload"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "blas": blas_library(),
                             "sample": f"one (batch, head) pair per step, {cfg.T * cfg.U} tokens"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# Softmax branch and the whole hybrid layer (--path softmax / hybrid)
# ----------------------------------------------------------------------------
def attention_pairs(cfg) -> int:
    """(query, visible key) token pairs of the window + anchor softmax per (b, h)."""
    from frame_level_delta_b200.inputs import CONFIGS  # noqa: F401 (keeps the import style of the module)
    c, T, U = cfg.chunk, cfg.T, cfg.U
    n = 0
    for t in range(T):
        if t in (0, T - 1):
            n += T
        else:
            j = t // c
            lo, hi = max(0, c * (j - 1)), min(T - 1, c * (j + 2) - 1)
            n += (hi - lo + 1) + (1 if lo > 0 else 0) + (1 if hi < T - 1 else 0)
    return n * U * U


def attention_flops(cfg) -> float:
    """Two d-deep products (Q K^T and P V) per visible pair: 4 d flops."""
    return 4.0 * cfg.d * attention_pairs(cfg) * cfg.B * cfg.H


def attention_bytes(cfg) -> float:
    """Q, K, V, gate read once and O written once (bf16)."""
    return 5.0 * cfg.B * cfg.T * cfg.U * cfg.H * cfg.d * 2


def merge_flops(cfg, n_model: int) -> float:
    return 2.0 * cfg.B * cfg.T * cfg.U * (2 * cfg.H * cfg.d) * n_model


def time_attention_oracle(cfg, inp, budget_s: float):
    """The float64 oracle's window softmax on query tokens of head 0, frame by
    frame from the middle of the clip, until the budget is spent."""
    import numpy as np
    from oracle.hybrid_oracle import softmax_gate, window_softmax_rows
    Q, K, V, g = (inp[k][0, :, 0].double().numpy() for k in ("Q", "K", "V", "gate"))
    done, t0 = 0, time.perf_counter()
    rows = list(range((cfg.T // 2) * cfg.U, cfg.T * cfg.U)) + list(range(0, (cfg.T // 2) * cfg.U))
    step = 64
    while time.perf_counter() - t0 < budget_s and done < len(rows):
        r = rows[done:done + step]
        softmax_gate(window_softmax_rows(Q, K, V, cfg.T, cfg.U, cfg.chunk, r), g[r])
        done += len(r)
    return done, time.perf_counter() - t0


def run_attention_path(args, cfg, rank, world, local, dist, dev):
    """One step = the softmax branch (--path softmax) or the whole hybrid layer's
    attention (--path hybrid: linear branch, softmax branch and the merge by the
    two output projections, model width H d) over one synthetic batch."""
    from frame_level_delta_b200 import vda as V
    from frame_level_delta_b200.inputs import make_attention_inputs, make_merge_inputs
    hybrid = args.path == "hybrid"
    inp_cpu = make_inputs(cfg, seed=rank_seed(cfg, rank)) if hybrid else {}
    att = make_attention_inputs(cfg, seed=rank_seed(cfg, rank))
    if hybrid:
        att = {k: att[k] for k in ("gate",)}
        att.update({k: inp_cpu[k] for k in ("Q", "K", "V")})
    n_model = cfg.H * cfg.d
    W = make_merge_inputs(1, n_model, cfg.H * cfg.d, seed=rank) if hybrid else {}
    host = {k: v.pin_memory() for k, v in {**inp_cpu, **att}.items()}
    dinp = {k: v.to(dev, non_blocking=True) for k, v in host.items()}
    Wd = {k: W[k].to(dev) for k in ("W_soft", "W_lin")} if hybrid else {}
    ctx = V.VDA(cfg, device=dev)
    # The linear branch runs on a side stream next to the softmax branch (its
    # middle kernels are latency-bound and fill the SMs the attention leaves).
    lin = V.VDA(cfg, device=dev) if hybrid else None
    side = torch.cuda.Stream(dev) if hybrid else None
    O_soft = ctx.new_output()
    O_lin = ctx.new_output() if hybrid else None
    M = cfg.B * cfg.T * cfg.U
    Y = torch.empty(M, n_model, dtype=torch.bfloat16, device=dev) if hybrid else None
    mstat = torch.zeros(256, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(d, o_soft, o_lin, y):
        if hybrid:
            side.wait_stream(stream)
            lin.run(d, o_lin, stream=side)
        ctx.window_attention(d["Q"], d["K"], d["V"], d["gate"], o_soft)
        if hybrid:
            stream.wait_stream(side)
            V.hybrid_merge(o_soft, Wd["W_soft"], o_lin, Wd["W_lin"], y, status=mstat)

    for _ in range(args.warmup):
        step(dinp, O_soft, O_lin, Y)
    torch.cuda.synchronize(dev)
    if ctx.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout during warm-up")
    n0 = ctx.launch_count() + (lin.launch_count() if hybrid else 0)
    clocks = ClockSampler(local)
    ctx.profile_enable(True)
    barrier(dist)
    torch.cuda.synchronize(dev)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step(dinp, O_soft, O_lin, Y)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(dist)
    ms = ev0.elapsed_time(ev1)
    prof = ctx.profile_read()
    ctx.profile_enable(False)
    launches = ctx.launch_count() + (lin.launch_count() if hybrid else 0) - n0 + (args.steps if hybrid else 0)
    if hybrid and lin.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the linear branch")
    if ctx.poll_device_status() != 0 or int(mstat[:4].view(torch.int32).item()) != 0:
        raise RuntimeError("device status reported a timeout in the timed region")
    ms_max = max_over_ranks(dist, ms, dev)
    value = whole_job_rate(world, cfg, args.steps, ms_max)

    # End to end: pinned host inputs up, the step, the result back, every step (serial).
    out_host = torch.empty((M, n_model) if hybrid else tuple(O_soft.shape), dtype=torch.bfloat16, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * 2
    ke = max(1, min(args.e2e_steps, args.steps, 5))
    barrier(dist)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ke):
        for k, v in host.items():
            dinp[k].copy_(v, non_blocking=True)
        step(dinp, O_soft, O_lin, Y)
        out_host.copy_(Y if hybrid else O_soft, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist)
    e2e_value = whole_job_rate(world, cfg, ke, max_over_ranks(dist, e0.elapsed_time(e1), dev))

    peaks, peak_src = load_peaks()
    att_n, att_ms = prof["window_attn_tc"]
    att_s = att_ms / att_n / 1e3
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    achieved = attention_flops(cfg) / att_s / 1e12
    step_s = ms_max / 1e3 / args.steps
    kernels = {k: {"launches": n, "avg_us": tot / n * 1e3} for k, (n, tot) in prof.items()}
    if rank == 0:
        metric = ("hybrid attention layer (VDA linear branch + window softmax + merge) head-tokens/s"
                  if hybrid else "window + anchor softmax branch head-tokens/s; % of B200 bf16 tensor peak")
        line = {
            "metric": metric, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "impl": "vda",
            "config": {"workload": workload_desc(cfg) + ("" if hybrid else ", softmax branch, logit std 1"),
                       "path": args.path, "model_width": n_model if hybrid else None,
                       "streams": ("linear branch on a side stream beside the softmax kernel; merge after both"
                                   if hybrid else "one stream"),
                       "l2": "no flush: each step reads > 1 GB of tokens, far above the 126 MB L2"},
            "roofline": {"bound": "tensor", "kernel": "window_attn_tc", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                         "peak_source": f"bf16_tflops_sustained of {peak_src} (each launch runs for tens of ms)",
                         "frac_of_burst": achieved / float(peaks["bf16_tflops"]),
                         "algorithmic_flops_per_launch": attention_flops(cfg),
                         "algorithmic_bytes_per_launch": attention_bytes(cfg)},
            "step_tflops": (attention_flops(cfg) + (merge_flops(cfg, n_model) + path_flops(cfg) if hybrid else 0))
                           / step_s / 1e12,
            "kernels": kernels, "gpu_launches": launches, "clocks": clocks.summary(),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": ke, "note": "serial copies: inputs up, step, result down"},
        }
        if world == 1 and args.cpu_budget > 0:
            done, dt = time_attention_oracle(cfg, att, args.cpu_budget)
            line["cpu_baseline"] = {
                "value": done / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                "blas": blas_library(),
                "sample": f"float64 oracle window softmax (+gate) of {done} query tokens of head 0, {dt:.2f} s"
                          + ("; the linear branch's oracle is timed by --path linear" if hybrid else "")}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def backward_flops(cfg) -> dict:
    """Per launch: the statistics (4 d^2 flops per token), the per-frame adjoints
    (the sweep's d^3 FMAs and three d x d x d products, S_t, Gx and GA, at 2 d^3
    flops each) and the per-token products (three d x d matrix-vector products,
    6 d^2 flops per token)."""
    B, H, d, T, U, L = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U, cfg.L
    F = T - 2
    return {"gram": B * H * (F * U + L) * 4 * d * d,
            "frame": B * H * F * (2 * d ** 3 + 3 * 2 * d ** 3),
            "token": B * H * F * U * 6 * d * d}


def backward_bytes(cfg) -> float:
    """K, V, beta read and dK, dV, dbeta written per token; S_prev, dS read and
    dS_prev written per frame; alpha and dalpha."""
    B, H, d, T, U = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U
    esz = 4 if cfg.dtype == "f32" else 2
    F = T - 2
    return B * H * F * (U * (4 * d * esz + 8) + 3 * d * d * 4 + 2 * d * 4)


def run_backward_path(args, cfg, rank, world, local, dist, dev):
    """--path backward: one step = vda_frame_solve_backward over every head and
    frame of one batch (the statistics recomputed, the per-frame adjoints, the
    per-token gradients)."""
    from frame_level_delta_b200 import vda as V
    from frame_level_delta_b200.inputs import make_backward_inputs
    inp = {k: v.to(dev) for k, v in make_inputs(cfg, seed=rank_seed(cfg, rank)).items()}
    bw = {k: v.to(dev) for k, v in make_backward_inputs(cfg, seed=rank_seed(cfg, rank)).items()}
    ctx = V.VDA(cfg, device=dev)
    out = None
    stream = torch.cuda.current_stream(dev)

    def step():
        return ctx.frame_solve_backward(inp["K"], inp["V"], inp["alpha"], inp["beta"], bw["S_prev"], bw["dS"],
                                        out=out)

    out = step()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    n0 = ctx.launch_count()
    ctx.profile_enable(True)
    clocks = ClockSampler(local)
    barrier(dist)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(dist)
    ms_max = max_over_ranks(dist, e0.elapsed_time(e1), dev)
    prof = ctx.profile_read()
    ctx.profile_enable(False)
    if ctx.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the timed region")
    tc_tokens = "token_bwd_tc" in prof
    # frame_bwd_simt is two launches per step when it also does the token part
    launches = ctx.launch_count() - n0 + (0 if tc_tokens else args.steps)
    value = whole_job_rate(world, cfg, args.steps, ms_max)
    fl = backward_flops(cfg)
    peaks, peak_src = load_peaks()
    sm_mhz = float(clocks.summary().get("sm_mhz") or 1965.0)
    dom = max(prof.items(), key=lambda kv: kv[1][1] / kv[1][0])[0]
    dn, dms = prof[dom]
    d_s = dms / dn / 1e3
    B_, H_, d_, T_, U_ = cfg.B, cfg.H, cfg.d, cfg.T, cfg.U
    esz = 4 if cfg.dtype == "f32" else 2
    token_bytes = B_ * H_ * (T_ - 2) * U_ * (4 * d_ * esz + 8)  # K, V, beta in; dK, dV, dbeta out
    if dom == "token_bwd_tc":
        bound, unit, peak = "hbm", "GB/s", float(peaks["hbm_gbs"])
        achieved = token_bytes / d_s / 1e9
        peak_note = f"hbm_gbs of {peak_src}"
    else:
        bound, unit, peak = "alu", "TFLOP/s", alu_peak_tflops(sm_mhz)
        achieved = (fl["frame"] + (0 if tc_tokens else fl["token"])) / d_s / 1e12
        peak_note = f"fp32 FMA peak derived: 148 SMs x 128 lanes x 2 flop x {sm_mhz:.0f} MHz"
    if rank == 0:
        line = {"metric": "frame-step backward head-tokens/s (dK, dV, dbeta, dalpha, dS_prev)", "value": value,
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic", "impl": "vda",
                "config": {"workload": workload_desc(cfg), "path": "backward"},
                "roofline": {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak,
                             "unit": unit, "frac": achieved / peak, "traffic": None, "peak_source": peak_note,
                             "algorithmic_flops_per_launch": fl["frame"] if dom != "token_bwd_tc" else fl["token"],
                             "algorithmic_bytes_per_launch": token_bytes if dom == "token_bwd_tc"
                             else backward_bytes(cfg)},
                "kernels": {k: {"launches": n, "avg_us": tot / n * 1e3} for k, (n, tot) in prof.items()},
                "gpu_launches": launches, "clocks": clocks.summary()}
        if world == 1 and args.cpu_budget > 0:
            from oracle.vda_oracle import frame_step_backward
            n, t0 = 0, time.perf_counter()
            U = cfg.U
            while time.perf_counter() - t0 < args.cpu_budget:
                h, t = n % cfg.H, 1 + (n // cfg.H) % (cfg.T - 2)
                frame_step_backward(bw["S_prev"][0, h, t].double().cpu().numpy(),
                                    inp["K"][0, t * U:(t + 1) * U, h].double().cpu().numpy(),
                                    inp["V"][0, t * U:(t + 1) * U, h].double().cpu().numpy(),
                                    inp["beta"][0, h, t].double().cpu().numpy(),
                                    inp["alpha"][0, h, t].double().cpu().numpy(),
                                    bw["dS"][0, h, t].double().cpu().numpy())
                n += 1
            dt = time.perf_counter() - t0
            line["cpu_baseline"] = {"value": n * U / dt, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                    "blas": blas_library(),
                                    "sample": f"float64 oracle frame_step_backward on {n} (head, frame) pairs, "
                                              f"{dt:.2f} s"}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_ulysses(args, cfg, rank, world, local, dist, dev):
    """--shard ulysses: the batch arrives sequence-sharded (rank r holds tokens
    r n .. (r+1) n - 1 of every head, n = T U / world); one step is the all-to-all
    of Q, K, V to head shards (every token of this rank's heads), the linear
    branch on those heads, and the all-to-all of O back to sequence shards. The
    per-head parameters (alpha, beta, text tokens) are this rank's heads' (they
    are small; their own exchange is the same operation). Strong scaling."""
    from frame_level_delta_b200 import vda as V
    from frame_level_delta_b200.shard import head_partition, heads_to_seq, seq_to_heads
    full = make_inputs(cfg)
    N = cfg.T * cfg.U
    if N % world:
        raise SystemExit(f"--shard ulysses needs T*U ({N}) divisible by the rank count ({world})")
    n = N // world
    parts = head_partition(cfg.H, world)
    h0, k = parts[rank]
    seq = {x: full[x][:, rank * n:(rank + 1) * n].contiguous().to(dev) for x in ("Q", "K", "V")}
    par = {x: full[x][:, :, h0:h0 + k].contiguous().to(dev) for x in ("K_txt", "V_txt")}
    par.update({x: full[x][:, h0:h0 + k].contiguous().to(dev) for x in ("alpha", "beta", "beta_txt")})
    lcfg = cfg.with_(H=k)
    lib = V.VDA(lcfg, device=dev)
    O = lib.new_output()
    stream = torch.cuda.current_stream(dev)

    def step():
        if world > 1:
            heads = {x: seq_to_heads(seq[x], parts) for x in ("Q", "K", "V")}
        else:
            heads = seq
        lib.run({**heads, **par}, O)
        return heads_to_seq(O, parts) if world > 1 else O

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    n0 = lib.launch_count()
    clocks = ClockSampler(local)
    barrier(dist)
    torch.cuda.synchronize(dev)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(dist)
    ms_max = max_over_ranks(dist, e0.elapsed_time(e1), dev)
    if lib.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the timed region")
    value = cfg.head_tokens * args.steps / (ms_max / 1e3)
    xbytes = 4 * cfg.B * n * cfg.H * cfg.d * (2 if cfg.dtype == "bf16" else 4) * (world - 1) / max(world, 1)
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
                "scaling": "strong", "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic",
                "config": {"workload": workload_desc(cfg), "global_batch": cfg.B,
                           "parallelism": f"ulysses{world}: sequence shards -> all-to-all -> heads {parts} "
                                          f"-> all-to-all back (NCCL)"},
                "exchange_bytes_per_rank_per_step": xbytes, "gpu_launches": lib.launch_count() - n0,
                "clocks": clocks.summary()}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="h3", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="vda", choices=["vda", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work (0: skip)")
    ap.add_argument("--solve", default="sweep", choices=["sweep", "cholesky"],
                    help="tensor-core frame solve: symmetric sweep (default) or blocked Cholesky")
    ap.add_argument("--scan", default="frames", choices=["frames", "chunked", "split"],
                    help="tensor-core scan frame by frame (default), over composed chunk maps, or frame "
                         "by frame on two-CTA clusters (each CTA half of every state's columns)")
    ap.add_argument("--heads", type=int, default=0,
                    help="override H (a smaller case of the same workload, e.g. for profiler captures)")
    ap.add_argument("--path", default="linear", choices=["linear", "softmax", "hybrid", "backward"],
                    help="linear: the VDA linear branch (the headline); softmax: the window + anchor "
                         "softmax branch; hybrid: both branches and the merge")
    ap.add_argument("--fp8", action="store_true",
                    help="linear path from e4m3 keys, values and queries with per-token scales")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads", "ulysses"],
                    help="N > 1: a batch per rank (weak scaling), one batch's heads split over the ranks, "
                         "or sequence-sharded inputs exchanged to head shards and back (all-to-all)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    if args.gpus > 1 and "RANK" not in os.environ:
        return relaunch_under_torchrun(sys.argv[1:], args.gpus)
    cfg = CONFIGS[args.config]
    if args.heads > 0:
        cfg = cfg.with_(H=args.heads)
    rank, world, local = rank_env()
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch one rank per GPU")
    if args.impl == "reference":
        return run_reference(args, cfg, rank, world)

    from frame_level_delta_b200 import vda as V
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_ranks(world, dev)
    if args.path == "backward":
        return run_backward_path(args, cfg, rank, world, local, dist, dev)
    if args.path != "linear":
        return run_attention_path(args, cfg, rank, world, local, dist, dev)
    if args.shard == "ulysses":
        return run_ulysses(args, cfg, rank, world, local, dist, dev)

    # Each rank draws its own batch (independent problems), or all draw the one
    # batch whose heads they split.
    if args.fp8:
        from frame_level_delta_b200.inputs import make_fp8_inputs
        x8 = make_fp8_inputs(cfg, seed=rank_seed(cfg, rank, args.shard))
        inp_cpu = {k: x8[k] for k in FP8_KEYS}
    else:
        inp_cpu = make_inputs(cfg, seed=rank_seed(cfg, rank, args.shard))
    heads = None
    if args.shard == "heads" and world > 1:
        from frame_level_delta_b200.shard import head_partition
        heads = head_partition(cfg.H, world)[rank]
    inp_host = {k: v.pin_memory() for k, v in inp_cpu.items()}
    inp_dev = {k: v.to(dev, non_blocking=True) for k, v in inp_host.items()}
    global SCAN_CHUNKED, SOLVE_CHOLESKY
    SCAN_CHUNKED = args.scan == "chunked"
    SOLVE_CHOLESKY = args.solve == "cholesky"
    lib = V.VDA(cfg, device=dev, cholesky=args.solve == "cholesky", chunked=SCAN_CHUNKED, heads=heads,
                split_scan=args.scan == "split")
    # Per-kernel accounting below is for the heads this rank serves.
    kcfg = cfg if heads is None else cfg.with_(H=heads[1])
    O = lib.new_output()
    stream = torch.cuda.current_stream(dev)
    if args.fp8:
        global FP8
        FP8 = True

        def run_fp8(inp, out, stream=None):
            lib.prepare_fp8(inp, stream=stream)
            lib.scan_bidir(stream=stream)
            lib.readout_fp8(inp["Q8"], inp["q_scale"], out, stream=stream)
            return out

        lib.run = run_fp8  # every step below goes through the FP8 entry points
    for _ in range(args.warmup):
        lib.run(inp_dev, O)
    torch.cuda.synchronize(dev)
    if lib.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout during warm-up")

    # ---- device-timed region: inputs resident in HBM (each step's working set,
    # ~1.5 GB at the H3-like clip, is larger than the 126 MB L2) -------------
    # The step time is taken without per-kernel events (an event pair around
    # every launch costs ~20 us per step here); a second pass of the same K
    # steps records one event pair per kernel launch for the per-kernel table
    # and the roofline.
    n0 = lib.launch_count()
    clocks = ClockSampler(local)
    barrier(dist)
    torch.cuda.synchronize(dev)
    clocks.start()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        lib.run(inp_dev, O)
    ev1.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier(dist)
    ms = ev0.elapsed_time(ev1)
    launches = lib.launch_count() - n0
    if lib.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the timed region")
    # ---- per-kernel pass: the same K steps with CUDA events around every launch
    lib.profile_enable(True)
    barrier(dist)
    torch.cuda.synchronize(dev)
    ep0, ep1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ep0.record(stream)
    for _ in range(args.steps):
        lib.run(inp_dev, O)
    ep1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist)
    ms_profiled = ep0.elapsed_time(ep1)
    prof = lib.profile_read()
    lib.profile_enable(False)
    if lib.poll_device_status() != 0:
        raise RuntimeError("device status reported a timeout in the per-kernel pass")
    ms_max = max_over_ranks(dist, ms, dev)
    value = whole_job_rate(world, cfg, args.steps, ms_max, args.shard)

    # ---- end to end through the public API: pinned host inputs -> device ->
    # prepare/scan/readout -> O back to pinned host memory, every step. The
    # steps are independent batches, so the copies are pipelined as a user
    # streaming batches would: step n+1's inputs go up on a copy stream while
    # step n computes and its output comes down on another (PCIe is full
    # duplex); inputs and outputs are double-buffered, and the compute (one
    # workspace) stays in order on the compute stream. Every step's copies lie
    # inside the timed region. --------------------------------------------------
    O_host = torch.empty(O.shape, dtype=O.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in inp_host.values())
    d2h = O.numel() * O.element_size()
    ke = max(1, min(args.e2e_steps, args.steps))
    inp_buf = [inp_dev, {k: torch.empty_like(v) for k, v in inp_dev.items()}]
    O_buf = [O, torch.empty_like(O)]
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    up_done = [ev() for _ in range(ke)]
    run_done = [ev() for _ in range(ke)]
    down_done = [ev() for _ in range(ke)]
    barrier(dist)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_stream(stream)
    down.wait_stream(stream)
    for n in range(ke):
        slot = n % 2
        with torch.cuda.stream(up):
            if n >= 2:
                up.wait_event(run_done[n - 2])  # step n-2 has finished reading this input buffer
            for k, v in inp_host.items():
                inp_buf[slot][k].copy_(v, non_blocking=True)
            up_done[n].record(up)
        stream.wait_event(up_done[n])
        if n >= 2:
            stream.wait_event(down_done[n - 2])  # step n-2's output has left this buffer
        lib.run(inp_buf[slot], O_buf[slot], stream=stream)
        run_done[n].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(run_done[n])
            O_host.copy_(O_buf[slot], non_blocking=True)
            down_done[n].record(down)
    stream.wait_stream(down)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist)
    e2e_value = whole_job_rate(world, cfg, ke, max_over_ranks(dist, e0.elapsed_time(e1), dev), args.shard)

    # ---- roofline of the dominant kernel (live per-kernel CUDA events) -------
    peaks, peak_src = load_peaks()
    dom = max(prof.items(), key=lambda kv: kv[1][1])
    dom_name, (dom_n, dom_ms) = dom
    dom_avg_s = dom_ms / dom_n / 1e3
    dom_bytes = kernel_bytes(dom_name, kcfg)
    traffic = traffic_for(dom_name, cfg.name) if heads is None else None
    if dom_name in ALU_BOUND:
        bound, unit = "alu", "TFLOP/s"
        sm_mhz = float(clocks.summary().get("sm_mhz") or 1965.0)
        achieved = kernel_alu_flops(dom_name, kcfg) / dom_avg_s / 1e12
        peak = alu_peak_tflops(sm_mhz)
        peak_note = (f"fp32 FMA peak derived: 148 SMs x 128 lanes x 2 flop x {sm_mhz:.0f} MHz "
                     f"(median SM clock in the timed region)")
    elif dom_name in TENSOR_BOUND:
        # timed inside a long step: the sustained bf16 figure is the denominator
        bound, unit = "tensor", "TFLOP/s"
        achieved = kernel_flops(dom_name, kcfg) / dom_avg_s / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
        peak_note = f"bf16_tflops_sustained of {peak_src}"
    else:
        bound, unit = "hbm", "GB/s"
        achieved = dom_bytes / dom_avg_s / 1e9
        peak = float(peaks["hbm_gbs"])
        peak_note = f"hbm_gbs of {peak_src}"
    hbm_peak = float(peaks["hbm_gbs"])
    kernels = {k: {"launches": n, "avg_us": tot / n * 1e3, "share": tot / sum(x[1] for x in prof.values()),
                   "algorithmic_GBps": kernel_bytes(k, kcfg) / (tot / n / 1e3) / 1e9,
                   "hbm_frac": kernel_bytes(k, kcfg) / (tot / n / 1e3) / 1e9 / hbm_peak,
                   "algorithmic_TFLOPs": kernel_flops(k, kcfg) / (tot / n / 1e3) / 1e12}
               for k, (n, tot) in prof.items()}

    if rank == 0:
        step_s = ms_max / 1e3 / args.steps
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak" if args.shard == "batch" else "strong", "vs_baseline": None,
            "dtype": ("e4m3 operands, fp32 accumulation and state, bf16 O" if FP8 else
                      "bf16" if cfg.dtype == "bf16" else "f32"),
            "data": "synthetic",
            "config": {"workload": workload_desc(cfg), "global_batch": cfg.B * (world if args.shard == "batch" else 1),
                       "parallelism": (f"dp{world} (independent batches, no collective)" if args.shard == "batch"
                                       else f"heads{world} (one batch, heads {heads} on rank 0, no collective)"),
                       "l2": "no flush: each step reads and writes > 1 GB, far above the 126 MB L2",
                       "path": V.describe(lib.c),
                       "stream": "one CUDA stream, kernels back to back"},
            "roofline": {"bound": bound, "kernel": dom_name, "achieved": achieved, "peak": peak,
                         "unit": unit, "frac": achieved / peak, "traffic": traffic,
                         "peak_source": peak_note,
                         "algorithmic_bytes_per_launch": dom_bytes,
                         "algorithmic_flops_per_launch": kernel_flops(dom_name, kcfg),
                         "alu_flops_per_launch": kernel_alu_flops(dom_name, kcfg) or None},
            "path_roofline": {"algorithmic_bytes_per_step": path_bytes(kcfg),
                              "hbm_GBps": path_bytes(kcfg) / step_s / 1e9,
                              "hbm_frac": path_bytes(kcfg) / step_s / 1e9 / hbm_peak,
                              "tflops": path_flops(kcfg) / step_s / 1e12,
                              "tensor_frac_of_bf16_burst": path_flops(kcfg) / step_s / 1e12 / float(peaks["bf16_tflops"])},
            "kernels": kernels,
            "kernel_pass": {"steps": args.steps, "ms_per_step": ms_profiled / args.steps,
                            "note": "per-kernel times, shares and the roofline come from this second pass of "
                                    "the same steps with a CUDA event pair around every launch; ms_per_step "
                                    "and value come from the first pass without them"},
            "gpu_launches": launches,
            "clocks": clocks.summary(),
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": ke},
        }
        if world == 1 and args.cpu_budget > 0:
            line["cpu_baseline"] = cpu_baseline(cfg, x8 if args.fp8 else inp_cpu, budget_s=args.cpu_budget)
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
