"""Benchmark: fused forward + backward of the full-vocabulary distillation loss.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl library|reference]

One step = nb_kl_forward + nb_kl_backward over one batch of the workload (every step of
the hot path: compaction, both block GEMMs with the online LSE/KL epilogue, split-V merge,
[JSD second sweep], masked mean, recompute sweep, dh_s and dW_s GEMMs). Inputs are resident
in HBM when the timed region starts; the unembeddings (>= 1 GB per step) are larger than
L2, so no explicit flush is needed between steps. The timed region is bracketed by a
barrier and a device synchronisation and timed with CUDA events on the launching stream;
with N > 1 every rank runs its own replica (no data-path collective) and the time is the
maximum over ranks.

Prints one JSON line. `value` is whole-job tokens/s (all B*T positions of every rank);
`e2e` repeats the measurement through the public API with the step's inputs copied from
pinned host memory and the loss read back each step; `roofline` describes the dominant
kernel; `cpu_baseline` times the fp64 oracle on a bounded sample on this host.
"""

from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "distill-loss tokens/sec (fwd+bwd) at V=151936; % of bf16 tensor peak"
DATASHEET_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DEFAULT_WORKLOAD = "opd_0p6b_4b"


# ----------------------------------------------------------------------------- helpers
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK), "fallback"


# SM clock of the sustained cuBLAS measurement when the peaks file does not record it (the
# median under load of the pool's sustained run) and the boost clock of the part
SUSTAINED_MHZ_DEFAULT = 1275.0
MAX_MHZ_DEFAULT = 1965.0


def _flat(d, prefix=""):
    for k, v in (d.items() if isinstance(d, dict) else []):
        key = f"{prefix}.{k}" if prefix else str(k)
        if isinstance(v, dict):
            yield from _flat(v, key)
        else:
            yield key.lower(), v


def peak_clocks(peaks):
    """(burst MHz, sustained MHz) of the peak measurements, from the peaks file's clock fields
    where it records them (a key naming a clock and the run), else the defaults."""
    burst, sustained = None, None
    for k, v in _flat(peaks):
        if not isinstance(v, (int, float)) or not ("mhz" in k or "clock" in k):
            continue
        if "sustained" in k and ("median" in k or sustained is None):
            sustained = float(v)
        elif "burst" in k and burst is None:
            burst = float(v)
    return burst, sustained if sustained is not None else SUSTAINED_MHZ_DEFAULT


def choose_peak(peaks, src, run_mhz, max_mhz):
    """The dense bf16 peak that applies at the clock the timed run held: the burst figure when
    the run's median SM clock under load is within 5% of the burst measurement's clock (the
    part's maximum when that is not recorded), the sustained figure when it is within 5% of the
    sustained measurement's clock, else the burst figure scaled by the clock ratio."""
    burst = float(peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"]))
    b_mhz, s_mhz = peak_clocks(peaks)
    b_mhz = b_mhz or max_mhz or MAX_MHZ_DEFAULT
    if not run_mhz:
        return burst, f"{src} bf16_tflops (burst; no clock record for this run)", b_mhz
    if run_mhz >= 0.95 * b_mhz:
        return burst, f"{src} bf16_tflops (burst, measured near {b_mhz:.0f} MHz)", b_mhz
    if abs(run_mhz - s_mhz) <= 0.05 * s_mhz:
        return sustained, f"{src} bf16_tflops_sustained (measured near {s_mhz:.0f} MHz)", s_mhz
    return burst * run_mhz / b_mhz, f"{src} bf16_tflops x {run_mhz:.0f} / {b_mhz:.0f} MHz (burst at the run's clock)", run_mhz


def algorithmic_flops(w, n_valid, V=None, proj=0.0):
    """FLOPs of the method on valid rows: forward sweep, [JSD second sweep], recompute sweep,
    dh_s and dW_s products (V: the vocabulary rows this rank holds), and the teacher-code
    projection of the spectral front end (`proj`, all positions)."""
    V = w.V if V is None else V
    sweep = 2.0 * n_valid * V * (w.d_s + w.d_t)
    jsd = 0.0 < w.beta < 1.0
    return {
        "sweep_fwd": sweep,
        "sweep_jsd": sweep if jsd else 0.0,
        "sweep_grad": sweep,
        "gemm_bwd": 4.0 * n_valid * V * w.d_s,
        "gemm_proj": proj,
    }


def model_flops(w, n_valid, V=None) -> float:
    """The stricter count with no recompute: one forward sweep over both models plus the dh_s and
    dW_s products (the JSD's second sweep and the backward's recompute sweep are left out)."""
    V = w.V if V is None else V
    return 2.0 * n_valid * V * (w.d_s + w.d_t) + 4.0 * n_valid * V * w.d_s


# headers that define the profiled tensor-core kernels (the vocabulary sweep and the GEMM)
PROFILED_SOURCES = ("common.cuh", "gemm.cuh", "ptx.cuh", "sweep.cuh")


def _code_only(text: str) -> str:
    """C++ source without comments and with whitespace collapsed: what the compiler sees."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha():
    """Hash of the sweep and GEMM device code (comments and layout ignored): a profile summary
    is only used while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "full_vocab_kl_b200", "csrc")
    for name in PROFILED_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


# profiling-size workload with the same token shape as a bench workload (its ncu summaries carry the
# per-launch DRAM bytes of each kernel)
PROFILE_OF = {"opd_0p6b_4b": "opd_0p6b_4b_v24k_prof"}


def profiled_traffic(kernel: str, workload: str, columns_per_launch: float):
    """DRAM bytes (read + write) of one launch of `kernel`, from the committed ncu summary of the
    workload's profiling-size twin (same tokens, smaller vocabulary), scaled by the vocabulary
    columns one launch covers: the unembedding rows, the gradient chunk and the dW_s rows grow in
    proportion to them. None unless that summary was taken from the current device code."""
    prof = PROFILE_OF.get(workload)
    if prof is None:
        return None
    p = os.path.join(ROOT, "profiles", f"{kernel}_{prof}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    m_c = re.search(r"profiled_vocab_columns_per_launch:\s*([0-9]+)", txt)
    if not (m_sha and m_b and m_c) or m_sha.group(1) != kernel_source_sha():
        return None
    return float(m_b.group(1)) * columns_per_launch / float(m_c.group(1))


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = f"/tmp/nbkl_clocks_{os.getpid()}.csv"

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.remove(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        busy = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": float(np.median(busy)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": float(max(power)) if power else None}


# ----------------------------------------------------------------------------- oracle timing
def oracle_sample_run(x, positions):
    """One oracle pass (forward + backward incl. dW_s) over the given positions only."""
    import oracle
    sub = np.full_like(x.labels, -100)
    sub[positions] = x.labels[positions]
    oracle.forward(x.h_s, x.W_s, x.h_t, x.W_t, sub, x.beta, x.tau)
    oracle.backward(x.h_s, x.W_s, x.h_t, x.W_t, sub, x.beta, x.tau, grad_out=x.grad_out)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:  # pragma: no cover
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(x, min_s=10.0, max_positions=None):
    """Oracle throughput on random positions of the workload: the sample doubles until one
    timed run takes at least `min_s` seconds (the oracle has a large fixed cost per call)."""
    rng = np.random.default_rng(7)
    N = x.labels.shape[0]
    cap = N if max_positions is None else min(N, max_positions)
    n = min(64, cap)
    while True:
        pos = np.sort(rng.choice(N, size=n, replace=False))
        t0 = time.perf_counter()
        oracle_sample_run(x, pos)
        dt = time.perf_counter() - t0
        if dt >= min_s or n >= cap:
            break
        n = min(cap, 2 * n)
    nv = int((x.labels[pos] != -100).sum())
    return {"value": n / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} of {N} positions ({nv} valid) of workload {x.workload.name}, "
                      f"forward + backward incl. dW_s, fp64 NumPy, {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from synthetic import make_inputs
    x = make_inputs(args.workload)
    N = x.labels.shape[0]
    rng = np.random.default_rng(11)
    budget = 150.0 / max(1, args.steps + args.warmup)
    t0 = time.perf_counter()
    oracle_sample_run(x, np.sort(rng.choice(N, size=32, replace=False)))
    per_pos = (time.perf_counter() - t0) / 32
    n = int(max(16, min(N, budget / max(per_pos, 1e-6))))
    for _ in range(args.warmup):
        oracle_sample_run(x, np.sort(rng.choice(N, size=n, replace=False)))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_run(x, np.sort(rng.choice(N, size=n, replace=False)))
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    w = x.workload
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, int((x.labels != -100).sum()), 1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{n} random positions of {N} per step, forward + backward incl. dW_s"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def max_over_ranks(value: float, world: int, device) -> float:
    """Maximum of a per-rank scalar (elapsed ms) over the process group."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: int, world: int, ms_per_step: float) -> float:
    """Units of all ranks per second (every rank runs its own replica of the step)."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def workload_config(w, n_valid, world):
    return {"workload": w.name, "global_batch": w.B * world, "seq_len": w.T, "tokens_per_rank": w.N,
            "valid_tokens_per_rank": n_valid, "vocab": w.V, "d_s": w.d_s, "d_t": w.d_t, "beta": w.beta,
            "tau": w.tau, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": "inputs larger than L2 (unembeddings >= 1 GB per step), no flush"}


# ----------------------------------------------------------------------------- other workloads
EXTRA_WORKLOADS = ("long_jsd", "large_vocab", "spectral")


def measure_workload(name, steps, warmup, dev, gpu_index):
    """Device-timed forward + backward of one more workload with its inputs resident, timed with
    CUDA events on the launching stream and with its own clock record (one GPU)."""
    import torch

    import full_vocab_kl_b200 as nb
    from synthetic import make_inputs
    x = make_inputs(name)
    w = x.workload
    nv = int((x.labels != -100).sum())

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    h_s, h_t, W_s, W_t = (to_dev(getattr(x, k)) for k in ("h_s", "h_t", "W_s", "W_t"))
    labels = torch.from_numpy(x.labels).to(dev)
    N = labels.shape[0]
    f32 = dict(dtype=torch.float32, device=dev)
    shape = nb.make_shape(h_s, W_s, h_t, W_t, labels)
    ws = torch.empty(nb.workspace_bytes(shape, w.beta), dtype=torch.uint8, device=dev)
    out = {"loss_tok": torch.empty(N, **f32), "lse_s": torch.empty(N, **f32), "lse_t": torch.empty(N, **f32),
           "aux": torch.empty(N, **f32), "loss_mean": torch.empty((), **f32),
           "n_valid": torch.empty((), dtype=torch.int64, device=dev)}
    dh = torch.empty((N, w.d_s), **f32)
    dW = (torch.from_numpy(x.dW_init).to(dev) if w.accumulate_dW else torch.empty((w.V, w.d_s), **f32))
    go = torch.ones((), **f32)

    def step():
        nb.kl_forward(h_s, W_s, h_t, W_t, labels, w.beta, w.tau, workspace=ws, out=out)
        nb.kl_backward(h_s, W_s, h_t, W_t, labels, w.beta, w.tau, out["lse_s"], out["lse_t"], out["aux"], go,
                       dh_s=dh, dW_s=dW, accumulate_dW=w.accumulate_dW, workspace=ws)

    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        step()
    clocks = ClockSampler(gpu_index)
    clocks.start()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    status = nb.device_status(ws)
    ms = e0.elapsed_time(e1) / steps
    flops = sum(algorithmic_flops(w, nv).values())
    tflops = flops / (ms * 1e-3) / 1e12
    res = {"workload": name, "tokens": N, "valid_tokens": nv, "vocab": w.V, "d_s": w.d_s, "d_t": w.d_t,
           "beta": w.beta, "tau": w.tau, "accumulate_dW": w.accumulate_dW, "steps": steps, "warmup": warmup,
           "ms_per_step": ms, "tokens_per_s": N / (ms * 1e-3), "tflops": tflops,
           "pct_bf16_peak_datasheet": 100.0 * tflops / DATASHEET_BF16_TFLOPS,
           "device_status": int(status), "clocks": clk}
    del h_s, h_t, W_s, W_t, ws, dW, dh
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- library arm
def run_library(args):
    import torch
    import torch.distributed as dist

    import full_vocab_kl_b200 as nb
    from full_vocab_kl_b200 import _abi
    from synthetic import make_inputs

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    x = make_inputs(args.workload)
    w = x.workload
    n_valid = int((x.labels != -100).sum())

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    h_s, h_t, W_s, W_t = (to_dev(getattr(x, k)) for k in ("h_s", "h_t", "W_s", "W_t"))
    labels = torch.from_numpy(x.labels).to(dev)
    N = labels.shape[0]
    f32 = dict(dtype=torch.float32, device=dev)
    lib = _abi.lib()
    grad_out = torch.ones((), **f32)
    V_rank, proj_flops, mode_cfg = w.V, 0.0, {}

    if args.front_end:
        # spectral front end: a full-width teacher (Gaussian unembedding, RMS-normalised hidden
        # states, drawn on the device from a seeded generator) compressed to the workload's rank
        from full_vocab_kl_b200 import spectral
        gen = torch.Generator(device=dev)
        gen.manual_seed(1000 + rank)
        d_full = args.teacher_width
        W_full = (torch.randn((w.V, d_full), generator=gen, device=dev) * (w.w_std / d_full ** 0.5)).to(
            torch.bfloat16)
        h_full = torch.randn((N, d_full), generator=gen, device=dev)
        h_full = (h_full / (h_full.pow(2).mean(1, keepdim=True) + 1e-6).sqrt()).to(torch.bfloat16)
        basis = spectral.spectral_factor(W_full, w.d_t)
        W_t = basis.W_code
        code = torch.empty((N, w.d_t), dtype=torch.bfloat16, device=dev)
        h_t = h_full
        del W_full
        proj_flops = 2.0 * N * d_full * w.d_t
        mode_cfg = {"front_end": "spectral", "teacher_width": d_full, "rank": w.d_t}

    if args.vocab_parallel:
        from full_vocab_kl_b200.vocab_parallel import LibraryKernels, shard_range, vp_backward, vp_forward
        v0, v1 = shard_range(w.V, rank, world)
        W_s, W_t = W_s[v0:v1].contiguous(), W_t[v0:v1].contiguous()
        V_rank = v1 - v0
        mode_cfg.update({"vocab_shard_rows": V_rank})

        class CountingKernels(LibraryKernels):
            launches = 0

            def _count(self, r):
                CountingKernels.launches += lib.nb_kl_last_launch_count()
                return r

            def state(self, *a, **k):
                return self._count(super().state(*a, **k))

            def combine(self, *a, **k):
                return self._count(super().combine(*a, **k))

            def jsd_partial(self, *a, **k):
                return self._count(super().jsd_partial(*a, **k))

            def jsd_combine(self, *a, **k):
                return self._count(super().jsd_combine(*a, **k))

            def backward(self, *a, **k):
                return self._count(super().backward(*a, **k))

        kern = CountingKernels()
        gather = (lambda t: t[None].contiguous()) if world == 1 else None
        reduce = (lambda t: t) if world == 1 else None
        vp_ws = {}

    if args.handoff:
        # the teacher's hidden rows arrive through the hand-off copy (valid rows only) into a
        # local buffer that the loss then reads; the buffer passed to `step` stands for the
        # teacher's memory (another GPU's, or an IPC mapping, in a two-GPU deployment)
        from full_vocab_kl_b200 import handoff
        ht_local = torch.zeros_like(h_t)
        handoff_bytes = n_valid * h_t.shape[1] * h_t.element_size()
        mode_cfg["handoff_bytes_per_step"] = handoff_bytes

    shape = nb.make_shape(h_s, W_s, code if args.front_end else h_t, W_t, labels, chunk_v=args.chunk_v)
    ws_bytes = nb.workspace_bytes(shape, w.beta)
    ws = None if args.vocab_parallel else torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    out = {"loss_tok": torch.empty(N, **f32), "lse_s": torch.empty(N, **f32), "lse_t": torch.empty(N, **f32),
           "aux": torch.empty(N, **f32), "loss_mean": torch.empty((), **f32),
           "n_valid": torch.empty((), dtype=torch.int64, device=dev)}
    if args.side:
        out["entropy_s"] = torch.empty(N, **f32)
        out["logp_label"] = torch.empty(N, **f32)
    dh = torch.empty((N, w.d_s), **f32)
    dW = torch.zeros((V_rank, w.d_s), **f32) if w.accumulate_dW else torch.empty((V_rank, w.d_s), **f32)

    def step(hs, ht, lab, marks=None):
        """One forward + backward; with `marks`, events on the launching stream bracket the
        backward call (its kernels, including any on the library's second stream, which the
        call joins back before it returns)."""
        if args.vocab_parallel:
            CountingKernels.launches = 0
            f = vp_forward(hs, W_s, ht, W_t, lab, w.beta, w.tau, vocab_offset=v0, side=args.side, kernels=kern,
                           all_gather=gather)
            vp_backward(hs, W_s, ht, W_t, lab, w.beta, w.tau, f["lse_s"], f["lse_t"], f["aux"], grad_out,
                        kernels=kern, workspace=f["workspace"], all_reduce=reduce)
            out["loss_mean"], out["n_valid"] = f["loss_mean"], f["n_valid"]
            return CountingKernels.launches
        n0 = 0
        if args.handoff:
            ht = handoff.receive_rows(ht, lab, out=ht_local)
            n0 += lib.nb_kl_last_launch_count()
        if args.front_end:
            spectral.project(ht, basis.V_k, out=code)
            n0 += lib.nb_kl_last_launch_count()
            ht = code
        nb.kl_forward(hs, W_s, ht, W_t, lab, w.beta, w.tau, workspace=ws, out=out, chunk_v=args.chunk_v,
                      side=args.side)
        n1 = lib.nb_kl_last_launch_count()
        if marks is not None:
            marks.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            marks[-1][0].record(stream)
        nb.kl_backward(hs, W_s, ht, W_t, lab, w.beta, w.tau, out["lse_s"], out["lse_t"], out["aux"], grad_out,
                       dh_s=dh, dW_s=dW, accumulate_dW=w.accumulate_dW, workspace=ws, chunk_v=args.chunk_v)
        if marks is not None:
            marks[-1][1].record(stream)
        return n0 + n1 + lib.nb_kl_last_launch_count()

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        step(h_s, h_t, labels)
    mem0 = torch.cuda.memory_allocated(dev)
    torch.cuda.reset_peak_memory_stats(dev)

    # ---- device-timed region (the headline): the library's per-launch timing hook is off
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    launches = 0
    for _ in range(args.steps):
        launches += step(h_s, h_t, labels)
    e1.record(stream)
    barrier()
    clk = clocks.stop() if rank == 0 else None
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    peak_extra = torch.cuda.max_memory_allocated(dev) - mem0

    # ---- per-kernel pass, after the headline and not part of it: the same number of steps
    # with the library's per-launch events on (each launch bracketed on its own stream) and
    # every backward call bracketed on the launching stream
    clocks_k = ClockSampler(local)
    if rank == 0:
        clocks_k.start()
    lib.nb_kl_timing_enable(1)
    barrier()
    marks = []
    ek0, ek1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ek0.record(stream)
    for _ in range(args.steps):
        step(h_s, h_t, labels, marks=None if args.vocab_parallel else marks)
    ek1.record(stream)
    barrier()
    lib.nb_kl_timing_enable(0)
    clk_k = clocks_k.stop() if rank == 0 else None
    ncat = len(_abi.KERNEL_CATEGORIES)
    ms_arr = (ctypes.c_double * ncat)()
    cnt_arr = (ctypes.c_int * ncat)()
    lib.nb_kl_timing_read(ctypes.cast(ms_arr, ctypes.c_void_p), ctypes.cast(cnt_arr, ctypes.c_void_p), ncat)
    ms_kpass = ek0.elapsed_time(ek1) / args.steps
    bwd_ms = (sum(a.elapsed_time(b) for a, b in marks) / len(marks)) if marks else None

    # ---- end-to-end through the public API with host buffers: every step copies its inputs
    # from pinned host memory and reads its loss back; the copy of step i + 1's inputs runs on
    # a second stream into the other of two device buffers while step i computes, and the host
    # reads step i - 1's loss while step i is queued (as a training loop that logs each step's
    # loss without stalling the device), the last one after the loop, inside the timed region
    pin = {}
    for k, t in (("h_s", h_s), ("h_t", h_t), ("labels", labels)):
        pin[k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        pin[k].copy_(t)
    loss_host = torch.empty((2, 2), dtype=torch.float64, pin_memory=True)   # [slot][loss, n_valid]
    bufs = [tuple(torch.empty_like(t) for t in (h_s, h_t, labels)) for _ in range(2)]
    ready = [torch.cuda.Event() for _ in range(2)]   # inputs of buffer b copied
    used = [torch.cuda.Event() for _ in range(2)]    # last step reading buffer b done
    read = [torch.cuda.Event() for _ in range(2)]    # loss of slot b copied to the host
    copy_stream = torch.cuda.Stream(dev)
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = out["loss_mean"].element_size() + out["n_valid"].element_size()
    e2e_steps = max(3, args.steps)   # as many steps as the device-timed region

    def issue_copy(i, first):
        # buffer i % 2 was last read by step i - 2: the copy waits for that step on the device
        b = i % 2
        with torch.cuda.stream(copy_stream):
            if not first:
                copy_stream.wait_event(used[b])
            for dst, k in zip(bufs[b], ("h_s", "h_t", "labels")):
                dst.copy_(pin[k], non_blocking=True)
            ready[b].record(copy_stream)

    def e2e_run(n, e_start=None):
        if e_start is not None:
            e_start.record(copy_stream)
        issue_copy(0, True)
        losses = []
        for i in range(n):
            b = i % 2
            stream.wait_event(ready[b])
            step(*bufs[b])
            used[b].record(stream)
            if i + 1 < n:
                issue_copy(i + 1, i + 1 < 2)
            loss_host[b, 0].copy_(out["loss_mean"], non_blocking=True)
            loss_host[b, 1].copy_(out["n_valid"], non_blocking=True)
            read[b].record(stream)
            if i >= 1:   # step i - 1's loss, read while step i is queued
                read[1 - b].synchronize()
                losses.append(float(loss_host[1 - b, 0]))
        read[(n - 1) % 2].synchronize()
        losses.append(float(loss_host[(n - 1) % 2, 0]))
        assert len(losses) == n
        return losses[-1]

    e2e_run(2)
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e2)
    e3.record(stream)
    barrier()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), world, dev)

    result = None
    if rank == 0:
        ms_step = ms / args.steps
        tokens = N * world
        # vocabulary-parallel ranks share one batch (strong scaling); otherwise each rank runs its own
        units = N if args.vocab_parallel else N * world
        value = units / (ms_step * 1e-3)
        flops = algorithmic_flops(w, n_valid, V=V_rank, proj=proj_flops)
        step_flops = sum(flops.values()) * world
        tflops = step_flops / (ms_step * 1e-3) / 1e12
        peaks, peak_src = measured_peaks()
        cats = _abi.KERNEL_CATEGORIES
        kms = {c: ms_arr[i] / args.steps for i, c in enumerate(cats)}
        kcount = {c: cnt_arr[i] / args.steps for i, c in enumerate(cats)}
        dom = max(("sweep_fwd", "sweep_jsd", "sweep_grad", "gemm_bwd", "gemm_proj"), key=lambda c: kms[c])
        per_launch_ms = kms[dom] / max(kcount[dom], 1)
        per_launch_flops = flops[dom] / max(kcount[dom], 1)
        achieved = per_launch_flops / (per_launch_ms * 1e-3) / 1e12
        run_mhz = (clk_k or {}).get("sm_mhz") or (clk or {}).get("sm_mhz")
        max_mhz = (clk or {}).get("sm_max_mhz")
        peak, peak_desc, peak_mhz = choose_peak(peaks, peak_src, run_mhz, max_mhz)
        step_peak, step_peak_desc, _ = choose_peak(peaks, peak_src, (clk or {}).get("sm_mhz"), max_mhz)
        # the backward as one unit: gradient sweeps and GEMMs over the backward call's span
        bwd_unit = None
        if bwd_ms:
            bwd_flops = flops["sweep_grad"] + flops["gemm_bwd"]
            bwd_unit = {"ms": bwd_ms, "flops": bwd_flops, "tflops": bwd_flops / (bwd_ms * 1e-3) / 1e12,
                        "frac": bwd_flops / (bwd_ms * 1e-3) / 1e12 / peak,
                        "note": "gradient sweeps + dh_s/dW_s GEMMs (+ the call's row kernels) between events "
                                "bracketing each backward call on the launching stream"}
        chunk_cols = lib.nb_kl_chunk_columns(_abi.shape_ptr(shape))
        cols_per_launch = V_rank / max(kcount[dom], 1) if dom != "gemm_proj" else 0.0
        traffic = (profiled_traffic(dom, w.name, cols_per_launch)
                   if not (args.vocab_parallel or args.front_end) else None)
        config = workload_config(w, n_valid, world)
        if args.vocab_parallel:
            config["parallelism"] = f"vocab{world}"
        if args.side:
            config["side_outputs"] = True
        config.update(mode_cfg)
        result = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if args.vocab_parallel else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; shapes of the workload)",
            "config": config,
            "tflops": tflops, "pct_bf16_peak_datasheet": 100.0 * tflops / DATASHEET_BF16_TFLOPS,
            "model_tflops": model_flops(w, n_valid, V_rank) * world / (ms_step * 1e-3) / 1e12,
            "pct_bf16_peak_measured": 100.0 * tflops / peaks.get("bf16_tflops", FALLBACK["bf16_tflops"]),
            "pct_bf16_peak_at_run_clock": 100.0 * tflops / step_peak, "step_peak_source": step_peak_desc,
            "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                         "peak_source": peak_desc, "peak_clock_mhz": peak_mhz, "run_sm_mhz": run_mhz,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_flops_per_launch": per_launch_flops, "launch_ms": per_launch_ms,
                         "traffic_source": ("ncu DRAM bytes of the profiling-size twin workload, scaled by the "
                                            "vocabulary columns per launch") if traffic else None,
                         "timed_in": "per-kernel pass after the headline (same steps, per-launch events on)"},
            "backward_unit": bwd_unit,
            "kernel_ms_per_step": kms, "kernel_launches_per_step": kcount,
            "kernel_pass": {"ms_per_step": ms_kpass, "kernel_ms_sum": sum(kms.values()), "clocks": clk_k},
            "kernel_tflops": {c: (flops[c] / (kms[c] * 1e-3) / 1e12 if kms[c] > 0 else None)
                              for c in ("sweep_fwd", "sweep_jsd", "sweep_grad", "gemm_bwd", "gemm_proj")},
            "e2e": {"value": units / (ms_e2e / e2e_steps * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "pipelining": "inputs of step i + 1 copied on a second stream during step i; the host reads step i's loss while step i + 1 is queued, the last one inside the timed region"},
            "gpu_launches": launches,
            **({"handoff": {"bytes_per_step": handoff_bytes, "ms_per_step": kms["handoff"],
                            "gbs": (2.0 * handoff_bytes / (kms["handoff"] * 1e-3) / 1e9) if kms["handoff"] else None,
                            "note": "read + write bytes over the copy's device time; one GPU: HBM to HBM"}}
               if args.handoff else {}),
            "clocks": clk,
            "scratch_bytes": ws_bytes, "peak_extra_alloc_bytes": int(peak_extra), "chunk_v": chunk_cols,
        }
    plain = not (args.vocab_parallel or args.front_end or args.handoff or args.side)
    if rank == 0 and world == 1 and plain and args.sustained > 0:
        result["sustained"] = measure_sustained(lambda: step(h_s, h_t, labels), ms / args.steps,
                                                step_flops, args.sustained, dev, local)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and world == 1 and plain and args.workload == DEFAULT_WORKLOAD and not args.no_workloads:
        # the other workloads of the method's configuration list, each timed on its own
        del ws, dW, dh, W_s, W_t
        torch.cuda.empty_cache()
        wl = [measure_workload(n, args.workload_steps, args.warmup, dev, local) for n in EXTRA_WORKLOADS]
        result["workloads"] = wl
        result["workloads_weakest"] = min(wl, key=lambda r: r["tflops"])["workload"]
    if rank == 0 and not args.no_cpu_baseline and not args.front_end:
        result["cpu_baseline"] = cpu_baseline(x)
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def measure_sustained(step, ms_step, step_flops, seconds, dev, gpu_index):
    """Throughput under the board's power cap: back-to-back steps for about `seconds`, then a
    cuBLAS bf16 GEMM (8192 x 8192 x 8192, torch.matmul) loop for as long, each device-timed with
    its own clock record. The GEMM is a reference point for the same power budget, measured in
    the same process; it is not part of the loss path."""
    import torch

    def loop(fn, iters):
        clocks = ClockSampler(gpu_index)
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / iters, clocks.stop()
    iters = max(3, int(seconds * 1e3 / ms_step))
    ms, clk = loop(step, iters)
    n = 8192
    A = torch.randn(n, n, device=dev).to(torch.bfloat16)
    B = torch.randn(n, n, device=dev).to(torch.bfloat16)
    torch.matmul(A, B)
    torch.cuda.synchronize()
    t0 = time.time()
    torch.matmul(A, B)
    torch.cuda.synchronize()
    g_ms, g_clk = loop(lambda: torch.matmul(A, B), max(3, int(seconds / max(time.time() - t0, 1e-4))))
    tf, g_tf = step_flops / (ms * 1e-3) / 1e12, 2.0 * n ** 3 / (g_ms * 1e-3) / 1e12
    return {"seconds": seconds, "steps": iters, "ms_per_step": ms, "tflops": tf, "clocks": clk,
            "cublas_bf16_gemm": {"shape": [n, n, n], "tflops": g_tf, "clocks": g_clk},
            "tflops_vs_cublas": tf / g_tf}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="a workload name (synthetic.WORKLOADS) or a profiling-size one (synthetic.PROFILE_WORKLOADS)")
    ap.add_argument("--impl", default="library", choices=["library", "reference"])
    ap.add_argument("--chunk-v", type=int, default=0, help="backward vocabulary chunk (0: library default)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sustained", type=float, default=0.0,
                    help="also run about this many seconds of back-to-back steps, then as long a cuBLAS "
                         "bf16 GEMM loop, under the power cap (0: off)")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the device-timed lines of the other workloads (long_jsd, large_vocab, spectral)")
    ap.add_argument("--workload-steps", type=int, default=10, help="timed steps of each other workload")
    ap.add_argument("--side", action="store_true",
                    help="forward with the student entropy / sampled-token log-prob side outputs")
    ap.add_argument("--vocab-parallel", action="store_true",
                    help="shard the unembeddings by rows over the ranks (one batch, strong scaling)")
    ap.add_argument("--front-end", choices=["spectral"], default=None,
                    help="time the teacher-code projection of a full-width teacher with the loss")
    ap.add_argument("--handoff", action="store_true",
                    help="the teacher's hidden rows reach the loss through the hand-off copy")
    ap.add_argument("--teacher-width", type=int, default=4096,
                    help="hidden width of the full teacher for --front-end spectral")
    args = ap.parse_args()
    if sum(map(bool, (args.front_end, args.vocab_parallel, args.handoff))) > 1:
        ap.error("--front-end, --vocab-parallel and --handoff are separate measurements")
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_library(args)


if __name__ == "__main__":
    sys.exit(main())
