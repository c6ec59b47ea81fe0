#!/usr/bin/env python
"""Benchmark of the Muon optimizer step (GPT-2 124M: 48 hidden matrices) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gpt2_124m]

One JSON line on stdout (rank 0).  A "step" is one full Muon optimizer step
over all matrices of the workload: momentum + Nesterov + Frobenius norm + bf16
cast (one kernel), 5 quintic Newton-Schulz iterations (Gram, polynomial and
X-update kernels, grouped over all matrices), and the fused parameter update.

* value     ms per step, inputs resident in HBM, CUDA events on the launching
            stream around exactly K steps (barrier + synchronize on both
            sides, max over ranks).  Gradients cycle through 4 pre-generated
            sets (1.36 GB, larger than L2), so no step reads a warm L2.
* e2e       the same step through the public API from pinned host memory:
            every step copies its gradients host->device and reads the
            updated parameters back device->host inside the timed region; the
            copies run on their own streams and overlap the optimizer work of
            the neighbouring steps (PCIe is full duplex).
* roofline  the dominant kernel (largest share of device time), timed live
            with CUDA events bracketing each of its launches in a timed pass
            of the same K steps run just before the headline pass (the
            bracketing events would add about 4% to the headline pass),
            against MEASURED_PEAKS.json.
* cpu_baseline  the CPU oracle (fp64 NumPy, emulated bf16) on a bounded sample
            (one GPT-2 block, 4 matrices), scaled to the full step.
* adamw     a side measurement, not part of the step above: one AdamW step
            over the GPT-2 124M parameters Muon leaves out (embeddings,
            LayerNorm and bias vectors; 100 tensors, 39.5M elements), timed
            the same way, with its HBM roofline (28 algorithmic bytes per
            element).

Under torchrun (N > 1) every rank runs its own independent 48-matrix step on
its own GPU with its own seed (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import (ADAMW_WORKLOADS, SQUARE_SWEEP, WORKLOADS, AdamWStream,  # noqa: E402
                       WorkloadStream, square_case)

METRIC = "Muon step ms, GPT-2 124M 48 mats; Newton-Schulz bf16 TFLOP/s vs tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
N_GRAD_SETS = 4
KINDS = ("momentum_norm_cast", "gram", "poly", "xupdate", "xupdate_final", "apply", "ns_chain")
ADAMW_BYTES_PER_ELEMENT = 28.0     # read p, g, m, v; write p, m, v (fp32)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="gpt2_124m",
                    choices=sorted(WORKLOADS) + [f"square_{n}" for n in SQUARE_SWEEP])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-adamw", action="store_true", help="skip the AdamW side measurement")
    ap.add_argument("--sharded", action="store_true",
                    help="matrix-sharded step: the ranks split one problem's matrices and "
                         "all-gather the parameters (strong scaling)")
    ap.add_argument("--adamw-only", action="store_true",
                    help="run only the AdamW side measurement (for profiling that kernel)")
    return ap.parse_args()


def workload_config(wl):
    shapes = sorted(set(wl.shapes), key=lambda s: wl.shapes.index(s))
    return {
        "workload": f"{wl.name}: {wl.n_matrices} fp32 matrices "
                    f"({', '.join(f'{r}x{c}' for r, c in shapes)}), "
                    f"grads rank-{wl.grad_rank} + {wl.grad_noise} noise, "
                    f"momentum N(0,{wl.buf_std}^2), lr {wl.lr}, beta {wl.beta}, "
                    f"nesterov, {wl.ns_steps} NS steps, coeffs {list(wl.coeffs)}",
        "matrices": wl.n_matrices,
        "elements": wl.n_elements,
        "ns_flop_per_step": wl.ns_flops(),
        "l2": f"inputs larger than L2: {N_GRAD_SETS} gradient sets cycled "
              f"({N_GRAD_SETS * wl.n_elements * 4 / 1e9:.2f} GB) + params + momentum",
        "precision": "fp32 momentum/norm/update; Newton-Schulz bf16 operands, fp32 accumulation",
    }


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"],
                    source="fallback")


# ---------------------------------------------------------------- algorithmic work per launch

def per_launch_work(wl):
    """Algorithmic FLOPs (tensor kernels) or bytes (HBM kernels) per launch."""
    g = p = u = 0.0
    for r, c in wl.shapes:
        m, n = min(r, c), max(r, c)
        g += m * m * n          # Gram, upper triangle
        p += m ** 3             # symmetric square
        u += 2 * m * m * n      # X update
    el = wl.n_elements
    k = wl.ns_steps
    return {
        "momentum_norm_cast": ("hbm", 14.0 * el),     # read g, buf; write buf (fp32); write X0 (bf16)
        "gram": ("tensor", g),
        "poly": ("tensor", p),
        "xupdate": ("tensor", u),
        "xupdate_final": ("tensor", u),
        "apply": ("hbm", 10.0 * el),
        # one launch: every Gram, polynomial and X-update phase but the last update
        "ns_chain": ("tensor", (g + p) * k + u * max(0, k - 1)),
    }


# The sources each kernel's code and launch configuration come from.
KIND_SOURCES = {
    "momentum_norm_cast": ("momentum.cu",),
    "gram": ("ns_gemm.cu",), "poly": ("ns_gemm.cu",), "xupdate": ("ns_gemm.cu",),
    "xupdate_final": ("ns_gemm.cu",), "apply": ("momentum.cu",), "ns_chain": ("ns_gemm.cu",),
    "adamw": ("adamw.cu",),
}
_SHARED_SOURCES = ("internal.h", "ptx.cuh", "muon_api.cu")


def _code_only(text: str) -> str:
    """Source text without comments and blank space, so that editing a
    comment does not mark a kernel as changed."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.strip() for line in text.splitlines() if line.strip())


def source_hash(kind):
    """Hash of the code that defines one kernel kind (its .cu file, the
    shared headers and the host file that configures its launches)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "newton_schulz_norm_b200", "csrc")
    for name in sorted(KIND_SOURCES[kind] + _SHARED_SOURCES):
        with open(os.path.join(csrc, name)) as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kind):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current sources of that kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic_gpt2_124m.txt")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    ent = d.get("kernels", {}).get(kind)
    if ent is None or ent.get("source_hash") != source_hash(kind):
        return None
    return float(ent["bytes_per_launch"])


# ---------------------------------------------------------------- clocks

def start_clocks(torch, dev):
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    clocks = ClockSampler(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
    clocks.start()
    return clocks


class ClockSampler:
    """SM clock, power and clock-event reasons read through NVML (read only)
    while the GPU runs the timed region: a background thread samples from
    ``begin()`` on (the host may spend the whole region queueing launches),
    and ``wait(event)`` goes on sampling from the calling thread until the
    region's last event has completed, so even a region of a few
    milliseconds holds samples.  Falls back to ``nvidia-smi -lms 100`` when
    NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.samples = []            # (sm_mhz, max_mhz, power_w, reasons_mask)
        self.proc = None
        self.nvml = None
        self.active = False
        self.done = False
        self.thread = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.nvml = (pynvml, h, get_reasons, smax)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            import threading

            def run():
                while not self.done:
                    if self.active:
                        self.sample()
                    time.sleep(0.001)

            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.gpu_id], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def sample(self):
        if self.nvml is None:
            return
        nv, h, get_reasons, smax = self.nvml
        try:
            power = nv.nvmlDeviceGetPowerUsage(h) / 1000.0 if len(self.samples) % 4 == 0 else \
                (self.samples[-1][2] if self.samples else 0.0)
            self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), smax, power,
                                 int(get_reasons(h))))
        except Exception:
            pass

    def begin(self):
        self.active = True

    def wait(self, event):
        """Sample until ``event`` (recorded after the timed work) completes."""
        while not event.query():
            self.sample()
            time.sleep(0.0005)
        self.active = False

    def stop(self):
        self.done = True
        if self.thread is not None:
            self.thread.join(timeout=5)
        if self.nvml is not None:
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
            sm = [x[0] for x in self.samples]
            reasons = sorted({nm for x in self.samples for nm, bit in self.REASONS if x[3] & bit})
            return {"sm_mhz": statistics.median(sm) if sm else None,
                    "sm_min_mhz": min(sm) if sm else None,
                    "sm_max_mhz": self.samples[0][1] if self.samples else None,
                    "power_w_max": max(x[2] for x in self.samples) if self.samples else None,
                    "samples": len(sm),
                    "source": "NVML, read back to back while the timed region runs",
                    "reasons": reasons}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "source": "nvidia-smi -lms 100 around the timed region",
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------- CPU oracle baseline

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads") for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def cpu_oracle_block(wl, params, grads, bufs, idx, keep=None):
    """Time the oracle on the given matrices (one step); returns seconds.
    With ``keep`` (a dict), also stores the oracle's new parameters and
    buffers there, for the parity spot check."""
    from oracle import muon_step_ref
    t0 = time.perf_counter()
    p_new, b_new = muon_step_ref([params[i] for i in idx], [grads[i] for i in idx],
                                 [bufs[i] for i in idx], lr=wl.lr, beta=wl.beta,
                                 nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
    secs = time.perf_counter() - t0
    if keep is not None:
        keep.update(idx=list(idx), p=p_new, b=b_new)
    return secs


def parity_spot_check(torch, muon, wl, params, grads, bufs, ref, dev):
    """The GPU step on the oracle's sample (same inputs, fresh copies): the
    relative Frobenius error of each matrix's update and the largest relative
    error of the momentum buffers, reported beside the timing."""
    idx = ref["idx"]
    P = [torch.from_numpy(params[i]).to(dev) for i in idx]
    G = [torch.from_numpy(grads[i]).to(dev) for i in idx]
    B = [torch.from_numpy(bufs[i]).to(dev) for i in idx]
    muon.step(P, G, B, lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps,
              coeffs=wl.coeffs)
    torch.cuda.synchronize()
    upd, buf = [], []
    for k, i in enumerate(idx):
        p0 = params[i].astype(np.float64)
        dg = P[k].cpu().numpy().astype(np.float64) - p0
        dr = ref["p"][k].astype(np.float64) - p0
        upd.append(float(np.linalg.norm(dg - dr) / max(np.linalg.norm(dr), 1e-300)))
        br = ref["b"][k].astype(np.float64)
        buf.append(float(np.max(np.abs(B[k].cpu().numpy() - br)) / max(np.max(np.abs(br)), 1e-300)))
    return {"matrices": idx, "update_rel_fro": upd, "buf_rel_max": max(buf),
            "bars": {"update": 1e-2 if wl.buf_std == 0 else 2e-2, "buf": 1e-6},
            "how": "one step of the GPU on the CPU baseline's sample (first gradient set), "
                   "against the oracle's result"}


def parallelism(world: int) -> str:
    return f"replicas x{world}" if world > 1 else "single GPU"


def run_reference(args, wl, rank, world):
    """Reference arm: the CPU oracle, as it stands, on the host cores.

    Each timed step is one real oracle call on a bounded sample of the
    workload: the matrices of one GPT-2 block (4 of the 48, one of each
    shape).  ``ms_per_step`` is the measured time of those calls, so
    steps x ms_per_step is the time actually spent; ``value`` scales the mean
    to the whole workload (x blocks), the metric's unit."""
    if rank != 0:
        return 0
    idx = [0, 1, 2, 3]
    st = WorkloadStream(wl, seed=0, subset=idx)
    params, bufs = st.init()
    grads = st.next_grads()
    local = list(range(len(idx)))
    times = []
    for k in range(args.warmup + args.steps):
        t = cpu_oracle_block(wl, params, grads, bufs, local)
        if k >= args.warmup:
            times.append(t)
    scale = wl.n_matrices / len(idx)
    call_ms = 1e3 * statistics.mean(times)
    ms = call_ms * scale
    cores = blas_threads()
    sample = (f"each step runs the oracle once on matrices {idx} (one GPT-2 block, every shape "
              f"once); {args.steps} timed calls after {args.warmup} untimed, "
              f"{sum(times):.1f} s timed; value = mean call x {scale:g}")
    out = {
        "impl": "reference", "metric": METRIC, "value": ms, "unit": "ms", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": call_ms,
        "sampled_calls": {"calls": args.steps, "matrices_per_call": len(idx),
                          "ms_per_call": call_ms, "seconds_timed": sum(times),
                          "scale_to_workload": scale},
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": dict(workload_config(wl), parallelism=parallelism(world)),
        "cpu_baseline": {"value": ms, "unit": "ms", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": ms, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------- GPU arm

def flat_views(torch, shapes, device, dtype, pinned=False):
    """One contiguous buffer with a 64-element-aligned view per matrix."""
    offs, tot = [], 0
    for r, c in shapes:
        offs.append(tot)
        tot += (r * c + 63) // 64 * 64
    if device == "cpu":
        flat = torch.empty(tot, dtype=dtype, pin_memory=pinned)
    else:
        flat = torch.empty(tot, dtype=dtype, device=device)
    views = [flat[o:o + r * c].view(r, c) for o, (r, c) in zip(offs, shapes)]
    return flat, views


# ---------------------------------------------------------------- ranks (weak scaling)

class Ranks:
    """Process-group plumbing of a multi-rank run: every rank times its own
    independent problem; the only collectives are barriers around the timed
    region and the max of the per-rank times.  There is no data-path
    collective.  backend 'nccl' on GPUs, 'gloo' for CPU tests."""

    def __init__(self, world: int, backend: str = "nccl", device=None, timeout_s: int = 120):
        import torch
        self.world = world
        self.device = device if device is not None else torch.device("cpu")
        self.dist = None
        if world > 1:
            import torch.distributed as dist
            kw = {"device_id": self.device} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.dist is None:
            return float(v)
        import torch
        t = torch.tensor([float(v)], dtype=torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()
            self.dist = None


def rank_seed(rank: int) -> int:
    """Each rank draws its own problem (seed = rank): the step is per-matrix
    independent, so N ranks run N independent problems (weak scaling)."""
    return int(rank)


def measure_adamw(args, rank, dev, stream, barrier, max_over_ranks, peaks):
    """Time one AdamW step over the non-hidden GPT-2 124M parameters."""
    import torch
    import newton_schulz_norm_b200 as muon

    aw = ADAMW_WORKLOADS["gpt2_124m_adamw"]
    st = AdamWStream(aw, seed=rank_seed(rank))
    params, us, vs = st.init()
    grad_sets = [st.next_grads() for _ in range(N_GRAD_SETS)]
    on_dev = lambda xs: [torch.from_numpy(x).to(dev) for x in xs]  # noqa: E731
    P, M, V = on_dev(params), on_dev(us), on_dev(vs)
    G = [on_dev(gs) for gs in grad_sets]
    decay = [t.decay for t in aw.tensors]
    kw = dict(lr=aw.lr, betas=(aw.beta1, aw.beta2), eps=aw.eps, weight_decay=aw.weight_decay,
              decay=decay)
    # one prepared group per gradient set: arguments checked and packed once
    groups = [muon.AdamWGroup(P, G[i], M, V, **kw) for i in range(N_GRAD_SETS)]
    for w in range(args.warmup):
        groups[w % N_GRAD_SETS].step(aw.step + w)
    torch.cuda.synchronize()
    barrier()
    muon.profile_begin()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clocks = start_clocks(torch, dev)
    clocks.begin()
    e0.record(stream)
    t0 = aw.step + args.warmup
    for k in range(args.steps):
        groups[k % N_GRAD_SETS].step(t0 + k)
    e1.record(stream)
    clocks.wait(e1)
    torch.cuda.synchronize()
    prof = muon.profile_end()
    clk = clocks.stop()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1) / args.steps)
    kern_ms, launches = prof["adamw"]
    per_launch = ADAMW_BYTES_PER_ELEMENT * aw.n_elements   # one launch per step (100 tensors)
    gbs = per_launch / (kern_ms / launches * 1e-3) / 1e9
    return {"workload": f"{aw.name}: {aw.n_tensors} fp32 tensors, {aw.n_elements} elements "
                        f"(wte 50257x768, wpe 1024x768 decayed; LayerNorm and bias vectors not), "
                        f"lr {aw.lr}, betas ({aw.beta1}, {aw.beta2}), eps {aw.eps}, "
                        f"weight decay {aw.weight_decay}",
            "ms_per_step": ms, "launches_per_step": launches / args.steps,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "traffic": recorded_traffic("adamw"),
                         "bytes_per_launch": per_launch, "avg_launch_ms": kern_ms / launches,
                         "peak_source": f"{peaks['source']} (burst)"},
            "clocks": clk,
            "l2": f"inputs larger than L2: {N_GRAD_SETS} gradient sets cycled "
                  f"({N_GRAD_SETS * aw.n_elements * 4 / 1e9:.2f} GB) + 3 state arrays "
                  f"({3 * aw.n_elements * 4 / 1e9:.2f} GB)"}


def run_adamw_only(args, rank, world):
    import torch

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(world, "nccl", dev)
    res = measure_adamw(args, rank, dev, torch.cuda.current_stream(), ranks.barrier, ranks.max,
                        load_peaks())
    if rank == 0:
        print(json.dumps({"n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "adamw": res}), flush=True)
    ranks.close()
    return 0


def run_sharded(args, wl, rank, world):
    """One problem (seed 0 on every rank) split across the ranks by matrix;
    each rank steps its own matrices, then one NCCL all-gather of the flat
    parameter buffer.  Strong scaling: the total work is fixed."""
    import torch
    from newton_schulz_norm_b200.sharded import ShardedMuon

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(world, "nccl", dev)
    st = WorkloadStream(wl, seed=0)
    params, _ = st.init()
    grad_sets = [st.next_grads() for _ in range(N_GRAD_SETS)]
    sm = ShardedMuon(wl.shapes, ns_steps=wl.ns_steps, device=dev)
    for v, a in zip(sm.params, params):
        v.copy_(torch.from_numpy(a))
    G = [[torch.from_numpy(g).to(dev) for g in gs] for gs in grad_sets]
    kw = dict(lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, coeffs=wl.coeffs)
    stream = torch.cuda.current_stream()
    for w in range(args.warmup):
        sm.step(G[w % N_GRAD_SETS], **kw)
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(args.steps):
        sm.step(G[k % N_GRAD_SETS], **kw)
    e1.record(stream)
    torch.cuda.synchronize()
    ranks.barrier()
    ms = ranks.max(e0.elapsed_time(e1) / args.steps)
    owned = len(sm.owned)
    if rank == 0:
        print(json.dumps({
            "metric": METRIC, "value": ms, "unit": "ms", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "mode": "sharded",
            "config": dict(workload_config(wl), parallelism=f"matrix-sharded x{world}",
                           matrices_on_rank0=owned),
        }), flush=True)
    ranks.close()
    return 0


def run_ours(args, wl, rank, world):
    import torch
    import newton_schulz_norm_b200 as muon

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(world, "nccl", dev)
    barrier = ranks.barrier
    max_over_ranks = ranks.max

    # ---- inputs (seeded per rank), resident in HBM
    st = WorkloadStream(wl, seed=rank_seed(rank))
    params, bufs = st.init()
    grad_sets = [st.next_grads() for _ in range(N_GRAD_SETS)]

    # CPU oracle baseline on a bounded sample (rank 0, N = 1 only), before GPU work
    cpu_base = None
    oracle_out = {}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        idx = list(range(min(4, wl.n_matrices)))
        secs = cpu_oracle_block(wl, params, grad_sets[0], bufs, idx, keep=oracle_out)
        cpu_base = {"value": 1e3 * secs * wl.n_matrices / len(idx), "unit": "ms",
                    "cores": blas_threads(), "kind": "oracle",
                    "sample": f"oracle on matrices {idx}, 1 step, {secs:.1f} s, "
                              f"scaled x{wl.n_matrices / len(idx):g} to the full step"}

    shapes = list(wl.shapes)
    p_flat, P = flat_views(torch, shapes, dev, torch.float32)
    b_flat, B = flat_views(torch, shapes, dev, torch.float32)
    g_flats, G = [], []
    for gs in grad_sets:
        f, v = flat_views(torch, shapes, dev, torch.float32)
        for t, a in zip(v, gs):
            t.copy_(torch.from_numpy(a))
        g_flats.append(f)
        G.append(v)
    for t, a in zip(P, params):
        t.copy_(torch.from_numpy(a))
    for t, a in zip(B, bufs):
        t.copy_(torch.from_numpy(a))
    torch.cuda.synchronize()

    kw = dict(lr=wl.lr, beta=wl.beta, nesterov=wl.nesterov, ns_steps=wl.ns_steps, coeffs=wl.coeffs)
    stream = torch.cuda.current_stream()

    for w in range(args.warmup):
        muon.step(P, G[w % N_GRAD_SETS], B, **kw)
    torch.cuda.synchronize()
    if muon.status() != 0:
        raise RuntimeError("device-side error during warm-up")

    # ---- per-kernel times: K steps with an event pair recorded around every
    # launch.  That bracketing costs about 4% of a step, so the headline pass
    # below runs the same K steps without it.  The two passes are separated by
    # a short idle pause so that each starts from the same power state.
    torch.cuda.synchronize()
    time.sleep(0.25)
    barrier()
    torch.cuda.synchronize()
    muon.profile_begin()
    for k in range(args.steps):
        muon.step(P, G[k % N_GRAD_SETS], B, **kw)
    torch.cuda.synchronize()
    prof = muon.profile_end()
    barrier()
    time.sleep(0.25)

    # ---- timed region (device-resident): the headline value
    clocks = start_clocks(torch, dev)
    barrier()
    torch.cuda.synchronize()
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    clocks.begin()
    evs[0].record(stream)
    for k in range(args.steps):
        muon.step(P, G[k % N_GRAD_SETS], B, **kw)
        evs[k + 1].record(stream)
    clocks.wait(evs[-1])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms_local = evs[0].elapsed_time(evs[-1]) / args.steps
    per_step = sorted(evs[k].elapsed_time(evs[k + 1]) for k in range(args.steps))
    pct = lambda q: per_step[min(len(per_step) - 1, int(q * len(per_step)))]  # noqa: E731
    ms = max_over_ranks(ms_local)
    if muon.status() != 0:
        raise RuntimeError("device-side error in the timed region")

    # ---- the same step replayed from CUDA graphs (one per gradient set)
    graphs = [muon.capture_step(P, G[i], B, **kw) for i in range(N_GRAD_SETS)]
    torch.cuda.synchronize()
    barrier()
    g0 = torch.cuda.Event(enable_timing=True)
    g1 = torch.cuda.Event(enable_timing=True)
    g0.record(stream)
    for k in range(args.steps):
        graphs[k % N_GRAD_SETS].replay()
    g1.record(stream)
    torch.cuda.synchronize()
    barrier()
    graph_ms = max_over_ranks(g0.elapsed_time(g1) / args.steps)
    if muon.status() != 0:
        raise RuntimeError("device-side error in the graph replays")
    del graphs

    # ---- end to end through the public API with host buffers
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    hg = []
    for gs in grad_sets:
        f, v = flat_views(torch, shapes, "cpu", torch.float32, pinned=True)
        for t, a in zip(v, gs):
            t.copy_(torch.from_numpy(a))
        hg.append(f)
    hp, _ = flat_views(torch, shapes, "cpu", torch.float32, pinned=True)
    p_snap = torch.empty_like(p_flat)
    # Three streams, so that the copies in and out overlap the optimizer work
    # of neighbouring steps (PCIe is full duplex): step k's gradients go in
    # on s_in while step k-1 computes; after step k the updated parameters
    # are snapshotted on the device (one D2D copy) and the snapshot goes out
    # on s_out while step k+1 computes.  Gradient buffers alternate between
    # two device sets.  Every step still copies its own gradients in and its
    # own parameters out.
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev() for _ in range(e2e_steps)]
    step_done = [ev() for _ in range(e2e_steps)]
    snap_done = [ev() for _ in range(e2e_steps)]
    out_done = [ev() for _ in range(e2e_steps)]
    torch.cuda.synchronize()
    barrier()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    s_in.wait_event(e2)
    s_out.wait_event(e2)
    for k in range(e2e_steps):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(step_done[k - 2])      # step k-2 is done reading this set
            g_flats[b].copy_(hg[k % N_GRAD_SETS], non_blocking=True)
            in_done[k].record(s_in)
        stream.wait_event(in_done[k])
        muon.step(P, G[b], B, **kw)
        step_done[k].record(stream)
        if k >= 1:
            stream.wait_event(out_done[k - 1])      # the snapshot of step k-1 has left
        p_snap.copy_(p_flat, non_blocking=True)
        snap_done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(snap_done[k])
            hp.copy_(p_snap, non_blocking=True)
            out_done[k].record(s_out)
    stream.wait_event(out_done[e2e_steps - 1])
    e3.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e2.elapsed_time(e3) / e2e_steps)
    # The link itself: one step's gradients in, and its parameters out, each alone.
    e4 = torch.cuda.Event(enable_timing=True)
    e5 = torch.cuda.Event(enable_timing=True)
    e6 = torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    g_flats[0].copy_(hg[0], non_blocking=True)
    e5.record(stream)
    hp.copy_(p_flat, non_blocking=True)
    e6.record(stream)
    torch.cuda.synchronize()
    link = {"h2d_gbs": 4 * wl.n_elements / (e4.elapsed_time(e5) * 1e-3) / 1e9,
            "d2h_gbs": 4 * wl.n_elements / (e5.elapsed_time(e6) * 1e-3) / 1e9}

    peaks = load_peaks()
    adamw = None if args.no_adamw else measure_adamw(args, rank, dev, stream, barrier,
                                                      max_over_ranks, peaks)
    parity = (parity_spot_check(torch, muon, wl, params, grad_sets[0], bufs, oracle_out, dev)
              if oracle_out else None)

    # ---- roofline of the dominant kernel
    work = per_launch_work(wl)
    dom = max((k for k in KINDS if prof[k][1] > 0), key=lambda k: prof[k][0])
    bound, per_launch = work[dom]
    avg_ms = prof[dom][0] / prof[dom][1]
    if bound == "tensor":
        achieved = per_launch / (avg_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = per_launch / (avg_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    roofline = {"bound": bound, "kernel": dom, "achieved": achieved, "peak": peak, "unit": unit,
                "frac": achieved / peak, "traffic": recorded_traffic(dom),
                "peak_source": f"{peaks['source']} (burst)",
                "work_per_launch": per_launch, "avg_launch_ms": avg_ms,
                "timing": "CUDA events around each launch, in a timed pass of the same K steps "
                          "run just before the headline pass"}

    kernels = {}
    for k in KINDS:
        tot, n = prof[k]
        if n == 0:
            continue
        b, wpl = work[k]
        rate = wpl / (tot / n * 1e-3)
        kernels[k] = {"launches": n, "ms_per_launch": tot / n, "share": None,
                      ("tflops" if b == "tensor" else "gbs"): rate / (1e12 if b == "tensor" else 1e9)}
    tot_all = sum(prof[k][0] for k in KINDS)
    for k in kernels:
        kernels[k]["share"] = prof[k][0] / tot_all
    ns_ms = sum(prof[k][0] for k in ("gram", "poly", "xupdate", "xupdate_final", "ns_chain")) / args.steps
    ns_tflops = wl.ns_flops() / (ns_ms * 1e-3) / 1e12
    launches = sum(prof[k][1] for k in KINDS)

    out = {
        "metric": METRIC, "value": ms, "unit": "ms", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl), parallelism=parallelism(world)),
        "ns_tflops": ns_tflops, "ns_frac_of_peak": ns_tflops / peaks["bf16_tflops"],
        "ns_ms_per_step": ns_ms,
        "step_ms_percentiles": {"p10": pct(0.1), "median": statistics.median(per_step),
                                "p90": pct(0.9), "rank": "0"},
        "graph": {"ms_per_step": graph_ms,
                  "how": "the same step captured once per gradient set (capture_step) and "
                         "replayed; not the headline value"},
        "roofline": roofline, "kernels": kernels,
        "cpu_baseline": cpu_base,
        "e2e": {"value": e2e_ms, "unit": "ms", "h2d_bytes_per_step": 4 * wl.n_elements,
                "d2h_bytes_per_step": 4 * wl.n_elements, "steps": e2e_steps,
                "how": "pinned host gradients in and updated parameters out every step, on two "
                       "copy streams overlapping neighbouring steps' optimizer work",
                "link": link},
        "gpu_launches": launches,
        "clocks": clk,
        "adamw": adamw,
        "parity": parity,
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    ranks.close()
    return 0


def run_square(args, n, rank, world):
    """The square sweep: one Newton-Schulz orthogonalisation (muon_orthogonalize,
    5 quintic steps, bf16) of an n x n matrix U diag(sigma) V^T with log-uniform
    sigma (condition number 1e3) per step; fp32 in, bf16 out.  Rank r of N
    orthogonalises its own matrix (seed = rank): weak scaling."""
    import torch
    import newton_schulz_norm_b200 as muon

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    ranks = Ranks(world, "nccl", dev)
    case = square_case(n, seed=rank_seed(rank))
    flops = 20.0 * n ** 3                     # (3 m^2 n + m^3) x 5 with m = n
    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import orthogonalize_ref
        m = min(n, 4096)                      # the oracle on the same matrix size up to 4096
        sub = square_case(m, seed=0)
        t0 = time.perf_counter()
        orthogonalize_ref(sub.g, 5, (3.4445, -4.7750, 2.0315))
        secs = time.perf_counter() - t0
        scale = (n / m) ** 3
        cpu_base = {"value": 1e3 * secs * scale, "unit": "ms", "cores": blas_threads(),
                    "kind": "oracle",
                    "sample": f"oracle on one {m} x {m} orthogonalisation, {secs:.1f} s"
                              + (f", scaled x{scale:g} (n^3)" if scale != 1 else "")}
    x = torch.from_numpy(case.g).to(dev)
    out = torch.empty((n, n), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        muon.orthogonalize(x, out=out)
    torch.cuda.synchronize()
    muon.profile_begin()
    for _ in range(args.steps):
        muon.orthogonalize(x, out=out)
    torch.cuda.synchronize()
    prof = muon.profile_end()
    time.sleep(0.25)
    ranks.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    clocks = start_clocks(torch, dev)
    clocks.begin()
    e0.record(stream)
    for _ in range(args.steps):
        muon.orthogonalize(x, out=out)
    e1.record(stream)
    clocks.wait(e1)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ranks.barrier()
    ms = ranks.max(e0.elapsed_time(e1) / args.steps)
    if muon.status() != 0:
        raise RuntimeError("device-side error")
    # e2e: fp32 matrix in from pinned host memory, bf16 result out, every step
    hx = torch.from_numpy(case.g).pin_memory()
    hout = torch.empty((n, n), dtype=torch.bfloat16).pin_memory()
    torch.cuda.synchronize()
    e2 = torch.cuda.Event(enable_timing=True)
    e3 = torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for _ in range(args.steps):
        x.copy_(hx, non_blocking=True)
        muon.orthogonalize(x, out=out)
        hout.copy_(out, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks.max(e2.elapsed_time(e3) / args.steps)
    peaks = load_peaks()
    # the dominant kernel: the chain launch (small n) or the per-phase X update
    work = {"gram": float(n) ** 3, "poly": float(n) ** 3, "xupdate": 2.0 * n ** 3,
            "xupdate_final": 2.0 * n ** 3, "ns_chain": flops - 2.0 * n ** 3}
    dom = max((k for k in work if prof[k][1] > 0), key=lambda k: prof[k][0])
    dom_ms, dom_n = prof[dom]
    ach = work[dom] / (dom_ms / dom_n * 1e-3) / 1e12
    kernels = {k: {"launches": v[1], "ms_per_launch": v[0] / v[1]} for k, v in prof.items() if v[1]}
    out_line = {
        "metric": f"Newton-Schulz orthogonalisation ms, {n}x{n}; bf16 TFLOP/s vs tensor peak",
        "value": ms, "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"square_{n}: one {n} x {n} fp32 matrix U diag(sigma) V^T, sigma "
                               f"log-uniform on [1e-3, 1], 5 NS steps, coeffs [3.4445, -4.775, 2.0315], "
                               f"bf16 output", "parallelism": parallelism(world),
                   "ns_flop_per_step": flops,
                   "l2": f"input {4 * n * n / 1e6:.0f} MB fp32, iterates {2 * 2 * n * n / 1e6:.0f} MB bf16"},
        "tflops": flops / (ms * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": ach,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": ach / peaks["bf16_tflops"], "traffic": None,
                     "peak_source": f"{peaks['source']} (burst)", "work_per_launch": work[dom],
                     "avg_launch_ms": dom_ms / dom_n},
        "kernels": kernels,
        "clocks": clk,
        "cpu_baseline": cpu_base,
        "e2e": {"value": e2e_ms, "unit": "ms", "h2d_bytes_per_step": 4 * n * n,
                "d2h_bytes_per_step": 2 * n * n},
        "gpu_launches": sum(v[1] for v in prof.values()) // max(1, args.steps) * args.steps,
    }
    if rank == 0:
        print(json.dumps(out_line), flush=True)
    ranks.close()
    return 0


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.workload.startswith("square_"):
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the square sweep's oracle "
                                  "time is reported in the GPU line's cpu_baseline"}))
            return 0
        return run_square(args, int(args.workload.split("_")[1]), rank, world)
    wl = WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl, rank, world)
    if args.adamw_only:
        return run_adamw_only(args, rank, world)
    if args.sharded:
        return run_sharded(args, wl, rank, world)
    return run_ours(args, wl, rank, world)


if __name__ == "__main__":
    sys.exit(main())
