#!/usr/bin/env python3
"""Benchmark of the fused norm + RoPE hot path on B200 (one JSON line on stdout).

A step is one pass of the whole path over the bf16 long-sequence workloads, every kernel
launched through the C ABI of libgn:

  RMSNorm x[15360, 5120] fwd + bwd, plain and Gemma weight offset (1% outlier rows x50)
  LayerNorm + tanh-GeLU x[32768, 5120] fwd + bwd
  interleaved RoPE in place on q, k [1, 32760, 40, 128] fwd + bwd (sin negated)
  qk-norm + RoPE on q, k [2, 76800, 40, 128] fwd + bwd

`value` is the algorithmic HBM bytes of a step (each input read once, each output written
once) divided by the device time of a step, in GB/s (1e9 bytes), summed over all ranks.
Every input is larger than the 126 MB L2, and consecutive kernels touch different tensors,
so no L2 flush is inserted. Launch with torchrun for several GPUs: the ranks share one global
problem of N times the per-GPU rows and tokens, and rank r owns the r-th contiguous range of
rows (norms) and tokens (RoPE, qk-norm; with the table rows of its positions), generated from
the same seed (weak scaling: the work per GPU is fixed). No activation crosses GPUs; the step's
weight gradients (views of one fp32 bucket) are summed over the ranks by one NCCL all-reduce
per step inside the timed region.

Besides the step, the line carries per-kernel times, GB/s, roofline fractions and ncu DRAM
traffic, the end-to-end figure through host buffers (`e2e`), the fp64 CPU oracle on one and on
all host cores (`cpu_baseline`), SM clocks sampled during the timed region, and (one GPU only,
outside the step) the fused norm + linear layer (TFLOP/s, forward and training backward) and
TiledLinear (time and extra peak memory) beside torch autograd.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--only KERNEL[,KERNEL]] [--scale F] [--no-e2e] [--no-cpu-baseline] [--no-next]
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from transformer_norm_rope_b200 import workloads as wl  # noqa: E402

METRIC = "achieved HBM GB/s (% of B200 peak) for norm+RoPE fwd/bwd, bf16, 1 GPU"
ORDER = ["rmsnorm_fwd", "layernorm_fwd", "rmsnorm_gemma_fwd", "rope_fwd", "qknorm_rope_fwd",
         "rmsnorm_bwd", "layernorm_bwd", "rmsnorm_gemma_bwd", "rope_bwd", "qknorm_rope_bwd"]
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--only", default="", help="comma list of kernels to time (default: all)")
    ap.add_argument("--scale", type=float, default=1.0, help="fraction of rows/tokens (profiling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next", action="store_true", help="skip the norm + linear and TiledLinear measurements")
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args()


# ---------------------------------------------------------------- workload and byte counts

def sizes(scale):
    s = lambda n: max(1, int(round(n * scale)))  # noqa: E731
    return {
        "rms": dict(M=s(wl.RMSNORM_MAIN["M"]), N=wl.RMSNORM_MAIN["N"]),
        "ln": dict(M=s(wl.LAYERNORM_MAIN["M"]), N=wl.LAYERNORM_MAIN["N"]),
        "rope": dict(B=1, S=s(wl.ROPE_MAIN["S"]), H=40, D=128),
        "qk": dict(B=2, S=s(wl.QKNORM_MAIN["S"]), H=40, D=128),
    }


def algorithmic_bytes(z):
    """Minimum HBM bytes per launch: every input read once, every output written once."""
    e = 2  # bf16
    M, N = z["rms"]["M"], z["rms"]["N"]
    rms_f = 2 * M * N * e + 4 * M + N * e
    rms_b = 3 * M * N * e + 4 * M + N * e + 4 * N
    M, N = z["ln"]["M"], z["ln"]["N"]
    ln_f = 2 * M * N * e + 8 * M + 2 * N * e
    ln_b = 3 * M * N * e + 8 * M + 2 * N * e + 8 * N
    r = z["rope"]
    E = r["B"] * r["S"] * r["H"] * r["D"]
    rope = 2 * 2 * E * e + 2 * r["S"] * r["D"] // 2 * 4
    q = z["qk"]
    E = q["B"] * q["S"] * q["H"] * q["D"]
    R = q["B"] * q["S"] * q["H"]
    tab = 2 * q["S"] * q["D"] // 2 * 4
    qk_f = 2 * (2 * E * e + 4 * R + q["D"] * e) + tab
    qk_b = 2 * (3 * E * e + 4 * R + q["D"] * e + 4 * q["D"]) + tab
    return {"rmsnorm_fwd": rms_f, "rmsnorm_gemma_fwd": rms_f, "rmsnorm_bwd": rms_b, "rmsnorm_gemma_bwd": rms_b,
            "layernorm_fwd": ln_f, "layernorm_bwd": ln_b, "rope_fwd": rope, "rope_bwd": rope,
            "qknorm_rope_fwd": qk_f, "qknorm_rope_bwd": qk_b}


def rows_of(z):
    return {"rmsnorm_fwd": z["rms"]["M"], "rmsnorm_gemma_fwd": z["rms"]["M"], "rmsnorm_bwd": z["rms"]["M"],
            "rmsnorm_gemma_bwd": z["rms"]["M"], "layernorm_fwd": z["ln"]["M"], "layernorm_bwd": z["ln"]["M"],
            "rope_fwd": 2 * z["rope"]["S"] * z["rope"]["H"], "rope_bwd": 2 * z["rope"]["S"] * z["rope"]["H"],
            "qknorm_rope_fwd": 2 * z["qk"]["B"] * z["qk"]["S"] * z["qk"]["H"],
            "qknorm_rope_bwd": 2 * z["qk"]["B"] * z["qk"]["S"] * z["qk"]["H"]}


def workload_config(z, l2_note=True):
    return {
        "workload": "norm+RoPE bf16 suite: RMSNorm fwd+bwd plain and Gemma x[%d,%d]; LayerNorm+tanh-GeLU "
                    "fwd+bwd x[%d,%d]; interleaved RoPE fwd+bwd in place q,k[1,%d,40,128]; qk-norm+RoPE "
                    "fwd+bwd q,k[2,%d,40,128]" % (z["rms"]["M"], z["rms"]["N"], z["ln"]["M"], z["ln"]["N"],
                                                  z["rope"]["S"], z["qk"]["S"]),
        "l2": "no flush: every input tensor is larger than the 126 MB L2 and consecutive kernels touch "
              "different tensors" if l2_note else "n/a",
        "seed": "seed 0 on every rank; rank r holds shard r of one global problem",
    }


FAMILY = {"rmsnorm_fwd": "rms", "rmsnorm_gemma_fwd": "rms", "rmsnorm_bwd": "rms", "rmsnorm_gemma_bwd": "rms",
          "layernorm_fwd": "ln", "layernorm_bwd": "ln", "rope_fwd": "rope", "rope_bwd": "rope",
          "qknorm_rope_fwd": "qk", "qknorm_rope_bwd": "qk"}


def global_sizes(z, ws):
    """The global problem of a run on ws ranks: ws times the per-GPU rows and tokens."""
    return {"rms": dict(z["rms"], M=z["rms"]["M"] * ws), "ln": dict(z["ln"], M=z["ln"]["M"] * ws),
            "rope": dict(z["rope"], S=z["rope"]["S"] * ws), "qk": dict(z["qk"], S=z["qk"]["S"] * ws)}


def shard_ranges(z, ws, rank):
    """Rank `rank`'s contiguous shard of the global problem (the token partition of the path):
    rows of the norm workloads, tokens of the rotary workloads (each with the table rows of its
    positions). With the global sizes ws times the per-GPU ones, every shard has the per-GPU
    size."""
    from transformer_norm_rope_b200.shard import shard_bounds

    g = global_sizes(z, ws)
    return {"rms": shard_bounds(g["rms"]["M"], ws, rank), "ln": shard_bounds(g["ln"]["M"], ws, rank),
            "rope": shard_bounds(g["rope"]["S"], ws, rank), "qk": shard_bounds(g["qk"]["S"], ws, rank)}


def gen_inputs(z, seed, families=("rms", "ln", "rope", "qk"), ws=1, rank=0):
    """Host inputs of rank `rank` of `ws`: its shard of the global problem, from `seed`."""
    g, sh = global_sizes(z, ws), shard_ranges(z, ws, rank)
    r, l, o, q = g["rms"], g["ln"], g["rope"], g["qk"]
    d = {}
    if "rms" in families:
        d["rms"] = wl.rmsnorm(M=r["M"], N=r["N"], dtype="bf16", seed=seed, rows=sh["rms"])
        d["rms_gemma_w"] = wl.normal(seed, wl.S_W, r["N"], "bf16", scale=0.1)
    if "ln" in families:
        d["ln"] = wl.layernorm(M=l["M"], N=l["N"], dtype="bf16", seed=seed, rows=sh["ln"])
    if "rope" in families:
        d["rope"] = wl.rope(**o, dtype="bf16", seed=seed, tokens=sh["rope"])
    if "qk" in families:
        d["qk"] = wl.qknorm_rope(**q, dtype="bf16", seed=seed, tokens=sh["qk"])
    return d


# ---------------------------------------------------------------- our arm

class Suite:
    """Device buffers and C-ABI launch closures for one step of the path (only the workloads
    of the selected kernels are generated and allocated)."""

    def __init__(self, gn, torch, z, host, dev, kernels):
        from transformer_norm_rope_b200.shard import GradBucket

        self.gn, self.torch, self.z, self.dev = gn, torch, z, dev
        self.kernels = list(kernels)
        fams = {FAMILY[k] for k in kernels}
        T = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)  # noqa
        F = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
        h = {}  # host tensors (pageable): the inputs of the step
        if "rms" in fams:
            r = host["rms"]
            h.update(rx=T(r["x"]), rdy=T(r["dy"]), rw=T(r["w"]), rwg=T(host["rms_gemma_w"]))
        if "ln" in fams:
            l = host["ln"]  # noqa: E741
            h.update(lx=T(l["x"]), ldy=T(l["dy"]), lw=T(l["w"]), lb=T(l["b"]))
        if "rope" in fams:
            o = host["rope"]
            h.update(oq=T(o["q"]), ok=T(o["k"]), ocos=F(o["cos"]), osin=F(o["sin"]))
        if "qk" in fams:
            q = host["qk"]
            h.update(qq=T(q["q"]), qk=T(q["k"]), qwq=T(q["wq"]), qwk=T(q["wk"]), qcos=F(q["cos"]),
                     qsin=F(q["sin"]), qdq=T(q["dq_out"]), qdk=T(q["dk_out"]))
        self.h = h
        self.inputs = list(h)
        self.d = d = {k: v.to(dev) for k, v in h.items()}
        f32 = torch.float32
        E = lambda ref, dt=None: torch.empty_like(ref) if dt is None else torch.empty(ref.shape[:-1], dtype=dt, device=dev)  # noqa
        # the weight gradients of the step are views of one bucket: with several ranks one
        # all-reduce per step sums them (the data-parallel exchange of a training step)
        gsz = {}
        if "rms" in fams:
            gsz.update(rdw=z["rms"]["N"], rdwg=z["rms"]["N"])
        if "ln" in fams:
            gsz.update(ldw=z["ln"]["N"], ldb=z["ln"]["N"])
        if "qk" in fams:
            gsz.update(qdwq=z["qk"]["D"], qdwk=z["qk"]["D"])
        self.grads = GradBucket(gsz, dev) if gsz else None
        if self.grads is not None:
            d.update(self.grads.views)
        if "rms" in fams:
            d.update(ry=E(d["rx"]), rr=E(d["rx"], f32), rdx=E(d["rx"]), ryg=E(d["rx"]), rrg=E(d["rx"], f32),
                     rdxg=E(d["rx"]))
        if "ln" in fams:
            d.update(ly=E(d["lx"]), lmu=E(d["lx"], f32), lrs=E(d["lx"], f32), ldx=E(d["lx"]))
        if "qk" in fams:
            d.update(qqo=E(d["qq"]), qko=E(d["qk"]), qrq=E(d["qq"], f32), qrk=E(d["qk"], f32), qdxq=E(d["qq"]),
                     qdxk=E(d["qk"]))
        r, l, q = z["rms"], z["ln"], z["qk"]
        self.ws_r = gn.gn_rmsnorm_bwd_workspace(r["M"], r["N"], gn.GN_BF16) if "rms" in fams else 0
        self.ws_l = gn.gn_layernorm_bwd_workspace(l["M"], l["N"], gn.GN_BF16) if "ln" in fams else 0
        self.ws_q = gn.gn_qknorm_rope_bwd_workspace(q["B"], q["S"], q["H"], q["D"], gn.GN_BF16) if "qk" in fams else 0
        self.ws = torch.empty(max(self.ws_r, self.ws_l, self.ws_q, 16), dtype=torch.uint8, device=dev)
        # outputs read back by the end-to-end measurement (final value of each output tensor)
        self.outputs = [k for k in ("ry", "rr", "rdx", "rdw", "ryg", "rrg", "rdxg", "rdwg", "ly", "lmu", "lrs", "ldx",
                                    "ldw", "ldb", "oq", "ok", "qqo", "qko", "qrq", "qrk", "qdxq", "qdxk", "qdwq",
                                    "qdwk") if k in d]
        self.stream = torch.cuda.current_stream(dev)

    def reduce_grads(self):
        """Sum the step's weight gradients over the ranks (one collective; no-op on one rank)."""
        if self.grads is not None and any(k.endswith("_bwd") for k in self.kernels):
            self.grads.allreduce()

    def launch(self, name):
        gn, d, z, s = self.gn, self.d, self.z, self.stream.cuda_stream
        P = lambda k: d[k].data_ptr()  # noqa: E731
        r, l, o, q = z["rms"], z["ln"], z["rope"], z["qk"]
        bf = gn.GN_BF16
        if name in ("rmsnorm_fwd", "rmsnorm_gemma_fwd"):
            g = name == "rmsnorm_gemma_fwd"
            st = gn.gn_rmsnorm_fwd(P("rx"), P("rwg" if g else "rw"), P("ryg" if g else "ry"), P("rrg" if g else "rr"),
                                   r["M"], r["N"], r["N"], r["N"], 1e-6, int(g), 0, bf, s)
        elif name in ("rmsnorm_bwd", "rmsnorm_gemma_bwd"):
            g = name == "rmsnorm_gemma_bwd"
            st = gn.gn_rmsnorm_bwd(P("rx"), P("rwg" if g else "rw"), P("rrg" if g else "rr"), P("rdy"),
                                   P("rdxg" if g else "rdx"), P("rdwg" if g else "rdw"), self.ws.data_ptr(),
                                   self.ws_r, r["M"], r["N"], r["N"], r["N"], r["N"], int(g), 0, bf, s)
        elif name == "layernorm_fwd":
            st = gn.gn_layernorm_fwd(P("lx"), P("lw"), P("lb"), P("ly"), P("lmu"), P("lrs"), l["M"], l["N"], l["N"],
                                     l["N"], 1e-5, gn.GN_EPI_GELU_TANH, bf, s)
        elif name == "layernorm_bwd":
            st = gn.gn_layernorm_bwd(P("lx"), P("lw"), P("lb"), P("lmu"), P("lrs"), P("ldy"), P("ldx"), P("ldw"),
                                     P("ldb"), self.ws.data_ptr(), self.ws_l, l["M"], l["N"], l["N"], l["N"], l["N"],
                                     gn.GN_EPI_GELU_TANH, bf, s)
        elif name in ("rope_fwd", "rope_bwd"):
            st = gn.gn_rope_apply_inplace(P("oq"), P("ok"), P("ocos"), P("osin"), o["B"], o["S"], o["H"], o["D"],
                                          1 if name == "rope_fwd" else -1, bf, s)
        elif name == "qknorm_rope_fwd":
            st = gn.gn_qknorm_rope_fwd(P("qq"), P("qk"), P("qwq"), P("qwk"), P("qcos"), P("qsin"), P("qqo"),
                                       P("qko"), P("qrq"), P("qrk"), q["B"], q["S"], q["H"], q["D"], 1e-6, 0, bf, s)
        elif name == "qknorm_rope_bwd":
            st = gn.gn_qknorm_rope_bwd(P("qq"), P("qk"), P("qwq"), P("qwk"), P("qcos"), P("qsin"), P("qrq"),
                                       P("qrk"), P("qdq"), P("qdk"), P("qdxq"), P("qdxk"), P("qdwq"), P("qdwk"),
                                       self.ws.data_ptr(), self.ws_q, q["B"], q["S"], q["H"], q["D"], 0, bf, s)
        else:
            raise KeyError(name)
        gn.check(st, name)


class ClockSampler:
    """Samples SM clocks and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz, self.ok = [], set(), None, False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = str(e)

    def __enter__(self):
        self.stop = threading.Event()
        if self.ok:
            self.t = threading.Thread(target=self.run, daemon=True)
            self.t.start()
        return self

    def run(self):
        while not self.stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                m = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.reasons |= {n for b, n in self.REASONS.items() if m & b and n != "gpu_idle"}
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.01)

    def __exit__(self, *a):
        self.stop.set()
        if self.ok:
            self.t.join()

    def report(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        return float(json.load(open(p))["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        return FALLBACK_HBM_GBS, "fallback"


def ncu_traffic(kernel, z):
    """dram bytes per launch of `kernel` from the committed ncu summary, scaled to this
    workload, or None when there is none or the kernel sources changed since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        t = json.load(open(p))
        from transformer_norm_rope_b200 import _build

        if t.get("sources_sha") != _build.sources_digest(step_only=True):
            return None
        e = t["kernels"][kernel]
        return e["dram_bytes_per_launch"] * (algorithmic_bytes(z)[kernel] / e["algorithmic_bytes"])
    except Exception:  # noqa: BLE001
        return None


def dist_setup(args):
    import torch

    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))
    return ws, rank, local


def barrier(ws, device):
    """All ranks meet; the device is idle on return."""
    import torch

    if ws > 1:
        import torch.distributed as dist

        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def reduce_over_ranks(v, ws, device, op):
    """Combine one float over the ranks ("max" or "sum")."""
    import torch

    if ws == 1:
        return float(v)
    import torch.distributed as dist

    t = torch.tensor([float(v)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def throughput_gbs(bytes_per_rank, elapsed_s, ws, device):
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's device time."""
    tot = reduce_over_ranks(bytes_per_rank, ws, device, "sum")
    el = reduce_over_ranks(elapsed_s, ws, device, "max")
    return tot / el / 1e9, el


def parallelism(ws):
    if ws == 1:
        return "single GPU"
    return (f"token-sharded data parallel x{ws} (weak): one global problem of {ws}x the per-GPU rows and "
            "tokens; rank r owns its r-th contiguous range of rows and tokens (RoPE tables sliced to its "
            "positions); the step's weight gradients are summed by one NCCL all-reduce")


def norm_linear_measure(gn, torch, dev, scale, seed, reps=10):
    """The fused LayerNorm + linear + SiLU (tcgen05 tensor cores) on x[32768, 5120] and a
    5120 x 5120 layer, timed alone with CUDA events (median of `reps` after 3 warm-ups), beside
    the unfused sequence it replaces: the LayerNorm kernel writing bf16 activations, a cuBLAS
    matmul (torch) and the bias + SiLU (torch). Tensor-bound: reported against the measured bf16
    burst peak. Not part of the HBM step."""
    M, N, K = max(256, int(32768 * scale)), 5120, 5120
    d = wl.norm_linear(M, N, K, seed)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa
    x, g, beta, W, bias = T(d["x"]), T(d["g"]), T(d["beta"]), T(d["W"]), T(d["bias"])
    Wf, c, dd = gn.norm_linear_prepare(W, g, beta, bias, norm="ln")
    stream = torch.cuda.current_stream(dev)

    def fused():
        gn.norm_linear_fwd(x, Wf, c, dd, eps=d["eps"], norm="ln", epilogue="silu", save_stats=False)

    def unfused():
        xn, _, _ = gn.layernorm_fwd(x, g, beta, d["eps"], save_stats=False)
        torch.nn.functional.silu(torch.addmm(bias, xn, W.t()))

    def timed(*fns):
        """Median seconds of each fn over `reps` rounds that run the fns in turn: tensor-core timings
        drift with the power state within seconds, so variants compared with each other are
        interleaved rather than timed one after another."""
        for _ in range(3):
            for fn in fns:
                fn()
        torch.cuda.synchronize(dev)
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in fns]
              for _ in range(reps)]
        for r in ev:
            for fn, (a, b) in zip(fns, r):
                a.record(stream)
                fn()
                b.record(stream)
        torch.cuda.synchronize(dev)
        out = [statistics.median(r[i][0].elapsed_time(r[i][1]) for r in ev) * 1e-3 for i in range(len(fns))]
        return out if len(fns) > 1 else out[0]

    t_f, t_u = timed(fused, unfused)
    # the training backward (this library's kernels only) beside torch autograd of the unfused
    # layer (torch LayerNorm, cuBLAS, SiLU), both from the same upstream gradient
    from transformer_norm_rope_b200 import norm_linear as nl

    dy = torch.randn(M, N, device=dev, dtype=torch.bfloat16)
    _, mu, rs = nl.forward(x, g, beta, W, bias, d["eps"], "ln", False, "silu")

    def bwd():
        nl.backward(x, g, beta, W, bias, mu, rs, dy, d["eps"], "ln", False, "silu")

    leaves = [t.detach().clone().requires_grad_() for t in (x, g, beta, W, bias)]

    def autograd_fwd_bwd():
        xa, ga, ba, Wa, bia = leaves
        ya = torch.nn.functional.silu(torch.nn.functional.linear(
            torch.nn.functional.layer_norm(xa, (K,), ga, ba, d["eps"]), Wa, bia))
        ya.backward(dy)

    def fwd_bwd_keep_z():  # the training form that stores the pre-activation instead of recomputing it
        yk, muk, rsk, zk = nl.forward_keeping_z(x, g, beta, W, bias, d["eps"], "ln", False, "silu")
        nl.backward(x, g, beta, W, bias, muk, rsk, dy, d["eps"], "ln", False, "silu", z=zk)

    t_b, t_ab, t_kz = timed(bwd, autograd_fwd_bwd, fwd_bwd_keep_z)
    flops = 2.0 * M * N * K
    tf = flops / t_f / 1e12
    peak = None
    try:
        peak = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        kind = "measured bf16_tflops (burst)"
    except Exception:  # noqa: BLE001
        peak, kind = 1590.0, "fallback"
    gn.check(0 if gn.device_error(clear=True) == 0 else gn.GN_ERR_CUDA, "norm_linear device error")
    return {"workload": f"LayerNorm + linear {K}->{N} + SiLU, x[{M},{K}] bf16 (statistics pre-pass + tcgen05 GEMM on pairs of SMs)",
            "ms": round(t_f * 1e3, 4), "TFLOP_s": round(tf, 1),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4), "peak_source": kind},
            "unfused_ms": round(t_u * 1e3, 4),
            "unfused": "LayerNorm kernel (bf16 activations) + cuBLAS addmm + SiLU (torch)",
            "speedup_vs_unfused": round(t_u / t_f, 3),
            "backward_ms": round(t_b * 1e3, 4),
            "fwd_bwd_ms": round((t_f + t_b) * 1e3, 4),
            "torch_autograd_fwd_bwd_ms": round(t_ab * 1e3, 4),
            "keep_z_fwd_bwd_ms": round(t_kz * 1e3, 4),
            "keep_z": "forward keeps the pre-activation (product with no activation, then the activation "
                      "elementwise); backward forms dz from it instead of recomputing the product",
            "backward": "normalized rows recomputed, activation gradient in the product epilogue, dx and fp32 dW "
                        "on the tensor cores with MN-major operands, column sums, LayerNorm backward"}


def tiled_linear_measure(gn, torch, dev, scale, seed, reps=5):
    """The token-chunked linear + SiLU (TiledLinear) on x[32768, 5120] and a 5120 x 5120 layer:
    forward + backward time and the peak memory the step allocates beyond its inputs, for the
    default chunk count (ceil(tokens / hidden) = 7), one chunk, and torch autograd keeping the
    pre-activation (the layer TiledLinear replaces)."""
    from transformer_norm_rope_b200 import tiled_linear as tl

    M, N, K = max(256, int(32768 * scale)), 5120, 5120
    d = wl.norm_linear(M, N, K, seed)
    T = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)  # noqa
    x, W, bias = T(d["x"]), T(d["W"]), T(d["bias"])
    dy = torch.randn((M, N), device=dev).to(torch.bfloat16)
    stream = torch.cuda.current_stream(dev)
    Wf, dd = tl.prepare(W, bias)

    def tiled(chunks):
        def f():
            tl.forward(x, Wf, dd, "silu", chunks)
            tl.backward(x, Wf, dd, dy, "silu", chunks)
        return f

    def autograd():
        xa, Wa, ba = x.detach().requires_grad_(), W.detach().requires_grad_(), bias.detach().requires_grad_()
        torch.nn.functional.silu(torch.nn.functional.linear(xa, Wa, ba)).backward(dy)

    variants = (("tiled", tiled(None)), ("one_chunk", tiled(1)), ("torch_autograd", autograd))
    peaks = {}
    for name, fn in variants:  # extra peak memory of one call, after a warm-up call
        fn()
        torch.cuda.synchronize(dev)
        base = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        fn()
        torch.cuda.synchronize(dev)
        peaks[name] = (torch.cuda.max_memory_allocated(dev) - base) / 2**20
    # times: the variants in turn over `reps` rounds (tensor-core timings drift with the power
    # state within seconds, so variants compared with each other are interleaved)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in variants]
          for _ in range(reps)]
    for r in ev:
        for (_, fn), (a, b) in zip(variants, r):
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize(dev)
    out = {"workload": f"linear {K}->{N} + SiLU forward + backward, x[{M},{K}] bf16",
           "default_chunks": tl.default_chunks(M, K)}
    for i, (name, _) in enumerate(variants):
        ms = statistics.median(r[i][0].elapsed_time(r[i][1]) for r in ev)
        out[name] = {"ms": round(ms, 3), "peak_extra_MiB": round(peaks[name], 1)}
    gn.check(0 if gn.device_error(clear=True) == 0 else gn.GN_ERR_CUDA, "tiled_linear device error")
    return out


def run_ours(args):
    import torch

    import transformer_norm_rope_b200 as gn

    ws, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)

    torch.cuda.set_device(dev)
    gn.load()
    z = sizes(args.scale)
    kernels = [k for k in ORDER if not args.only or k in args.only.split(",")]
    host = gen_inputs(z, args.seed, {FAMILY[k] for k in kernels}, ws, rank)
    suite = Suite(gn, torch, z, host, dev, kernels)
    nbytes = algorithmic_bytes(z)
    step_bytes = sum(nbytes[k] for k in kernels)
    # the backward kernels read the forward statistics: run each forward once before timing
    for k in ORDER:
        if k.endswith("_fwd") and k.replace("_fwd", "_bwd") in kernels and k not in kernels:
            suite.launch(k)
    stream = suite.stream

    def step(ev=None):
        for i, k in enumerate(kernels):
            if ev is not None:
                ev[i][0].record(stream)
            suite.launch(k)
            if ev is not None:
                ev[i][1].record(stream)
        if ws > 1:
            suite.reduce_grads()

    for _ in range(args.warmup):
        step()
        if "rope_fwd" in kernels and "rope_bwd" not in kernels:  # keep rotated tensors bounded
            suite.launch("rope_bwd")
    barrier(ws, dev)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in kernels]
          for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = gn.gn_launch_count()
    with ClockSampler(dev.index) as clk:
        barrier(ws, dev)
        t0.record(stream)
        for i in range(args.steps):
            step(ev[i])
        t1.record(stream)
        t1.synchronize()
        barrier(ws, dev)
    launches = gn.gn_launch_count() - n0
    value, elapsed = throughput_gbs(step_bytes * args.steps, t0.elapsed_time(t1) * 1e-3, ws, dev)
    per_kernel = {k: statistics.mean(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(args.steps)) * 1e-3
                  for j, k in enumerate(kernels)}
    peak, peak_kind = peaks()
    dom = max(kernels, key=lambda k: per_kernel[k])
    ach = nbytes[dom] / per_kernel[dom] / 1e9
    traffic = ncu_traffic(dom, z)
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded generator, seed 0; rank r generates shard r of one global problem)",
        "config": dict(workload_config(z), parallelism=parallelism(ws), bytes_per_step_per_gpu=step_bytes),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(ach / peak, 4), "traffic": traffic, "peak_source": f"{peak_kind} hbm_gbs"},
        "kernels": {k: {"ms": round(per_kernel[k] * 1e3, 4), "GB_s": round(nbytes[k] / per_kernel[k] / 1e9, 1),
                        "frac_of_peak": round(nbytes[k] / per_kernel[k] / 1e9 / peak, 4),
                        "rows_per_s": round(rows_of(z)[k] / per_kernel[k], 1),
                        "algorithmic_bytes": nbytes[k], "traffic": ncu_traffic(k, z)} for k in kernels},
        "frac_of_peak": round(value / ws / peak, 4),
        "frac_of_8TBs": round(value / ws / 8000.0, 4),
        "clocks": clk.report(),
        "gpu_launches": int(launches),
    }
    if not args.no_e2e:
        out["e2e"] = e2e(args, suite, kernels, step_bytes, ws, dev)
    if not args.no_next and not args.only and ws == 1:  # single-GPU measurements, not part of the step
        del suite  # free the step's buffers first
        torch.cuda.empty_cache()
        out["next_norm_linear"] = norm_linear_measure(gn, torch, dev, args.scale, args.seed)
        torch.cuda.empty_cache()
        out["next_tiled_linear"] = tiled_linear_measure(gn, torch, dev, args.scale, args.seed)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(host, z, kernels, budget_s=15.0, seed=args.seed)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def e2e(args, suite, kernels, step_bytes, ws, dev):
    """Same metric through host buffers: each step copies its inputs from pinned host memory,
    runs the path, and copies every output back to pinned host memory, as a caller streaming
    batches through the API would. Uploads, kernels and downloads run on three streams over two
    sets of device buffers used by alternate steps, so that step i+1's upload overlaps step i's
    download (PCIe moves both directions at once) and neither waits for the other: a set is
    overwritten only after the step that used it two steps earlier has been read by its
    kernels (inputs) and by its download (outputs, in-place tensors included)."""
    import torch

    from transformer_norm_rope_b200.shard import GradBucket

    steps = max(1, min(args.steps, 5))
    need = set()
    for k in kernels:
        need |= set(INPUTS[k])
    ins = [k for k in suite.inputs if k in need]
    outs = [k for k in suite.outputs if any(k in OUTPUTS[x] for x in kernels)]
    inplace = [k for k in ins if k in outs]
    pin_in = {k: suite.h[k].pin_memory() for k in ins}
    pin_out = {k: torch.empty(suite.d[k].shape, dtype=suite.d[k].dtype, pin_memory=True) for k in outs}
    h2d = sum(v.numel() * v.element_size() for v in pin_in.values())
    d2h = sum(v.numel() * v.element_size() for v in pin_out.values())
    # the second buffer set: its own copy of every tensor a step uploads or downloads, and its
    # own gradient bucket (the all-reduce of a step sums that step's gradients)
    grad_names = set(suite.grads.names()) if suite.grads is not None else set()
    alt = dict(suite.d)
    for k in set(ins) | set(outs):
        if k not in grad_names:
            alt[k] = torch.empty_like(suite.d[k])
    alt_grads = None
    if suite.grads is not None:
        alt_grads = GradBucket({k: suite.grads[k].numel() for k in suite.grads.names()}, dev)
        alt.update(alt_grads.views)
    sets = [(suite.d, suite.grads), (alt, alt_grads)]
    comp = suite.stream
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    Ev = lambda: torch.cuda.Event(enable_timing=False)  # noqa: E731

    def run(n, t0=None, t1=None):
        done = [None, None]  # per set: (kernels read its inputs, download read its outputs)
        last_out = None
        if t0 is not None:
            t0.record(comp)
            s_in.wait_event(t0)
        for i in range(n):
            d, grads = sets[i % 2]
            prev = done[i % 2]
            ev_in, ev_comp, ev_out = Ev(), Ev(), Ev()
            with torch.cuda.stream(s_in):
                if prev is not None:
                    s_in.wait_event(prev[0])  # the set's last kernels have read its inputs
                for k in ins:
                    if k not in inplace:
                        d[k].copy_(pin_in[k], non_blocking=True)
                if prev is not None and inplace:
                    s_in.wait_event(prev[1])  # ... and its download has read the in-place tensors
                for k in inplace:
                    d[k].copy_(pin_in[k], non_blocking=True)
                ev_in.record(s_in)
            comp.wait_event(ev_in)
            if prev is not None:
                comp.wait_event(prev[1])  # the set's outputs are overwritten only after their download
            suite.d, suite.grads = d, grads
            for k in kernels:
                suite.launch(k)
            if ws > 1:
                suite.reduce_grads()
            ev_comp.record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp)
                for k in outs:
                    pin_out[k].copy_(d[k], non_blocking=True)
                ev_out.record(s_out)
            done[i % 2] = (ev_comp, ev_out)
            last_out = ev_out
        comp.wait_event(last_out)
        if t1 is not None:
            t1.record(comp)

    try:
        run(2)
        torch.cuda.synchronize(dev)
        barrier(ws, dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run(steps, a, b)
        b.synchronize()
        barrier(ws, dev)
    finally:
        suite.d, suite.grads = sets[0]
    v, _ = throughput_gbs(step_bytes * steps, a.elapsed_time(b) * 1e-3, ws, dev)
    return {"value": round(v, 2), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": steps,
            "schedule": "two device buffer sets on alternate steps; uploads of step i+1 overlap downloads of step i (3 streams)"}


INPUTS = {
    "rmsnorm_fwd": ["rx", "rw"], "rmsnorm_gemma_fwd": ["rx", "rwg"],
    "rmsnorm_bwd": ["rx", "rw", "rdy"], "rmsnorm_gemma_bwd": ["rx", "rwg", "rdy"],
    "layernorm_fwd": ["lx", "lw", "lb"], "layernorm_bwd": ["lx", "lw", "lb", "ldy"],
    "rope_fwd": ["oq", "ok", "ocos", "osin"], "rope_bwd": ["ocos", "osin"],
    "qknorm_rope_fwd": ["qq", "qk", "qwq", "qwk", "qcos", "qsin"],
    "qknorm_rope_bwd": ["qq", "qk", "qwq", "qwk", "qcos", "qsin", "qdq", "qdk"],
}
OUTPUTS = {
    "rmsnorm_fwd": ["ry", "rr"], "rmsnorm_gemma_fwd": ["ryg", "rrg"], "rmsnorm_bwd": ["rdx", "rdw"],
    "rmsnorm_gemma_bwd": ["rdxg", "rdwg"], "layernorm_fwd": ["ly", "lmu", "lrs"], "layernorm_bwd": ["ldx", "ldw", "ldb"],
    "rope_fwd": [], "rope_bwd": ["oq", "ok"], "qknorm_rope_fwd": ["qqo", "qko", "qrq", "qrk"],
    "qknorm_rope_bwd": ["qdxq", "qdxk", "qdwq", "qdwk"],
}


# ---------------------------------------------------------------- the fp64 CPU oracle arm

def _units(z, k):
    fam = FAMILY[k]
    return z[fam]["M"] if fam in ("rms", "ln") else z[fam]["S"]


def oracle_range(host, z, k, lo, hi):
    """Runs the oracle for kernel k on rows (norms) or tokens (rotary) [lo, hi) of the host
    inputs; returns the algorithmic bytes of that range (the kernel's bytes pro rata)."""
    import oracle

    if hi <= lo:
        return 0.0
    if k.startswith("rmsnorm"):
        r = host["rms"]
        w = host["rms_gemma_w"] if "gemma" in k else r["w"]
        g = "gemma" in k
        if k.endswith("fwd"):
            oracle.rmsnorm_fwd(r["x"][lo:hi], w, 1e-6, gemma=g)
        else:
            oracle.rmsnorm_bwd(r["x"][lo:hi], w, r["dy"][lo:hi], 1e-6, gemma=g)
    elif k.startswith("layernorm"):
        l = host["ln"]  # noqa: E741
        if k.endswith("fwd"):
            oracle.layernorm_fwd(l["x"][lo:hi], l["w"], l["b"], 1e-5, act="gelu_tanh")
        else:
            oracle.layernorm_bwd(l["x"][lo:hi], l["w"], l["b"], l["dy"][lo:hi], 1e-5, act="gelu_tanh")
    elif k.startswith("rope"):
        o = host["rope"]
        sign = 1 if k == "rope_fwd" else -1
        oracle.rope(o["q"][:, lo:hi], o["cos"][lo:hi], o["sin"][lo:hi], sign)
        oracle.rope(o["k"][:, lo:hi], o["cos"][lo:hi], o["sin"][lo:hi], sign)
    else:
        q = host["qk"]
        for x, w, dy in (("q", "wq", "dq_out"), ("k", "wk", "dk_out")):
            if k.endswith("fwd"):
                oracle.qknorm_rope_fwd(q[x][:, lo:hi], q[w], q["cos"][lo:hi], q["sin"][lo:hi], 1e-6)
            else:
                oracle.qknorm_rope_bwd(q[x][:, lo:hi], q[w], q["cos"][lo:hi], q["sin"][lo:hi], q[dy][:, lo:hi], 1e-6)
    return algorithmic_bytes(z)[k] * (hi - lo) / _units(z, k)


def oracle_step(host, z, kernels, frac):
    """Runs the oracle on the first `frac` of the rows/tokens of each kernel; returns
    (seconds, algorithmic bytes of the sample)."""
    done, t = 0.0, 0.0
    for k in kernels:
        m = max(1, int(_units(z, k) * frac))
        s = time.perf_counter()
        done += oracle_range(host, z, k, 0, m)
        t += time.perf_counter() - s
    return t, done


def _oracle_worker(conn, z, seed, jobs):
    """One host core of the all-cores oracle run: generates the inputs of its (kernel, lo, hi)
    ranges, reports ready, then for every start signal runs the oracle on them and reports
    (seconds, bytes), until told to stop."""
    try:
        local = []
        for k, lo, hi in jobs:
            fam = FAMILY[k]
            if fam == "rms":
                h = {"rms": wl.rmsnorm(M=z["rms"]["M"], N=z["rms"]["N"], dtype="bf16", seed=seed, rows=(lo, hi)),
                     "rms_gemma_w": wl.normal(seed, wl.S_W, z["rms"]["N"], "bf16", scale=0.1)}
            elif fam == "ln":
                h = {"ln": wl.layernorm(M=z["ln"]["M"], N=z["ln"]["N"], dtype="bf16", seed=seed, rows=(lo, hi))}
            elif fam == "rope":
                h = {"rope": wl.rope(**z["rope"], dtype="bf16", seed=seed, tokens=(lo, hi))}
            else:
                h = {"qk": wl.qknorm_rope(**z["qk"], dtype="bf16", seed=seed, tokens=(lo, hi))}
            local.append((k, h, hi - lo))
        conn.send("ready")
        while conn.recv() == "go":
            s = time.perf_counter()
            done = sum(oracle_range(h, z, k, 0, n) for k, h, n in local)
            conn.send((time.perf_counter() - s, done))
    except Exception as e:  # noqa: BLE001 - reported to the parent, which raises
        conn.send(("error", repr(e)))
    finally:
        conn.close()


class OraclePool:
    """The unchanged oracle on `cores` spawned host processes: the first `frac` of every kernel's
    rows/tokens split into `cores` contiguous ranges, one per process, each process holding the
    inputs of its ranges (generated once, before any clock starts). run() starts all processes
    together and returns (wall seconds from the common start to the last one's end, bytes)."""

    def __init__(self, z, seed, kernels, frac, cores):
        import multiprocessing as mp

        jobs = [[] for _ in range(cores)]
        for k in kernels:
            m = max(1, int(_units(z, k) * frac))
            for i in range(cores):
                lo, hi = m * i // cores, m * (i + 1) // cores
                if hi > lo:
                    jobs[i].append((k, lo, hi))
        ctx = mp.get_context("spawn")
        self.procs, self.conns = [], []
        try:
            for i in range(cores):
                a, b = ctx.Pipe()
                p = ctx.Process(target=_oracle_worker, args=(b, z, seed, jobs[i]), daemon=True)
                p.start()
                self.procs.append(p)
                self.conns.append(a)
            for c in self.conns:
                msg = c.recv()
                if msg != "ready":
                    raise RuntimeError(f"oracle worker failed: {msg}")
        except BaseException:
            self.close()
            raise

    def run(self):
        t0 = time.perf_counter()
        for c in self.conns:
            c.send("go")
        res = [c.recv() for c in self.conns]
        wall = time.perf_counter() - t0
        bad = [r for r in res if r[0] == "error"]
        if bad:
            raise RuntimeError(f"oracle worker failed: {bad[0][1]}")
        return wall, sum(r[1] for r in res)

    def close(self):
        for c in self.conns:
            try:
                c.send("stop")
            except (OSError, ValueError):
                pass
        for p in self.procs:
            p.join(60)


def oracle_all_cores(z, seed, kernels, frac, cores):
    """One all-cores run of the oracle (OraclePool) on the first `frac` of every kernel's
    rows/tokens. Returns (seconds, bytes)."""
    pool = OraclePool(z, seed, kernels, frac, cores)
    try:
        return pool.run()
    finally:
        pool.close()


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(host, z, kernels, budget_s, seed=0):
    """The oracle as it stands on the host cores: one thread on a sample sized to about
    `budget_s`, then every core at once (one process per core) on a sample sized to about
    budget_s / 2 per core."""
    t, done = oracle_step(host, z, kernels, 1.0 / 4096)
    frac = min(1.0, (1.0 / 4096) * max(1.0, budget_s / max(t, 1e-3)))
    t, done = oracle_step(host, z, kernels, frac)
    single = done / t / 1e9
    cores = host_cores()
    frac_all = min(1.0, frac * cores * 0.5)
    t_all, done_all = oracle_all_cores(z, seed, kernels, frac_all, cores)
    multi = done_all / t_all / 1e9
    return {"value": round(multi, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "single_core": {"value": round(single, 4), "cores": 1,
                            "sample": f"first {frac:.5f} of the rows/tokens of every kernel of the step "
                                      f"({t:.1f} s of fp64 C oracle, one thread)"},
            "all_cores": {"value": round(multi, 4), "cores": cores,
                          "sample": f"first {frac_all:.5f} of the rows/tokens of every kernel of the step, split "
                                    f"into {cores} contiguous ranges run at once by {cores} processes "
                                    f"({t_all:.1f} s wall)"},
            "sample": f"all {cores} host cores (one oracle process each) on the first {frac_all:.5f} of the "
                      f"rows/tokens of every kernel of the step; same seeded inputs"}


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands on every host core (one spawned process
    per core, OraclePool), each step one all-cores pass over a bounded sample of the workload sized
    so that warm-up and steps take about a minute and a half; rank 0 only."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    z = sizes(args.scale)
    kernels = [k for k in ORDER if not args.only or k in args.only.split(",")]
    cores = host_cores()
    probe_frac = min(1.0, cores / 8192)
    t, _ = oracle_all_cores(z, args.seed, kernels, probe_frac, cores)
    budget = max(0.5, min(20.0, 90.0 / max(1, args.steps + args.warmup)))
    # at most a quarter of the workload per step keeps the processes' inputs to a few GB of host memory
    frac = min(0.25, probe_frac * budget / max(t, 1e-3))
    pool = OraclePool(z, args.seed, kernels, frac, cores)
    try:
        for _ in range(args.warmup):
            pool.run()
        tot_t, tot_b = 0.0, 0.0
        for _ in range(args.steps):
            t, b = pool.run()
            tot_t += t
            tot_b += b
    finally:
        pool.close()
    v = tot_b / tot_t / 1e9
    sample = (f"first {frac:.6f} of the rows/tokens of every kernel per step, split into {cores} contiguous "
              f"ranges run at once by {cores} processes (fp64 C oracle, one process per host core)")
    out = {"metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 3), "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator, seed 0)",
           "config": dict(workload_config(z), parallelism="host oracle on all host cores, rank 0 only"),
           "impl": "reference",
           "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
