#!/usr/bin/env python
"""Throughput of the partitioned Transformer layer on B200 (libtp).

One step = the whole hot path over one batch of synthetic input: head-wise
attention forward + backward and the partitioned MLP forward + backward
(tp_attn_fwd, tp_attn_bwd, tp_mlp_fwd, tp_mlp_bwd) on the 175B-shaped layer
(b=1, s=2048, h=12288, f=49152, 96 heads of 128, t=8 logical shards, bf16
with fp32 accumulation, weights ~ N(0, 0.006^2), random-init, synthetic data).

Prints one JSON line (rank 0).  `value` is algorithmic TFLOP/s of the whole
job (2*M*N*K per GEMM; causal attention counts the unmasked half; backward
core = 2.5x forward core), timed on the device with CUDA events over exactly
`--steps` steps after `--warmup` steps, max over ranks.  The weights (2.7 GB
per step) are larger than L2, so every step streams them from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl libtp|reference]

--impl reference times the CPU oracle (the reference arm of this build) on
the host cores on a bounded sample of the same workload.  Under torchrun,
each rank runs an independent replica (the layer does not shard across GPUs
here: replicas only); rank 0 prints.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from megatron_tensor_transformer_logical_b200.inputs import WORKLOADS  # noqa: E402

METRIC = "partitioned MLP+attn fwd+bwd TFLOP/s and tokens/s, % of B200 BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# --------------------------------------------------------------- FLOP model
def layer_flops(b, s, h, f, heads, causal=True):
    M = b * s
    d = h // heads
    g = lambda m, n, k: 2.0 * m * n * k
    pairs = 0.5 * s * s if causal else float(s * s)
    core = 4.0 * d * pairs * b * heads
    mlp_f = g(M, f, h) + g(M, h, f)
    mlp_b = 2 * mlp_f
    att_f = g(M, 3 * h, h) + core + g(M, h, h)
    att_b = g(M, h, h) + g(h, h, M) + 2.5 * core + g(h, 3 * h, M) + g(M, h, 3 * h)
    return {"mlp_fwd": mlp_f, "mlp_bwd": mlp_b, "attn_fwd": att_f, "attn_bwd": att_b,
            "total": mlp_f + mlp_b + att_f + att_b}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_hash():
    p = os.path.join(ROOT, "megatron_tensor_transformer_logical_b200", "csrc", "tp_gemm_sm100.cu")
    with open(p, "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def traffic_per_launch():
    """DRAM bytes per GEMM launch from the committed ncu capture (and the
    launches it covers, with their algorithmic bytes), if it was taken on the
    current kernel source; otherwise (None, None, None)."""
    p = os.path.join(ROOT, "profiles", "gemm_tcgen05_traffic.json")
    if not os.path.exists(p):
        return None, None, None
    with open(p) as fh:
        d = json.load(fh)
    if d.get("source_sha256_16") != gemm_source_hash():
        return None, None, None
    return (d.get("dram_bytes_per_launch"), d.get("scope"),
            d.get("algorithmic_bytes_per_launch"))


# ------------------------------------------------------------ clock sampling
class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(suffix=".csv")
        self.proc = None
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark(self):
        return time.time()

    def stop(self, t0, t1):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        inside = [r for r in rows if t0 - 0.15 <= r[0] <= t1 + 0.15] or rows
        if not inside:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside), "reasons": reasons,
                "samples": len(inside)}


# ------------------------------------------------------------------- ranks
class Ranks:
    """The job's ranks: one process per GPU, each running an independent
    replica of the step (no collective on the data path).  torch.distributed
    carries only the barriers around the timed regions and the max over
    ranks of each timing.  A single process needs no process group."""

    def __init__(self, rank: int = 0, world: int = 1, local_rank: int = 0, dist=None,
                 backend: str = ""):
        self.rank, self.world, self.local_rank = rank, world, local_rank
        self.dist, self.backend = dist, backend

    @classmethod
    def from_env(cls, backend: str = "nccl", timeout_s: int = 600):
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        if world == 1:
            return cls(rank, world, local_rank)
        import datetime

        import torch.distributed as tdist
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
            kw["device_id"] = torch.device("cuda", local_rank)
        tdist.init_process_group(backend, **kw)
        return cls(rank, world, local_rank, tdist, backend)

    def barrier(self):
        if self.dist is None:
            return
        if self.backend == "nccl":
            self.dist.barrier(device_ids=[self.local_rank])
        else:
            self.dist.barrier()

    def max(self, x):
        """The maximum of x over the ranks (None stays None on every rank)."""
        if self.dist is None or x is None:
            return x
        dev = torch.device("cuda", self.local_rank) if self.backend == "nccl" else "cpu"
        t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.destroy_process_group()


def job_rate(units_per_rank: float, world: int, ms_max: float, steps: int) -> float:
    """Whole-job throughput: the units every rank processed in `steps` steps,
    divided by the slowest rank's time (weak scaling: each rank's work is
    fixed as the job grows)."""
    return world * units_per_rank / (ms_max / steps * 1e-3)


# ------------------------------------------------------------- libtp arm
class LayerStep:
    """Device buffers and the four libtp calls of one layer step."""

    def __init__(self, wl, dev):
        from megatron_tensor_transformer_logical_b200 import binding as L
        from megatron_tensor_transformer_logical_b200.inputs import make_attn_inputs, make_mlp_inputs
        self.L = L
        self.wl = wl
        mi = make_mlp_inputs(wl)
        ai = make_attn_inputs(wl)
        bf = torch.bfloat16
        M, h, f = wl.M, wl.h, wl.f
        self.X = mi["X"].to(dev)
        self.dZ = mi["dZ"].to(dev)
        self.A, self.B = mi["A"].to(dev), mi["B"].to(dev)
        self.Wqkv, self.Wo = ai["Wqkv"].to(dev), ai["Wo"].to(dev)
        e = lambda *s, dt=bf: torch.empty(*s, dtype=dt, device=dev)
        self.Zm, self.Y = e(M, h), e(M, f)
        self.dXm, self.dA, self.dB = e(M, h), e(h, f), e(f, h)
        self.Za, self.QKV, self.O = e(M, h), e(M, 3 * h, dt=torch.float16), e(M, h)
        self.LSE = e(wl.b, wl.heads, wl.s, dt=torch.float32)
        self.dXa, self.dWqkv, self.dWo = e(M, h), e(h, 3 * h), e(h, h)
        self.ws = {op: L.workspace(op, M, h, f, wl.heads, wl.t, L.TP_BF16, device=dev)
                   for op in (L.TP_OP_MLP_FWD, L.TP_OP_MLP_BWD, L.TP_OP_ATTN_FWD,
                              L.TP_OP_ATTN_BWD)}

    def attn(self):
        L, wl = self.L, self.wl
        L.tp_attn_fwd(self.X, self.Wqkv, self.Wo, self.Za, self.QKV, self.O, self.LSE, wl.b, wl.s,
                      wl.heads, wl.t, True, self.ws[L.TP_OP_ATTN_FWD])
        L.tp_attn_bwd(self.X, self.Wqkv, self.Wo, self.QKV, self.O, self.LSE, self.dZ, self.dXa,
                      self.dWqkv, self.dWo, wl.b, wl.s, wl.heads, wl.t, True,
                      self.ws[L.TP_OP_ATTN_BWD])

    def mlp(self, save_y=True):
        """MLP forward + backward.  save_y: keep the pre-activation Y from the
        forward for the backward (default); otherwise the backward recomputes
        it with one more GEMM (the activation-recompute policy)."""
        L, wl = self.L, self.wl
        Y = self.Y if save_y else None
        L.tp_mlp_fwd(self.X, self.A, None, self.B, None, self.Zm, Y, wl.t,
                     self.ws[L.TP_OP_MLP_FWD])
        L.tp_mlp_bwd(self.X, self.A, None, self.B, Y, self.dZ, self.dXm, self.dA, None,
                     self.dB, None, wl.t, self.ws[L.TP_OP_MLP_BWD])

    def step(self):
        self.attn()
        self.mlp()

    def make_block(self, dev):
        """Buffers of the full Transformer block (LayerNorm + residual around
        the same attention and MLP weights)."""
        L, wl = self.L, self.wl
        M, h, f = wl.M, wl.h, wl.f
        bf, f32 = torch.bfloat16, torch.float32
        e = lambda *sh, dt=bf: torch.empty(*sh, dtype=dt, device=dev)
        ones, zeros = torch.ones(h, dtype=bf, device=dev), torch.zeros(h, dtype=bf, device=dev)
        self.bw = {"ln1_g": ones, "ln1_b": zeros, "Wqkv": self.Wqkv, "Wo": self.Wo,
                   "ln2_g": ones, "ln2_b": zeros, "A": self.A, "B": self.B}
        self.bsv = {"Xn1": e(M, h), "mean1": e(M, dt=f32), "rstd1": e(M, dt=f32),
                    "QKV": self.QKV, "O": self.O, "LSE": self.LSE, "X1": e(M, h), "Xn2": e(M, h),
                    "mean2": e(M, dt=f32), "rstd2": e(M, dt=f32), "Y": self.Y}
        self.bg = {"dln1_g": e(h), "dln1_b": e(h), "dWqkv": self.dWqkv, "dWo": self.dWo,
                   "dln2_g": e(h), "dln2_b": e(h), "dA": self.dA, "dB": self.dB}
        self.bX2, self.bdX = e(M, h), e(M, h)
        self.bws_f = L.workspace(L.TP_OP_BLOCK_FWD, M, h, f, wl.heads, wl.t, L.TP_BF16, device=dev)
        self.bws_b = L.workspace(L.TP_OP_BLOCK_BWD, M, h, f, wl.heads, wl.t, L.TP_BF16, device=dev)

    def block(self):
        L, wl = self.L, self.wl
        L.tp_block_fwd(self.X, self.bw, self.bX2, self.bsv, wl.b, wl.s, wl.f, wl.heads, wl.t, 1e-5,
                       self.bws_f)
        L.tp_block_bwd(self.X, self.bw, self.bsv, self.dZ, self.bdX, self.bg, wl.b, wl.s, wl.f,
                       wl.heads, wl.t, 1e-5, self.bws_b)

    def outputs(self):
        return (self.Za, self.Zm, self.dXa, self.dXm)

    def make_library_gemms(self, dev):
        """The step's twelve GEMMs as plain torch.matmul calls (cuBLAS) with
        the same shapes and operand layouts, no epilogues: a library yardstick
        for the tcgen05 GEMMs, not part of the step."""
        wl = self.wl
        M, h, f = wl.M, wl.h, wl.f
        e = lambda *sh: torch.empty(*sh, dtype=torch.bfloat16, device=dev)
        self.lib_dqkv = e(M, 3 * h)
        self.lib_out = {"qkv": e(M, 3 * h), "mh": e(M, h), "hh": e(h, h), "h3h": e(h, 3 * h),
                        "mf": e(M, f), "fh": e(f, h), "hf": e(h, f)}
        flops = 0.0
        for (a, b, c) in ((M, 3 * h, h), (M, h, h), (M, h, h), (h, h, M), (h, 3 * h, M),
                          (M, h, 3 * h), (M, f, h), (M, h, f), (M, f, h), (f, h, M), (h, f, M),
                          (M, h, f)):
            flops += 2.0 * a * b * c
        self.lib_flops = flops

    def library_gemms(self):
        o, X, dZ, Y = self.lib_out, self.X, self.dZ, self.Y
        torch.matmul(X, self.Wqkv, out=o["qkv"])                 # QKV
        torch.matmul(self.O, self.Wo, out=o["mh"])               # Z = O Wo
        torch.matmul(dZ, self.Wo.t(), out=o["mh"])               # dO
        torch.matmul(self.O.t(), dZ, out=o["hh"])                # dWo
        torch.matmul(X.t(), self.lib_dqkv, out=o["h3h"])         # dWqkv
        torch.matmul(self.lib_dqkv, self.Wqkv.t(), out=o["mh"])  # dX (attention)
        torch.matmul(X, self.A, out=o["mf"])                     # Y = X A
        torch.matmul(Y, self.B, out=o["mh"])                     # Z = H B
        torch.matmul(dZ, self.B.t(), out=o["mf"])                # dH
        torch.matmul(Y.t(), dZ, out=o["fh"])                     # dB
        torch.matmul(X.t(), Y, out=o["hf"])                      # dA
        torch.matmul(Y, self.A.t(), out=o["mh"])                 # dX (MLP)


class VocabStep:
    """The vocabulary-parallel embedding and loss with tied weights, forward
    and backward: Y = embed(ids); loss = CE(X @ E^T, targets);
    dE = CE's dE + scatter(dY) (X and dY stand for the hidden states and
    gradient of the layers in between, which this step does not run)."""

    VOCAB_NAMES = {1: "embed_gather", 2: "embed_scatter_add", 3: "loss_combine",
                   4: "softmax_grad"}

    def __init__(self, wl, dev):
        from megatron_tensor_transformer_logical_b200 import binding as L
        from megatron_tensor_transformer_logical_b200.inputs import make_vocab_inputs
        self.L, self.wl = L, wl
        d = {k: v.to(dev) for k, v in make_vocab_inputs(wl).items()}
        self.ids, self.targets, self.E, self.X, self.dY = (d[k] for k in
                                                           ("ids", "targets", "E", "X", "dY"))
        M, h, V = wl.M, wl.h, wl.vocab
        bf, f32 = torch.bfloat16, torch.float32
        self.Y = torch.empty(M, h, dtype=bf, device=dev)
        self.logits = torch.empty(M, V, dtype=bf, device=dev)
        self.lse = torch.empty(M, dtype=f32, device=dev)
        self.loss = torch.empty(M, dtype=f32, device=dev)
        self.total = torch.empty(1, dtype=f32, device=dev)
        self.dX = torch.empty(M, h, dtype=bf, device=dev)
        self.dE = torch.empty(V, h, dtype=bf, device=dev)
        self.ws = L.workspace(L.TP_OP_VOCAB_CE_FWD, M, h, V, 0, wl.t, L.TP_BF16, device=dev)
        self.ws_e = L.workspace(L.TP_OP_VOCAB_EMBED_BWD, M, h, V, 0, wl.t, L.TP_BF16, device=dev)

    def step(self):
        L, t = self.L, self.wl.t
        L.tp_vocab_embed_fwd(self.ids, self.E, self.Y, t)
        L.tp_vocab_ce_fwd(self.X, self.E, self.targets, self.logits, self.lse, self.loss,
                          self.total, t, self.ws)
        L.tp_vocab_ce_bwd(self.X, self.E, self.targets, self.logits, self.lse, None, self.logits,
                          self.dX, self.dE, t)
        L.tp_vocab_embed_bwd(self.ids, self.dY, self.dE, self.dE, t, self.ws_e)

    def flops(self):
        wl = self.wl
        return 3 * 2.0 * wl.M * wl.vocab * wl.h


def vocab_report(vs, steps, ms, records, peaks, world):
    """Per-kernel times of the vocabulary step from the launch trace."""
    per = {}
    for r in records:
        if r["kind"] == "vocab":
            name = VocabStep.VOCAB_NAMES.get(r["tile"], str(r["tile"]))
        elif r["kind"] == "gemm_tcgen05":
            name = f'gemm {r["m"]}x{r["n"]}x{r["k"]}'
        else:
            name = r["kind"]
        p = per.setdefault(name, {"ms": 0.0, "n": 0, "bytes": 0.0, "flops": 0.0})
        p["ms"] += r["ms"]
        p["n"] += 1
        p["bytes"] += r["bytes"]
        p["flops"] += r["flops"]
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    kernels = {}
    for name, p in per.items():
        k = {"ms_per_step": round(p["ms"] / steps, 4), "share": round(p["ms"] / ms, 4)}
        if name.startswith("gemm"):
            k["tflops"] = round(p["flops"] / (p["ms"] * 1e-3) / 1e12, 1)
        else:
            gbs = p["bytes"] / (p["ms"] * 1e-3) / 1e9
            k["gbs"] = round(gbs, 1)
            k["frac_of_measured_hbm"] = round(gbs / hbm, 4)
        kernels[name] = k
    wl = vs.wl
    per_step = ms / steps
    return {"what": "tied embedding + vocabulary-parallel cross-entropy, forward and backward",
            "M": wl.M, "h": wl.h, "V": wl.vocab, "t": wl.t,
            "ms_per_step": round(per_step, 4),
            "tflops": round(world * vs.flops() / (per_step * 1e-3) / 1e12, 2),
            "tokens_per_s": round(world * wl.M / (per_step * 1e-3), 1),
            "kernels": kernels}


def timed(fn, steps, stream):
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    return ev0.elapsed_time(ev1)


def timed_interleaved(fns, steps, stream):
    """Times each of `fns` over `steps` rounds with the calls interleaved
    round by round (a, b, a, b, ...), so that all of them run under the same
    clocks; returns the total ms of each."""
    tot = [0.0] * len(fns)
    torch.cuda.synchronize()
    for _ in range(steps):
        evs = []
        for fn in fns:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        torch.cuda.synchronize()
        for i, (e0, e1) in enumerate(evs):
            tot[i] += e0.elapsed_time(e1)
    return tot


def e2e_pipelined(st, steps, stream, barrier):
    """Times `steps` layer steps end to end: host inputs -> device -> step ->
    results back to the host, double-buffered over two slots."""
    dev = st.X.device
    host_in = [(torch.empty_like(st.X, device="cpu").pin_memory(),
                torch.empty_like(st.dZ, device="cpu").pin_memory()) for _ in range(2)]
    for hX, hdZ in host_in:
        hX.copy_(st.X.cpu())
        hdZ.copy_(st.dZ.cpu())
    slots = [{"X": torch.empty_like(st.X), "dZ": torch.empty_like(st.dZ),
              "out": [torch.empty_like(o) for o in st.outputs()]} for _ in range(2)]
    host_out = [[torch.empty_like(o, device="cpu").pin_memory() for o in st.outputs()]
                for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_ready, step_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    saved = (st.X, st.dZ, st.Za, st.Zm, st.dXa, st.dXm)

    def run(n):
        for k in range(n):
            i = k & 1
            sl = slots[i]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(step_done[i])  # slot i's inputs no longer read
                sl["X"].copy_(host_in[i][0], non_blocking=True)
                sl["dZ"].copy_(host_in[i][1], non_blocking=True)
                in_ready[i].record(s_in)
            stream.wait_event(in_ready[i])
            if k >= 2:
                stream.wait_event(out_done[i])  # slot i's results have left
            st.X, st.dZ = sl["X"], sl["dZ"]
            st.Za, st.Zm, st.dXa, st.dXm = sl["out"]
            st.step()
            step_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(step_done[i])
                for ho, o in zip(host_out[i], sl["out"]):
                    ho.copy_(o, non_blocking=True)
                out_done[i].record(s_out)
        stream.wait_stream(s_out)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def run_timed(n):
        e0.record(stream)
        s_in.wait_event(e0)   # no copy starts before the timed region
        s_out.wait_event(e0)
        run(n)

    run(2)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    run_timed(steps)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    barrier()
    st.X, st.dZ, st.Za, st.Zm, st.dXa, st.dXm = saved
    h2d = sum(t.numel() * t.element_size() for t in host_in[0])
    d2h = sum(t.numel() * t.element_size() for t in host_out[0])
    return ms, h2d, d2h


def other_configs(dev, stream, steps, barrier, peak):
    """Throughput of the other workloads of the build, each on its own
    buffers, timed with CUDA events over `steps` calls after two warm-up calls:
    GPT-2-small MLP fwd+bwd with biases (t = 4), the standalone column- and
    row-split linears at t = 1, 2, 4, 8, and head-wise attention fwd+bwd
    (b = 4, s = 2048, h = 4096, 32 heads, t = 8)."""
    from megatron_tensor_transformer_logical_b200 import binding as L
    from megatron_tensor_transformer_logical_b200.inputs import (make_attn_inputs,
                                                                 make_linear_inputs,
                                                                 make_mlp_inputs)
    bf = torch.bfloat16
    out = {}

    def rate(flops, ms):
        tf = flops / (ms / steps * 1e-3) / 1e12
        return {"tflops": round(tf, 2), "frac_of_nominal_2250": round(tf / NOMINAL_BF16_TFLOPS, 4),
                "frac_of_measured_sustained": round(tf / peak, 4)}

    def run(fn):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        L.tp_device_status()
        barrier()
        L.tp_profile_enable(True)
        ms = timed(fn, steps, stream)
        prof = {name: L.tp_profile_read(k) for k, name in L.KIND_NAMES.items()}
        L.tp_profile_enable(False)
        barrier()
        return ms, prof

    def kernel_split(prof, ms):
        return {name: {"ms_per_step": round(p["total_ms"] / steps, 4),
                       "share": round(p["total_ms"] / ms, 4)}
                for name, p in prof.items() if p["launches"]}

    # Workload 2: GPT-2-small MLP with biases, fwd + bwd (both bias gradients).
    wl = WORKLOADS[2]
    d = {k: v.to(dev) for k, v in make_mlp_inputs(wl).items()}
    M, h, f = wl.M, wl.h, wl.f
    e = lambda *sh: torch.empty(*sh, dtype=bf, device=dev)
    Z, Y, dX, dA, dB, dbA, dbB = e(M, h), e(M, f), e(M, h), e(h, f), e(f, h), e(f), e(h)
    wsf = L.workspace(L.TP_OP_MLP_FWD, M, h, f, 0, wl.t, L.TP_BF16, device=dev)
    wsb = L.workspace(L.TP_OP_MLP_BWD, M, h, f, 0, wl.t, L.TP_BF16, device=dev)

    def mlp2():
        L.tp_mlp_fwd(d["X"], d["A"], d["bA"], d["B"], d["bB"], Z, Y, wl.t, wsf)
        L.tp_mlp_bwd(d["X"], d["A"], d["bA"], d["B"], Y, d["dZ"], dX, dA, dbA, dB, dbB, wl.t, wsb)
    ms, prof = run(mlp2)
    fl = 3 * (2.0 * M * f * h * 2)
    out["2"] = {"workload": f"{wl.name}: MLP fwd+bwd with biases (dbA, dbB), t={wl.t}",
                "M": M, "h": h, "f": f, "ms_per_step": round(ms / steps, 4),
                "tokens_per_s": round(M / (ms / steps * 1e-3), 1), **rate(fl, ms),
                "kernels": kernel_split(prof, ms)}
    del d, Z, Y, dX, dA, dB, dbA, dbB, wsf, wsb

    # Workload 3: standalone column- and row-split linears.
    wl = WORKLOADS[3]
    d = {k: v.to(dev) for k, v in make_linear_inputs(wl).items()}
    M, K, N = wl.M, wl.h, wl.n_out
    Yc, Zr = e(M, N), e(M, N)
    sweep = {}
    for t in (1, 2, 4, 8):
        msc, _ = run(lambda: L.tp_linear_col(d["X"], d["W"], None, Yc, t))
        msr, _ = run(lambda: L.tp_linear_row(d["X"], d["W"], None, Zr, t))
        fl = 2.0 * M * N * K
        sweep[f"t{t}"] = {"col": {"ms_per_call": round(msc / steps, 4), **rate(fl, msc)},
                          "row": {"ms_per_call": round(msr / steps, 4), **rate(fl, msr)}}
    out["3"] = {"workload": f"{wl.name}: X[{M},{K}] @ W[{K},{N}]", "tokens_per_call": M,
                "sweep": sweep}
    del d, Yc, Zr

    # Workload 4: head-wise attention fwd + bwd.
    wl = WORKLOADS[4]
    d = {k: v.to(dev) for k, v in make_attn_inputs(wl).items()}
    M, h = wl.M, wl.h
    Za, Os, dXa, dWo = e(M, h), e(M, h), e(M, h), e(h, h)
    QKV = torch.empty(M, 3 * h, dtype=torch.float16, device=dev)
    LSE = torch.empty(wl.b, wl.heads, wl.s, dtype=torch.float32, device=dev)
    dWqkv = e(h, 3 * h)
    wsf = L.workspace(L.TP_OP_ATTN_FWD, M, h, 0, wl.heads, wl.t, L.TP_BF16, device=dev)
    wsb = L.workspace(L.TP_OP_ATTN_BWD, M, h, 0, wl.heads, wl.t, L.TP_BF16, device=dev)

    def attn4():
        L.tp_attn_fwd(d["X"], d["Wqkv"], d["Wo"], Za, QKV, Os, LSE, wl.b, wl.s, wl.heads, wl.t,
                      True, wsf)
        L.tp_attn_bwd(d["X"], d["Wqkv"], d["Wo"], QKV, Os, LSE, d["dZ"], dXa, dWqkv, dWo, wl.b,
                      wl.s, wl.heads, wl.t, True, wsb)
    ms, prof = run(attn4)
    lf = layer_flops(wl.b, wl.s, wl.h, 4 * wl.h, wl.heads)
    fl = lf["attn_fwd"] + lf["attn_bwd"]
    core = {}
    for name in ("attn_fwd", "attn_bwd"):
        p = prof[name]
        if p["launches"]:
            core[name] = {"ms_per_step": round(p["total_ms"] / steps, 4),
                          "tflops": round(p["flops"] / (p["total_ms"] * 1e-3) / 1e12, 1)}
    out["4"] = {"workload": f"{wl.name}: attention fwd+bwd, b={wl.b}, s={wl.s}, h={wl.h}, "
                            f"{wl.heads} heads, t={wl.t}, causal",
                "ms_per_step": round(ms / steps, 4),
                "tokens_per_s": round(M / (ms / steps * 1e-3), 1), **rate(fl, ms),
                "attention_core": core, "kernels": kernel_split(prof, ms)}
    return out


def run_libtp(args, ranks: Ranks):
    from megatron_tensor_transformer_logical_b200 import binding as L
    rank, world, local_rank = ranks.rank, ranks.world, ranks.local_rank
    barrier = ranks.barrier
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    st = LayerStep(wl, dev)
    stream = torch.cuda.current_stream()
    fl = layer_flops(wl.b, wl.s, wl.h, wl.f, wl.heads)

    for _ in range(args.warmup):
        st.step()
    torch.cuda.synchronize()
    L.tp_device_status()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    time.sleep(0.3 if sampler else 0.0)
    barrier()
    L.tp_profile_enable(True)
    n0 = L.tp_launch_count()
    t0 = time.time()
    ms = timed(st.step, args.steps, stream)
    t1 = time.time()
    launches = L.tp_launch_count() - n0
    prof = {name: L.tp_profile_read(k) for k, name in L.KIND_NAMES.items()}
    records = L.tp_profile_records()
    L.tp_profile_enable(False)
    barrier()
    clocks = sampler.stop(t0, t1) if sampler else None
    L.tp_device_status()

    # MLP fwd+bwd alone, and the activation policy that recomputes Y in the
    # backward instead of keeping it; the two interleaved step by step, so
    # the comparison sees the same (power-capped) clocks.
    recompute = lambda: st.mlp(save_y=False)
    for _ in range(2):
        st.mlp()
        recompute()
    barrier()
    mlp_ms, mlp_rec_ms = timed_interleaved([st.mlp, recompute], args.steps, stream)
    barrier()
    # The full Transformer block: LayerNorm and residual around both sublayers.
    st.make_block(dev)
    for _ in range(2):
        st.block()
    barrier()
    block_ms = timed(st.block, args.steps, stream)
    barrier()
    # Library yardstick: the same twelve GEMMs as plain cuBLAS calls,
    # interleaved step by step with the layer step (whose GEMM launches are
    # timed by libtp's trace), so both see the same clocks.
    st.make_library_gemms(dev)
    for _ in range(2):
        st.library_gemms()
    barrier()
    lib_ms = own_gemm_ms = 0.0
    L.tp_profile_enable(True)
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st.library_gemms()
        e1.record(stream)
        st.step()
        torch.cuda.synchronize()
        lib_ms += e0.elapsed_time(e1)
    own_gemm_ms = L.tp_profile_read(L.TP_KIND_GEMM_TCGEN05)["total_ms"]
    L.tp_profile_enable(False)
    barrier()
    del st.lib_out, st.lib_dqkv
    # The vocabulary-parallel embedding and loss (a second workload).
    vocab_ms = vocab_records = None
    vs = None
    if not args.no_vocab:
        del st.bsv, st.bg, st.bX2, st.bdX, st.bws_f, st.bws_b
        vs = VocabStep(WORKLOADS[6], dev)
        for _ in range(3):
            vs.step()
        torch.cuda.synchronize()
        L.tp_device_status()
        barrier()
        L.tp_profile_enable(True)
        vocab_ms = timed(vs.step, args.steps, stream)
        vocab_records = L.tp_profile_records()
        L.tp_profile_enable(False)
        barrier()
        del vs.logits

    # The build's other workloads (MLP with biases, linear sweep, attention).
    others = None
    if not args.no_configs:
        peaks_, _ = load_peaks()
        others = other_configs(dev, stream, args.steps, barrier,
                               float(peaks_.get("bf16_tflops_sustained",
                                                FALLBACK_PEAKS["bf16_tflops_sustained"])))
        L.tp_device_status()

    # End to end through the public API: per step, the step's inputs (X, dZ)
    # copied from pinned host memory and its results (Z and dX of both
    # sublayers) read back into pinned host memory, inside the timed region.
    # The copies run on their own streams with two buffer slots, so step k's
    # inputs arrive and step k-1's results leave while step k-1 / k compute
    # (a data loader's prefetch); every byte still crosses PCIe every step.
    e2e_ms = None
    h2d = d2h = 0
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_pipelined(st, args.steps, stream, barrier)
    L.tp_device_status()

    maxall = ranks.max

    ms, mlp_ms, mlp_rec_ms = maxall(ms), maxall(mlp_ms), maxall(mlp_rec_ms)
    block_ms = maxall(block_ms)
    lib_ms, own_gemm_ms = maxall(lib_ms), maxall(own_gemm_ms)
    vocab_ms = maxall(vocab_ms)
    e2e_ms = maxall(e2e_ms)
    if rank != 0:
        return None

    per_step = ms / args.steps
    tflops = job_rate(fl["total"], world, ms, args.steps) / 1e12
    tokens = job_rate(wl.M, world, ms, args.steps)
    peaks, peak_src = load_peaks()
    g = prof["gemm_tcgen05"]
    achieved = g["flops"] / (g["total_ms"] * 1e-3) / 1e12 if g["total_ms"] > 0 else 0.0
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    traffic, traffic_scope, traffic_alg = traffic_per_launch()
    mlp_tflops = world * (fl["mlp_fwd"] + fl["mlp_bwd"]) / (mlp_ms / args.steps * 1e-3) / 1e12
    gemms = {}
    for r in records:
        if r["kind"] != "gemm_tcgen05":
            continue
        key = f'{r["m"]}x{r["n"]}x{r["k"]}'
        g_ = gemms.setdefault(key, {"tile": r["tile"], "ms": 0.0, "flops": 0.0, "n": 0})
        g_["ms"] += r["ms"]
        g_["flops"] += r["flops"]
        g_["n"] += 1
    gemm_shapes = {k: {"tile": v["tile"], "ms_per_launch": round(v["ms"] / v["n"], 4),
                       "tflops": round(v["flops"] / (v["ms"] * 1e-3) / 1e12, 1)}
                   for k, v in gemms.items()}
    kernels = {}
    for name, p in prof.items():
        if p["launches"]:
            kernels[name] = {"launches_per_step": p["launches"] / args.steps,
                             "ms_per_step": p["total_ms"] / args.steps,
                             "share": p["total_ms"] / ms,
                             "tflops": p["flops"] / (p["total_ms"] * 1e-3) / 1e12}
    out = {
        "metric": METRIC,
        "value": round(tflops, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,0.006^2) random-init weights)",
        "config": {"workload": f"{wl.name}: attention + MLP fwd+bwd", "b": wl.b, "s": wl.s,
                   "h": wl.h, "f": wl.f, "heads": wl.heads, "head_dim": wl.h // wl.heads,
                   "t": wl.t, "causal": True, "global_batch_tokens": world * wl.M,
                   "parallelism": f"replicas{world} (t={wl.t} logical shards per GPU)",
                   "l2": "no flush: weights (2.7 GB per step) exceed the 126 MB L2"},
        "tokens_per_s": round(tokens, 1),
        "frac_of_nominal_bf16_peak": round(tflops / world / NOMINAL_BF16_TFLOPS, 4),
        "mlp_fwd_bwd": {"tflops": round(mlp_tflops, 2), "ms_per_step": round(mlp_ms / args.steps, 4),
                        "frac_of_nominal_2250": round(mlp_tflops / world / NOMINAL_BF16_TFLOPS, 4),
                        "frac_of_measured_sustained": round(mlp_tflops / world / peak, 4)},
        "block_fwd_bwd": {
            "what": "LN1 -> attention -> +residual -> LN2 -> MLP -> +residual, forward and backward",
            "ms_per_step": round(block_ms / args.steps, 4),
            "tflops": round(world * fl["total"] / (block_ms / args.steps * 1e-3) / 1e12, 2),
            "overhead_vs_layer_step": round(block_ms / ms - 1.0, 4)},
        "library_gemm_yardstick": {
            "what": "the step's 12 GEMMs as plain torch.matmul (cuBLAS), same shapes and layouts, "
                    "no epilogues, interleaved step by step with the layer step; context only, "
                    "not on the measured path",
            "cublas_ms_per_step": round(lib_ms / args.steps, 4),
            "cublas_tflops": round(st.lib_flops / (lib_ms / args.steps * 1e-3) / 1e12, 2),
            "libtp_gemm_ms_per_step": round(own_gemm_ms / args.steps, 4),
            "libtp_gemm_tflops": round(st.lib_flops / (own_gemm_ms / args.steps * 1e-3) / 1e12, 2),
            "libtp_over_cublas": round(lib_ms / own_gemm_ms, 4) if own_gemm_ms else None},
        "activation_policy": {
            "measured": "the two MLP steps interleaved step by step, same clocks",
            "save_y": {"mlp_ms_per_step": round(mlp_ms / args.steps, 4),
                       "bytes_kept_fwd_to_bwd": wl.M * wl.f * 2},
            "recompute_y": {"mlp_ms_per_step": round(mlp_rec_ms / args.steps, 4),
                            "bytes_kept_fwd_to_bwd": 0,
                            "extra_flops": 2.0 * wl.M * wl.h * wl.f}},
        "roofline": {"bound": "tensor", "kernel": "gemm_bf16_tcgen05",
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_src} bf16_tflops_sustained",
                     "traffic": traffic,
                     "traffic_scope": traffic_scope,
                     "traffic_algorithmic_bytes_per_launch": traffic_alg,
                     "algorithmic_bytes_per_launch": (g["bytes"] / g["launches"]) if g["launches"] else None,
                     "flops_per_launch": (g["flops"] / g["launches"]) if g["launches"] else None},
        "kernels": kernels,
        "gemm_shapes": gemm_shapes,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if vocab_ms is not None:
        out["vocab_fwd_bwd"] = vocab_report(vs, args.steps, vocab_ms, vocab_records, peaks, world)
    if others is not None:
        out["other_workloads"] = others
    if e2e_ms is not None:
        out["e2e"] = {"value": round(job_rate(fl["total"], world, e2e_ms, args.steps) / 1e12, 2),
                      "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "ms_per_step": round(e2e_ms / args.steps, 4)}
    if not args.no_cpu_baseline and world == 1:  # the oracle baseline: rank 0 at N = 1 only
        out["cpu_baseline"] = cpu_baseline(wl, tokens=args.cpu_sample_tokens)
    return out


# ----------------------------------------------------- the oracle (CPU) arm
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:  # noqa: BLE001
        return os.cpu_count()


def oracle_layer_sample(wl, tokens: int, mi=None, ai=None):
    """Returns (fn, flops): one oracle pass (attention and MLP, forward and
    backward) over the first `tokens` tokens of the workload, full width."""
    import numpy as np  # noqa: F401

    from megatron_tensor_transformer_logical_b200.inputs import make_attn_inputs, make_mlp_inputs
    from oracle import tp_oracle as O
    mi = mi or make_mlp_inputs(wl)
    ai = ai or make_attn_inputs(wl)
    f64 = lambda t: t.float().numpy().astype("float64")
    X, dZ = f64(mi["X"][:tokens]), f64(mi["dZ"][:tokens])
    A, B = f64(mi["A"]), f64(mi["B"])
    Wqkv, Wo = f64(ai["Wqkv"]), f64(ai["Wo"])

    def fn():
        O.attn_fwd(X, Wqkv, Wo, 1, tokens, wl.heads)
        O.attn_bwd(X, Wqkv, Wo, dZ, 1, tokens, wl.heads)
        O.mlp_fwd(X, A, None, B, None)
        O.mlp_bwd(X, A, None, B, dZ)

    return fn, layer_flops(1, tokens, wl.h, wl.f, wl.heads)["total"]


def cpu_baseline(wl, tokens=768):
    """The oracle as it stands, timed once on the host's cores on the first
    `tokens` tokens of the layer (exact under the causal mask)."""
    tokens = int(tokens)
    fn, flops = oracle_layer_sample(wl, tokens)
    t0 = time.perf_counter()
    fn()
    dt = time.perf_counter() - t0
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": _blas_threads(),
            "kind": "oracle",
            "sample": f"first {tokens} of {wl.M} tokens of the same layer (full h, f, heads), "
                      f"attention + MLP fwd+bwd in fp64 numpy, {dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    wl = WORKLOADS[args.workload]
    tokens = args.ref_sample_tokens
    fn, flops = oracle_layer_sample(wl, tokens)
    for _ in range(args.warmup):
        fn()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fn()
    dt = (time.perf_counter() - t0) / args.steps
    value = flops / dt / 1e12
    cores = _blas_threads()
    sample = f"first {tokens} of {wl.M} tokens per step (full h, f, heads), fp64 numpy oracle"
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: attention + MLP fwd+bwd", "b": wl.b, "s": wl.s,
                   "h": wl.h, "f": wl.f, "heads": wl.heads, "t": wl.t,
                   "sample_tokens": tokens},
        "cpu_baseline": {"value": round(value, 5), "unit": "TFLOP/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 5), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["libtp", "reference"], default="libtp")
    ap.add_argument("--workload", type=int, default=5, choices=[5])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-vocab", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (MLP with biases, linear sweep, attention)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=768)
    ap.add_argument("--ref-sample-tokens", type=int, default=64)
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "libtp":
        ap.error("--warmup must be at least 3")

    if args.impl == "reference":
        # Rank 0 alone times the oracle; the other ranks exit without work.
        world = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, int(os.environ.get("RANK", "0")), world)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    ranks = Ranks.from_env("nccl")
    try:
        out = run_libtp(args, ranks)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        ranks.close()


if __name__ == "__main__":
    main()
