#!/usr/bin/env python
"""Benchmark of the B200 attention library (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Default workload: MQA decode at head_dim 512 (B=32, Hq=16, Hkv=1, per-sequence
KV length uniform in [1024, 8192], bf16): one step = one decode forward of
the whole batch (split-KV kernel, whose last CTA per sequence merges the
pieces, after a small kernel that zeroes its arrival counters).  The metric is the
KV-cache bytes read per second (each cached K/V byte counted once).  The
same line carries, measured in the same run and each in an object of its
own: the d=512 MQA causal prefill (B=2, Hq=16, S=4096; key "prefill"),
absorbed-MLA decode ("mla_decode"), GQA d=128 decode ("gqa_decode") and GQA
causal prefill ("gqa_prefill") -- each with its dominant kernel's roofline
fraction against the measured and the datasheet peaks, the prefill ones with
the CPU oracle on a sample -- plus the CPU oracle's throughput on a bounded
sample of the main workload and an end-to-end figure through the C ABI with
host buffers.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronize on both sides, replayed from CUDA graphs of two
steps that hold the steps' C-ABI launches; CUDA events on the replay stream
(one between consecutive replays for the step-time percentiles).  The dominant kernel's
duration is timed the same way on graphs of 20 back-to-back launches of that
kernel alone (a top-k step is one attn_topk_fwd: the decode kernel gathers
the selected rows itself).  With N GPUs
(torchrun) every rank runs its own replica of the workload and the time is
the max over ranks.  Inputs are larger than L2 for the decode workloads (the
KV cache alone is 302 MB vs 126 MB L2).  Other workloads: --workload
gqa_decode, mla_decode, gqa_extend, mla_topk_decode, mqa_prefill,
gqa_prefill, mla_prefill, mqa_prefill_tiny.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attention_mqa_gqa_b200 import workloads as wl  # noqa: E402

_CSRC = "attention_mqa_gqa_b200/csrc/"
# the sources each kernel is built from (a committed ncu traffic figure is
# used only while these are unchanged)
KERNEL_SOURCES = {
    "decode_split_kernel": [_CSRC + "sm100.cuh", _CSRC + "decode_kernel.cuh", _CSRC + "attn_api.cu"],
    "mla_pair_kernel": [_CSRC + "sm100.cuh", _CSRC + "decode_kernel.cuh", _CSRC + "mla_pair_kernel.cuh",
                        _CSRC + "attn_api.cu"],
    "prefill_kernel": [_CSRC + "sm100.cuh", _CSRC + "prefill_kernel.cuh", _CSRC + "attn_api.cu"],
    "prefill_ab_kernel": [_CSRC + "sm100.cuh", _CSRC + "prefill_kernel.cuh", _CSRC + "prefill_ab_kernel.cuh",
                          _CSRC + "attn_api.cu"],
    "gather_rows_kernel": [_CSRC + "sm100.cuh", _CSRC + "gather_rows.cuh", _CSRC + "attn_api.cu"],
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures: ~8 TB/s HBM3e, 2.25 PFLOP/s dense bf16/fp16 (no sparsity)
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


# ----------------------------------------------------------------- accounting

def keys_of(w, inp):
    """Keys each sequence attends to: its length, or for a top-k workload
    the number of selected positions."""
    return inp["n_sel"] if w.topk else inp["skv"]


def kv_bytes(w, skv) -> int:
    """Cached K/V bytes one decode step must read: every key row of every
    sequence once (MLA: the 576-wide row once, V aliases its first 512).
    For a top-k workload pass the selected counts: the selected rows once."""
    n = int(sum(int(x) for x in skv))
    el = 2
    if w.mla:
        return n * w.d_k * el
    return n * w.Hkv * (w.d_k + w.d_v) * el


def visible_pairs(w, skv) -> int:
    """Number of (query row, key) pairs the softmax covers, over all heads.
    Causal rows are bottom-right aligned: row i of Sq sees
    max(0, i + L - Sq + 1) of a sequence's L keys, so the last min(Sq, L)
    rows see L - c + 1 .. L keys (c = that count)."""
    tot = 0
    for L in skv:
        L = int(L)
        if not w.causal:
            tot += w.Sq * L
        else:
            c = min(w.Sq, L)
            tot += (2 * L - c + 1) * c // 2
    return tot * w.Hq


def flops(w, skv) -> int:
    return 2 * (w.d_k + w.d_v) * visible_pairs(w, skv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def code_tokens(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace runs collapsed
    (string and character literals kept verbatim): what the compiler sees,
    so that editing a comment does not void a recorded measurement."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == "/" and text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
            out.append(" ")
        elif c == "/" and text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def sources_hash(kernel: str) -> str:
    """Hash of the code (comments and layout ignored) a kernel is built from."""
    h = hashlib.sha256()
    for s in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, s), encoding="utf-8") as f:
            h.update(code_tokens(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("sources_sha") != sources_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"attn_bench_clocks_{os.getpid()}.csv")
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.id = None

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.id:
                cmd += ["--id", self.id]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not rows:
            return None
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(mhz) if mhz else None,
                "sm_max_mhz": float(rows[0][2]) if rows[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- GPU arm

def steps_per_graph(steps: int) -> int:
    """Steps captured in one CUDA graph: two (one if K is odd), so that K
    timed steps give K/2 replays and the step-time percentiles come from
    many samples rather than one."""
    return 2 if steps % 2 == 0 else 1


class GpuRunner:
    """Holds one workload's device tensors and launches steps through the C ABI."""

    def __init__(self, w, inp, device):
        from attention_mqa_gqa_b200 import binding

        self.b = binding
        self.w = w
        self.dev = device
        self.skv_host = inp["skv"]
        self.max_skv = inp["max_skv"]
        self.q = inp["q"].to(device)
        if w.mla:
            cache = inp["cache"].to(device)
            B, S, dk = cache.shape
            self.k = cache.view(B, 1, S, dk)
            self.v = cache.view(B, 1, S, dk)[..., : w.d_v]
            self._keep = cache
        else:
            self.k = inp["k"].to(device)
            self.v = inp["v"].to(device)
        self.skv = inp["skv"].to(device)
        self.topk = w.topk
        if self.topk:
            # the step: attn_topk_fwd, the MLA decode that gathers the
            # selected rows of the latent cache itself (one pass)
            if not w.mla:
                raise ValueError("top-k workloads are defined on the MLA latent cache")
            self.cache_rows = self.max_skv
            self.idx = inp["idx"].to(device)
            self.n_sel = inp["n_sel"].to(device)
            self.max_skv = self.topk
        self.out = torch.empty(w.B, w.Hq, w.Sq, w.d_v, dtype=w.dtype, device=device)
        self.lse = torch.empty(w.B, w.Hq, w.Sq, dtype=torch.float32, device=device)
        nws = binding.workspace_bytes(w.B, w.Hq, w.Hkv, w.Sq, self.max_skv, w.d_k, w.d_v)
        self.ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=device)
        self.plan = binding.plan(w.B, w.Hq, w.Hkv, w.Sq, self.max_skv, w.d_k, w.d_v, w.dtype)
        self.stream = torch.cuda.current_stream(device)
        self._args = None

    def args(self):
        if self._args is None and self.topk:
            b, w = self.b, self.w
            st = lambda t: b.Strides(t.stride(0), t.stride(1), t.stride(2))
            self._args = (self.q.data_ptr(), self.k.data_ptr(), self.out.data_ptr(),
                          self.lse.data_ptr(), w.B, w.Hq, self.idx.data_ptr(), self.idx.stride(0),
                          self.n_sel.data_ptr(), self.skv.data_ptr(), self.topk, self.cache_rows,
                          w.d_k, w.d_v, w.scale, b.dtype_code(w.dtype), st(self.q), st(self.k),
                          st(self.out), self.ws.data_ptr(), self.ws.numel(),
                          self.stream.cuda_stream)
        if self._args is None:
            b, w = self.b, self.w
            st = lambda t: b.Strides(t.stride(0), t.stride(1), t.stride(2))
            self._args = (self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(),
                          self.out.data_ptr(), self.lse.data_ptr(), w.B, w.Hq, w.Hkv, w.Sq,
                          self.skv.data_ptr(), self.max_skv, w.d_k, w.d_v, w.scale,
                          int(w.causal), b.dtype_code(w.dtype), st(self.q), st(self.k),
                          st(self.v), st(self.out), self.ws.data_ptr(), self.ws.numel(),
                          self.stream.cuda_stream)
        return self._args

    def call(self, entry="attn_fwd"):
        """One launch group: "attn_fwd" = "forward" (a whole step: attn_fwd,
        or attn_topk_fwd for a top-k workload)."""
        if self.topk:
            rc = self.b.topk_raw(*self.args())
            if rc != 0:
                raise self.b.AttnError(rc, "attn_topk_fwd")
            return
        if entry == "forward":
            entry = "attn_fwd"
        rc = self.b.fwd_raw(*self.args(), entry=entry)
        if rc != 0:
            raise self.b.AttnError(rc, entry)

    @property
    def decode(self):
        return self.plan["path"] == 1

    def launches_per_step(self):
        return 2 if self.decode else 1

    def _graph(self, nsteps, entry="attn_fwd"):
        """Capture `nsteps` launches of `entry` (a whole step for attn_fwd)
        into one CUDA graph on a side stream."""
        side = torch.cuda.Stream(self.dev)
        saved, self.stream, self._args = self.stream, side, None
        graph = torch.cuda.CUDAGraph()
        torch.cuda.synchronize(self.dev)
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                for _ in range(nsteps):
                    self.call(entry)
        torch.cuda.synchronize(self.dev)
        self.stream, self._args = saved, None
        return graph, side

    def _replay_ms(self, graph, side, reps, warmup_reps, per_replay=None):
        """Total ms of `reps` back-to-back replays (events on the replay
        stream); with a list in `per_replay`, also each replay's ms (an event
        between consecutive replays, so the replays still run back to back)."""
        with torch.cuda.stream(side):  # replays run on the current stream
            for _ in range(warmup_reps):
                graph.replay()
            torch.cuda.synchronize(self.dev)
            ev = [torch.cuda.Event(enable_timing=True)
                  for _ in range(reps + 1 if per_replay is not None else 2)]
            ev[0].record(side)
            for r in range(reps):
                graph.replay()
                if per_replay is not None:
                    ev[r + 1].record(side)
            ev[-1].record(side)
            torch.cuda.synchronize(self.dev)
        if per_replay is not None:
            per_replay.extend(ev[r].elapsed_time(ev[r + 1]) for r in range(reps))
        return ev[0].elapsed_time(ev[-1])

    def timed(self, steps, warmup):
        """Warm up, then time exactly `steps` steps replayed from CUDA graphs
        (captured two steps at a time); CUDA events on the replay stream.
        Returns (total_ms, dominant kernel mean ms, other kernel mean ms).
        The dominant kernel's duration is timed the same way over graphs of
        20 back-to-back launches of it alone: for decode, attn_fwd's split
        kernel with the merge of the pieces inside it (with the few-
        microsecond kernel that zeroes its arrival counters and lets it start
        early); for a top-k step the same, the kernel gathering the rows."""
        per = steps_per_graph(steps)
        graph, side = self._graph(per)
        reps = []
        total = self._replay_ms(graph, side, steps // per, max(1, warmup // per), reps)
        self.step_ms_samples = [r / per for r in reps]  # mean step time of each replay
        del graph
        if not self.decode:
            return total, total / steps, 0.0
        kg, kside = self._graph(20, "forward")
        k_ms = self._replay_ms(kg, kside, 10, 1) / 200
        del kg
        return total, k_ms, max(total / steps - k_ms, 0.0)

    def e2e(self, steps, warmup, inp):
        """Same step through the C ABI with the step's inputs in pinned host
        memory: H2D copy of the inputs, the forward, D2H copy of out and lse,
        synchronised every step.  Decode keeps the KV cache resident (it is
        state, not a per-step input); prefill copies q, k and v every step;
        a top-k step also copies the selection (idx, n_sel)."""
        pin = lambda t: t.pin_memory()
        hq = pin(inp["q"])
        hskv = pin(inp["skv"])
        hk = hv = hidx = hnsel = None
        dskv = self.skv
        if not self.decode:  # prefill shapes have separate K and V tensors
            hk, hv = pin(inp["k"]), pin(inp["v"])
        if self.topk:
            hidx, hnsel = pin(inp["idx"]), pin(inp["n_sel"])
        hout = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        hlse = torch.empty(self.lse.shape, dtype=self.lse.dtype).pin_memory()
        h2d = hq.numel() * hq.element_size() + hskv.numel() * 4
        if hk is not None:
            h2d += hk.numel() * hk.element_size() + hv.numel() * hv.element_size()
        if hidx is not None:
            h2d += hidx.numel() * 4 + hnsel.numel() * 4
        d2h = hout.numel() * hout.element_size() + hlse.numel() * 4

        def step():
            self.q.copy_(hq, non_blocking=True)
            dskv.copy_(hskv, non_blocking=True)
            if hidx is not None:
                self.idx.copy_(hidx, non_blocking=True)
                self.n_sel.copy_(hnsel, non_blocking=True)
            if hk is not None:
                self.k.copy_(hk, non_blocking=True)
                self.v.copy_(hv, non_blocking=True)
            self.call()
            hout.copy_(self.out, non_blocking=True)
            hlse.copy_(self.lse, non_blocking=True)
            self.stream.synchronize()

        for _ in range(warmup):
            step()
        torch.cuda.synchronize(self.dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(self.stream)
        for _ in range(steps):
            step()
        b_.record(self.stream)
        torch.cuda.synchronize(self.dev)
        return a.elapsed_time(b_), h2d, d2h


def metric_of(w):
    if w.is_decode:
        return "kv_cache_read_GBps", "GB/s", True
    return "attention_TFLOPs", "TFLOP/s", True


def value_of(w, skv, ms):
    if w.is_decode:
        return kv_bytes(w, skv) / (ms * 1e-3) / 1e9
    return flops(w, skv) / (ms * 1e-3) / 1e12


def roofline(w, skv, kernel_ms, peaks, peak_src, long_run, traffic):
    """Roofline of the dominant kernel: `frac` against the measured B200
    peaks (MEASURED_PEAKS.json, else the fallback figures), and
    `frac_nominal` against the datasheet figure (~8 TB/s HBM, 2.25 PFLOP/s
    dense bf16), each labelled with its denominator."""
    if w.is_decode:
        achieved = kv_bytes(w, skv) / (kernel_ms * 1e-3) / 1e9
        peak = float(peaks["hbm_gbs"])
        nom = NOMINAL_PEAKS["hbm_gbs"]
        return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": traffic,
                "peak_source": f"hbm_gbs ({peak_src})",
                "peak_nominal": nom, "frac_nominal": round(achieved / nom, 4),
                "peak_nominal_source": "B200 datasheet HBM3e ~8 TB/s"}
    key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
    peak = float(peaks[key])
    if w.dtype == torch.float16:
        key += " (fp16 = bf16 dense rate)"
    achieved = flops(w, skv) / (kernel_ms * 1e-3) / 1e12
    nom = NOMINAL_PEAKS["bf16_tflops"]
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": f"{key} ({peak_src})",
            "peak_nominal": nom, "frac_nominal": round(achieved / nom, 4),
            "peak_nominal_source": "B200 datasheet dense bf16/fp16 2.25 PFLOP/s"}


def config_of(w, inp):
    """The workload (the same for the GPU arm and the reference arm; where it
    runs is reported beside it, in the line's `parallelism`)."""
    skv = inp["skv"]
    d = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq, "d_k": w.d_k,
         "d_v": w.d_v, "causal": w.causal, "scale": round(w.scale, 6), "mla_absorbed": w.mla,
         "skv": f"U[{w.skv_lo},{w.skv_hi}] seed {w.seed}" if w.skv_lo != w.skv_hi else w.skv_lo,
         "skv_total": int(skv.sum())}
    if w.topk:
        sel = kv_bytes(w, inp["n_sel"])
        d["topk"] = w.topk
        d["selection"] = ("per sequence min(topk, skv) distinct positions, uniform, ascending "
                          f"(seed {w.seed}); {int(inp['n_sel'].sum())} rows selected")
        d["l2"] = (f"inputs larger than L2: selected rows {sel / 1e6:.0f} MB > 126 MB, gathered "
                   "from a {:.1f} GB cache".format(kv_bytes(w, skv) / 1e9))
    elif w.is_decode:
        d["l2"] = f"inputs larger than L2: KV {kv_bytes(w, skv) / 1e6:.0f} MB > 126 MB"
    else:
        qb = w.B * w.Hq * w.Sq * w.d_k * 2
        d["l2"] = (f"no flush: Q {qb / 1e6:.0f} MB and O stream through; K/V "
                   f"{kv_bytes(w, skv) / 1e6:.1f} MB are meant to stay in L2 (prefill reuses them)")
    return d


# ----------------------------------------------------------------- CPU oracle

def oracle_sample(w, inp, budget_s):
    """The first n sequences (all heads) whose estimated oracle cost fits the
    budget (the fp64 C oracle runs at roughly 1 GFLOP/s per thread; the
    numpy top-k oracle is timed on one sequence)."""
    if w.topk:
        t1 = max(run_oracle(w, inp, 1), 1e-3)
        return max(1, min(w.B, int(budget_s / t1)))
    rate = 1.0e9 * (os.cpu_count() or 1)
    skv = inp["skv"].tolist()
    n, acc = 0, 0.0
    for b in range(w.B):
        cost = flops(w.scaled(B=1), [skv[b]]) / rate
        if n > 0 and acc + cost > budget_s:
            break
        n += 1
        acc += cost
    return n


def run_oracle(w, inp, n, nthreads=None):
    """Seconds the oracle takes on the first n sequences (all heads); the C
    oracle on `nthreads` host threads (default: all cores)."""
    from oracle import c_oracle

    t0 = time.perf_counter()
    if w.topk:
        from oracle import attention as npo

        npo.topk_attention_fwd(inp["q"][:n], inp["k"][:n], inp["v"][:n], inp["skv"][:n].tolist(),
                               inp["idx"][:n], inp["n_sel"][:n].tolist(), w.scale)
    else:
        c_oracle.attention_fwd(inp["q"][:n], inp["k"][:n], inp["v"][:n],
                               inp["skv"][:n].tolist(), w.scale, w.causal, nthreads=nthreads)
    return time.perf_counter() - t0


def cpu_value(w, inp, n, secs):
    skv = keys_of(w, inp)[:n].tolist()
    wb = w.scaled(B=n)
    if w.is_decode:
        return kv_bytes(wb, skv) / secs / 1e9
    return flops(wb, skv) / secs / 1e12


# ----------------------------------------------------------------- main

def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def allreduce(x, op, world, device):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def reference_arm(args, world, rank):
    """The oracle as it stands, timed on the host cores; rank 0 only."""
    if rank != 0:
        return 0
    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(w)
    n = oracle_sample(w, inp, budget_s=args.ref_step_budget)
    from oracle import c_oracle

    c_oracle.build()
    steps = args.steps if args.steps else 3
    for _ in range(args.warmup):
        run_oracle(w, inp, n)
    t = 0.0
    for _ in range(steps):
        t += run_oracle(w, inp, n)
    val = cpu_value(w, inp, n, t / steps)
    metric, unit, hib = metric_of(w)
    cores = os.cpu_count() or 1
    sample = f"first {n} of {w.B} sequences, all {w.Hq} heads, per step" + (
        " (numpy fp64 top-k oracle)" if w.topk else "")
    line = {"impl": "reference", "metric": f"{w.name}_{metric}", "value": round(val, 4),
            "unit": unit, "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(t / steps * 1e3, 3), "higher_is_better": hib,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(w, inp), "parallelism": f"host cores x{cores}",
            "cpu_baseline": {"value": round(val, 4), "unit": unit, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(val, 4), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def measure_workload(w, inp, device, steps, warmup, world):
    g = GpuRunner(w, inp, device)
    if steps is None:  # size the timed region to about 2 s (a multiple of 20 steps)
        t_ms, _, _ = g.timed(20, 3)
        steps = int(min(20000, max(20, 2000.0 / max(t_ms / 20, 1e-3)))) // 20 * 20
    barrier(world)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(device)
    sampler.start()
    total_ms, k_ms, other_ms = g.timed(steps, warmup)
    clocks = sampler.stop()
    barrier(world)
    return g, steps, total_ms, k_ms, other_ms, clocks


def step_dist_of(g, steps):
    samples = sorted(g.step_ms_samples)
    pct = lambda q: samples[min(len(samples) - 1, int(q * (len(samples) - 1) + 0.5))]
    return {"p10": round(pct(0.1), 5), "p50": round(pct(0.5), 5), "p90": round(pct(0.9), 5),
            "replays": len(samples), "steps_per_replay": steps // len(samples)}


def kernel_name(w, g):
    if not g.decode:
        # d_k = 512: SM pairs that split the two matmuls
        return "prefill_ab_kernel" if w.d_k == 512 else "prefill_kernel"
    return "mla_pair_kernel" if w.mla else "decode_split_kernel"


def dominant_roofline(w, g, keys, k_ms, other_ms, total_ms, peaks, peak_src):
    kname = kernel_name(w, g)
    roof = roofline(w, keys, k_ms, peaks, peak_src, total_ms > 1000.0, traffic_for(kname, w.name))
    roof["kernel"] = kname
    roof["kernel_ms"] = round(k_ms, 5)
    if g.decode:
        # the pieces of each (sequence, kv head) are merged inside the split
        # kernel by the CTA that finishes the unit; kernel_ms covers the
        # launch with its small counter-zeroing kernel (launched just before
        # it, overlapping its start)
        roof["merge"] = "in kernel (last CTA of a unit)"
        roof["other_ms"] = round(other_ms, 5)
    return roof


def cpu_leg(w, inp, budget_s, one_core=True):
    """The fp64 C oracle (numpy for top-k) as it stands, on a bounded sample of
    the workload, on all host cores and (if asked) on one thread."""
    from oracle import c_oracle

    c_oracle.build()
    cores = os.cpu_count() or 1
    metric, unit, _ = metric_of(w)
    which = "numpy fp64 top-k oracle" if w.topk else "fp64 C oracle"
    if w.is_decode:
        n = oracle_sample(w, inp, budget_s=budget_s)
        secs = run_oracle(w, inp, n)
        d = {"value": round(cpu_value(w, inp, n, secs), 4), "unit": unit, "cores": cores,
             "kind": "oracle",
             "sample": f"first {n} of {w.B} sequences, all {w.Hq} heads ({secs:.1f} s, {which})"}
        if one_core and not w.topk:  # the same oracle on one host thread, first sequence
            s1 = run_oracle(w, inp, 1, nthreads=1)
            d["value_1core"] = round(cpu_value(w, inp, 1, s1), 4)
            d["sample_1core"] = f"first sequence, all {w.Hq} heads, one thread ({s1:.2f} s)"
        return d
    # prefill: the oracle threads over (sequence, query head); one head per
    # host thread, every query row of each
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hq)][:cores]
    work = flops(w.scaled(B=1, Hq=1), inp["skv"][:1].tolist())  # one head's FLOPs
    t0 = time.perf_counter()
    c_oracle.attention_fwd(inp["q"], inp["k"], inp["v"], inp["skv"].tolist(), w.scale, w.causal,
                           pairs=pairs)
    secs = time.perf_counter() - t0
    d = {"value": round(work * len(pairs) / secs / 1e12, 6), "unit": unit, "cores": cores,
         "kind": "oracle",
         "sample": f"{len(pairs)} of {w.B * w.Hq} (sequence, head) pairs, every query row "
                   f"({secs:.1f} s, {which})"}
    if one_core:
        t0 = time.perf_counter()
        c_oracle.attention_fwd(inp["q"], inp["k"], inp["v"], inp["skv"].tolist(), w.scale,
                               w.causal, nthreads=1, pairs=pairs[:1])
        s1 = time.perf_counter() - t0
        d["value_1core"] = round(work / s1 / 1e12, 6)
        d["sample_1core"] = f"one (sequence, head) pair, every query row, one thread ({s1:.2f} s)"
    return d


# Workloads whose figures the default line carries beside its own (key in
# the line: workload), each measured in the same run the same way.
SECONDARY = (("prefill", "mqa_prefill"), ("mla_decode", "mla_decode"),
             ("gqa_decode", "gqa_decode"), ("gqa_prefill", "gqa_prefill"))


def secondary(name, rank, world, device, args, peaks, peak_src, with_cpu):
    import torch.distributed as dist_mod

    w = wl.WORKLOADS[name]
    if rank:
        w = w.scaled(seed=w.seed + 1000 * rank)
    inp = wl.make_inputs(w)
    g, steps, tot, k_ms, other_ms, clocks = measure_workload(w, inp, device, args.steps,
                                                             args.warmup, world)
    mx = allreduce(tot, dist_mod.ReduceOp.MAX if world > 1 else None, world, device)
    keys = keys_of(w, inp)
    work = kv_bytes(w, keys) if w.is_decode else flops(w, keys)
    work = allreduce(work, dist_mod.ReduceOp.SUM if world > 1 else None, world, device)
    metric, unit, _ = metric_of(w)
    scale_div = 1e9 if w.is_decode else 1e12
    d = {"metric": f"{w.name}_{metric}", "value": round(work * steps / (mx * 1e-3) / scale_div, 3),
         "unit": unit, "steps": steps, "ms_per_step": round(mx / steps, 5),
         "ms_per_step_dist": step_dist_of(g, steps), "config": config_of(w, inp),
         "roofline": dominant_roofline(w, g, keys, k_ms, other_ms, tot, peaks, peak_src),
         "gpu_launches": g.launches_per_step() * steps, "clocks": clocks}
    del g
    if with_cpu and not w.is_decode:
        d["cpu_baseline"] = cpu_leg(w, inp, budget_s=10.0)
    return d


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mqa_decode", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the other workloads' figures in the default line")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--ref-step-budget", type=float, default=2.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_setup(args.gpus)
    if args.impl == "reference":
        rc = reference_arm(args, world, rank)
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return rc

    from attention_mqa_gqa_b200 import binding, build

    if not os.path.exists(binding.LIB_PATH):
        build.build()
    binding.load()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()

    w = wl.WORKLOADS[args.workload]
    if rank:
        w = w.scaled(seed=w.seed + 1000 * rank)  # each replica its own batch
    inp = wl.make_inputs(w)
    g, steps, total_ms, k_ms, other_ms, clocks = measure_workload(w, inp, device, args.steps,
                                                                  args.warmup, world)
    import torch.distributed as dist_mod

    max_ms = allreduce(total_ms, dist_mod.ReduceOp.MAX if world > 1 else None, world, device)
    keys = keys_of(w, inp)
    work = kv_bytes(w, keys) if w.is_decode else flops(w, keys)
    work_all = allreduce(work, dist_mod.ReduceOp.SUM if world > 1 else None, world, device)
    ms_step = max_ms / steps
    scale_div = 1e9 if w.is_decode else 1e12
    value = work_all * steps / (max_ms * 1e-3) / scale_div
    metric, unit, hib = metric_of(w)
    roof = dominant_roofline(w, g, keys, k_ms, other_ms, total_ms, peaks, peak_src)
    if w.topk:
        roof["gather"] = "in kernel (cp.async rows into the decode kernel's ring)"

    # end to end through the C ABI with host buffers
    e2e_steps = max(10, min(steps, 200))
    e_ms, h2d, d2h = g.e2e(e2e_steps, 3, inp)
    e_ms = allreduce(e_ms, dist_mod.ReduceOp.MAX if world > 1 else None, world, device)
    e_val = work_all * e2e_steps / (e_ms * 1e-3) / scale_div
    assert binding.last_device_error() == binding.ATTN_OK, "device-side wait timed out"

    line = {"metric": f"{w.name}_{metric}", "value": round(value, 3), "unit": unit,
            "n_gpus": world, "steps": steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 5), "ms_per_step_dist": step_dist_of(g, steps),
            "higher_is_better": hib, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.dtype == torch.bfloat16 else "fp16",
            "data": "synthetic (seeded N(0,1), rounded once to the element type)",
            "config": config_of(w, inp),
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "roofline": roof, "gpu_launches": g.launches_per_step() * steps,
            "clocks": clocks,
            "e2e": {"value": round(e_val, 3), "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps}}
    del g

    with_cpu = rank == 0 and world == 1 and not args.no_cpu
    if not args.no_secondary and args.workload == "mqa_decode":
        for key, name in SECONDARY:
            line[key] = secondary(name, rank, world, device, args, peaks, peak_src, with_cpu)
            torch.cuda.empty_cache()
        assert binding.last_device_error() == binding.ATTN_OK, "device-side wait timed out"

    if with_cpu:
        line["cpu_baseline"] = cpu_leg(w, inp, budget_s=15.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
