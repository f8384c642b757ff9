#!/usr/bin/env python
"""Benchmark of the tensor-parallel sharded-linear path on B200.

One step is one pass of the whole hot path over one batch of synthetic input
(workload ``block``, the default):

  1. GQA fused-QKV column-parallel linear  x[4,1024,4096] bf16, 32 q + 8 kv
     heads of 128, tp 8, bias                      (sub-parameter partition)
  2. RMSNorm (eps 1e-6, centred scale) fused into c_fc 4096->14336
     column-parallel + GELU(erf) -> c_proj 14336->4096 row-parallel with the
     partial-sum reduction in the epilogue         x[8,1024,4096] bf16, tp 8
  3. decode LM head x[32,4096] over W[128256,4096] bf16, 8 vocab shards x 4
     chunks, fp32 logits kept on chip, per-shard + global argmax

``value`` is the sharded-linear FLOP rate of the step (algorithmic FLOPs of
the three contractions / step time).  ``--workload stack`` runs the 4-layer
residual stack x[4,4096,8192], 8192->28672->8192 instead (``stack_layer``: one
of its layers on x[1,4096,8192], the same GEMM shapes in K and N, small enough
for a multi-pass profiler capture); the other workloads (``qkv``, ``mlp``,
``lmhead``, ``swiglu``, ``seqpar``, ``embed``, ``tp_ranks``) time one part or a
next-step variant of the path.

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload, on the host cores, without loading the CUDA library.  Under torchrun
(N > 1) every rank runs an independent replica (the single-GPU path has no
exchange) and the step time is the max over ranks; ``--workload tp_ranks``
instead runs one tensor-parallel rank per GPU, exchanging through peer memory.
"""
from __future__ import annotations

import argparse
import datetime
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

from workloads import configs as C  # noqa: E402
from workloads import gen  # noqa: E402

METRIC = "sharded-linear TFLOP/s (% bf16 peak); LM-head decode GB/s (% HBM) at 1 B200"
DECODE_LAUNCHES = 50
PARTS_PAUSE_S = 0.3


def lmhead_kernel(batch: int) -> str:
    """The LM-head kernel the library runs for this batch (TPL_LMHEAD_TN, read
    the way the library reads it: 2 by default)."""
    mode = os.environ.get("TPL_LMHEAD_TN", "2").strip() or "2"
    if batch <= 32 and mode in ("1", "2"):
        return "lmhead_argmax_tn<64>" if mode == "2" else "lmhead_argmax_tn<128>"
    return "lmhead_argmax_tcgen05"
FUSED_NORM = True   # the block's RMSNorm runs inside its c_fc GEMM
ALONE_LAUNCHES = 30
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ ncu traffic

def _src_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "tensor_transformer_linear_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def ncu_traffic(kernel: str, workload: str, sources):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.txt")
    if not os.path.exists(p):
        return None
    cur = _src_hash(sources)
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == kernel and f[1] == workload:
            return float(f[2]) if f[3] == cur else None
    return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and throttle reasons during the timed region, from two sources:
    nvidia-smi every 100 ms, and NVML read every ~2 ms by a host thread.  A
    block region of a few ms holds no nvidia-smi sample, but NVML samples fall
    inside it; the record prefers the samples taken inside the region."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h: nvmlClocksEventReason*)
    NVML_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                 "hw_thermal_slowdown": 0x40}
    POLL_S = 0.002

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None
        self.thread = None
        self.polls = []
        self.nvml_max = None

    def _nvml_handle(self):
        import pynvml as N
        N.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.index).uuid)
            return N, N.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
        except Exception:
            return N, N.nvmlDeviceGetHandleByIndex(self.index)

    def _poll(self, N, h):
        while not self.halt.is_set():
            try:
                t = datetime.datetime.now()
                sm = N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)
                r = N.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.polls.append((t, float(sm), int(r)))
            except Exception:
                return
            self.halt.wait(self.POLL_S)

    def start(self):
        import threading
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        try:
            N, h = self._nvml_handle()
            self.nvml_max = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
            self.halt = threading.Event()
            self.thread = threading.Thread(target=self._poll, args=(N, h), daemon=True)
            self.thread.start()
        except Exception:
            self.thread = None

    def _smi_rows(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 10:
                try:
                    ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                except ValueError:
                    continue
                rows.append((ts, f[1:]))
        os.unlink(self.path)
        return rows

    def stop(self, t0=None, t1=None):
        """Median SM clock and the throttle reasons seen; with a host-time window
        [t0, t1] (datetime.now() values) only the samples taken inside it count
        (all samples if none falls inside)."""
        if self.thread is not None:
            self.halt.set()
            self.thread.join(timeout=5)
        rows = self._smi_rows()
        polls = list(self.polls)
        if t0 is not None and t1 is not None:
            rows_in = [r for ts, r in rows if t0 <= ts <= t1]
            polls_in = [p for p in polls if t0 <= p[0] <= t1]
        else:
            rows_in, polls_in = [r for _, r in rows], polls
        if not rows and not polls:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        smi = rows_in if (rows_in or polls_in) else [r for _, r in rows]
        reasons = {names[i] for r in smi for i in range(4) if r[5 + i] == "Active"}
        reasons |= {n for _, _, bits in polls_in for n, b in self.NVML_BITS.items() if bits & b}
        if polls_in:
            sm = [p[1] for p in polls_in]
            source = "NVML every 2 ms inside the timed region"
        else:
            sm = [float(r[1]) for r in smi if r[1].replace(".", "").isdigit()]
            source = ("nvidia-smi inside the timed region" if rows_in
                      else "nvidia-smi around the timed region (no sample inside it)")
        mx = [float(r[2]) for _, r in rows if r[2].replace(".", "").isdigit()]
        if self.nvml_max:
            mx.append(self.nvml_max)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm), "smi_samples_inside": len(rows_in), "source": source}


def clocks_rejected(clk) -> bool:
    """A hardware or thermal slowdown, or SM clocks held far below max with no
    reason given (a leftover clock lock), invalidates a timing."""
    if not clk:
        return False
    if set(clk["reasons"]) & {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}:
        return True
    sm, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    return bool(sm and mx and not clk["reasons"] and sm < 0.6 * mx)


def tensor_peak(pk, pk_kind, clk):
    """The bf16 GEMM peak that matches the regime the timed region ran in: the
    seconds-long power-capped figure when the clock record shows the power cap
    active, the burst figure otherwise.  Returns (peak, label)."""
    if clk and "sw_power_cap" in clk.get("reasons", ()):
        return pk["bf16_tflops_sustained"], f"{pk_kind} bf16 sustained (power cap active in the timed region)"
    return pk["bf16_tflops"], f"{pk_kind} bf16 burst"


# ------------------------------------------------------------------ end to end

E2E_SETS = 3


class E2EPipeline:
    """Steps end to end through pinned host buffers, as a serving loop runs them.

    Step k uploads its inputs from pinned host memory on an upload stream,
    computes on the launching stream and downloads its results into pinned host
    memory on a download stream, using device buffer set k % E2E_SETS.  Step
    k+1's upload and step k-1's download therefore overlap step k's compute;
    events order the reuse of each set (its upload waits for the download
    E2E_SETS steps back).  Every step's copies are inside the timed region.
    """

    def __init__(self, wl, stream):
        self.wl, self.stream = wl, stream
        names = list(dict.fromkeys(wl.io_in + wl.io_out))
        base = {a: getattr(wl, a) for a in names}
        self.sets = [base] + [{a: torch.empty_like(t) for a, t in base.items()}
                              for _ in range(E2E_SETS - 1)]
        src = wl.host_inputs() if hasattr(wl, "host_inputs") else base
        pin = lambda t: torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t.cpu())
        self.h_in = {a: pin(src[a]) for a in wl.io_in}
        self.h_out = [{a: torch.empty(base[a].shape, dtype=base[a].dtype, pin_memory=True)
                       for a in wl.io_out} for _ in range(E2E_SETS)]
        self.bytes_in = sum(t.numel() * t.element_size() for t in self.h_in.values())
        self.bytes_out = sum(t.numel() * t.element_size() for t in self.h_out[0].values())
        self.up, self.down = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: [torch.cuda.Event() for _ in range(E2E_SETS)]
        self.ev_up, self.ev_cmp, self.ev_down = ev(), ev(), ev()
        self.k = 0

    def step(self):
        wl, b = self.wl, self.k % E2E_SETS
        bufs = self.sets[b]
        if self.k >= E2E_SETS:
            self.up.wait_event(self.ev_down[b])
        with torch.cuda.stream(self.up):
            for a, h in self.h_in.items():
                bufs[a].copy_(h, non_blocking=True)
        self.ev_up[b].record(self.up)
        self.stream.wait_event(self.ev_up[b])
        if self.k >= E2E_SETS:
            self.stream.wait_event(self.ev_down[b])
        for a, t in bufs.items():
            setattr(wl, a, t)
        if hasattr(wl, "inputs_replaced"):
            wl.inputs_replaced()   # fresh inputs: nothing computed from the last ones holds
        wl.step(self.stream)
        self.ev_cmp[b].record(self.stream)
        self.down.wait_event(self.ev_cmp[b])
        with torch.cuda.stream(self.down):
            for a, h in self.h_out[b].items():
                h.copy_(bufs[a], non_blocking=True)
        self.ev_down[b].record(self.down)
        self.k += 1

    def close(self):
        torch.cuda.synchronize()
        for a, t in self.sets[0].items():
            setattr(self.wl, a, t)
        if hasattr(self.wl, "inputs_replaced"):
            self.wl.inputs_replaced()


# ------------------------------------------------------------------ workloads

class Block:
    """The default step: fused QKV + RMSNorm/MLP + decode LM head (or a subset, for profiling)."""

    def __init__(self, dev, parts=("qkv", "mlp", "lmhead")):
        import tensor_transformer_linear_b200 as T
        self.T = T
        q, m, l = C.GQA_QKV, C.TP_MLP, C.LM_HEAD
        self.q, self.m, self.l = q, m, l
        self.sel = parts
        names = {"qkv": q.name, "mlp": m.name, "lmhead": l.name}
        self.name = ("tp-block: " if len(parts) > 1 else "") + " + ".join(names[p] for p in parts)
        self.flops = 0.0
        self.gemm_flops = 0.0
        self.launches = []        # (part name, callable(stream)), in launch order
        # Attributes holding each step's inputs and results; every launch reads
        # them at call time, so the end-to-end pipeline can rotate buffer sets.
        self.io_in, self.io_out = [], []
        if "qkv" in parts:
            # inputs and weights, generated on the device by the seeded generator
            self.qx = C.qkv_x(q, dev)
            self.qw = C.qkv_w(q, dev)
            self.qb = C.qkv_bias(q, dev)
            self.qpart = T.tpl_partition_subparams(q.sub_sizes, q.tp, q.align)
            self.qy = torch.empty(q.M * q.out, dtype=torch.bfloat16, device=dev)
            self.launches.append(("qkv_column", lambda s: T.tpl_column_linear(
                self.qpart, self.qx, self.qw, self.qb, "none", y=self.qy, stream=s)))
            self.flops += q.flops()
            self.gemm_flops += q.flops()
            self.io_in.append("qx")
            self.io_out.append("qy")
        if "mlp" in parts:
            self.mx = C.mlp_x(m, dev)
            self.mlp = T.TPMLP(C.mlp_w1(m, 0, dev), C.mlp_w2(m, 0, dev), m.tp, m.act,
                               scale=C.mlp_scale(m, 0, dev), centered=True, norm=True,
                               fused_norm=FUSED_NORM)
            self.my = torch.empty((m.M, m.hidden), dtype=torch.bfloat16, device=dev)
            self.xn = torch.empty_like(self.mx)
            self.h = torch.empty(m.M * m.inter, dtype=torch.bfloat16, device=dev)
            mlp = self.mlp
            # the RMSNorm kernel on its own (an L2-flushed launch outside the step)
            self.alone_launches = {"rmsnorm": lambda s: T.tpl_rmsnorm(
                self.mx, mlp.scale, True, 1e-6, y=self.xn, stream=s)}
            if FUSED_NORM:
                # RMSNorm inside the c_fc GEMM: no normalised copy of x
                self.norm_ws = mlp.norm_workspace(m.M, dev)
                self.launches += [
                    ("mlp_column_rmsnorm_gelu", lambda s: T.tpl_column_linear_rmsnorm(
                        mlp.part, self.mx, mlp.w1, None, 1e-6, m.act, self.norm_ws, y=self.h,
                        stream=s))]
            else:
                self.launches += [
                    ("rmsnorm", self.alone_launches["rmsnorm"]),
                    ("mlp_column_gelu", lambda s: T.tpl_column_linear(
                        mlp.part, self.xn, mlp.w1, None, m.act, y=self.h, stream=s))]
            self.launches += [
                ("mlp_row_reduce", lambda s: T.tpl_row_linear_reduce(
                    self.h, mlp.k_w, m.M, mlp.w2, None, None, y=self.my, stream=s))]
            self.flops += m.flops()
            self.gemm_flops += m.flops()
            self.io_in.append("mx")
            self.io_out.append("my")
        if "lmhead" in parts:
            self.lx = C.lm_x(l, dev)
            self.lw = C.lm_w(l, dev)
            self.ws = T.lmhead_workspace(l.batch, l.vocab, l.tp, l.n_chunks, dev)
            self.ids = torch.empty(l.batch, dtype=torch.int32, device=dev)
            self.smax = torch.empty((l.tp, l.batch), dtype=torch.float32, device=dev)
            self.sidx = torch.empty((l.tp, l.batch), dtype=torch.int32, device=dev)
            self.launches.append(("lmhead_argmax", lambda s: T.tpl_lmhead_argmax(
                self.lx, self.lw, l.tp, l.n_chunks, self.ws, ids=self.ids, shard_max=self.smax,
                shard_idx=self.sidx, stream=s)))
            self.flops += l.flops()
            self.io_in.append("lx")
            self.io_out += ["ids", "smax", "sidx"]
        self.parts = [n for n, _ in self.launches]

    def step(self, stream, events=None, skip=()):
        for i, (name, fn) in enumerate(self.launches):
            if events is not None:
                events[i].record(stream)
            if name not in skip:
                fn(stream)
        if events is not None:
            events[len(self.launches)].record(stream)

    def gemm_part_ids(self):
        return [i for i, n in enumerate(self.parts)
                if n in ("qkv_column", "mlp_column_gelu", "mlp_column_rmsnorm_gelu",
                         "mlp_row_reduce")]

    def lmhead_bytes(self):
        return self.l.algorithmic_bytes() if "lmhead" in self.sel else None

    def hbm_parts(self):
        if "mlp" not in self.sel:
            return []
        return [("roofline_rmsnorm", "rmsnorm_cta", "rmsnorm", 2 * 2 * self.m.M * self.m.hidden)]


class Stack:
    """The 4-layer residual TP stack (or another MLPWorkload of residual layers)."""

    def __init__(self, dev, w=C.STACK4):
        import tensor_transformer_linear_b200 as T
        self.T = T
        self.w = w
        self.name = w.name
        self.x0 = C.mlp_x(w, dev)
        self.x = self.x0.clone()
        self.io_in, self.io_out = ["x"], ["x"]   # the residual stream is updated in place
        self.layers = [T.TPMLP(C.mlp_w1(w, l, dev), C.mlp_w2(w, l, dev), w.tp, w.act,
                               norm=True, residual=True, fused_norm=FUSED_NORM)
                       for l in range(w.layers)]
        # the fused norm's workspace, one for every layer (they run one after another)
        self.ws = self.layers[0].norm_workspace(w.M, dev) if FUSED_NORM else None
        self.flops = w.flops()
        self.gemm_flops = w.flops()
        self.parts = []
        for l in range(w.layers):
            if FUSED_NORM:
                self.parts += [f"l{l}_column_rmsnorm_gelu", f"l{l}_row_reduce_residual"]
            else:
                self.parts += [f"l{l}_rmsnorm", f"l{l}_column_gelu", f"l{l}_row_reduce_residual"]
        self.launches_per_step = len(self.parts)

    def step(self, stream, events=None):
        T = self.T
        mark = (lambda i: events[i].record(stream)) if events is not None else (lambda i: None)
        i = 0
        for layer in self.layers:
            M = self.x.shape[0]
            h = layer._buf("h", M * layer.inter, self.x)
            if FUSED_NORM:
                mark(i)
                T.tpl_column_linear_rmsnorm(layer.part, self.x, layer.w1, None, 1e-6, layer.act,
                                            self.ws, y=h, stream=stream)
                i += 1
            else:
                xn = layer._buf("xn", self.x.numel(), self.x).view(M, -1)
                mark(i)
                T.tpl_rmsnorm(self.x, None, False, 1e-6, y=xn, stream=stream)
                mark(i + 1)
                T.tpl_column_linear(layer.part, xn, layer.w1, None, layer.act, y=h,
                                    stream=stream)
                i += 2
            mark(i)
            T.tpl_row_linear_reduce(h, layer.k_w, M, layer.w2, None, self.x, y=self.x,
                                    stream=stream)
            i += 1
        mark(i)

    def host_inputs(self):
        return {"x": self.x0}

    def lmhead_bytes(self):
        return None

    def hbm_parts(self):
        return []

    def gemm_part_ids(self):
        return [i for i, n in enumerate(self.parts) if not n.endswith("_rmsnorm")]


class NextRows:
    """Workloads of the path's next rows, one at a time (measured like the block).

    swiglu: fused [wi0; wi1] column projection x[8192,4096] -> 2 x 14336, tp 8
            (full d_ff per gate, as the PaLM note on the page says).
    embed:  vocab-sharded lookup of 8192 token ids in W[128256,4096] bf16, tp 8.
    seqpar: the RMSNorm + TP MLP block in sequence-parallel form (x[8,1024,4096],
            tp 8): RMSNorm of the rank-major slices -> all-gather c_fc + GELU ->
            c_proj with the reduce-scatter and residual.
    """

    def __init__(self, dev, kind):
        import tensor_transformer_linear_b200 as T
        self.T, self.kind = T, kind
        m, l = C.TP_MLP, C.LM_HEAD
        self.m, self.l = m, l
        self.flops = 0.0
        self.gemm_flops = 0.0
        self.hbm_bytes = 0
        self.launches = []
        if kind == "swiglu":
            self.F = m.inter
            self.name = WORKLOAD_NAMES["swiglu"]
            self.x = C.mlp_x(m, dev)
            self.w = gen.normal((2 * self.F, m.hidden), m.w_sigma, tensor_id=gen.TID_W1,
                                device=dev)
            self.h = torch.empty(m.M * self.F, dtype=torch.bfloat16, device=dev)
            self.launches.append(("swiglu_column", lambda s: T.tpl_swiglu_column_linear(
                self.x, self.w, self.F, m.tp, h=self.h, stream=s)))
            self.flops = self.gemm_flops = 2.0 * m.M * m.hidden * 2 * self.F
            self.io_in, self.io_out = ["x"], ["h"]
        elif kind == "embed":
            self.name = WORKLOAD_NAMES["embed"]
            g = torch.Generator(device=dev)
            g.manual_seed(0)
            self.ids = torch.randint(0, l.vocab, (m.M,), generator=g, device=dev,
                                     dtype=torch.int32)
            self.table = C.lm_w(l, dev)
            self.out = torch.empty((m.M, l.hidden), dtype=torch.bfloat16, device=dev)
            self.launches.append(("embed_lookup", lambda s: T.tpl_embedding_lookup(
                self.ids, self.table, l.tp, out=self.out, stream=s)))
            self.hbm_bytes = m.M * l.hidden * 2 * 2 + m.M * 4
            self.io_in, self.io_out = ["ids"], ["out"]
        elif kind == "seqpar":
            b, sq = m.batch, m.seq
            self.name = WORKLOAD_NAMES["seqpar"]
            self.x = C.mlp_x(m, dev)      # read as the rank-major [tp][b][s/tp][H] layout
            self.scale = C.mlp_scale(m, 0, dev)
            self.w1 = C.mlp_w1(m, 0, dev)
            self.part = T.tpl_partition_subparams([m.inter], m.tp, 1)
            self.k_w = [self.part.shard_width[r] for r in range(m.tp)]
            self.w2 = T.pack_row_weight(C.mlp_w2(m, 0, dev), self.k_w)
            self.xn = torch.empty_like(self.x)
            self.hbuf = torch.empty(m.M * m.inter, dtype=torch.bfloat16, device=dev)
            self.y = torch.empty_like(self.x)
            self.launches += [
                ("sp_rmsnorm", lambda s: T.tpl_rmsnorm(self.x, self.scale, True, 1e-6,
                                                       y=self.xn, stream=s)),
                ("sp_column_gelu", lambda s: T.tpl_column_linear_allgather(
                    self.part, self.xn, b, sq, self.w1, None, m.act, y=self.hbuf, stream=s)),
                ("sp_row_scatter", lambda s: T.tpl_row_linear_reduce_scatter(
                    self.hbuf, self.k_w, b, sq, self.w2, None, self.x, y=self.y, stream=s))]
            self.flops = self.gemm_flops = m.flops()
            self.io_in, self.io_out = ["x"], ["y"]
        elif kind == "tp_ranks":
            # The RMSNorm + MLP block as tp rank-local shares, the ranks run one
            # after another on this GPU, their peers' buffers standing in as
            # local tensors: each rank normalises its token slice, runs c_fc +
            # GELU over all tokens reading every rank's slice (peer gather),
            # scatters its c_proj partials into every rank's receive buffer,
            # and sums its slots into its slice of the residual stream.
            tp, b, sq, N, I = m.tp, m.batch, m.seq, m.hidden, m.inter
            M, kr = m.M, m.inter // m.tp
            rows = b * (sq // tp)
            self.name = WORKLOAD_NAMES["tp_ranks"]
            self.xs = C.mlp_x(m, dev).view(b, tp, sq // tp, N).transpose(0, 1).contiguous()
            self.scale = C.mlp_scale(m, 0, dev)
            self.xn = torch.empty_like(self.xs)
            self.w1 = C.mlp_w1(m, 0, dev)
            self.w2p = T.pack_row_weight(C.mlp_w2(m, 0, dev), [kr] * tp)
            self.p_rank = T.tpl_partition_subparams([kr], 1, 1)
            self.hbuf = torch.empty(tp * M * kr, dtype=torch.bfloat16, device=dev)
            self.recv = [torch.empty(tp * rows * N, dtype=torch.bfloat16, device=dev)
                         for _ in range(tp)]

            def norm_all(s):
                for q in range(tp):
                    T.tpl_rmsnorm(self.xs[q], self.scale, True, 1e-6, y=self.xn[q], stream=s)

            def gather_all(s):
                hs = self.hbuf.view(tp, M * kr)
                slices = [self.xn[q] for q in range(tp)]
                for r in range(tp):
                    T.tpl_column_linear_gather(self.p_rank, slices, b, sq,
                                               self.w1[r * kr:(r + 1) * kr], None, m.act,
                                               y=hs[r], stream=s)

            def scatter_all(s):
                hs, ws = self.hbuf.view(tp, M, kr), self.w2p.view(tp, N, kr)
                for r in range(tp):
                    T.tpl_row_linear_scatter(hs[r], ws[r], b, sq, r, tp, self.recv, stream=s)

            def reduce_all(s):
                # each rank's slots summed into its slice of the residual stream,
                # with the RMSNorm of the result written for the next step
                for q in range(tp):
                    x_q = self.xs[q].view(rows, N)
                    T.tpl_reduce_slots_rmsnorm(self.recv[q], tp, N, self.xn[q].view(rows, N),
                                               self.scale, True, 1e-6, None, x_q, y=x_q,
                                               stream=s)
                self.xn_ready = True

            # A step is the block applied again to its own output (a stack of
            # identical layers), so each step's slot reductions also produce the
            # next step's normalised slices; the RMSNorm launches run only after
            # new inputs (first step, or every end-to-end step).
            self.norm_all = norm_all
            self.xn_ready = False
            self.alone_launches = {"rank_rmsnorm": norm_all}
            self.launches += [("rank_gather_gemms", gather_all),
                              ("rank_scatter_gemms", scatter_all),
                              ("rank_slot_reductions", reduce_all)]
            self.flops = self.gemm_flops = m.flops()
            self.gemm_launches = 2 * tp         # one gather and one scatter GEMM per rank
            # per rank: tp slots and the residual read, y and xn written
            self.reduce_bytes = tp * (tp + 3) * rows * N * 2
            self.io_in, self.io_out = ["xs"], ["xs"]   # the residual stream, in place
        else:
            raise ValueError(kind)
        self.parts = [n for n, _ in self.launches]

    def step(self, stream, events=None, skip=()):
        if self.kind == "tp_ranks" and not self.xn_ready:
            self.norm_all(stream)
        for i, (name, fn) in enumerate(self.launches):
            if events is not None:
                events[i].record(stream)
            if name not in skip:
                fn(stream)
        if events is not None:
            events[len(self.launches)].record(stream)

    def inputs_replaced(self):
        self.xn_ready = False

    def gemm_part_ids(self):
        return [i for i, n in enumerate(self.parts)
                if n in ("swiglu_column", "sp_column_gelu", "sp_row_scatter",
                         "rank_gather_gemms", "rank_scatter_gemms")]

    def lmhead_bytes(self):
        return None

    def hbm_parts(self):
        if self.kind == "embed":
            return [("roofline_embed", "embedding_lookup_kernel", "embed_lookup", self.hbm_bytes)]
        if self.kind == "seqpar":
            return [("roofline_rmsnorm", "rmsnorm_cta", "sp_rmsnorm",
                     2 * 2 * self.m.M * self.m.hidden)]
        if self.kind == "tp_ranks":
            return [("roofline_rmsnorm", "rmsnorm_cta", "rank_rmsnorm",
                     2 * 2 * self.m.M * self.m.hidden, self.m.tp),
                    ("roofline_reduce", "reduce_slots_rmsnorm_kernel", "rank_slot_reductions",
                     self.reduce_bytes, self.m.tp)]
        return []


class RankTP:
    """One rank of the RMSNorm + TP MLP block split over GPUs: x[8,1024,4096],
    4096->14336->4096, GELU(erf), tp = the number of processes, one per GPU.

    Each rank holds its token slice of the residual stream ``[batch, seq/tp,
    hidden]`` and its weight shards; a step is TPRankMLP: RMSNorm of the slice ->
    c_fc + GELU over every rank's slice (each token tile read from the rank that
    owns it, through a CUDA IPC mapping) -> c_proj, its partials written into
    the owners' receive buffers -> the slots summed with the residual, in
    place.  Barriers are one-element all-reduces on the launching stream.  The
    whole job computes one block per step (strong scaling).  ``ops``,
    ``exchange`` and ``barrier`` replace the library calls, the CUDA IPC mapping
    and the stream barrier (host tests run the same orchestration on CPU)."""

    kind = "tp_ranks"

    def __init__(self, dev, rank, world, ops=None, exchange=None, barrier=None,
                 workload=None):
        from tensor_transformer_linear_b200 import path
        m = workload or C.TP_MLP
        self.m, self.rank, self.tp = m, rank, world
        b, sq, H, I = m.batch, m.seq, m.hidden, m.inter
        kr = I // world
        self.rows = path.sp_rows(b, sq, world)
        self.name = WORKLOAD_NAMES_RANKS(world)
        full_x = C.mlp_x(m, dev)
        self.x = path.sp_slice(full_x, b, sq, world, rank).reshape(self.rows, H)
        del full_x
        w1 = C.mlp_w1(m, 0, dev)[rank * kr:(rank + 1) * kr].contiguous()
        w2 = C.mlp_w2(m, 0, dev)[:, rank * kr:(rank + 1) * kr].contiguous()
        exchange = exchange or path.exchange_peer_buffers
        xn = exchange(torch.empty_like(self.x))
        recv = exchange(torch.empty(path.recv_buffer_numel(world, b, sq, H), dtype=self.x.dtype,
                                    device=self.x.device))
        barrier = barrier or path.stream_barrier(device=dev)
        self.block = path.TPRankMLP(w1, w2, rank, world, m.act, xn, recv, barrier,
                                    scale=C.mlp_scale(m, 0, dev), centered=True, ops=ops)
        self.parts = ["rank_" + s for s in path.TPRankMLP.STEPS]
        self.flops = m.flops()                 # the whole job's work per step
        self.gemm_flops = m.flops() / world   # this rank's GEMMs
        self.io_in, self.io_out = ["x"], ["x"]   # the residual slice, in place
        self.batch, self.seq = b, sq
        self.xn_ready = False

    def step(self, stream, events=None):
        # a step is the layer applied again to its own output (a stack of
        # identical layers): the slot reduction also writes the next step's
        # normalised slice, so only the first step after new inputs normalises
        mark = None if events is None else (lambda i: events[i].record(stream))
        self.block(self.x, self.batch, self.seq, stream=stream, on_step=mark,
                   normed=self.xn_ready, norm_next=self.block)
        self.xn_ready = True
        if events is not None:
            events[len(self.parts)].record(stream)

    def inputs_replaced(self):
        self.xn_ready = False

    def gemm_part_ids(self):
        return [self.parts.index("rank_column_gather"), self.parts.index("rank_row_scatter")]

    def lmhead_bytes(self):
        return None

    def hbm_parts(self):
        return []


def WORKLOAD_NAMES_RANKS(world):
    """Name of the TP MLP block split over `world` ranks, one per GPU."""
    m = C.TP_MLP
    return (f"tp-ranks rmsnorm-tp-mlp x[{m.batch},{m.seq},{m.hidden}] bf16 "
            f"{m.hidden}->{m.inter}->{m.hidden} gelu-erf, {world} ranks, one per GPU "
            "(peer-gather c_fc, peer-scatter c_proj, slot reduction)")


# ------------------------------------------------------------------ the oracle
#
# The CPU baseline and the reference arm time the fp64 oracle on a bounded
# sample of a workload.  The sample's tensors are generated on the host by the
# seeded generator (bit-identical to the device copies); nothing here imports
# the library or touches CUDA.  Each job returns (run, work, description) with
# work in FLOP (or bytes, for the embedding).

def _f64(t):
    import numpy as np
    return t.to(torch.float32).numpy().astype(np.float64)


def _sample_rows(M, n):
    """n token rows spread evenly over [0, M)."""
    return [int(i * M // n) for i in range(n)]


def oracle_job_block(parts=("qkv", "mlp", "lmhead"), rows_qkv=256, rows_mlp=96,
                     lm_rows=16032):
    import oracle as O
    q, m, l = C.GQA_QKV, C.TP_MLP, C.LM_HEAD
    jobs, flops, desc = [], 0.0, []
    if "qkv" in parts:
        xq = _f64(gen.rows((q.M, q.hidden), _sample_rows(q.M, rows_qkv), 1.0,
                           tensor_id=gen.TID_X))
        wq, bq = _f64(C.qkv_w(q)), _f64(C.qkv_bias(q))
        part = O.partition_subparams(list(q.sub_sizes), q.tp, q.align)
        jobs.append(lambda: O.column_linear(xq, wq, bq, part))
        flops += 2.0 * rows_qkv * q.hidden * q.out
        desc.append(f"{rows_qkv} token rows of the fused QKV")
    if "mlp" in parts:
        xm = _f64(gen.rows((m.M, m.hidden), _sample_rows(m.M, rows_mlp), 1.0,
                           tensor_id=gen.TID_X))
        w1, w2, sc = _f64(C.mlp_w1(m)), _f64(C.mlp_w2(m)), _f64(C.mlp_scale(m))
        jobs.append(lambda: O.tp_mlp(xm, w1, w2, m.tp, m.act, scale=sc, centered=True,
                                     norm=True))
        flops += 4.0 * rows_mlp * m.hidden * m.inter
        desc.append(f"{rows_mlp} token rows of the RMSNorm+MLP")
    if "lmhead" in parts:
        xl = _f64(C.lm_x(l))
        wl = _f64(gen.normal((lm_rows, l.hidden), l.w_sigma, tensor_id=gen.TID_W1))
        jobs.append(lambda: O.lmhead_argmax(xl, wl, 1, 1))
        flops += 2.0 * l.batch * l.hidden * lm_rows
        desc.append(f"{lm_rows} vocab rows x {l.batch} batch rows of the LM head")

    def run():
        for j in jobs:
            j()
    return run, flops, ", ".join(desc)


def oracle_job_stack(rows=8, w=C.STACK4):
    import oracle as O
    xs = _f64(gen.rows((w.M, w.hidden), _sample_rows(w.M, rows), 1.0, tensor_id=gen.TID_X))
    layers = [(C.mlp_w1(w, i).to(torch.float32).numpy(),
               C.mlp_w2(w, i).to(torch.float32).numpy()) for i in range(w.layers)]

    def run():
        # fp32 holds the bf16 weights exactly; each layer is widened to fp64 as it is used
        x = xs
        for w1, w2 in layers:
            x = O.tp_mlp(x, w1.astype("float64"), w2.astype("float64"), w.tp, w.act,
                         norm=True, residual=True)
    return run, w.layers * 4.0 * rows * w.hidden * w.inter, \
        f"{rows} token rows through all {w.layers} layers"


def oracle_job_next(kind, rows=64):
    import oracle as O
    m, l = C.TP_MLP, C.LM_HEAD
    if kind == "swiglu":
        F = m.inter
        xs = _f64(gen.rows((m.M, m.hidden), _sample_rows(m.M, rows), 1.0, tensor_id=gen.TID_X))
        w = _f64(gen.normal((2 * F, m.hidden), m.w_sigma, tensor_id=gen.TID_W1))
        return (lambda: O.swiglu_column_linear(xs, w, F, m.tp),
                2.0 * rows * m.hidden * 2 * F, f"{rows} token rows")
    if kind == "embed":
        sub = 16032
        table = _f64(gen.normal((sub, l.hidden), l.w_sigma, tensor_id=gen.TID_W1))
        g = torch.Generator()
        g.manual_seed(0)
        ids = torch.randint(0, sub, (4096,), generator=g).numpy()
        return (lambda: O.embedding_lookup(ids, table, l.tp),
                ids.size * l.hidden * 2 * 2 + ids.size * 4,
                f"{ids.size} ids over a {sub}-row slice of the table")
    # seqpar / tp_ranks: the RMSNorm + MLP block with the residual, per token
    rows = 128 if kind == "tp_ranks" else rows
    xs = _f64(gen.rows((m.M, m.hidden), _sample_rows(m.M, rows), 1.0, tensor_id=gen.TID_X))
    w1, w2, sc = _f64(C.mlp_w1(m)), _f64(C.mlp_w2(m)), _f64(C.mlp_scale(m))
    return (lambda: O.tp_mlp(xs, w1, w2, m.tp, m.act, scale=sc, centered=True, norm=True,
                             residual=True),
            4.0 * rows * m.hidden * m.inter, f"{rows} tokens through the block")


ORACLE_JOBS = {"block": oracle_job_block, "stack": oracle_job_stack,
               "stack_layer": lambda: oracle_job_stack(w=C.STACK_LAYER),
               "qkv": lambda: oracle_job_block(("qkv",)),
               "mlp": lambda: oracle_job_block(("mlp",)),
               "lmhead": lambda: oracle_job_block(("lmhead",)),
               "swiglu": lambda: oracle_job_next("swiglu"),
               "embed": lambda: oracle_job_next("embed"),
               "seqpar": lambda: oracle_job_next("seqpar"),
               "tp_ranks": lambda: oracle_job_next("tp_ranks")}

# Workload names for the reference arm's line, without building the workload.
WORKLOAD_NAMES = {
    "block": "tp-block: " + " + ".join((C.GQA_QKV.name, C.TP_MLP.name, C.LM_HEAD.name)),
    "stack": C.STACK4.name, "stack_layer": C.STACK_LAYER.name,
    "qkv": C.GQA_QKV.name, "mlp": C.TP_MLP.name,
    "lmhead": C.LM_HEAD.name,
    "swiglu": "fused-swiglu-column x[8,1024,4096] bf16 4096->2x14336 tp8",
    "embed": "vocab-sharded-embedding ids[8,1024] W[128256,4096] bf16 tp8",
    "seqpar": "sequence-parallel rmsnorm-tp-mlp x[8,1024,4096] bf16 4096->14336->4096 tp8",
    "tp_ranks": "tp-ranks rmsnorm-tp-mlp x[8,1024,4096] bf16 4096->14336->4096 gelu-erf, 8 ranks "
                "(peer-gather c_fc, peer-scatter c_proj, slot reduction)",
}


PARALLELISM = {
    "tp_ranks": "8 TP ranks emulated in sequence on one GPU: each rank's c_fc reads every "
                "rank's token slice, its c_proj writes into every rank's receive buffer, then "
                "every rank reduces its slots"}
L2_NOTE = ("not flushed: one step streams ~1.5 GB (block) / ~4 GB (stack), far above the "
           "126 MB L2")


def workload_config(kind, world):
    """The ``config`` of a line: the same for both arms of one workload and N."""
    if kind == "tp_ranks" and world > 1:
        return {"workload": WORKLOAD_NAMES_RANKS(world),
                "parallelism": f"tp{world}: one TP rank per GPU, peer memory over NVLink "
                               "(CUDA IPC), no replicas",
                "l2": L2_NOTE}
    par = PARALLELISM.get(kind, "tp shards of each linear computed on one GPU, cross-shard sum "
                                "in the GEMM epilogue")
    return {"workload": WORKLOAD_NAMES[kind], "parallelism": f"{world} replica(s); " + par,
            "l2": L2_NOTE}


WORKLOADS = {"block": Block, "stack": Stack,
             "stack_layer": lambda dev: Stack(dev, C.STACK_LAYER),
             "qkv": lambda dev: Block(dev, ("qkv",)),
             "mlp": lambda dev: Block(dev, ("mlp",)),
             "lmhead": lambda dev: Block(dev, ("lmhead",)),
             "swiglu": lambda dev: NextRows(dev, "swiglu"),
             "embed": lambda dev: NextRows(dev, "embed"),
             "seqpar": lambda dev: NextRows(dev, "seqpar"),
             "tp_ranks": lambda dev: NextRows(dev, "tp_ranks")}


# ------------------------------------------------------------------ timing

def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else cpu_cores()
    except Exception:
        return cpu_cores()


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (every rank calls this at the same point)."""
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def replica_rate(world, flops_per_step, step_ms):
    """Whole-job TFLOP/s of ``world`` replicas that each ran one step in ``step_ms`` (max)."""
    return world * flops_per_step / (step_ms * 1e-3) / 1e12


def time_oracle(run, flops, target_s=15.0, max_reps=50):
    """Repeat the oracle sample for about target_s seconds; returns TFLOP/s and reps."""
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    reps = max(1, min(max_reps, int(target_s / max(one, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = time.perf_counter() - t0
    return flops * reps / dt / 1e12, reps, dt


def oracle_rate(workload, work, seconds):
    """(value, unit) of the oracle's work over the given time: TFLOP/s, or GB/s
    for the bandwidth-only embedding."""
    if workload == "embed":
        return work / seconds / 1e9, "GB/s"
    return work / seconds / 1e12, "TFLOP/s"


def run_reference(args, rank, world):
    """The fp64 CPU oracle as the reference arm (rank 0 only).

    Its inputs come from the host generator; it neither loads the library nor
    initialises CUDA."""
    if rank != 0:
        return
    run, work, desc = ORACLE_JOBS[args.workload]()
    for _ in range(max(1, args.warmup)):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    v, unit = oracle_rate(args.workload, work * args.steps, dt)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args.workload, world),
            "runs_on": "host cores: the fp64 oracle on a bounded sample of the workload",
            "cpu_baseline": {"value": v, "unit": unit, "cores": blas_threads(),
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def step_region_ms(wl, stream, steps, skip=()):
    """Device time of ``steps`` steps with events only around the region (no
    event between launches, so programmatic dependent launches overlap as in a
    real run)."""
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(steps):
        wl.step(stream, skip=skip) if skip else wl.step(stream)
    stop.record(stream)
    torch.cuda.synchronize()
    return start.elapsed_time(stop)


def timed_steps(wl, stream, steps, pg, dev):
    """Times ``steps`` steps of ``wl`` on ``stream`` with CUDA events, sampling the
    SM clock meanwhile.  The step time comes from a region with events only at
    its ends; the time of each launch from a second pass with an event between
    every two launches.  (An event between two kernels stops the next one from
    starting its prologue during the previous one's tail, so the parts of the
    second pass can add up to slightly more than a step.)  A run under a
    hardware or thermal slowdown (or a stale clock lock) is taken again once;
    every rank makes the same decision.  Returns (region ms, mean ms per part,
    library launches in the region, clock record)."""
    import tensor_transformer_linear_b200 as T
    n_ev = len(wl.parts) + 1

    def region():
        clocks = ClockSampler(torch.cuda.current_device())
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.3)   # nvidia-smi is sampling before the timed steps start
        n0 = T.tpl_launch_count()
        t0 = datetime.datetime.now()
        ms = step_region_ms(wl, stream, steps)
        t1 = datetime.datetime.now()
        launches = T.tpl_launch_count() - n0
        clk = clocks.stop(t0, t1)
        if pg is not None:
            pg.barrier()
        if T.tpl_get_device_status(stream) != 0:
            raise RuntimeError("a kernel reported a pipeline timeout in the timed region")
        # per-launch times: a second pass with an event between every two
        # launches, after an idle pause so that it starts from the power state
        # the timed region started from (the power limit lowers the clock
        # within tens of milliseconds of load)
        time.sleep(PARTS_PAUSE_S)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
               for _ in range(steps)]
        for k in range(steps):
            wl.step(stream, evs[k])
        torch.cuda.synchronize()
        if pg is not None:
            pg.barrier()
        part_ms = [statistics.mean(evs[k][i].elapsed_time(evs[k][i + 1])
                                   for k in range(steps)) for i in range(n_ev - 1)]
        return ms, part_ms, launches, clk

    ms, part_ms, launches, clk = region()
    bad = torch.tensor([1.0 if clocks_rejected(clk) else 0.0], device=dev)
    if pg is not None:
        pg.all_reduce(bad, op=pg.ReduceOp.MAX)
    remeasured = bool(bad.item() > 0)
    if remeasured:
        ms, part_ms, launches, clk = region()
    if clk is not None:
        clk["remeasured"] = remeasured
    return ms, part_ms, launches, clk


def marginal_part_ms(wl, stream, steps, part, rounds=5):
    """A part's cost inside the step as it really runs (no events around it):
    the median, over ``rounds`` interleaved pairs, of (step time) - (step time
    without that launch), per step."""
    with_p, without = [], []
    for _ in range(rounds):
        with_p.append(step_region_ms(wl, stream, steps) / steps)
        without.append(step_region_ms(wl, stream, steps, skip=(part,)) / steps)
    return statistics.median(w - o for w, o in zip(with_p, without))

TENSOR_FLOP_PER_CYCLE_SM = 8192   # dense bf16 tcgen05, per SM


def kernel_clocks(wl, stream, steps=3, decode=10):
    """The SM clock each launch really ran at, from the library's per-CTA
    timing records (tpl_trace_set: %clock64 and %globaltimer of every CTA), on
    an untimed pass of ``steps`` steps (the first is dropped: it starts from
    idle) and a decode loop of ``decode`` LM-head launches.  nvidia-smi and NVML
    sample a clock that a launch of a few hundred microseconds does not show.
    Per part: median over launches of the median CTA clock, the span (first
    CTA start to last CTA end) and the median CTA duration."""
    import tensor_transformer_linear_b200 as T
    launches = getattr(wl, "launches", None)
    dev = torch.cuda.current_device()
    seq_of = []
    with T.Trace(16384, dev) as tr:
        with torch.cuda.stream(stream):
            for k in range(steps):
                if launches:
                    for name, fn in launches:
                        n0 = T.tpl_launch_count()
                        fn(stream)
                        seq_of.append((n0, T.tpl_launch_count(), name, k))
                else:
                    # one library launch per part, in order (the stack)
                    n0 = T.tpl_launch_count()
                    wl.step(stream)
                    for q in range(n0, min(T.tpl_launch_count(), n0 + len(wl.parts))):
                        seq_of.append((q, q + 1, wl.parts[q - n0], k))
            lm = dict(launches or []).get("lmhead_argmax")
            if lm is not None:
                for k in range(decode):
                    n0 = T.tpl_launch_count()
                    lm(stream)
                    seq_of.append((n0, T.tpl_launch_count(), "lmhead_decode_loop", k))
        torch.cuda.synchronize()
    by_seq = {l["seq"]: l for l in tr.launches()}
    per, total = {}, {}
    for n0, n1, name, k in seq_of:
        if k == 0:
            continue            # the first step starts from idle
        # a part may be several launches (one per rank); element-wise kernels leave no record
        ls = [by_seq[q] for q in range(n0, n1) if q in by_seq]
        if ls:
            per.setdefault(name, []).extend(ls)
            total.setdefault(name, []).append(sum(l["span_us"] for l in ls))
    out = {}
    for name, ls in per.items():
        out[name] = {"sm_mhz": round(statistics.median(l["sm_mhz"] for l in ls), 1),
                     "span_us": round(statistics.median(l["span_us"] for l in ls), 1),
                     "cta_us": round(statistics.median(l["cta_us"] for l in ls), 1),
                     "launches": len(ls),
                     "span_us_per_call": round(statistics.median(total[name]), 1)}
    return out


def tensor_pipe_at_clock(wl, kclk, dev):
    """The GEMM launches' rate over their traced spans against the tensor
    pipe's peak at the (span-weighted) SM clock they ran at."""
    gids = wl.gemm_part_ids()
    g = [wl.parts[i] for i in gids if wl.parts[i] in kclk]
    if not g or len(g) != len(gids):
        return None
    span_us = sum(kclk[n]["span_us_per_call"] for n in g)
    mhz = sum(kclk[n]["span_us_per_call"] * kclk[n]["sm_mhz"] for n in g) / span_us
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    pipe = sms * TENSOR_FLOP_PER_CYCLE_SM * mhz * 1e6 / 1e12
    a_span = wl.gemm_flops / (span_us * 1e-6) / 1e12
    return {"sm_mhz": round(mhz, 1), "peak": round(pipe, 1),
            "achieved_in_span": round(a_span, 1), "frac": round(a_span / pipe, 4),
            "note": f"{sms} SMs x {TENSOR_FLOP_PER_CYCLE_SM} bf16 FLOP/cycle at the "
                    "span-weighted SM clock the GEMM launches ran at; achieved from "
                    "their traced spans"}


def measure_stack(args, dev, stream, pg, world, pk, pk_kind):
    """The 4-layer residual stack x[4,4096,8192] at full size, timed in the same
    process: long enough (about a second) to run in the power-capped regime."""
    wl = Stack(dev)
    steps = max(20, min(args.steps, 40))
    for _ in range(3):
        wl.step(stream)
    torch.cuda.synchronize()
    ms, part_ms, launches, clk = timed_steps(wl, stream, steps, pg, dev)
    kclk = kernel_clocks(wl, stream, steps=3)   # untimed, right after the timed steps
    if pg is not None:
        ms = max_over_ranks([ms], dev)[0]
        part_ms = max_over_ranks(part_ms, dev)
    step_ms = ms / steps
    gids = wl.gemm_part_ids()
    gemm_ms = sum(part_ms[i] for i in gids)
    achieved = wl.gemm_flops / (gemm_ms * 1e-3) / 1e12
    peak_t, peak_label = tensor_peak(pk, pk_kind, clk)
    norm_ms = sum(part_ms[i] for i in range(len(part_ms)) if i not in gids)
    norm_bytes = wl.w.layers * 2 * 2 * wl.w.M * wl.w.hidden
    rec = {
        "workload": wl.name, "steps": steps, "warmup": 3, "ms_per_step": round(step_ms, 4),
        "value": round(replica_rate(world, wl.flops, step_ms), 2), "unit": "TFLOP/s",
        "flops_per_step": wl.flops,
        "kernel": "gemm_bf16_tcgen05_pair", "bound": "tensor",
        "gemm_launches_per_step": len(gids), "gemm_flops_per_launch": wl.flops / len(gids),
        "gemm_ms_per_step": round(gemm_ms, 4), "achieved": round(achieved, 2),
        "peak": peak_t, "peak_kind": peak_label, "frac": round(achieved / peak_t, 4),
        "frac_of_burst": round(achieved / pk["bf16_tflops"], 4),
        "frac_of_sustained": round(achieved / pk["bf16_tflops_sustained"], 4),
        "rmsnorm": ({"kernel": "rmsnorm_cta", "bytes_per_step": norm_bytes,
                     "ms_per_step": round(norm_ms, 4),
                     "achieved_gbs": round(norm_bytes / (norm_ms * 1e-3) / 1e9, 1)}
                    if norm_ms > 0 else "fused into each layer's c_fc GEMM "
                                        "(tpl_column_linear_rmsnorm)"),
        "parts_ms": {n: round(v, 4) for n, v in zip(wl.parts, part_ms)},
        "gpu_launches": int(launches), "clocks": clk,
        "l2": "not flushed: one step streams ~4 GB of weights and activations, far above "
              "the 126 MB L2",
        "measured": "CUDA events around every launch on the launching stream, mean over "
                    "the timed steps; the GEMM rate is the step's GEMM FLOPs over the sum "
                    "of its GEMM launch times"}
    if kclk:
        rec["kernel_clocks"] = {
            "parts": kclk,
            "measured": "per-CTA %clock64 / %globaltimer records (tpl_trace_set) of an untimed "
                        "pass of 3 steps right after the timed ones, the first dropped"}
        tp_clk = tensor_pipe_at_clock(wl, kclk, dev)
        if tp_clk:
            rec["tensor_pipe_at_kernel_clock"] = tp_clk
    del wl
    torch.cuda.empty_cache()
    return rec


def host_link_ms(dev, bytes_in, bytes_out, reps=5):
    """Time to move one step's upload and download bytes over the host link at
    once (pinned buffers, one stream per direction, no compute): the floor of
    the end-to-end step."""
    try:
        h_in = torch.empty(int(bytes_in), dtype=torch.uint8, pin_memory=True)
        h_out = torch.empty(int(bytes_out), dtype=torch.uint8, pin_memory=True)
        d_in = torch.empty(int(bytes_in), dtype=torch.uint8, device=dev)
        d_out = torch.empty(int(bytes_out), dtype=torch.uint8, device=dev)
    except RuntimeError:
        return None
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ts = []
    for _ in range(reps + 1):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(up)
        down.wait_event(a)
        with torch.cuda.stream(up):
            d_in.copy_(h_in, non_blocking=True)
        with torch.cuda.stream(down):
            h_out.copy_(d_out, non_blocking=True)
        up.wait_stream(down)
        b.record(up)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    del h_in, h_out, d_in, d_out
    return statistics.median(ts[1:])


def measure_tiny(dev, stream, reps=200):
    """The tiny fp32 TP MLP (x[2,16,256], 256->1024->256, tp 4, GELU tanh): the
    latency of one block.  Median over ``reps`` blocks, each bracketed by CUDA
    events, two ways: replays of the block captured once in a CUDA graph (device
    latency, no host work in between) and eager calls through the Python
    binding (each launch also waits for its host-side argument marshalling).
    The block runs as one fused launch (tpl_tp_mlp_fp32); the two-launch form
    (c_fc, then c_proj with the partial-sum reduction) is timed beside it."""
    import tensor_transformer_linear_b200 as T
    w = C.TINY_MLP
    x = C.mlp_x(w, dev)
    y = torch.empty((w.M, w.hidden), dtype=w.dtype, device=dev)

    def timed(run):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        with torch.cuda.stream(stream):
            for e0, e1 in evs:
                e0.record(stream)
                run()
                e1.record(stream)
        torch.cuda.synchronize()
        return sorted(e0.elapsed_time(e1) * 1e3 for e0, e1 in evs)

    out = {}
    for key, fused in (("fused", True), ("two_launch", False)):
        blk = T.TPMLP(C.mlp_w1(w, 0, dev), C.mlp_w2(w, 0, dev), w.tp, w.act, norm=False,
                      fused_fp32=fused)
        with torch.cuda.stream(stream):
            for _ in range(10):
                blk(x, out=y)
        torch.cuda.synchronize()
        n0 = T.tpl_launch_count()
        with torch.cuda.stream(stream):
            blk(x, out=y)
        launches = T.tpl_launch_count() - n0
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            blk(x, out=y)
        torch.cuda.synchronize()
        tg = timed(graph.replay)
        te = timed(lambda: blk(x, out=y))
        del graph
        out[key] = (tg, te, launches, blk.fused_fp32)
    tg, te, launches, fused = out["fused"]
    us = statistics.median(tg)
    return {"workload": w.name, "dtype": "f32", "us_per_block": round(us, 2),
            "p10_us": round(tg[len(tg) // 10], 2), "p90_us": round(tg[9 * len(tg) // 10], 2),
            "eager_us_per_block": round(statistics.median(te), 2),
            "launches_per_block": launches,
            "kernel": "mlp_fp32_fused" if fused else "gemm_fp32_simt",
            "flops_per_block": w.flops(),
            "gflops": round(w.flops() / (us * 1e-6) / 1e9, 1), "bound": "latency",
            "two_launch": {"us_per_block": round(statistics.median(out["two_launch"][0]), 2),
                           "eager_us_per_block": round(statistics.median(out["two_launch"][1]), 2),
                           "launches_per_block": out["two_launch"][2],
                           "kernel": "gemm_fp32_simt"},
            "measured": f"median of {reps} blocks, CUDA events around each block on the "
                        "launching stream; us_per_block replays the block captured in a CUDA "
                        "graph, eager_us_per_block calls it through the Python binding"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="block", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="block workload: skip the 4-layer stack and tiny-MLP records")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl_cls = WORKLOADS[args.workload]

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    import tensor_transformer_linear_b200 as T
    ranks = args.workload == "tp_ranks" and world > 1
    wl = RankTP(dev, rank, world) if ranks else wl_cls(dev)
    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            wl.step(stream)
    torch.cuda.synchronize()
    if T.tpl_get_device_status(stream) != 0:
        raise RuntimeError("a kernel reported a pipeline timeout during warm-up")

    # ---- device-timed region: K steps, per-launch events on the launching stream
    ms, part_ms, launches, clk = timed_steps(wl, stream, args.steps, pg, dev)

    # ---- the LM head's cost inside the step as it runs (no events around it)
    lm_marginal_ms = None
    if "lmhead_argmax" in getattr(wl, "parts", []) and len(wl.parts) > 1:
        lm_marginal_ms = marginal_part_ms(wl, stream, args.steps, "lmhead_argmax")
        if pg is not None:
            lm_marginal_ms = max_over_ranks([lm_marginal_ms], dev)[0]

    # ---- the LM head in a decode loop: back-to-back launches, as once per decode step
    decode_ms = None
    lm = dict(getattr(wl, "launches", [])).get("lmhead_argmax")
    if lm is not None:
        for _ in range(3):
            lm(stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        for _ in range(DECODE_LAUNCHES):
            lm(stream)
        d1.record(stream)
        torch.cuda.synchronize()
        decode_ms = d0.elapsed_time(d1) / DECODE_LAUNCHES
        if pg is not None:
            decode_ms = max_over_ranks([decode_ms], dev)[0]

    # ---- the SM clock inside each launch (per-CTA timing records, untimed pass)
    kclk = None if ranks else kernel_clocks(wl, stream)

    # ---- the HBM-bound parts alone: each launch after a read-only L2 flush (a
    # 256 MiB sum, which evicts earlier kernels' dirty lines and leaves L2
    # clean), timed with events around that launch alone; median of ALONE_LAUNCHES
    alone_ms = {}
    launch_of = dict(getattr(wl, "launches", []))
    launch_of.update(getattr(wl, "alone_launches", {}))
    parts_alone = [h for h in wl.hbm_parts() if h[2] in launch_of]
    if parts_alone:
        flush = torch.ones(256 * 2**20 // 4, dtype=torch.float32, device=dev)
        with torch.cuda.stream(stream):
            for key, _, part, *_ in parts_alone:
                fn = launch_of[part]
                evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                       for _ in range(ALONE_LAUNCHES)]
                for _ in range(3):
                    fn(stream)
                for e0, e1 in evs:
                    flush.sum()
                    e0.record(stream)
                    fn(stream)
                    e1.record(stream)
                torch.cuda.synchronize()
                t = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
                alone_ms[key] = max_over_ranks([t], dev)[0] if pg is not None else t
        del flush

    # ---- end to end through pinned host buffers, copies inside the timed region
    e2e = E2EPipeline(wl, stream)
    b_in, b_out = e2e.bytes_in, e2e.bytes_out
    for _ in range(E2E_SETS + 1):
        e2e.step()
    torch.cuda.synchronize()
    # The timed region starts and ends with the pipeline empty: the first
    # upload and the last download are not overlapped, so take enough steps
    # (about 0.1 s) that this fill and drain is a small part of it.
    e_steps = max(40, args.steps)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize()
    e0.record(e2e.up)
    for _ in range(e_steps):
        e2e.step()
    e1.record(e2e.down)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    e2e.close()
    link_ms = host_link_ms(dev, b_in, b_out)

    if pg is not None:
        ms, e_ms = max_over_ranks([ms, e_ms], dev)

    # ---- the other single-GPU configurations, in the same process: the 4-layer
    # stack (the largest, seconds-long, power-capped) and the tiny fp32 MLP (latency)
    extra = {}
    if args.workload == "block" and not args.no_extra:
        pk, pk_kind = peaks()
        extra["roofline_stack"] = measure_stack(args, dev, stream, pg, world, pk, pk_kind)
        extra["tiny_mlp_us"] = measure_tiny(dev, stream)
        if pg is not None:
            extra["tiny_mlp_us"]["us_per_block"] = max_over_ranks(
                [extra["tiny_mlp_us"]["us_per_block"]], dev)[0]

    if rank == 0:
        pk, pk_kind = peaks()
        step_ms = ms / args.steps
        # replicas: every rank did a whole step; TP ranks: the job did one step
        copies = 1 if ranks else world
        value = replica_rate(copies, wl.flops, step_ms)
        e2e_val = replica_rate(copies, wl.flops, e_ms / e_steps)
        # dominant kernel: the tcgen05 GEMM (all launches of it in the step)
        gids = wl.gemm_part_ids()
        n_gemm = getattr(wl, "gemm_launches", len(gids)) if gids else 0
        gemm_ms = sum(part_ms[i] for i in gids)
        gemm_launch_flops = wl.gemm_flops / max(1, n_gemm)
        gemm_achieved = wl.gemm_flops / (gemm_ms * 1e-3) / 1e12 if n_gemm else 0.0
        peak_t, peak_label = tensor_peak(pk, pk_kind, clk)
        traffic = ncu_traffic("gemm_bf16_tcgen05_pair", args.workload,
                              ["gemm_bf16.cuh", "gemm_bf16_pair.cuh", "ptx.cuh", "common.cuh",
                               "trace.cuh"])
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "strong" if ranks else "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded SplitMix64 / Irwin-Hall normal, the pages' shapes)",
            "config": workload_config(args.workload, world),
            "roofline": {"kernel": "gemm_bf16_tcgen05_pair", "bound": "tensor",
                         "achieved": round(gemm_achieved, 2), "peak": peak_t,
                         "unit": "TFLOP/s", "frac": round(gemm_achieved / peak_t, 4),
                         "peak_kind": peak_label,
                         "frac_of_burst": round(gemm_achieved / pk["bf16_tflops"], 4),
                         "frac_of_sustained": round(gemm_achieved / pk["bf16_tflops_sustained"], 4),
                         "launches_per_step": n_gemm,
                         "flops_per_launch_avg": gemm_launch_flops,
                         "traffic": traffic},
            "parts_ms": {n: round(v, 4) for n, v in zip(wl.parts, part_ms)},
            "gpu_launches": int(launches),
            "clocks": clk,
            "e2e": {"value": round(e2e_val, 2), "unit": "TFLOP/s",
                    "h2d_bytes_per_step": int(b_in), "d2h_bytes_per_step": int(b_out),
                    "steps": e_steps,
                    "method": f"pinned host buffers; upload, compute and download on three "
                              f"streams over {E2E_SETS} device buffer sets, so step k+1's "
                              "upload and step k-1's download overlap step k's compute; "
                              "timed from an empty pipeline to an empty one (the first upload "
                              "and the last download overlap nothing)"},
        }
        if link_ms:
            bound = replica_rate(copies, wl.flops, max(link_ms, step_ms))
            line["e2e"]["host_link_bound"] = {
                "value": round(bound, 2), "frac": round(e2e_val / bound, 4),
                "copy_ms_per_step": round(link_ms, 4),
                "measured": "one step's upload and download bytes copied at the same time "
                            "between pinned host buffers and the device, no compute, median "
                            "of 5; the bound is the step's FLOPs over the longer of that "
                            "and the device step time"}
        if kclk:
            line["kernel_clocks"] = {
                "parts": kclk,
                "measured": "per-CTA %clock64 / %globaltimer records (tpl_trace_set) of an "
                            "untimed pass of 3 steps, the first dropped, and a 10-launch LM-head "
                            "decode loop; sm_mhz = median CTA cycles / duration"}
            tp_clk = tensor_pipe_at_clock(wl, kclk, dev)
            if tp_clk:
                line["roofline"]["tensor_pipe_at_kernel_clock"] = tp_clk
        lb = wl.lmhead_bytes()
        if lb is not None:
            lm_kernel = lmhead_kernel(C.LM_HEAD.batch)
            lm_ms = part_ms[wl.parts.index("lmhead_argmax")]
            gbs = lb / (lm_ms * 1e-3) / 1e9
            line["roofline_lmhead"] = {
                "kernel": lm_kernel, "bound": "hbm", "achieved": round(gbs, 1),
                "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(gbs / pk["hbm_gbs"], 4),
                "frac_of_8000": round(gbs / 8000.0, 4), "bytes_per_launch": lb,
                "ms": round(lm_ms, 4),
                "measured": "inside the block steps, right after the GEMMs, from CUDA events "
                            "around the launch",
                "traffic": ncu_traffic(lm_kernel, "lmhead",
                                       ["lmhead.cuh", "lmhead_tn.cuh", "ptx.cuh", "common.cuh",
                                        "trace.cuh"])}
            if lm_marginal_ms is not None and lm_marginal_ms > 0:
                gm = lb / (lm_marginal_ms * 1e-3) / 1e9
                line["roofline_lmhead"]["in_step_marginal"] = {
                    "achieved": round(gm, 1), "frac": round(gm / pk["hbm_gbs"], 4),
                    "frac_of_8000": round(gm / 8000.0, 4), "ms": round(lm_marginal_ms, 4),
                    "measured": "step time minus the step time without the LM head launch, "
                                "each from events around 20-step regions with no event "
                                "between launches (the launch overlaps the GEMM's tail as it "
                                "does in a real step), median of 5 interleaved pairs"}
            if decode_ms is not None:
                dg = lb / (decode_ms * 1e-3) / 1e9
                line["roofline_lmhead_decode"] = {
                    "kernel": lm_kernel, "bound": "hbm", "achieved": round(dg, 1),
                    "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": round(dg / pk["hbm_gbs"], 4),
                    "frac_of_8000": round(dg / 8000.0, 4), "ms_per_launch": round(decode_ms, 4),
                    "measured": f"{DECODE_LAUNCHES} back-to-back launches (a decode loop), "
                                "CUDA events on the launching stream"}
        for key, kern, part, nbytes, *n_l in wl.hbm_parts():
            n_l = n_l[0] if n_l else 1
            if part in wl.parts:
                p_ms = part_ms[wl.parts.index(part)]
                gb = nbytes / (p_ms * 1e-3) / 1e9
                line[key] = {"kernel": kern, "bound": "hbm", "achieved": round(gb, 1),
                             "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": round(gb / pk["hbm_gbs"], 4),
                             "bytes_per_launch": nbytes // n_l, "launches_per_step": n_l,
                             "measured": "inside the timed steps, after the kernel before it, "
                                         "whose dirty output lines in L2 it evicts"}
            else:
                # not a launch of the step (the norm is fused into the GEMM there):
                # the kernel timed on its own
                line[key] = {"kernel": kern, "bound": "hbm", "unit": "GB/s",
                             "peak": pk["hbm_gbs"], "bytes_per_launch": nbytes // n_l,
                             "in_step": False}
            if key in alone_ms:
                ga = nbytes / (alone_ms[key] * 1e-3) / 1e9
                line[key]["alone"] = {
                    "achieved": round(ga, 1), "frac": round(ga / pk["hbm_gbs"], 4),
                    "ms": round(alone_ms[key], 4),
                    "measured": f"median of {ALONE_LAUNCHES} launches, each after a read-only "
                                "256 MiB L2 flush, CUDA events around the launch alone"}
                if not line[key].get("in_step", True):
                    line[key].update(achieved=line[key]["alone"]["achieved"],
                                     frac=line[key]["alone"]["frac"])
        if not gids:
            first = "roofline_lmhead" if "roofline_lmhead" in line else wl.hbm_parts()[0][0]
            line["roofline"] = line.pop(first)
        if wl.flops == 0:
            # a bandwidth-only workload: the rate is bytes moved per second
            line["value"] = round(wl.hbm_bytes / (step_ms * 1e-3) / 1e9 * world, 1)
            line["unit"] = "GB/s"
            line["e2e"]["value"] = round(wl.hbm_bytes / (e_ms / e_steps * 1e-3) / 1e9 * world, 1)
            line["e2e"]["unit"] = "GB/s"
        if world == 1 and not args.no_cpu_baseline:
            run, work, desc = ORACLE_JOBS[args.workload]()
            _, reps, dt = time_oracle(run, work)
            v, unit = oracle_rate(args.workload, work * reps, dt)
            line["cpu_baseline"] = {"value": round(v, 6), "unit": unit,
                                    "cores": blas_threads(), "kind": "oracle",
                                    "sample": f"{desc}; {reps} reps in {dt:.1f} s"}
        line.update(extra)
        print(json.dumps(line), flush=True)

    if pg is not None:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
