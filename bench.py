#!/usr/bin/env python
"""Benchmark of the FP8 blockwise linear-layer hot path on B200.

One step = the four linear GEMMs of a Qwen2-1.5B-shaped decoder layer (QKV
2048x1536, O 1536x1536, gate+up 17920x1536, down 1536x8960), each run
forward, data-gradient and weight-gradient at 16384 tokens per GPU, with
every quantisation the pass needs inside the step (24 kernels):

    per linear layer (X [T,K], W [N,K], dY [T,N]):
      quantize_act_1x128(X, BOTH)          row-wise for FWD, along tokens for WGRAD
      quantize_weight_128x128_both(W)      FWD operand and (transposed) DGRAD operand
      gemm FWD    Y  = X . W^T
      quantize_act_1x128(dY, BOTH)
      gemm DGRAD  dX = dY . W
      gemm WGRAD  dW = dY^T . X

value = GEMM FLOPs of all ranks / device time of the step (quantisation included),
in TFLOP/s.  With --gpus N > 1 every rank runs its own 16384-token batch
(weak scaling) and the weight gradients are summed over ranks with NCCL
all-reduce inside the step (the data-parallel exchange).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload layer|qkv_fwd|mlp_fwd|down_bwd] [--tokens T] [--sweep]

`--impl reference` times the CPU oracle (the slow, plain implementation the
parity tests check against) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "blockwise-FP8 GEMM TFLOP/s incl. quantize (fraction of dense FP8 peak); quant GB/s"
SPEC_FP8_TFLOPS = 4500.0          # B200 dense FP8, NVIDIA's published figure
FP8_PER_BF16 = 2.0                # nominal dense FP8 / BF16 tensor throughput ratio
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20
# DRAM traffic of the 12 GEMM launches of one decoder-layer step at 16384 tokens
# (dram__bytes_read.sum + dram__bytes_write.sum, one ncu pass over the launches of
# one step; profiles/gemm_dram_layer_16384.md); algorithmic minimum 2.59 GB (codes
# read once, bf16 outputs written once).  It describes the GEMM source whose
# SHA-256 prefix is given; for any other source the bench reports no traffic.
GEMM_STEP_DRAM = {"bytes": 2.881e9, "gemm_cu_sha256": "56f0202c9d77f700"}
GEMM_SOURCE = os.path.join(ROOT, "fp8_blockwise_scaled_b200", "csrc", "gemm.cu")

WORKLOAD_DESC = {
    "layer": "qwen2-1.5b-shaped decoder layer linears (qkv 2048x1536, o 1536x1536, gate_up 17920x1536, "
             "down 1536x8960), fwd+dgrad+wgrad, all quantisation included",
    "qkv_fwd": "qkv projection fwd, X[Tx1536] with 0.1% outlier channels x20, W[2048x1536]",
    "mlp_fwd": "mlp fwd: gate_up X[Tx1536].W[17920x1536]^T then down X[Tx8960].W[1536x8960]^T",
    "down_bwd": "mlp down backward: dgrad dX=dY.W, wgrad dW=dY^T.X, dY[Tx1536], X[Tx8960]",
}


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def gemm_source_sha() -> str:
    import hashlib
    with open(GEMM_SOURCE, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def fp8_peaks(peaks: dict) -> dict:
    """Dense FP8 denominators: the measured bf16 GEMM rate times the nominal FP8/BF16 ratio,
    burst (for kernels timed on their own) and sustained, and NVIDIA's dense FP8 figure."""
    return {"burst": peaks["bf16_tflops"] * FP8_PER_BF16,
            "sustained": peaks["bf16_tflops_sustained"] * FP8_PER_BF16,
            "spec": SPEC_FP8_TFLOPS}


# --------------------------------------------------------------------------- workload programs
def workload_tensors(name: str, tokens: int) -> list[dict]:
    """[{name, X, W, dY, passes}] with bf16 host arrays; passes in {"fwd", "dgrad", "wgrad"}."""
    if name == "layer":
        L = workloads.layer(seed=4, tokens=tokens)
        return [{"name": g, **L[g], "passes": ("fwd", "dgrad", "wgrad")} for g, _, _ in workloads.LAYER_GEMMS]
    if name == "qkv_fwd":
        d = workloads.qkv_fwd(seed=1, tokens=tokens)
        return [{"name": "qkv", "X": d["X"], "W": d["W"], "dY": None, "passes": ("fwd",)}]
    if name == "mlp_fwd":
        d = workloads.mlp_fwd(seed=2, tokens=tokens)
        return [{"name": "gate_up", "X": d["X_gate_up"], "W": d["W_gate_up"], "dY": None, "passes": ("fwd",)},
                {"name": "down", "X": d["X_down"], "W": d["W_down"], "dY": None, "passes": ("fwd",)}]
    if name == "down_bwd":
        d = workloads.down_bwd(seed=3, tokens=tokens)
        return [{"name": "down", "X": d["X"], "W": d["W"], "dY": d["dY"], "passes": ("dgrad", "wgrad")}]
    raise ValueError(name)


class Program:
    """Device buffers and the ordered kernel launches of one step."""

    def __init__(self, specs, device, world, grad_e5m2=False, recipe="blockwise"):
        import torch
        import fp8_blockwise_scaled_b200 as fb
        self.fb, self.torch, self.world = fb, torch, world
        self.ops = []          # (label, kind, units, fn); kind "quant" (units = bytes) or "gemm" (units = flops)
        self.inputs = []       # (device tensor, host array) copied in by the end-to-end run
        self.outputs = []      # device tensors read back by the end-to-end run
        self.grads = []        # weight gradients all-reduced across ranks
        self.named = {}        # "<linear>.<buffer>" -> device tensor (the parity tests read them)
        self.splits = {}       # GEMM label -> split-K count the library chose (1 = none)
        self.gemm_flops = 0
        E4 = torch.float8_e4m3fn
        if recipe == "delayed":
            self._build_delayed(specs, device)
            specs = []
        # A layer whose every linear runs forward and data-gradient quantises all its weights (both
        # block layouts) in one launch at the start of the step.
        group_w = len(specs) > 1 and all("fwd" in sp["passes"] and "dgrad" in sp["passes"] for sp in specs)
        grouped = []           # (w, q, s, qT, sT) of each linear when group_w
        for sp in specs:
            x = self._dev(sp["X"], device)
            w = self._dev(sp["W"], device)
            T, K = x.shape
            N = w.shape[0]
            passes = sp["passes"]
            need_row_x = "fwd" in passes
            need_colt_x = "wgrad" in passes
            g = sp["name"]
            f = lambda *s, dt=E4: torch.empty(s, dtype=dt, device=device)  # noqa: E731
            qx = f(T, K) if need_row_x else None
            sx = f(K // 128, T, dt=torch.float32) if need_row_x else None
            qxT = f(K, T) if need_colt_x else None
            sxT = f(T // 128, K, dt=torch.float32) if need_colt_x else None
            mode = (fb.ROWWISE if need_row_x else 0) | (fb.COLWISE_T if need_colt_x else 0)
            self.named.update({f"{g}.X": x, f"{g}.W": w, f"{g}.qx": qx, f"{g}.sx": sx, f"{g}.qxT": qxT,
                               f"{g}.sxT": sxT})
            qbytes = T * K * (2 + (1 + 4 / 128) * (int(need_row_x) + int(need_colt_x)))
            self._op(f"{g}.quant_x", "quant", qbytes,
                     lambda x=x, m=mode, a=qx, b=sx, c=qxT, d=sxT: fb.fp8blk_quantize_act_1x128(x, m, a, b, c, d))
            if "fwd" in passes:
                qw, sw = f(N, K), f(N // 128, K // 128, dt=torch.float32)
            if "dgrad" in passes:
                qwT, swT = f(K, N), f(K // 128, N // 128, dt=torch.float32)
            if group_w:
                grouped.append((w, qw, sw, qwT, swT))
            elif "fwd" in passes and "dgrad" in passes:     # both block layouts from one read of W
                self._op(f"{g}.quant_w", "quant", N * K * (2 + 2 * (1 + 4 / 16384)),
                         lambda w=w, q=qw, s=sw, qT=qwT, sT=swT: fb.fp8blk_quantize_weight_128x128_both(w, q, s, qT, sT))
            elif "fwd" in passes:
                self._op(f"{g}.quant_w", "quant", N * K * (3 + 4 / 16384),
                         lambda w=w, q=qw, s=sw: fb.fp8blk_quantize_weight_128x128(w, q, s))
            elif "dgrad" in passes:
                self._op(f"{g}.quant_wt", "quant", N * K * (3 + 4 / 16384),
                         lambda w=w, q=qwT, s=swT: fb.fp8blk_quantize_weight_128x128_t(w, q, s))
            self.named.update({f"{g}.qw": qw if "fwd" in passes else None, f"{g}.sw": sw if "fwd" in passes else None,
                               f"{g}.qwT": qwT if "dgrad" in passes else None,
                               f"{g}.swT": swT if "dgrad" in passes else None})
            if "fwd" in passes:
                y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
                self.named[f"{g}.Y"] = y
                self._gemm_op(f"{g}.gemm_fwd", fb.FWD, qx, sx, qw, sw, y)
                self.outputs.append(y)
            if "dgrad" in passes or "wgrad" in passes:
                dy = self._dev(sp["dY"], device)
                need_row_d = "dgrad" in passes
                need_colt_d = "wgrad" in passes
                gdt = torch.float8_e5m2 if grad_e5m2 else E4      # E5M2 gradients: the DGRAD/WGRAD A operand
                qd = f(T, N, dt=gdt) if need_row_d else None
                sd = f(N // 128, T, dt=torch.float32) if need_row_d else None
                qdT = f(N, T, dt=gdt) if need_colt_d else None
                sdT = f(T // 128, N, dt=torch.float32) if need_colt_d else None
                self.named.update({f"{g}.dY": dy, f"{g}.qd": qd, f"{g}.sd": sd, f"{g}.qdT": qdT, f"{g}.sdT": sdT})
                mode_d = ((fb.ROWWISE if need_row_d else 0) | (fb.COLWISE_T if need_colt_d else 0)
                          | (fb.E5M2 if grad_e5m2 else 0))
                self._op(f"{g}.quant_dy", "quant", T * N * (2 + (1 + 4 / 128) * (int(need_row_d) + int(need_colt_d))),
                         lambda x=dy, m=mode_d, a=qd, b=sd, c=qdT, d=sdT:
                         fb.fp8blk_quantize_act_1x128(x, m, a, b, c, d))
                if need_row_d:
                    dx = torch.empty(T, K, dtype=torch.bfloat16, device=device)
                    self.named[f"{g}.dX"] = dx
                    self._gemm_op(f"{g}.gemm_dgrad", fb.DGRAD, qd, sd, qwT, swT, dx)
                    self.outputs.append(dx)
                if need_colt_d:
                    dw = torch.empty(N, K, dtype=torch.bfloat16, device=device)
                    self.named[f"{g}.dW"] = dw
                    # Data parallel: this rank's partial dW in fp32, summed across ranks, rounded once.
                    part = torch.empty(N, K, dtype=torch.float32, device=device) if world > 1 else dw
                    self._gemm_op(f"{g}.gemm_wgrad", fb.WGRAD, qdT, sdT, qxT, sxT, part)
                    self.outputs.append(dw)
                    if world > 1:
                        self.grads.append((part, dw))
        if grouped:
            ws = [e[0] for e in grouped]
            outs = [e[1:] for e in grouped]
            self.ops.insert(0, ("weights.quant_w", "quant",
                                sum(w.shape[0] * w.shape[1] * (2 + 2 * (1 + 4 / 16384)) for w in ws),
                                lambda ws=ws, outs=outs: fb.fp8blk_quantize_weights_128x128_both(ws, outs)))
        self.gemm_flops = sum(u for _, k, u, _ in self.ops if k == "gemm")
        self.quant_bytes = sum(u for _, k, u, _ in self.ops if k == "quant")

    def _build_delayed(self, specs, device):
        """The pages' per-tensor delayed-scaling FP8Linear forward for every linear: amax EMA of X and
        of W (buffers persist across steps), both tensors quantised with their one scale, one GEMM."""
        torch, fb = self.torch, self.fb
        for sp in specs:
            x, w = self._dev(sp["X"], device), self._dev(sp["W"], device)
            T, K = x.shape
            N = w.shape[0]
            g = sp["name"]
            amax = {k: torch.ones(1, dtype=torch.float32, device=device) for k in "xw"}
            scale = {k: torch.empty(1, dtype=torch.float32, device=device) for k in "xw"}
            ws = {k: torch.empty(max(16, fb.fp8blk_amax_ema_workspace_bytes(r)), dtype=torch.uint8, device=device)
                  for k, r in (("x", T), ("w", N))}
            qx = torch.empty(T, K, dtype=torch.float8_e4m3fn, device=device)
            qw = torch.empty(N, K, dtype=torch.float8_e4m3fn, device=device)
            y = torch.empty(T, N, dtype=torch.bfloat16, device=device)
            self._op(f"{g}.amax_x", "quant", T * K * 2,
                     lambda x=x, a=amax["x"], s=scale["x"], w=ws["x"]: fb.fp8blk_amax_ema(x, a, s, w))
            self._op(f"{g}.amax_w", "quant", N * K * 2,
                     lambda x=w, a=amax["w"], s=scale["w"], w=ws["w"]: fb.fp8blk_amax_ema(x, a, s, w))
            self._op(f"{g}.quant_x", "quant", T * K * 3, lambda x=x, s=scale["x"], q=qx: fb.fp8blk_quantize_tensor(x, s, q))
            self._op(f"{g}.quant_w", "quant", N * K * 3, lambda x=w, s=scale["w"], q=qw: fb.fp8blk_quantize_tensor(x, s, q))
            self._op(f"{g}.gemm_fwd", "gemm", 2 * T * N * K,
                     lambda a=qx, sa=scale["x"], b=qw, sb=scale["w"], d=y: fb.fp8blk_gemm_tensor_scaled(a, sa, b, sb, d))
            self.outputs.append(y)

    def _dev(self, host, device):
        t = self.torch.from_numpy(np.ascontiguousarray(host)).view(self.torch.bfloat16).to(device)
        self.inputs.append((t, host))
        return t

    def _op(self, label, kind, units, fn):
        self.ops.append((label, kind, units, fn))

    def _gemm_op(self, label, layout, a, sa, b, sb, d):
        """One blockwise GEMM op, split-K where the library's count for the shape says so (its
        fp32 partial-tile workspace allocated here, once)."""
        fb, torch = self.fb, self.torch
        m, n, k = d.shape[0], d.shape[1], a.shape[1]
        splits = fb.fp8blk_gemm_splitk_count(layout, m, n, k)
        ws = (torch.empty(fb.fp8blk_gemm_splitk_workspace_bytes(layout, m, n, k, splits) // 4, dtype=torch.float32,
                          device=d.device) if splits > 1 else None)
        self.splits[label] = splits
        self._op(label, "gemm", 2 * m * n * k,
                 lambda: fb.fp8blk_gemm(layout, a, sa, b, sb, d, splits=splits, workspace=ws))

    def run(self, events=None, reduce=True):
        """One step.  events: list of (start, end) CUDA event pairs, one per op, or None.
        reduce: sum the weight gradients over ranks (data parallel) at the end."""
        for i, (_, _, _, fn) in enumerate(self.ops):
            if events is not None:
                events[i][0].record()
            fn()
            if events is not None:
                events[i][1].record()
        if reduce:
            self.reduce()

    def run_overlapped(self, quant_stream):
        """One step with the quantisers on `quant_stream` and the GEMMs on the
        current stream; each GEMM waits only for the quantisers whose outputs
        it reads (FWD: X and W; DGRAD: dY and W; WGRAD: dY and X)."""
        torch = self.torch
        main = torch.cuda.current_stream()
        quant_stream.wait_stream(main)
        done = {}
        for label, kind, _, fn in self.ops:
            if kind == "quant":
                with torch.cuda.stream(quant_stream):
                    fn()
                    done[label] = torch.cuda.Event()
                    done[label].record(quant_stream)
        for label, kind, _, fn in self.ops:
            if kind == "gemm":
                g, which = label.split(".")
                needs = {"gemm_fwd": ("quant_x", "quant_w"), "gemm_dgrad": ("quant_dy", "quant_w"),
                         "gemm_wgrad": ("quant_dy", "quant_x")}[which]
                for q in needs:
                    ev = done.get(f"{g}.{q}")
                    if ev is None and q == "quant_w":          # all of a layer's weights in one launch,
                        ev = done.get("weights.quant_w") or done.get(f"{g}.quant_wt")   # or W^T alone

                    if ev is not None:
                        main.wait_event(ev)
                fn()
        main.wait_stream(quant_stream)

    def reduce(self):
        if self.world > 1:
            from fp8_blockwise_scaled_b200.dp import allreduce_weight_grads
            allreduce_weight_grads(self.grads)


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        # Raw nvidia-smi samples; BENCH_CLOCKS_DIR keeps them somewhere chosen.
        out_dir = os.environ.get("BENCH_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_bench_gpu{gpu_index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        loaded = [r for r in rows if _num(r[4]) is not None and _num(r[4]) >= 50] or rows
        sm = [_num(r[1]) for r in loaded if _num(r[1]) is not None]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": _num(rows[0][2]) if rows else None,
                "reasons": reasons, "samples": len(loaded),
                "power_w_max": max((_num(r[3]) or 0.0) for r in loaded) if loaded else None}


def _num(s):
    try:
        return float(s)
    except (TypeError, ValueError):
        return None


# --------------------------------------------------------------------------- CPU oracle
def oracle_pass(specs, tokens: int, col_frac: float = 1.0) -> tuple[float, float, str]:
    """Runs the oracle over the first `tokens` tokens (and a fraction of each weight's rows)
    of every GEMM of the workload.  Returns (flops, seconds, description)."""
    import oracle
    flops = 0
    t0 = time.perf_counter()
    for sp in specs:
        n_all = sp["W"].shape[0]
        n = max(128, int(n_all * col_frac) // 128 * 128)
        x = sp["X"][:tokens]
        w = sp["W"][:n]
        k = x.shape[1]
        passes = sp["passes"]
        if "fwd" in passes:
            qx, sx = oracle.quantize_act_rowwise(x)
            qw, sw = oracle.quantize_weight(w)
            oracle.gemm(oracle.FWD, qx, sx, qw, sw)
            flops += 2 * tokens * n * k
        if "dgrad" in passes or "wgrad" in passes:
            dy = np.ascontiguousarray(sp["dY"][:tokens, :n])
            if "dgrad" in passes:
                qd, sd = oracle.quantize_act_rowwise(dy)
                qwt, swt = oracle.quantize_weight_t(w)
                oracle.gemm(oracle.DGRAD, qd, sd, qwt, swt)
                flops += 2 * tokens * n * k
            if "wgrad" in passes:
                qdt, sdt = oracle.quantize_act_colwise_t(dy)
                qxt, sxt = oracle.quantize_act_colwise_t(x)
                oracle.gemm(oracle.WGRAD, qdt, sdt, qxt, sxt)
                flops += 2 * tokens * n * k
    dt = time.perf_counter() - t0
    desc = (f"first {tokens} tokens of every GEMM of the workload"
            + (f", first {col_frac:.0%} of each weight's output rows" if col_frac < 1 else "")
            + ", quantisation + fp64 GEMM, all passes")
    return flops, dt, desc


def cpu_baseline(specs) -> dict:
    import oracle
    flops, dt, desc = oracle_pass(specs, tokens=256)
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": desc, "seconds": round(dt, 3)}


# --------------------------------------------------------------------------- extra measurements
def host_enqueue_seconds(prog) -> float:
    """Host time to enqueue one step (every launch of the program), measured once."""
    import torch
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    prog.run(reduce=False)
    t = time.perf_counter() - t0
    torch.cuda.synchronize()
    return t


def hold_device(host_seconds: float) -> None:
    """Keeps the stream busy (a spin kernel) for about twice the host's enqueue time of a step,
    so that the per-op events recorded next measure the kernels back to back on the device,
    without the host's launch gaps.  The spin counts clock cycles; 2e9 per second is above the
    B200's maximum SM clock, so the spin lasts at least that long."""
    import torch
    torch.cuda._sleep(int(2.0 * host_seconds * 2.0e9) + 100000)


def time_program(prog, flush, steps: int, warmup: int) -> dict:
    """Median per-op event times of eager launches, and the median device time of the
    whole step replayed as one CUDA graph (L2 flushed before every step)."""
    import torch
    for _ in range(warmup):
        flush.zero_()
        prog.run(reduce=False)
    torch.cuda.synchronize()
    ahead = host_enqueue_seconds(prog)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in prog.ops]
          for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        hold_device(ahead)
        prog.run(ev[i], reduce=False)
    torch.cuda.synchronize()
    op_ms = [statistics.median(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(steps))
             for j in range(len(prog.ops))]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        prog.run(reduce=False)
    graph.replay()
    torch.cuda.synchronize()
    st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        st[i][0].record()
        graph.replay()
        st[i][1].record()
    torch.cuda.synchronize()
    step_ms = statistics.median(a.elapsed_time(b) for a, b in st)
    del graph
    gemm_ms = sum(ms for ms, (_, kind, _, _) in zip(op_ms, prog.ops) if kind == "gemm")
    quant_ms = sum(ms for ms, (_, kind, _, _) in zip(op_ms, prog.ops) if kind == "quant")
    return {"op_ms": op_ms, "step_ms": step_ms, "gemm_ms": gemm_ms, "quant_ms": quant_ms}


def time_configs_8192(dev, flush, fp8: dict, steps: int) -> dict:
    """The 8192-token configs (QKV forward, MLP forward, MLP down backward), each one step of its
    quantisers and GEMMs: the GEMM kernel alone and the sequential step including quantisation."""
    import torch
    out = {}
    for name in ("qkv_fwd", "mlp_fwd", "down_bwd"):
        prog = Program(workload_tensors(name, 8192), dev, 1)
        t = time_program(prog, flush, steps, 3)
        gemm = prog.gemm_flops / (t["gemm_ms"] * 1e-3) / 1e12
        incl = prog.gemm_flops / (t["step_ms"] * 1e-3) / 1e12
        out[name] = {"gemm_tflops": round(gemm, 1), "gemm_frac": round(gemm / fp8["burst"], 3),
                     "gemm_frac_of_spec": round(gemm / fp8["spec"], 3),
                     "incl_quant_tflops": round(incl, 1), "incl_quant_frac": round(incl / fp8["burst"], 3),
                     "incl_quant_frac_of_spec": round(incl / fp8["spec"], 3),
                     "quant_gbs": round(prog.quant_bytes / (t["quant_ms"] * 1e-3) / 1e9, 1),
                     "step_ms": round(t["step_ms"], 4)}
        del prog
        torch.cuda.empty_cache()
    return out


def time_sweep(dev, flush, fp8: dict, steps: int) -> dict:
    """Token sweep of the decoder layer (all 12 GEMMs and their quantisers) at every count in
    workloads.TOKEN_SWEEP: the step including quantisation (one graph) and the GEMMs alone."""
    import torch
    rows = []
    for m in workloads.TOKEN_SWEEP:
        prog = Program(workload_tensors("layer", m), dev, 1)
        t = time_program(prog, flush, steps, 3)
        incl = prog.gemm_flops / (t["step_ms"] * 1e-3) / 1e12
        gemm = prog.gemm_flops / (t["gemm_ms"] * 1e-3) / 1e12
        rows.append({"tokens": m, "incl_quant_tflops": round(incl, 1), "gemm_tflops": round(gemm, 1),
                     "incl_quant_frac_of_spec": round(incl / fp8["spec"], 3)})
        del prog
        torch.cuda.empty_cache()
    best = max(r["incl_quant_tflops"] for r in rows)
    knee = next(r["tokens"] for r in rows if r["incl_quant_tflops"] >= 0.95 * best)
    return {"points": rows, "knee_tokens": knee,
            "knee_rule": "smallest token count within 5% of the best step rate including quantisation"}


def time_fp8_proxy(dev) -> dict:
    """Context only: the library's per-tensor-scaled FP8 GEMM (torch._scaled_mm, cuBLASLt) at
    8192^3, best of 10 launches.  No 1x128 / 128x128 blockwise library kernel exists on sm_100
    to compare against; this is the plain FP8 tensor-core rate on this GPU."""
    import torch
    try:
        a = torch.randn(8192, 8192, device=dev).to(torch.float8_e4m3fn)
        b = torch.randn(8192, 8192, device=dev).to(torch.float8_e4m3fn)
        one = torch.ones((), device=dev)
        for _ in range(3):
            torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return {"kernel": "torch._scaled_mm per-tensor FP8 8192^3", "tflops": round(2 * 8192**3 / (best * 1e-3) / 1e12, 1)}
    except Exception as e:     # context only: never fails the bench
        return {"kernel": "torch._scaled_mm per-tensor FP8 8192^3", "unavailable": str(e)[:200]}


# --------------------------------------------------------------------------- arms
def run_reference(args, rank: int, world: int):
    """The oracle, as it stands, on the host cores: each step a bounded sample of the workload."""
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    tokens = args.tokens or (16384 if args.workload == "layer" else 8192)
    specs = workload_tensors(args.workload, 256)
    budget = 150.0 / max(1, args.steps + args.warmup)       # seconds per step
    _, t_full, _ = oracle_pass(specs, tokens=128)
    frac = min(1.0, budget / t_full) if t_full > 0 else 1.0
    for _ in range(max(0, args.warmup - 1)):
        oracle_pass(specs, 128, frac)
    times, flops, desc = [], 0, ""
    for _ in range(args.steps):
        flops, dt, desc = oracle_pass(specs, 128, frac)
        times.append(dt)
    total = sum(times)
    value = flops * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD_DESC[args.workload], "tokens": tokens,
                                        "sample_tokens": 128},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    tokens = args.tokens or (16384 if args.workload == "layer" else 8192)
    specs = workload_tensors(args.workload, tokens)
    prog = Program(specs, dev, world, grad_e5m2=args.grad_format == "e5m2", recipe=args.recipe)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        flush.zero_()
        prog.run()
    barrier()

    nops = len(prog.ops)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nops)]
          for _ in range(args.steps)]
    st = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # Per-op device times: eager launches, one event pair around each op, the whole step
    # enqueued behind a spin kernel so that the kernels run back to back on the device.
    ahead = host_enqueue_seconds(prog)
    for i in range(args.steps):
        flush.zero_()
        hold_device(ahead)
        prog.run(ev[i], reduce=False)
    barrier()
    per_op_ms = [[a.elapsed_time(b) for a, b in ev[i]] for i in range(args.steps)]
    # The timed steps: the step's kernels as one CUDA graph (with FP8BLK_PDL=1, consecutive
    # kernels linked by programmatic dependent launch), replayed once per step.
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            prog.run(reduce=False)
        graph.replay()                         # one untimed replay
    barrier()
    sampler = ClockSampler(local_rank)
    time.sleep(0.3)
    barrier()
    for i in range(args.steps):
        flush.zero_()                          # L2 flush, outside the timed events
        st[i][0].record(stream)
        if graph is not None:
            graph.replay()
        else:
            prog.run(reduce=False)
        prog.reduce()
        st[i][1].record(stream)
    barrier()
    clocks = sampler.stop()
    step_ms = [a.elapsed_time(b) for a, b in st]
    total_ms = sum(step_ms)
    # The same steps with the quantisers on a second stream (one graph holding both streams).
    overlapped_ms = None
    partitioned = []
    if graph is not None:
        qs = torch.cuda.Stream()
        graph2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph2):
            prog.run_overlapped(qs)
        graph2.replay()
        barrier()
        so = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            so[i][0].record(stream)
            graph2.replay()
            prog.reduce()
            so[i][1].record(stream)
        barrier()
        overlapped_ms = sum(a.elapsed_time(b) for a, b in so)
        del graph2
        # The same two-stream step with the SMs partitioned: the GEMMs capped at SMs - k CTAs,
        # the quantisers at 2k CTAs, so that quantisers run beside a GEMM instead of in its tail.
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        for k in (() if world > 1 or args.no_extra else (8, 16, 24)):
            os.environ["FP8BLK_GEMM_MAX_CTAS"] = str(sms - k)
            os.environ["FP8BLK_QUANT_MAX_CTAS"] = str(2 * k)
            graph3 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph3):
                prog.run_overlapped(qs)
            del os.environ["FP8BLK_GEMM_MAX_CTAS"], os.environ["FP8BLK_QUANT_MAX_CTAS"]
            graph3.replay()
            barrier()
            sp = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
            for i in range(args.steps):
                flush.zero_()
                sp[i][0].record(stream)
                graph3.replay()
                sp[i][1].record(stream)
            barrier()
            part_ms = sum(a.elapsed_time(b) for a, b in sp)
            partitioned.append({"quant_sms": k, "gemm_ctas": sms - k,
                                "value": prog.gemm_flops * world * args.steps / (part_ms * 1e-3) / 1e12,
                                "ms_per_step": part_ms / args.steps})
            del graph3
        if world > 1:
            t = torch.tensor([overlapped_ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            overlapped_ms = t.item()
    gemm_ms = sum(per_op_ms[i][j] for i in range(args.steps) for j in range(nops) if prog.ops[j][1] == "gemm")
    quant_ms = sum(per_op_ms[i][j] for i in range(args.steps) for j in range(nops) if prog.ops[j][1] == "quant")
    if world > 1:
        t = torch.tensor([total_ms, gemm_ms, quant_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms, gemm_ms, quant_ms = t.tolist()

    # End to end through the public API: pinned host inputs in, outputs back, every step.
    # Two sets of device buffers alternate between steps, and the copies use both copy
    # engines: step i+1's inputs come in on one stream while step i computes and step i-1's
    # outputs go out on another.  A step's kernels wait for its inputs and for the outputs of
    # the step two back (the same buffers) to be out; the inputs of a buffer set are rewritten
    # only after the step two back has read them.  Every step copies all of its inputs in and
    # all of its outputs back.
    progs = [prog, Program(specs, dev, world, grad_e5m2=args.grad_format == "e5m2", recipe=args.recipe)]
    h_in = [[(d, torch.from_numpy(np.ascontiguousarray(h)).view(torch.bfloat16).pin_memory()) for d, h in p.inputs]
            for p in progs]
    h_out = [[(d, torch.empty(d.shape, dtype=d.dtype, pin_memory=True)) for d in p.outputs] for p in progs]
    h2d = sum(h.numel() * h.element_size() for _, h in h_in[0])
    d2h = sum(h.numel() * h.element_size() for _, h in h_out[0])
    e2e_steps = max(3, args.steps)                   # the same steps as the device-timed value
    progs[1].run()                                   # set-up of the second buffer set, outside the timing
    copy_in, copy_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in.wait_stream(stream)
    computed, sent = [None, None], [None, None]
    for i in range(e2e_steps):
        b = i % 2
        with torch.cuda.stream(copy_in):
            if computed[b] is not None:
                copy_in.wait_event(computed[b])      # the step two back has read these inputs
            for d, h in h_in[b]:
                d.copy_(h, non_blocking=True)
            arrived = torch.cuda.Event()
            arrived.record(copy_in)
        stream.wait_event(arrived)
        if sent[b] is not None:
            stream.wait_event(sent[b])               # the outputs this step overwrites are out
        progs[b].run()
        computed[b] = torch.cuda.Event()
        computed[b].record(stream)
        with torch.cuda.stream(copy_out):
            copy_out.wait_event(computed[b])
            for d, h in h_out[b]:
                h.copy_(d, non_blocking=True)
            sent[b] = torch.cuda.Event()
            sent[b].record(copy_out)
    for ev in sent:
        if ev is not None:
            stream.wait_event(ev)
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
    err = prog.fb.fp8blk_get_device_error()

    peaks, peak_src = load_peaks()
    fp8 = fp8_peaks(peaks)
    fp8_peak = fp8["burst"]
    flops_all = prog.gemm_flops * world
    value = flops_all * args.steps / (total_ms * 1e-3) / 1e12
    gemm_tflops = prog.gemm_flops * args.steps / (gemm_ms * 1e-3) / 1e12
    quant_gbs = prog.quant_bytes * args.steps / (quant_ms * 1e-3) / 1e9
    per_op = {}
    for j, (label, kind, units, _) in enumerate(prog.ops):
        ms = statistics.median(per_op_ms[i][j] for i in range(args.steps))
        rate = units / (ms * 1e-3) / (1e12 if kind == "gemm" else 1e9)
        per_op[label] = {"us": round(ms * 1e3, 1), ("tflops" if kind == "gemm" else "gbs"): round(rate, 1),
                         "frac": round(rate / (fp8_peak if kind == "gemm" else peaks["hbm_gbs"]), 3)}
        if prog.splits.get(label, 1) > 1:
            per_op[label]["split_k"] = prog.splits[label]
    traffic_ok = args.workload == "layer" and tokens == 16384 and gemm_source_sha() == GEMM_STEP_DRAM["gemm_cu_sha256"]
    extra = {}
    if rank == 0 and world == 1 and args.workload == "layer" and not args.no_extra:
        extra["configs_8192"] = time_configs_8192(dev, flush, fp8, max(3, min(args.steps, 10)))
        extra["token_sweep"] = time_sweep(dev, flush, fp8, 5)
        extra["fp8_library_proxy"] = time_fp8_proxy(dev)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "e4m3" if args.grad_format == "e4m3" else "e4m3+e5m2",
        "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC[args.workload], "tokens_per_gpu": tokens,
                   "l2": "flushed between steps (256 MiB write outside the timed events)",
                   "streams": 1, "seed": {"layer": 4, "qkv_fwd": 1, "mlp_fwd": 2, "down_bwd": 3}[args.workload],
                   "grad_format": args.grad_format,
                   "recipe": args.recipe if args.recipe == "blockwise" else
                             "delayed: per-tensor scales from an amax EMA, forward GEMMs only",
                   "launch": ("eager" if graph is None else "one CUDA graph per step")
                             + (", programmatic dependent launch" if os.environ.get("FP8BLK_PDL") == "1" else ""),
                   "parallelism": f"dp{world}" if world > 1 else "single-gpu"},
        "frac_of_spec_fp8_peak": value / SPEC_FP8_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": "gemm_blockwise_kernel", "achieved": gemm_tflops,
                     "peak": fp8_peak, "unit": "TFLOP/s", "frac": gemm_tflops / fp8_peak,
                     "traffic": GEMM_STEP_DRAM["bytes"] if traffic_ok else None,
                     "traffic_scope": "bytes per step, the GEMM launches together (12 GEMMs, the split-K sums included; "
                                      "achieved is over the same launches)",
                     "traffic_note": "ncu capture of this GEMM source" if traffic_ok else
                                     "no capture of this GEMM source (or another workload): not reported",
                     "peak_source": f"{peak_src} bf16 burst x {FP8_PER_BF16:g} (nominal fp8/bf16 ratio); each GEMM "
                                    "is timed on its own by CUDA events, so the burst figure applies",
                     "frac_of_sustained_derived_peak": gemm_tflops / fp8["sustained"],
                     "frac_of_spec_fp8": gemm_tflops / SPEC_FP8_TFLOPS},
        "quant": {"kernel": "quant_tile_kernel", "achieved_gbs": quant_gbs, "peak_gbs": peaks["hbm_gbs"],
                  "frac": quant_gbs / peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm copy"},
        "overlapped": None if overlapped_ms is None else {
            "value": flops_all * args.steps / (overlapped_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "ms_per_step": overlapped_ms / args.steps, "streams": 2,
            "note": "quantisers on a second stream; each GEMM waits for the quantisers it reads",
            "partitioned": partitioned},
        "per_op_median": per_op,
        "per_op_timing": "CUDA events around each eager launch, the step enqueued behind a spin kernel "
                         "(kernels back to back on the device, no host launch gaps); L2 flushed once per step",
        "e2e": {"value": flops_all * e2e_steps / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "copies": "pinned host buffers, two device buffer sets alternating between steps; the next "
                          "step's inputs come in on one stream while a step computes and the previous step's "
                          "outputs go out on another"},
        # one kernel per op, two for an amax EMA (partial maxima, then the EMA) and for a
        # split-K GEMM (the units, then the sum of their partials), and with data parallelism
        # one rounding kernel per weight gradient after its all-reduce
        "gpu_launches": (sum(2 if ".amax_" in label or prog.splits.get(label, 1) > 1 else 1
                             for label, _, _, _ in prog.ops) + len(prog.grads)) * args.steps,
        "clocks": clocks,
        "device_error": prog.fb.status_string(err),
        **extra,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(workload_tensors(args.workload, 256) if tokens != 256 else specs)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if err == 0 else 1


def run_sweep(args, local_rank: int):
    """Token sweep: each linear layer fwd (quantise X, W + GEMM) at M in the sweep list."""
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    results = []
    for m in workloads.TOKEN_SWEEP:
        specs = [dict(s, passes=("fwd", "dgrad", "wgrad")) for s in workload_tensors("layer", m)]
        prog = Program(specs, dev, 1)
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        for _ in range(3):
            prog.run()
        torch.cuda.synchronize()
        n = max(5, min(args.steps, 20))
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in prog.ops] for _ in range(n)]
        for i in range(n):
            flush.zero_()
            prog.run(ev[i])
        torch.cuda.synchronize()
        row = {"tokens": m}
        for j, (label, kind, units, _) in enumerate(prog.ops):
            if kind == "gemm":
                ms = statistics.median(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(n))
                row[label] = round(units / (ms * 1e-3) / 1e12, 1)
        tot = sum(statistics.median(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(n))
                  for j in range(len(prog.ops)))
        row["layer_tflops_incl_quant"] = round(prog.gemm_flops / (tot * 1e-3) / 1e12, 1)
        results.append(row)
        del prog
        torch.cuda.empty_cache()
    print(json.dumps({"sweep": results, "unit": "TFLOP/s (median per-kernel events, L2 flushed)"}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOAD_DESC), default="layer")
    ap.add_argument("--tokens", type=int, default=0, help="tokens per GPU (default 16384 for layer, else 8192)")
    ap.add_argument("--sweep", action="store_true", help="token sweep of the layer GEMMs (one JSON line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the 8192-token configs, the token sweep and the library FP8 proxy")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches instead of the step's CUDA graph")
    ap.add_argument("--recipe", choices=["blockwise", "delayed"], default="blockwise",
                    help="blockwise 1x128 / 128x128 scaling (fwd+dgrad+wgrad), or the per-tensor delayed-scaling "
                         "forward")
    ap.add_argument("--grad-format", choices=["e4m3", "e5m2"], default="e4m3",
                    help="code format of the output gradient dY (the DGRAD/WGRAD A operand)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch N>1 with torch.distributed.run")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.sweep:
            return run_sweep(args, local_rank) if rank == 0 else 0
        return run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
