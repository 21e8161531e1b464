"""Benchmark of the NVFP4 quantize + linear hot path on B200.

One step = one pass of the hot path over one batch: for each of the four
Qwen2.5-VL-7B-shaped projections (qkv 3584->4608, o 3584->3584, gate_up
3584->37888, down 18944->3584) the fused activation prologue
(vlaq_quantize_act_nvfp4) followed by the block-scaled FP4 GEMM
(vlaq_linear_nvfp4), M = 1024 tokens, weights quantized offline beforehand
(vlaq_quantize_weight_nvfp4, outside the timed region).  The step is
captured once in a CUDA graph and replayed.

Reported (one JSON line on rank 0):
  value      GEMM TFLOP/s of the whole job (sum 2MNK / step time, all ranks)
  e2e        same metric through the public API with host buffers: pinned
             host -> device copy of X, prologue + GEMM, device -> host copy
             of Y, every step
  roofline   the dominant kernel (the NVFP4 GEMM) timed with CUDA events on
             its stream: algorithmic FLOPs / launch duration vs the measured
             dense FP4 peak (bf16 burst peak x 4, the nominal FP4:BF16 ratio)
  prologue   the activation prologue: algorithmic bytes / duration vs HBM
  decode     M = 1, 4, 8 (weight-bandwidth-bound): GB/s of algorithmic
             bytes, weights rotated over copies so the working set exceeds L2
  fused      the fused-prologue step (RMSNorm + block-64 rotation on the
             qkv / gate_up inputs, rotation + residual add on o / down,
             rotated weights), NVFP4 and FP8 W8A8
  fp8, int8  the FP8 and INT8 W8A8 variants of the plain step (TFLOP/s;
             INT8 multiply-accumulates counted as FLOPs)
  stack      the 28-layer stack (196 projections, one graph), all NVFP4 and
             mixed (o / down FP8), at M = 1024 and M = 1: us per token
  cpu_baseline  the CPU oracle on a bounded sample of the same workload,
             with one entry per workload above
Kernel durations: CUDA events recorded as nodes inside the captured step
("in_step": includes the node-to-node launch gap, which is a large share of
a few-microsecond kernel), and for the prologue and the decode GEMMs also a
graph of the same kernel launched back to back over buffers larger than L2
("back_to_back": per-launch time in a stream of such launches).
Inputs: seeded synthetic bf16 (synthetic_inputs.py); the per-step working set
(X 61 MB + W 131 MB + Y 102 MB) exceeds the 126 MB L2.

Multi-GPU: one process per GPU (torchrun), each rank runs the same per-GPU
batch (token batches are independent: weak scaling, no collective on the
data path); the step time is the max over ranks.

`--impl reference` runs the CPU oracle as the reference arm on the same
workload (bounded token sample per step), rank 0 only.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synthetic_inputs as si  # noqa: E402

METRIC = "W4A4 NVFP4 linear TFLOP/s @M=1024, GB/s @M=1; % of B200 roofline"
PROJ = ["qkv", "o", "gate_up", "down"]
M_PREFILL = 1024
FP4_PER_BF16 = 9.0 / 2.25   # nominal dense FP4 : BF16 tensor throughput
FP8_PER_BF16 = 4.5 / 2.25


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def traffic_source_sha(sources):
    """sha256 (16 hex digits) of the source the traffic counters depend on:
    a list of {"file": path, optional "from" / "to" markers bounding a
    region of the file}."""
    import hashlib
    h = hashlib.sha256()
    for src in sources:
        txt = open(os.path.join(ROOT, src["file"]), encoding="utf-8").read()
        if "from" in src:
            a = txt.index(src["from"])
            txt = txt[a:txt.index(src["to"], a)]
        h.update(txt.encode())
    return h.hexdigest()[:16]


def load_traffic(kernel_key):
    """dram bytes per launch from the committed ncu summary, valid only while
    the kernel's source is unchanged (hash recorded beside the counters)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        ent = json.load(open(p)).get(kernel_key)
        if not ent or traffic_source_sha(ent["sources"]) != ent["source_sha"]:
            return None
        return ent["bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled during the timed region."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index),
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        smax = float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for nm, v in zip(names, r[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        loaded = [s for s in sm if smax and s > 0.3 * smax] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------ setup
RANK_SEED_STRIDE = 1000  # activation seed offset per rank


def make_inputs(M, device, seed_offset=0):
    data = {}
    for name in PROJ:
        K, N, seed = si.PROJECTIONS[name]
        X = si.projection_activations(K, M, seed + seed_offset)
        W = si.projection_weight(K, N, seed)
        data[name] = (K, N, X, W)
    return data


FUSED = {c.name: c for c in si.FUSED_CASES}


class Step:
    """Device buffers and launch sequence of one hot-path step.  fused: the
    fused-prologue workload (RMSNorm + block-64 rotation on the qkv /
    gate_up inputs, rotation only plus a residual add on o / down, weights
    rotated too)."""

    def __init__(self, vq, data, M, device, fmt="nvfp4", weight_copies=1, fused=False):
        assert fmt in ("nvfp4", "fp8", "int8"), fmt
        self.vq = vq
        self.M = M
        self.fmt = fmt
        self.fp8 = fmt != "nvfp4"  # an 8-bit W8A8 format (FP8 or INT8)
        self.fused = fused
        self.layers = []
        for name in PROJ:
            K, N, X, W = data[name]
            # the library reads M rows of X through a raw pointer
            if X.shape[0] < M or X.shape[1] != K:
                raise ValueError(f"{name}: X is {tuple(X.shape)}, the step needs at least {M} x {K}")
            case = FUSED[name]
            flags = (3 if case.rmsnorm else 2) if fused else 0
            wflags = flags & 2
            Wd = W.to(device)
            copies = []
            for c in range(weight_copies):
                if c > 0:  # further copies: the same bytes in other buffers
                    copies.append(tuple(None if t is None else t.clone() for t in copies[0]))
                elif fmt == "fp8":
                    wq, sw = vq.alloc_fp8(N, K, device)
                    vq.vlaq_quantize_weight_fp8(Wd, N, K, wflags, wq, sw)
                    copies.append((wq, None, sw))
                elif fmt == "int8":
                    wq, sw = vq.alloc_int8(N, K, device)
                    vq.vlaq_quantize_weight_int8(Wd, N, K, wflags, wq, sw)
                    copies.append((wq, None, sw))
                else:
                    wq, ws, wg = vq.alloc_nvfp4(N, K, device, per_tensor=True)
                    vq.vlaq_quantize_weight_nvfp4(Wd, N, K, wflags, wq, ws, wg)
                    copies.append((wq, ws, wg))
            del Wd
            Xd = X.to(device)
            if self.fp8:
                xq, sx = (vq.alloc_fp8 if fmt == "fp8" else vq.alloc_int8)(M, K, device)
                act = (xq, None, sx)
            else:
                act = vq.alloc_nvfp4(M, K, device)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
            wsp, nb = vq.alloc_workspace(M, N, K, device)
            gam = si.norm_gain(K, FUSED[name].seed).to(device) if flags & 1 else None
            R = si.residual(M, N, FUSED[name].seed).to(device) if fused and case.residual else None
            self.layers.append(dict(name=name, K=K, N=N, X=Xd, act=act, W=copies, Y=Y, ws=wsp, nb=nb,
                                    flags=flags, gamma=gam, R=R))
        torch.cuda.synchronize()
        self.flops = sum(2.0 * M * L["N"] * L["K"] for L in self.layers)

    def run(self, copy=0, events=None):
        for i, L in enumerate(self.layers):
            if events is not None:
                events[i][0].record()
            self.prologue(L)
            if events is not None:
                events[i][1].record()
            self.gemm(L, copy)
            if events is not None:
                events[i][2].record()

    def prologue(self, L, X=None):
        vq, M, K = self.vq, self.M, L["K"]
        X = L["X"] if X is None else X
        xq, xs, xg = L["act"]
        if self.fmt == "fp8":
            vq.vlaq_quantize_act_fp8(X, M, K, L["gamma"], 1e-6, L["flags"], xq, xg)
        elif self.fmt == "int8":
            vq.vlaq_quantize_act_int8(X, M, K, L["gamma"], 1e-6, L["flags"], xq, xg)
        else:
            vq.vlaq_quantize_act_nvfp4(X, M, K, L["gamma"], 1e-6, L["flags"], xq, xs, xg)

    def gemm(self, L, copy=0):
        vq, M, K, N = self.vq, self.M, L["K"], L["N"]
        xq, xs, xg = L["act"]
        wq, ws, wg = L["W"][copy % len(L["W"])]
        if self.fmt == "fp8":
            vq.vlaq_linear_fp8(xq, xg, wq, wg, L["R"], L["Y"], M, N, K, L["ws"], L["nb"])
        elif self.fmt == "int8":
            vq.vlaq_linear_int8(xq, xg, wq, wg, L["R"], L["Y"], M, N, K, L["ws"], L["nb"])
        else:
            vq.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, L["R"], L["Y"], M, N, K, L["ws"], L["nb"])

    def gemm_bytes(self, L):
        """Algorithmic HBM bytes of one GEMM launch (residual read included)."""
        M, N, K = self.M, L["N"], L["K"]
        res = 2 * M * N if L["R"] is not None else 0
        if self.fp8:
            return N * K + 4 * N + M * K + 4 * M + 2 * M * N + res
        return N * K // 2 + N * K // 16 + 4 + M * K // 2 + M * K // 16 + 4 * M + 2 * M * N + res

    def prologue_bytes(self, L):
        M, K = self.M, L["K"]
        if self.fp8:
            return M * K * 2 + M * K + 4 * M
        return M * K * 2 + M * K // 2 + M * K // 16 + 4 * M


# the mixed-precision stack: these projections in FP8 W8A8, the rest NVFP4
MIXED_FP8 = ("o", "down")


def stack_weights(vq, device, layers=si.STACK_LAYERS, fp8=(), reuse=None):
    """Weights of the 28-layer stack in (layer, projection) order, each
    quantized on the device right after it is generated (only the quantized
    copy stays: about 3.7 GB all NVFP4).  Projections named in fp8 get FP8
    codes and per-row scales (2-tuples), the others NVFP4 (3-tuples).
    reuse: an all-NVFP4 list from an earlier call whose NVFP4 entries are
    shared instead of regenerated."""
    out = []
    for l in range(layers):
        for p, (name, K, N) in enumerate(si.STACK_PROJECTIONS):
            if reuse is not None and name not in fp8:
                out.append(reuse[7 * l + p])
                continue
            W = si.projection_weight(K, N, si.stack_seed(l, p)).to(device)
            if name in fp8:
                wq, sw = vq.alloc_fp8(N, K, device)
                vq.vlaq_quantize_weight_fp8(W, N, K, 0, wq, sw)
                out.append((wq, sw))
            else:
                wq, ws, wg = vq.alloc_nvfp4(N, K, device, per_tensor=True)
                vq.vlaq_quantize_weight_nvfp4(W, N, K, 0, wq, ws, wg)
                out.append((wq, ws, wg))
            del W
    torch.cuda.synchronize()
    return out


class Stack:
    """The 28-layer stack of seven unfused projections (196 GEMMs): every
    (layer, projection) has its own seeded weight and its own seeded
    activations [M, K]; run() is one prologue + GEMM per entry.  All NVFP4
    by default; with fp8 = MIXED_FP8 the o and down projections run FP8
    W8A8 (per-row scales) and q/k/v/gate/up NVFP4."""

    def __init__(self, vq, M, device, layers=si.STACK_LAYERS, weights=None, fp8=()):
        self.vq = vq
        self.M = M
        self.entries = []
        if weights is None:
            weights = stack_weights(vq, device, layers, fp8)
        for l in range(layers):
            for p, (name, K, N) in enumerate(si.STACK_PROJECTIONS):
                seed = si.stack_seed(l, p)
                W = weights[7 * l + p]
                is8 = name in fp8
                assert len(W) == (2 if is8 else 3), (name, len(W))
                X = si.projection_activations(K, M, seed).to(device)
                wsp, nb = vq.alloc_workspace(M, N, K, device)
                act = vq.alloc_fp8(M, K, device) if is8 else vq.alloc_nvfp4(M, K, device)
                self.entries.append(dict(layer=l, proj=p, name=name, K=K, N=N, W=W, X=X, fp8=is8, act=act,
                                         Y=torch.empty(M, N, dtype=torch.bfloat16, device=device), ws=wsp, nb=nb))
        torch.cuda.synchronize()
        self.flops = sum(2.0 * M * e["N"] * e["K"] for e in self.entries)
        self.weight_bytes = sum(sum(t.numel() * t.element_size() for t in e["W"]) for e in self.entries)

    def run(self, copy=0):
        vq, M = self.vq, self.M
        for e in self.entries:
            if e["fp8"]:
                xq, sx = e["act"]
                wq, sw = e["W"]
                vq.vlaq_quantize_act_fp8(e["X"], M, e["K"], None, 1e-6, 0, xq, sx)
                vq.vlaq_linear_fp8(xq, sx, wq, sw, None, e["Y"], M, e["N"], e["K"], e["ws"], e["nb"])
            else:
                xq, xs, xg = e["act"]
                wq, ws, wg = e["W"]
                vq.vlaq_quantize_act_nvfp4(e["X"], M, e["K"], None, 1e-6, 0, xq, xs, xg)
                vq.vlaq_linear_nvfp4(xq, xs, xg, wq, ws, wg, None, e["Y"], M, e["N"], e["K"], e["ws"], e["nb"])


def capture(step, copies=1):
    """CUDA graph of `copies` consecutive steps (rotating weight copies)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for c in range(copies):
            step.run(c)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in range(copies):
            step.run(c)
    torch.cuda.synchronize()
    return g


def barrier(dist_on):
    if dist_on:
        torch.distributed.barrier()


def max_over_ranks(v, dist_on, device):
    if not dist_on:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def time_graph(g, reps, dist_on, device):
    barrier(dist_on)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier(dist_on)
    return max_over_ranks(e0.elapsed_time(e1) / reps, dist_on, device)


class _Rt:
    """CUDA runtime calls for timing events that live inside a graph: an
    event recorded with cudaEventRecordExternal during stream capture
    becomes an event-record node that timestamps every replay (a plain
    record would only become a dependency edge)."""
    lib = None

    @classmethod
    def get(cls):
        if cls.lib is None:
            import ctypes
            for name in ("libcudart.so.12", "libcudart.so"):
                try:
                    lib = ctypes.CDLL(name)
                    break
                except OSError:
                    lib = None
            if lib is None:
                raise OSError("CUDA runtime library not found")
            P = ctypes.c_void_p
            lib.cudaEventCreate.argtypes = [ctypes.POINTER(P)]
            lib.cudaEventRecordWithFlags.argtypes = [P, P, ctypes.c_uint]
            lib.cudaEventElapsedTime.argtypes = [ctypes.POINTER(ctypes.c_float), P, P]
            lib.cudaEventDestroy.argtypes = [P]
            cls.lib = lib
        return cls.lib


class GraphEvent:
    def __init__(self):
        import ctypes
        self.h = ctypes.c_void_p()
        rc = _Rt.get().cudaEventCreate(ctypes.byref(self.h))
        if rc != 0:
            raise RuntimeError(f"cudaEventCreate failed ({rc})")

    def record(self):
        rc = _Rt.get().cudaEventRecordWithFlags(self.h, ctypes_stream(), 1)  # cudaEventRecordExternal
        if rc != 0:
            raise RuntimeError(f"cudaEventRecordWithFlags failed ({rc})")

    def elapsed_time(self, other):
        import ctypes
        ms = ctypes.c_float()
        rc = _Rt.get().cudaEventElapsedTime(ctypes.byref(ms), self.h, other.h)
        if rc != 0:
            raise RuntimeError(f"cudaEventElapsedTime failed ({rc})")
        return ms.value


def ctypes_stream():
    import ctypes
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def kernel_durations(step, reps, copies=1):
    """Per-launch durations (ms) of the prologue and the GEMM of each
    projection from CUDA events on the launching stream, recorded as event
    nodes inside a CUDA graph of the step (host launch overhead cannot leak
    into the kernel times).  Falls back to eager event pairs if the runtime
    refuses.  Returns (prologue[i][r], gemm[i][r], mode)."""
    pro = [[] for _ in step.layers]
    gem = [[] for _ in step.layers]

    def collect(evs):
        for c in range(copies):
            for i in range(len(step.layers)):
                pro[i].append(evs[c][i][0].elapsed_time(evs[c][i][1]))
                gem[i].append(evs[c][i][1].elapsed_time(evs[c][i][2]))

    try:
        evs = [[[GraphEvent() for _ in range(3)] for _ in step.layers] for _ in range(copies)]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for c in range(copies):
                step.run(c, evs[c])
        torch.cuda.synchronize()
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize()
        for _ in range(reps):
            g.replay()
            torch.cuda.synchronize()
            collect(evs)
        del g
        return pro, gem, "graph"
    except Exception as exc:  # noqa: BLE001
        torch.cuda.synchronize()
        print(f"bench: in-graph event timing unavailable ({exc}); using eager events", file=sys.stderr)
        pro = [[] for _ in step.layers]
        gem = [[] for _ in step.layers]
        for _ in range(reps):
            evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in step.layers]
                   for _ in range(copies)]
            for c in range(copies):
                step.run(c, evs[c])
            torch.cuda.synchronize()
            collect(evs)
        return pro, gem, "eager"


# -------------------------------------------------------------- CPU oracle
def cpu_oracle_sample(data, rows_per_proj, fp8=False, decoded_w=None):
    """Runs the oracle on `rows_per_proj` token rows of every projection;
    returns (seconds, GEMM flops of the sample, decoded weights)."""
    import oracle
    if decoded_w is None:
        decoded_w = {}
        for name in PROJ:
            K, N, X, W = data[name]
            cw, sw, gw = oracle.quantize_nvfp4(si.to_bits(W), per_tensor=True)
            decoded_w[name] = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
    t0 = time.perf_counter()
    flops = 0.0
    for name in PROJ:
        K, N, X, W = data[name]
        xb = si.to_bits(X[:rows_per_proj])
        cx, sx, gx = oracle.quantize_nvfp4(xb)
        dx = oracle.decode_nvfp4(cx, sx, gx, K)
        oracle.linear_f64(dx, decoded_w[name])
        flops += 2.0 * rows_per_proj * N * K
    return time.perf_counter() - t0, flops, decoded_w


# -------------------------------------------------------------------- main
def run_reference(args, rank):
    """Reference arm: the CPU oracle, as it stands, on the host cores."""
    if rank != 0:
        return
    import oracle
    data = make_inputs(M_PREFILL, "cpu")
    rows = args.ref_rows
    _, _, dec = cpu_oracle_sample(data, 1)
    for _ in range(args.warmup):
        cpu_oracle_sample(data, 1, decoded_w=dec)
    times, flops = [], 0.0
    for _ in range(args.steps):
        t, flops, _ = cpu_oracle_sample(data, rows, decoded_w=dec)
        times.append(t)
    ms = 1000.0 * sum(times) / len(times)
    value = flops / (ms / 1000.0) / 1e12
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"NVFP4 W4A4 prefill projections qkv/o/gate_up/down, M={M_PREFILL} "
                               f"(oracle sample: {rows} token rows per projection per step)",
                   "global_batch": M_PREFILL, "parallelism": "host cores"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"{rows} token rows x 4 projections per step: NVFP4 quantize + fp64 GEMM"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


SECTIONS = ("decode", "fused", "w8a8", "e2e", "variants", "weight_quant", "stack")


class Launches:
    """run() issues the given launches in order (a graph of them is timed
    back to back)."""

    def __init__(self, fns):
        self.fns = fns

    def run(self, c=0):
        for f in self.fns:
            f()


def back_to_back_ms(fns, reps, warmup, dist_on, device):
    """Per-launch time of `fns` launched back to back in one graph."""
    g = capture(Launches(fns))
    for _ in range(warmup):
        g.replay()
    ms = time_graph(g, reps, dist_on, device) / len(fns)
    del g
    return ms


L2_BYTES = 126 * 2 ** 20


def copies_beyond_l2(nbytes, least=2):
    """Buffer copies whose total exceeds L2 (so every launch reads HBM)."""
    return max(least, -(-int(1.25 * L2_BYTES) // max(int(nbytes), 1)))


def prologue_back_to_back(step, args, dist_on, device):
    """Per-projection prologue launch time, back to back over input copies
    larger than L2 in total (ms)."""
    out = {}
    for L in step.layers:
        xb = L["X"].numel() * L["X"].element_size()
        Xs = [L["X"]] + [L["X"].clone() for _ in range(copies_beyond_l2(xb) - 1)]
        fns = [(lambda X=X, L=L: step.prologue(L, X)) for X in Xs]
        out[L["name"]] = back_to_back_ms(fns, args.steps, args.warmup, dist_on, device)
        del Xs
    return out


def gemm_back_to_back(step, args, dist_on, device):
    """Per-projection GEMM launch time, back to back over weight copies
    larger than L2 in total (ms)."""
    out = {}
    for L in step.layers:
        wb = sum(t.numel() * t.element_size() for t in L["W"][0] if t is not None)
        need = copies_beyond_l2(wb)
        extra = [tuple(None if t is None else t.clone() for t in L["W"][0]) for _ in range(need - len(L["W"]))]
        W = L["W"] + extra
        fns = []
        for c in range(len(W)):
            def f(c=c, L=L, W=W):
                saved = L["W"]
                L["W"] = W
                step.gemm(L, c)
                L["W"] = saved
            fns.append(f)
        out[L["name"]] = back_to_back_ms(fns, args.steps, args.warmup, dist_on, device)
        del extra, W
    return out


def step_section(vq, step, args, dist_on, device, peaks, world, copies=1):
    """Graph-timed step plus in-step kernel durations."""
    graph = capture(step, copies)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    ms = time_graph(graph, args.steps, dist_on, device) / copies
    del graph
    pro, gem, tmode = kernel_durations(step, max(args.steps // 2, 3), copies=copies)
    return ms, pro, gem, tmode


def prefill_section(vq, data, args, dist_on, device, peaks, world):
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    step = Step(vq, data, M_PREFILL, device)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    graph = capture(step)
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ms = time_graph(graph, args.steps, dist_on, device)
    pro, gem, tmode = kernel_durations(step, max(args.steps // 2, 3))
    clocks = sampler.stop()
    del graph
    value = world * step.flops / (ms / 1e3) / 1e12
    # dominant kernel: the gate_up GEMM launch (about half of the step);
    # achieved: per-launch time back to back over weight copies larger than
    # L2 (as for the prologue), in_step: event nodes around it in the step
    gi = PROJ.index("gate_up")
    GL = step.layers[gi]
    gflop = lambda L: 2.0 * M_PREFILL * L["N"] * L["K"]
    gb2b = gemm_back_to_back(step, args, dist_on, device)
    g_ach = gflop(GL) / (gb2b["gate_up"] / 1e3) / 1e12
    g_ach_step = gflop(GL) / (statistics.mean(gem[gi]) / 1e3) / 1e12
    gemm_all = step.flops / (sum(gb2b.values()) / 1e3) / 1e12
    gemm_all_step = step.flops / (sum(statistics.mean(x) for x in gem) / 1e3) / 1e12
    pro_ms = sum(statistics.mean(x) for x in pro)
    pro_bytes = sum(step.prologue_bytes(L) for L in step.layers)
    b2b = prologue_back_to_back(step, args, dist_on, device)
    b2b_ms = sum(b2b.values())
    per_proj = {L["name"]: {"gemm_us": 1e3 * gb2b[L["name"]],
                            "gemm_tflops": gflop(L) / (gb2b[L["name"]] / 1e3) / 1e12,
                            "gemm_us_in_step": 1e3 * statistics.mean(gem[i]),
                            "gemm_tflops_in_step": gflop(L) / (statistics.mean(gem[i]) / 1e3) / 1e12,
                            "prologue_us_in_step": 1e3 * statistics.mean(pro[i]),
                            "prologue_us": 1e3 * b2b[L["name"]],
                            "prologue_gbs": step.prologue_bytes(L) / (b2b[L["name"]] / 1e3) / 1e9}
                for i, L in enumerate(step.layers)}
    traffic = load_traffic("gemm_nvfp4_prefill")
    out = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1/e4m3 (fp32 accumulate, bf16 out)", "data": "synthetic",
        "config": {"workload": "NVFP4 W4A4 prefill: act prologue + block-scaled FP4 GEMM for qkv 3584->4608, "
                               "o 3584->3584, gate_up 3584->37888, down 18944->3584 (Qwen2.5-VL-7B shapes)",
                   "global_batch": M_PREFILL * world, "seq_len": M_PREFILL, "parallelism": f"dp{world}",
                   "l2": "inputs larger than L2 (per-step working set ~294 MB)", "graph": True},
        "roofline": {"bound": "tensor", "achieved": g_ach, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": g_ach / fp4_peak, "traffic": traffic,
                     "kernel": "gemm_fp4_pair_kernel gate_up 1024x37888x3584 (2MNK = 278.1 GFLOP per launch)",
                     "achieved_in_step": g_ach_step, "frac_in_step": g_ach_step / fp4_peak,
                     "all_gemms_tflops": gemm_all, "all_gemms_frac": gemm_all / fp4_peak,
                     "all_gemms_tflops_in_step": gemm_all_step, "all_gemms_frac_in_step": gemm_all_step / fp4_peak,
                     "timing": "achieved: back to back over weight copies > L2 (per-launch time, CUDA events around "
                               f"the graph); in_step: event nodes around each launch inside a {tmode} capture of the step",
                     "peak_note": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} TFLOP/s x 4 (nominal FP4:BF16)"},
        "prologue": {"bound": "hbm", "achieved": pro_bytes / (b2b_ms / 1e3) / 1e9, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": pro_bytes / (b2b_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "achieved_in_step": pro_bytes / (pro_ms / 1e3) / 1e9,
                     "frac_in_step": pro_bytes / (pro_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                     "kernel": "quant_rows_kernel (NVFP4 activation prologue), qkv / o / gate_up / down inputs",
                     "timing": "achieved: back to back over input copies > L2 (per-launch time, CUDA events around "
                               "the graph); in_step: event nodes around each launch inside the step"},
        "per_projection": per_proj,
        "clocks": clocks,
    }
    return step, out


def decode_section(vq, data, args, dist_on, device, peaks, world):
    """M = 1, 4, 8: the step over two weight copies, plus the GEMMs back to
    back over weight copies larger than L2."""
    res = {}
    for M in (1, 4, 8):
        ddata = {n: (K, N, X[:M].contiguous(), W) for n, (K, N, X, W) in data.items()}
        dstep = Step(vq, ddata, M, device, weight_copies=2)
        dms, dpro, dgem, _ = step_section(vq, dstep, args, dist_on, device, peaks, world, copies=2)
        dbytes = sum(dstep.gemm_bytes(L) + dstep.prologue_bytes(L) for L in dstep.layers)
        gem_bytes = {L["name"]: dstep.gemm_bytes(L) for L in dstep.layers}
        b2b = gemm_back_to_back(dstep, args, dist_on, device)
        tot_bytes = sum(gem_bytes.values())
        b2b_ach = tot_bytes / (sum(b2b.values()) / 1e3) / 1e9
        ins_ms = sum(sum(x) for x in dgem) / len(dgem[0])
        res[str(M)] = {
            "value": world * dbytes / (dms / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": dms,
            "bytes_per_step": dbytes, "M": M,
            "gemm_roofline": {"bound": "hbm", "achieved": b2b_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": b2b_ach / peaks["hbm_gbs"],
                              "achieved_in_step": tot_bytes / (ins_ms / 1e3) / 1e9,
                              "frac_in_step": tot_bytes / (ins_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
                              "timing": "achieved: each GEMM back to back over weight copies > L2; in_step: "
                                        "event nodes inside the step"},
            "per_projection": {L["name"]: {"gemm_us": 1e3 * b2b[L["name"]],
                                           "gemm_gbs": gem_bytes[L["name"]] / (b2b[L["name"]] / 1e3) / 1e9,
                                           "gemm_us_in_step": 1e3 * statistics.mean(dgem[i]),
                                           "prologue_us_in_step": 1e3 * statistics.mean(dpro[i])}
                               for i, L in enumerate(dstep.layers)}}
        del dstep
        torch.cuda.empty_cache()
    return res


GEMM_TIMING = ("gemm_achieved: the four GEMMs back to back over weight copies > L2 (per-launch times, CUDA "
               "events around the graph); in_step: event nodes around each launch inside the step")


def w8a8_section(vq, data, args, dist_on, device, peaks, world, fmt, fused=False):
    fstep = Step(vq, data, M_PREFILL, device, fmt=fmt, fused=fused)
    fms, _, fgem, _ = step_section(vq, fstep, args, dist_on, device, peaks, world)
    fgem_ms = sum(sum(x) for x in fgem) / len(fgem[0])
    gb2b = gemm_back_to_back(fstep, args, dist_on, device)
    gb_ms = sum(gb2b.values())
    fp8_peak = peaks["bf16_tflops"] * FP8_PER_BF16
    out = {"value": world * fstep.flops / (fms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": fms,
           "gemm_achieved": fstep.flops / (gb_ms / 1e3) / 1e12, "peak": fp8_peak,
           "frac": fstep.flops / (gb_ms / 1e3) / 1e12 / fp8_peak,
           "gemm_achieved_in_step": fstep.flops / (fgem_ms / 1e3) / 1e12,
           "frac_in_step": fstep.flops / (fgem_ms / 1e3) / 1e12 / fp8_peak,
           "gemm_us": {k: 1e3 * v for k, v in gb2b.items()}, "timing": GEMM_TIMING}
    del fstep
    return out


def fused_section(vq, data, args, dist_on, device, peaks, world):
    """The fused-prologue step at M = 1024: NVFP4 and FP8 W8A8."""
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    step = Step(vq, data, M_PREFILL, device, fused=True)
    ms, pro, gem, _ = step_section(vq, step, args, dist_on, device, peaks, world)
    b2b = prologue_back_to_back(step, args, dist_on, device)
    gb2b = gemm_back_to_back(step, args, dist_on, device)
    pro_bytes = sum(step.prologue_bytes(L) for L in step.layers)
    gemm_ms = sum(statistics.mean(x) for x in gem)
    gb_ms = sum(gb2b.values())
    out = {"nvfp4": {
        "value": world * step.flops / (ms / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ms,
        "gemm_tflops": step.flops / (gb_ms / 1e3) / 1e12, "gemm_frac": step.flops / (gb_ms / 1e3) / 1e12 / fp4_peak,
        "gemm_tflops_in_step": step.flops / (gemm_ms / 1e3) / 1e12,
        "gemm_frac_in_step": step.flops / (gemm_ms / 1e3) / 1e12 / fp4_peak, "timing": GEMM_TIMING,
        "prologue_gbs": pro_bytes / (sum(b2b.values()) / 1e3) / 1e9,
        "prologue_frac": pro_bytes / (sum(b2b.values()) / 1e3) / 1e9 / peaks["hbm_gbs"],
        "per_projection": {L["name"]: {"flags": L["flags"], "residual": L["R"] is not None,
                                       "prologue_us": 1e3 * b2b[L["name"]],
                                       "gemm_us": 1e3 * gb2b[L["name"]],
                                       "gemm_us_in_step": 1e3 * statistics.mean(gem[i])}
                           for i, L in enumerate(step.layers)},
        "workload": "RMSNorm (gain U(0.5,1.5), eps 1e-6) + block-64 WHT on qkv / gate_up inputs, WHT + residual "
                    "add on o / down, WHT-rotated weights; M = 1024"}}
    del step
    out["fp8"] = w8a8_section(vq, data, args, dist_on, device, peaks, world, "fp8", fused=True)
    return out


def stack_section(vq, args, dist_on, device, world):
    """28-layer stack, one graph of 196 prologue + GEMM pairs: all NVFP4,
    then mixed (o / down FP8 W8A8, the rest NVFP4)."""
    out = {}
    sw = stack_weights(vq, device)
    variants = (("", (), sw), ("mixed_", MIXED_FP8, None))
    for prefix, fp8, w in variants:
        if w is None:
            w = stack_weights(vq, device, fp8=fp8, reuse=sw)
        for sm in (M_PREFILL, 1):
            st = Stack(vq, sm, device, weights=w, fp8=fp8)
            sg = capture(st)
            for _ in range(args.warmup):
                sg.replay()
            torch.cuda.synchronize()
            sms = time_graph(sg, max(args.steps // 4, 3), dist_on, device)
            key = prefix + ("prefill" if sm > 1 else "decode")
            out[key] = {"M": sm, "ms": sms, "us_per_token": 1e3 * sms / sm,
                        "tflops": world * st.flops / (sms / 1e3) / 1e12,
                        "weight_gbs": world * st.weight_bytes / (sms / 1e3) / 1e9,
                        "gemms": len(st.entries), "fp8_projections": list(fp8)}
            del sg, st
            torch.cuda.empty_cache()
        del w
    del sw
    torch.cuda.empty_cache()
    return out


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


class _OmpThreads:
    """Sets the OpenMP thread count of this process (the oracle's GEMM is
    parallel over output rows) for a single-core timing, then restores it."""

    def __init__(self, n):
        import ctypes
        self.n = n
        try:
            self.lib = ctypes.CDLL("libgomp.so.1")
        except OSError:
            self.lib = None

    def __enter__(self):
        if self.lib:
            self.prev = self.lib.omp_get_max_threads()
            self.lib.omp_set_num_threads(self.n)
        return self

    def __exit__(self, *exc):
        if self.lib:
            self.lib.omp_set_num_threads(self.prev)


def cpu_baselines(data, args):
    """The CPU oracle, as it stands, on bounded samples of every workload."""
    import oracle
    cores = oracle.num_threads()
    out = {"cores": cores, "cpu": cpu_model()}
    # prefill: a token sample of each projection
    t, fl, dec = cpu_oracle_sample(data, 1)
    t, fl, _ = cpu_oracle_sample(data, args.cpu_rows, decoded_w=dec)
    out["prefill"] = {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                      "sample": f"{args.cpu_rows} token rows of each projection: NVFP4 quantize + fp64 GEMM "
                                f"({t:.1f} s)"}
    # decode M = 1, 4, 8: every token, all four projections; GB/s of the
    # same algorithmic bytes as the GPU line (the fp64 GEMM runs in parallel
    # over output rows only, so M = 1 is one core)
    dec_out = {}
    for M in (1, 4, 8):
        t0 = time.perf_counter()
        nbytes = 0
        for name in PROJ:
            K, N, X, W = data[name]
            cx, sx, gx = oracle.quantize_nvfp4(si.to_bits(X[:M]))
            oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, K), dec[name])
            nbytes += N * K // 2 + N * K // 16 + M * K * 2 + 2 * M * N
        tt = time.perf_counter() - t0
        dec_out[str(M)] = {"value": nbytes / tt / 1e9, "unit": "GB/s", "s": tt,
                           "cores": 1 if M == 1 else min(M, cores)}
    out["decode"] = dec_out
    # tiny workload (16 x 256 x 128), all cores and one core
    X, W = si.tiny_inputs(0)
    cw, sw, gw = oracle.quantize_nvfp4(si.to_bits(W), per_tensor=True)
    dw = oracle.decode_nvfp4(cw, sw, gw, 256, per_tensor=True)

    def tiny():
        cx, sx, gx = oracle.quantize_nvfp4(si.to_bits(X))
        oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, 256), dw)

    reps = 200
    t0 = time.perf_counter()
    for _ in range(reps):
        tiny()
    ta = (time.perf_counter() - t0) / reps
    with _OmpThreads(1):
        t0 = time.perf_counter()
        for _ in range(reps):
            tiny()
        t1 = (time.perf_counter() - t0) / reps
    out["tiny"] = {"unit": "GFLOP/s", "value": 2 * 16 * 128 * 256 / ta / 1e9, "single_core": 2 * 16 * 128 * 256 / t1 / 1e9,
                   "us_per_call": 1e6 * ta, "us_per_call_single_core": 1e6 * t1}
    # single-core decode M = 1 (as above, pinned to one thread)
    with _OmpThreads(1):
        t0 = time.perf_counter()
        for name in PROJ:
            K, N, X, W = data[name]
            cx, sx, gx = oracle.quantize_nvfp4(si.to_bits(X[:1]))
            oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, K), dec[name])
        out["decode"]["1"]["single_core_s"] = time.perf_counter() - t0
    del dec
    # fused workload: rotated weights, RMSNorm + rotation (qkv, gate_up) or
    # rotation + residual (o, down) on a token sample
    rows = max(args.cpu_rows // 16, 4)
    t = fl = 0.0
    for name in PROJ:
        K, N, X, W = data[name]
        case = FUSED[name]
        flags = 3 if case.rmsnorm else 2
        cw, sw, gw = oracle.quantize_nvfp4(si.to_bits(W), flags=2, per_tensor=True)
        dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
        gam = si.to_bits(si.norm_gain(K, case.seed))
        R = si.to_bits(si.residual(rows, N, case.seed)) if case.residual else None
        t0 = time.perf_counter()
        cx, sx, gx = oracle.quantize_nvfp4(si.to_bits(X[:rows]), gam, 1e-6, flags)
        oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, K), dw, R)
        t += time.perf_counter() - t0
        fl += 2.0 * rows * N * K
        del dw
    out["fused"] = {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                    "sample": f"{rows} token rows of each projection, fused prologue + fp64 GEMM ({t:.1f} s)"}
    # 28-layer stack: layer 0 timed on a token sample, per token x 28 layers
    rows = 4
    t = 0.0
    for p, (name, K, N) in enumerate(si.STACK_PROJECTIONS):
        seed = si.stack_seed(0, p)
        cw, sw, gw = oracle.quantize_nvfp4(si.to_bits(si.projection_weight(K, N, seed)), per_tensor=True)
        dw = oracle.decode_nvfp4(cw, sw, gw, K, per_tensor=True)
        X = si.projection_activations(K, rows, seed)
        t0 = time.perf_counter()
        cx, sx, gx = oracle.quantize_nvfp4(si.to_bits(X))
        oracle.linear_f64(oracle.decode_nvfp4(cx, sx, gx, K), dw)
        t += time.perf_counter() - t0
        del dw
    out["stack"] = {"us_per_token": 1e6 * t / rows * si.STACK_LAYERS, "unit": "us/token", "cores": cores,
                    "kind": "oracle", "extrapolated": True,
                    "sample": f"layer 0 (7 projections) on {rows} token rows, x {si.STACK_LAYERS} layers"}
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="vlaq", choices=["vlaq", "reference"])
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="the prefill step only (no decode / fused / 8-bit / e2e / "
                                                        "stack sections)")
    ap.add_argument("--no-stack", action="store_true", help="skip the 28-layer stack (about a minute of setup)")
    ap.add_argument("--sections", default=",".join(SECTIONS),
                    help="comma-separated sections to run after the prefill step: " + ", ".join(SECTIONS))
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    sections = set() if args.quick else {x for x in args.sections.split(",") if x}
    if args.no_stack:
        sections.discard("stack")
    unknown = sections - set(SECTIONS)
    if unknown:
        ap.error(f"unknown sections {sorted(unknown)}")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1

    if args.impl == "reference":
        # rank 0 alone runs the oracle; the other ranks exit without work
        run_reference(args, rank)
        return

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=300))
    import vlaq_quantize_act_b200 as vq

    peaks = load_peaks()
    # weak scaling: every rank quantizes and multiplies its own tokens (its
    # own activation seeds) against the same weights
    data = make_inputs(M_PREFILL, "cpu", seed_offset=RANK_SEED_STRIDE * rank)

    step, out = prefill_section(vq, data, args, dist_on, device, peaks, world)
    launches_per_step = sum(2 + (1 if L["nb"] else 0) for L in step.layers)

    if "decode" in sections:
        out["decode"] = decode_section(vq, data, args, dist_on, device, peaks, world)
    if "fused" in sections:
        out["fused"] = fused_section(vq, data, args, dist_on, device, peaks, world)
    if "w8a8" in sections:
        for fmt in ("fp8", "int8"):
            out[fmt] = w8a8_section(vq, data, args, dist_on, device, peaks, world, fmt)
    if "e2e" in sections:
        # ---------------- e2e through the public API with host buffers
        hostX = [L["X"].cpu().pin_memory() for L in step.layers]
        hostY = [torch.empty(L["Y"].shape, dtype=torch.bfloat16).pin_memory() for L in step.layers]
        h2d = sum(x.numel() * 2 for x in hostX)
        d2h = sum(y.numel() * 2 for y in hostY)

        def e2e_step():
            for i, L in enumerate(step.layers):
                L["X"].copy_(hostX[i], non_blocking=True)
            step.run(0)
            for i, L in enumerate(step.layers):
                hostY[i].copy_(L["Y"], non_blocking=True)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        barrier(dist_on)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            e2e_step()
        e1.record()
        torch.cuda.synchronize()
        barrier(dist_on)
        ems = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist_on, device)
        out["e2e"] = {"value": world * step.flops / (ems / 1e3) / 1e12, "unit": "TFLOP/s", "ms_per_step": ems,
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if "variants" in sections:
        # ---------------- prologue variants over the four projection inputs:
        # fused RMSNorm + block-64 rotation, per-channel smoothing (divide,
        # before the rotation), both, and a static calibrated global scale
        # (no row-amax pass) plain and fused; same bytes as the plain
        # prologue (the gains and smoothing factors stay in cache)
        pro_bytes = sum(step.prologue_bytes(L) for L in step.layers)
        variants = {"fused_rmsnorm_wht": (3, False, None), "smooth": (0, True, None),
                    "fused_smooth": (3, True, None), "static": (0, False, 0.01),
                    "fused_static": (3, False, 0.01)}
        extra = {}
        for L in step.layers:
            K = L["K"]
            rng = np.random.default_rng(K)
            extra[L["name"]] = (si.norm_gain(K, 5).to(device),
                                torch.from_numpy(np.exp(rng.uniform(np.log(0.1553), np.log(6.4375), K))
                                                 .astype(np.float32)).to(device))
        out["prologue_variants"] = {}
        for vname, (vflags, vsmooth, vstatic) in variants.items():
            class _PV:
                def run(self, c=0):
                    for L in step.layers:
                        xq, xs, xg = L["act"]
                        gam, sm = extra[L["name"]]
                        if vstatic is not None:
                            vq.vlaq_quantize_act_nvfp4_static(L["X"], M_PREFILL, L["K"], gam, None, 1e-6, vflags,
                                                              vstatic, xq, xs, xg)
                        elif vsmooth:
                            vq.vlaq_quantize_act_nvfp4_smooth(L["X"], M_PREFILL, L["K"], gam, sm, 1e-6, vflags,
                                                              xq, xs, xg)
                        else:
                            vq.vlaq_quantize_act_nvfp4(L["X"], M_PREFILL, L["K"], gam, 1e-6, vflags, xq, xs, xg)

            pgraph = capture(_PV())
            for _ in range(args.warmup):
                pgraph.replay()
            torch.cuda.synchronize()
            pms = time_graph(pgraph, args.steps, dist_on, device)
            out["prologue_variants"][vname] = {"GB/s": pro_bytes / (pms / 1e3) / 1e9, "ms": pms,
                                               "frac": pro_bytes / (pms / 1e3) / 1e9 / peaks["hbm_gbs"]}
            del pgraph

    if "weight_quant" in sections:
        # ---------------- offline weight quantization (a1), gate_up weights:
        # HBM-bound; algorithmic bytes = one bf16 read + codes, scales, g
        K, N, _, W = data["gate_up"]
        Wd = W.to(device)
        wq, ws, wg = vq.alloc_nvfp4(N, K, device, per_tensor=True)

        class _WQ:
            def run(self, c=0):
                vq.vlaq_quantize_weight_nvfp4(Wd, N, K, 0, wq, ws, wg)

        wgraph = capture(_WQ())
        for _ in range(args.warmup):
            wgraph.replay()
        torch.cuda.synchronize()
        wms = time_graph(wgraph, args.steps, dist_on, device)
        wbytes = 2 * N * K + wq.numel() + ws.numel() + 4
        out["weight_quant"] = {"unit": "GB/s", "value": wbytes / (wms / 1e3) / 1e9, "ms": wms,
                               "bytes": wbytes, "frac": wbytes / (wms / 1e3) / 1e9 / peaks["hbm_gbs"],
                               "peak": peaks["hbm_gbs"],
                               "shape": f"gate_up W {N}x{K} bf16 -> NVFP4 (amax pass + quantize pass)"}
        del wgraph, Wd, wq, ws, wg

    if "stack" in sections:
        del step
        torch.cuda.empty_cache()
        step = None
        out["stack"] = stack_section(vq, args, dist_on, device, world)

    # launches of our kernels inside the headline timed region: per step 4
    # prologues + 4 GEMMs (+ split-K reductions when planned)
    out["gpu_launches"] = launches_per_step * args.steps

    if rank == 0 and not args.no_cpu_baseline:
        base = cpu_baselines(data, args)
        out["cpu_baseline"] = dict(base["prefill"])
        out["cpu_baseline"]["cpu"] = base["cpu"]
        out["cpu_baseline"]["workloads"] = {k: v for k, v in base.items() if k not in ("prefill", "cores", "cpu")}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist_on:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
