"""Benchmark of the BitNet b1.58 BitLinear forward on B200.

Default workload: the 70B-shaped decoder block projections at decode (T = 1): q,k,v
(attn_norm), o (attn_sub_norm, on a synthetic attention output), and the SiLU FFN
(ffn_norm -> gate/up -> SiLU -> ffn_sub_norm -> down, fed by o's output), the largest
configuration that runs on one GPU.  A step is one pass of that whole path; weights are
packed once before timing (offline step).  The same JSON line carries a `prefill` object
for the prefill half of the metric: the 32B-shaped FFN block at T = 4096 (int8 TOPS).

value  = packed-weight bytes read per step x steps x ranks / device time (max over ranks)
         [GB/s]; for prefill workloads (T >= 64) int8 TOPS = 2 T sum(N K) / time.
e2e    = the same metric with each step's activations copied from pinned host memory
         and its outputs copied back, inside the timed region.
L2     = the packed weights rotate over enough copies to exceed 2x the 126 MB L2, so
         every step reads its weights from HBM.

``--impl reference`` times the CPU oracle (numpy) on a bounded sample of the same
workload on this host's cores (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

L2_BYTES = 126 * 2 ** 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="proj_70b_decode_t1", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--prefill-workload", default="ffn_32b_t4096", choices=sorted(workloads.WORKLOADS) + ["none"],
                    help="prefill workload reported in the line's `prefill` object ('none' to skip)")
    ap.add_argument("--prefill-steps", type=int, default=30)
    ap.add_argument("--attention", default="70b", choices=["none"] + sorted(workloads.ATTN_SHAPES),
                    help="heads of the block whose decode attention is reported in the `attention` object")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying CUDA graphs")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU work of the oracle sample")
    ap.add_argument("--seed", type=int, default=0)
    return ap.parse_args()


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-i", str(self.index), "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        self.f.flush()
        self.f.seek(0)
        rows = [ln.split(",") for ln in self.f.read().strip().splitlines() if ln.strip()]
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for nm, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.f.name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel_key: str, sha: str):
    """DRAM bytes per launch of the dominant kernel ("<kernel> @ <workload>") from the
    committed ncu summary, if it was taken on the current kernel source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            d = json.load(f)
        e = d.get(kernel_key)
        if e and e.get("source_sha") == sha:
            return e["dram_bytes_per_launch"]
    except Exception:
        pass
    return None


def workload_units(name: str):
    """(packed bytes per step, int8 ops per step, tensor shapes) of a workload, from its shapes."""
    spec = workloads.WORKLOADS[name]
    if spec["kind"] == "bitlinear":
        tensors = {"w": (spec["N"], spec["K"])}
    else:
        sh = spec["shape"]
        names = ["gate", "up", "down"] if spec["kind"] == "ffn" else list(sh.tensors())
        tensors = {nm: sh.tensors()[nm] for nm in names}
    T = spec["T"]
    packed = sum(n * k // 4 + 32 for (n, k) in tensors.values())
    ops = sum(2 * T * n * k for (n, k) in tensors.values())
    return packed, ops, tensors


def workload_config(name: str, world: int, use_graph: bool) -> dict:
    """The `config` object of the JSON line (identical for both arms)."""
    packed, ops, _ = workload_units(name)
    n_copies = max(1, math.ceil(2 * L2_BYTES / packed) + 1)
    return {"workload": name, "T": workloads.WORKLOADS[name]["T"], "packed_bytes_per_step": packed,
            "int8_ops_per_step": ops, "parallelism": f"replicas x{world}",
            "l2": f"weights rotated over {n_copies} copies ({n_copies * packed / 1e6:.0f} MB > 2x L2)",
            "cuda_graphs": use_graph}


def max_over_ranks(values):
    """Element-wise maximum of per-rank timings over all ranks (identity with one process)."""
    t = torch.tensor(values, dtype=torch.float64)
    if torch.distributed.is_initialized():
        if torch.distributed.get_backend() == "nccl":
            t = t.cuda()
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def whole_job_rate(units_per_step: float, steps: int, world: int, ms: float) -> float:
    """Units processed by all ranks per second, over the slowest rank's time."""
    return world * units_per_step * steps / (ms / 1e3)


# ----------------------------------------------------------------------------- workload on the GPU

class Workload:
    def __init__(self, name: str, seed: int, device: str):
        import ternary_bitlinear_quantized_b200 as tb
        self.tb = tb
        self.name = name
        self.spec = workloads.WORKLOADS[name]
        self.kind = self.spec["kind"]
        self.T = self.spec["T"]
        dev = device
        self.dev = dev
        if self.kind == "bitlinear":
            N, K = self.spec["N"], self.spec["K"]
            self.tensors = {"w": (N, K)}
            W = {"w": workloads.latent_weight(N, K, seed, name, dev)}
            self.x = workloads.activations(self.T, K, seed, name + "/x", device=dev)
            self.g = workloads.gain(K, seed, name + "/g", dev)
        else:
            sh = self.spec["shape"]
            self.shape = sh
            ffn_only = self.kind == "ffn"
            d = workloads.block_inputs(sh, self.T, seed, self.spec.get("outliers", False), dev, ffn_only)
            self.d = d
            self.tensors = {nm: sh.tensors()[nm] for nm in (["gate", "up", "down"] if ffn_only else sh.tensors())}
            W = {nm: d["W_" + nm] for nm in self.tensors}
            self.act = tb.RELU2 if sh.act == "relu2" else tb.SILU
        self.packed_bytes = sum(tb.i2s_packed_bytes(n, k) for (n, k) in self.tensors.values())
        self.ops_per_step = sum(2 * self.T * n * k for (n, k) in self.tensors.values())
        # Pack once (offline), then replicate the bytes so that the copies exceed 2x L2.
        packed = {nm: tb.pack_i2s(W[nm]) for nm in self.tensors}
        del W
        self.n_copies = max(1, math.ceil(2 * L2_BYTES / self.packed_bytes) + 1)
        self.copies = [packed] + [{nm: p.clone() for nm, p in packed.items()} for _ in range(self.n_copies - 1)]
        self._alloc_outputs()

    def _alloc_outputs(self):
        T, dev = self.T, self.dev
        e = lambda *s, dt=torch.bfloat16: torch.empty(*s, dtype=dt, device=dev)
        if self.kind == "bitlinear":
            N, K = self.tensors["w"]
            self.qbuf = (e(T, K, dt=torch.int8), e(T, dt=torch.float32), e(T, dt=torch.int32))
            self.out = e(T, N)
            self.outputs = [self.out]
            self.inputs = [self.x]
            return
        sh = self.shape
        H, I = sh.hidden, sh.inter
        if self.kind == "block":
            self.qx = (e(T, H, dt=torch.int8), e(T, dt=torch.float32), e(T, dt=torch.int32))
            self.qa = (e(T, sh.n_q, dt=torch.int8), e(T, dt=torch.float32), e(T, dt=torch.int32))
            self.oq, self.ok_, self.ov = e(T, sh.n_q), e(T, sh.n_kv), e(T, sh.n_kv)
            self.oo = e(T, H)
            self.inputs = [self.d["x"], self.d["attn_out"]]
        else:
            self.inputs = [self.d["x"]]
        self.offn = e(T, H)
        # Zeroed once: the decode engine's grid-barrier counters live in the workspace.
        nws = (self.tb.block_workspace_bytes(T, H, sh.n_q, I) if self.kind == "block"
               else self.tb.ffn_workspace_bytes(T, H, I))
        self.ws = torch.zeros(nws, dtype=torch.uint8, device=self.dev)
        self.outputs = ([self.oq, self.ok_, self.ov, self.oo, self.offn] if self.kind == "block" else [self.offn])
        if self.kind == "block":
            self.gains = {k[2:]: v for k, v in self.d.items() if k.startswith("g_")}
            self.outs = {"q": self.oq, "k": self.ok_, "v": self.ov, "o": self.oo, "ffn": self.offn}

    def step(self, c: int):
        tb, p = self.tb, self.copies[c]
        if self.kind == "bitlinear":
            q, s, sq = tb.rmsnorm_quant_act(self.x, self.g, workloads.EPS, out=self.qbuf)
            tb.bitlinear(q, s, sq, p["w"], self.tensors["w"][0], out=self.out)
            return
        d, sh = self.d, self.shape
        if self.kind == "block":
            tb.decoder_block(d["x"], d["attn_out"], self.gains, p, sh.n_kv, sh.inter, self.act, workloads.EPS,
                             outs=self.outs, ws=self.ws)
            return
        tb.ffn_block(d["x"], d["g_ffn_norm"], p["gate"], p["up"], d["g_ffn_sub_norm"], p["down"], sh.inter,
                     self.act, workloads.EPS, out=self.offn, ws=self.ws)

    def launches_per_step(self) -> int:
        """Launches of this library's kernels per step (the decode engine runs a whole
        block or FFN in one launch; prefill launches quant + tensor-core product per layer)."""
        if self.kind == "bitlinear":
            return 2
        if self.T <= 16:
            return 1
        return 8 if self.kind == "block" else 4

    def dominant(self):
        """(label, callable(c), bytes per launch, ops per launch) of the dominant kernel: at
        decode the single engine launch of the whole step; at prefill the FFN's gate/up
        tensor-core launch (relu2/SiLU epilogue); for one BitLinear its product kernel."""
        tb = self.tb
        if self.kind != "bitlinear" and self.T <= 16:
            label = "k_engine (decoder block, one launch)" if self.kind == "block" else "k_engine (FFN, one launch)"
            return (label, lambda c: self.step(c), self.packed_bytes, self.ops_per_step)
        if self.kind == "bitlinear":
            N, K = self.tensors["w"]
            q, s, sq = self.qbuf
            return ("k_engine (bitlinear)" if self.T <= 16 else "k_gemm_tc (bitlinear)", lambda c: tb.bitlinear(q, s, sq, self.copies[c]["w"], N, out=self.out),
                    tb.i2s_packed_bytes(N, K), 2 * self.T * N * K)
        sh = self.shape
        H, I = sh.hidden, sh.inter
        off = tb.ffn_workspace_offsets(self.T, H, I)
        T = self.T
        q = self.ws[off[0]:off[0] + T * H].view(torch.int8).view(T, H)
        s = self.ws[off[1]:off[1] + 4 * T].view(torch.float32)
        sq = self.ws[off[2]:off[2] + 4 * T].view(torch.int32)
        h = self.ws[off[3]:off[3] + 4 * T * I].view(torch.float32).view(T, I)
        fn = lambda c: tb.bitlinear_gate_up_act(q, s, sq, self.copies[c]["gate"], self.copies[c]["up"], I, self.act,
                                                out=h)
        return ("k_gemm_tc<ffn> (gate/up + act)", fn, 2 * tb.i2s_packed_bytes(I, H), 4 * T * I * H)


def time_steps(wl: Workload, steps: int, warmup: int, use_graph: bool, e2e: bool):
    """Device time (ms) of `steps` steps, after `warmup` untimed ones."""
    R = wl.n_copies
    host_in = [t.cpu().pin_memory() for t in wl.inputs] if e2e else None
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in wl.outputs] if e2e else None

    def one(c):
        if e2e:
            for h, d in zip(host_in, wl.inputs):
                d.copy_(h, non_blocking=True)
        wl.step(c)
        if e2e:
            for h, d in zip(host_out, wl.outputs):
                h.copy_(d, non_blocking=True)

    for c in range(min(R, 2)):
        one(c)
    torch.cuda.synchronize()
    graphs = None
    if use_graph:
        graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        for c in range(R):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                one(c)
            graphs.append(g)
        torch.cuda.synchronize()
    run = (lambda i: graphs[i % R].replay()) if use_graph else (lambda i: one(i % R))
    for i in range(warmup):
        run(i)
    torch.cuda.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for i in range(steps):
        run(warmup + i)
    ev1.record()
    torch.cuda.synchronize()
    if torch.distributed.is_initialized():
        torch.distributed.barrier()
    ms = ev0.elapsed_time(ev1)
    del graphs
    h2d = sum(t.numel() * t.element_size() for t in wl.inputs) if e2e else 0
    d2h = sum(t.numel() * t.element_size() for t in wl.outputs) if e2e else 0
    return ms, h2d, d2h


def time_dominant(wl: Workload, steps: int, step_ms: float):
    """Average device duration (ms) of one launch of the dominant kernel, timed the way the
    step is timed: CUDA graphs replayed back to back on one stream, weights rotating.  At
    decode the step IS one launch of the decode engine, so its time is the step's."""
    label, fn, nbytes, ops = wl.dominant()
    if wl.kind != "bitlinear" and wl.T <= 16:
        return label, step_ms, nbytes, ops
    R = wl.n_copies
    for c in range(min(R, 2)):
        fn(c)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in range(R):
            fn(c)
    torch.cuda.synchronize()
    reps = max(1, steps // R)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * R)
    del g
    return label, ms, nbytes, ops


def int8_peak_probe():
    """Dense int8 tensor-core throughput of this GPU, measured now: torch._int_mm (cuBLASLt,
    int8 x int8 -> int32) at 8192^3, best of 10 launches after 3 warm-up ones (TOPS)."""
    n = 8192
    gen = torch.Generator(device="cuda").manual_seed(0)
    A = torch.randint(-128, 127, (n, n), dtype=torch.int8, device="cuda", generator=gen)
    B = torch.randint(-128, 127, (n, n), dtype=torch.int8, device="cuda", generator=gen).t().contiguous().t()
    for _ in range(3):
        torch._int_mm(A, B)
    torch.cuda.synchronize()
    best = None
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(A, B)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        best = ms if best is None else min(best, ms)
    del A, B
    return 2.0 * n ** 3 / (best / 1e3) / 1e12


# ----------------------------------------------------------------------------- CPU oracle leg

def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_sample(name: str, seed: int, seconds: float, single_thread_seconds: float = 0.0):
    """Time the numpy oracle on this workload (bounded sample) on all the host threads numpy
    uses, and optionally single-threaded.  Returns a dict: value, unit, sample, cores,
    and (if asked) single_thread_value."""
    import numpy as np
    from oracle import bitnet_oracle as O
    spec = workloads.WORKLOADS[name]
    T = spec["T"]
    decode = T < 64
    if spec["kind"] == "bitlinear":
        N, K = spec["N"], spec["K"]
        W = workloads.latent_weight(N, K, seed, name).numpy()
        packed = O.pack_i2s(W)
        x = workloads.activations(T, K, seed, name + "/x")
        xf = O.bf16_bits_to_f32(x.view(torch.int16).numpy().view(np.uint16))
        g = workloads.gain(K, seed, name + "/g").numpy()
        tensors = {"w": (N, K)}
        run = lambda xs, a=None: O.bitlinear_from_x(xs, g, workloads.EPS, packed, N, K, "bf16")
        af = None
    else:
        sh = spec["shape"]
        ffn_only = spec["kind"] == "ffn"
        d = workloads.block_inputs(sh, T, seed, spec.get("outliers", False), "cpu", ffn_only)
        tensors = {nm: sh.tensors()[nm] for nm in (["gate", "up", "down"] if ffn_only else sh.tensors())}
        packed = {nm: O.pack_i2s(d["W_" + nm].numpy()) for nm in tensors}
        gains = {k[2:]: v.numpy() for k, v in d.items() if k.startswith("g_")}
        xf = O.bf16_bits_to_f32(d["x"].view(torch.int16).numpy().view(np.uint16))
        af = None if ffn_only else O.bf16_bits_to_f32(d["attn_out"].view(torch.int16).numpy().view(np.uint16))
        H, I = sh.hidden, sh.inter
        if ffn_only:
            run = lambda xs, a=None: O.ffn_block(xs, gains["ffn_norm"], packed["gate"], packed["up"],
                                                 gains["ffn_sub_norm"], packed["down"], H, I, sh.act,
                                                 workloads.EPS, "bf16")
        else:
            run = lambda xs, a=None: O.decoder_block(xs, a, gains, packed, sh.tensors(), sh.act, workloads.EPS,
                                                     "bf16")
    pbytes = sum(n * k // 4 + 32 for (n, k) in tensors.values())
    # Tokens are independent through every step, so a prefill sample takes a few tokens.
    t_sample = T if decode else min(T, 8)
    xs = xf[:t_sample]
    a_s = None if af is None else af[:t_sample]

    def timed(limit):
        n, t0 = 0, time.perf_counter()
        while True:
            run(xs, a_s)
            n += 1
            el = time.perf_counter() - t0
            if el >= limit:
                return n, el

    def rate(n, el):
        if decode:
            return pbytes * n / el / 1e9
        return sum(2 * t_sample * nn * kk for (nn, kk) in tensors.values()) * n / el / 1e12

    n, el = timed(seconds)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    out = {"value": rate(n, el), "unit": "GB/s" if decode else "TOPS", "cores": cores, "kind": "oracle",
           "cpu_model": cpu_model()}
    if decode:
        out["sample"] = f"{n} full steps of the workload (T={T}) in {el:.1f} s on {cores} threads"
    else:
        out["sample"] = f"{n} steps on {t_sample} of the {T} tokens (tokens are independent) in {el:.1f} s"
    if single_thread_seconds > 0:
        try:
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                n1, el1 = timed(single_thread_seconds)
            out["single_thread_value"] = rate(n1, el1)
            out["single_thread_sample"] = f"{n1} steps in {el1:.1f} s on 1 thread"
        except Exception as e:  # threadpoolctl missing: report why
            out["single_thread_value"] = None
            out["single_thread_sample"] = f"not measured: {e}"
    return out


# ----------------------------------------------------------------------------- main

def roofline(wl: Workload, name: str, label: str, dom_ms: float, dom_bytes: int, dom_ops: int, int8_peak):
    """The `roofline` object of the dominant kernel (decode: HBM-bound on packed bytes;
    prefill: int8 tensor-core bound)."""
    hbm, bf16, src = peaks()
    decode = wl.T < 64
    kernel_files = (["ternary_bitlinear_quantized_b200/csrc/engine.cuh"] if decode else
                    ["ternary_bitlinear_quantized_b200/csrc/gemm_tc.cuh"]) + [
        "ternary_bitlinear_quantized_b200/csrc/gemv.cuh", "ternary_bitlinear_quantized_b200/csrc/common.cuh"]
    traffic = stored_traffic(f"{label} @ {name}", source_sha(kernel_files))
    if decode:
        achieved = dom_bytes / (dom_ms / 1e3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": traffic, "kernel": label, "bytes_per_launch": dom_bytes, "launch_us": dom_ms * 1e3,
                "peak_source": f"{src} hbm_gbs (copy bandwidth, burst)"}
    achieved = dom_ops / (dom_ms / 1e3) / 1e12
    nominal = bf16 * 2.0  # dense int8 = 2x dense bf16 (nominal ratio 4.5 / 2.25 PFLOP/s)
    peak = int8_peak if int8_peak else nominal
    return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TOPS", "frac": achieved / peak,
            "traffic": traffic, "kernel": label, "ops_per_launch": dom_ops, "launch_us": dom_ms * 1e3,
            "peak_source": ("int8 dense measured in this run (torch._int_mm, cuBLASLt, 8192^3, best of 10)"
                            if int8_peak else f"{src} bf16_tflops x 2 (nominal int8/bf16 ratio)"),
            "frac_of_bf16x2": achieved / nominal}


def measure(name: str, args, world: int, use_graph: bool, steps: int, int8_peak=None):
    """Device-timed throughput, end-to-end throughput and the dominant kernel of one
    workload (max over ranks).  Returns (line fields, clocks)."""
    spec = workloads.WORKLOADS[name]
    decode = spec["T"] < 64
    wl = Workload(name, args.seed + 0, f"cuda:{torch.cuda.current_device()}")  # same workload on every rank
    clk = ClockSampler(torch.cuda.current_device())
    clk.start()
    ms, _, _ = time_steps(wl, steps, args.warmup, use_graph, e2e=False)
    clocks = clk.stop()
    ms_e2e, h2d, d2h = time_steps(wl, steps, args.warmup, use_graph, e2e=True)
    label, dom_ms, dom_bytes, dom_ops = time_dominant(wl, steps, ms / steps)
    status = wl.tb.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    ms, ms_e2e, dom_ms = max_over_ranks([ms, ms_e2e, dom_ms])
    per_step_units = wl.packed_bytes / 1e9 if decode else wl.ops_per_step / 1e12
    fields = {
        "metric": "packed-weight HBM GB/s (decode)" if decode else "int8 TOPS (prefill)",
        "value": whole_job_rate(per_step_units, steps, world, ms),
        "unit": "GB/s" if decode else "TOPS",
        "steps": steps,
        "ms_per_step": ms / steps,
        "config": workload_config(name, world, use_graph),
        "roofline": roofline(wl, name, label, dom_ms, dom_bytes, dom_ops, int8_peak),
        "e2e": {"value": whole_job_rate(per_step_units, steps, world, ms_e2e), "unit": "GB/s" if decode else "TOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": wl.launches_per_step() * steps,
    }
    del wl
    torch.cuda.empty_cache()
    return fields, clocks


def measure_attention(shape: str, steps: int, warmup: int):
    """Decode attention of one block (T = 1): rotary embedding + cache append of the new token,
    then causal GQA attention over ATTN_CONTEXT cached positions.  Bound by the cache read:
    2 x Hkv x L x 256 bytes per step (keys and values, bf16)."""
    import ternary_bitlinear_quantized_b200 as tb
    Hq, Hkv = workloads.ATTN_SHAPES[shape]
    L = workloads.ATTN_CONTEXT
    T, pos0 = 1, L - 1
    dev = f"cuda:{torch.cuda.current_device()}"
    # several caches rotate so that the reads come from HBM (each 2 x Hkv x L x 256 bytes)
    cache_bytes = 2 * Hkv * L * 256
    R = max(2, math.ceil(2 * L2_BYTES / cache_bytes) + 1)
    d = workloads.attention_inputs(T, Hq, Hkv, L, pos0, seed=0, device=dev)
    caches = [(d["k_cache"].clone(), d["v_cache"].clone()) for _ in range(R)]
    q_rot = torch.empty(T, Hq, 128, dtype=torch.float32, device=dev)
    out = torch.empty(T, Hq, 128, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(tb.attention_workspace_bytes(T, Hq, Hkv, L), dtype=torch.uint8, device=dev)

    def one(c):
        kc, vc = caches[c]
        tb.rope_kv_append(d["q"], d["k"], d["v"], pos0, 10000.0, kc, vc, q_rot=q_rot)
        tb.attention_decode(q_rot, kc, vc, pos0, out=out, ws=ws)

    for c in range(R):
        one(c)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for c in range(R):
            one(c)
    torch.cuda.synchronize()
    reps = max(1, steps // R)
    for _ in range(max(1, warmup // R)):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * R)
    (ms,) = max_over_ranks([ms])
    hbm, _, src = peaks()
    gbs = cache_bytes / (ms / 1e3) / 1e9
    return {"workload": f"attention_{shape}_decode_t1_ctx{L}", "metric": "KV-cache HBM GB/s (decode attention)",
            "value": gbs, "unit": "GB/s", "us_per_step": ms * 1e3, "steps": reps * R,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "bytes_per_step": cache_bytes, "peak_source": f"{src} hbm_gbs",
                         "kernels": "k_rope_append + k_attn_partial + k_attn_combine"},
            "l2": f"caches rotated over {R} copies ({R * cache_bytes / 1e6:.0f} MB > 2x L2)",
            "gpu_launches": 3 * reps * R}


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    spec = workloads.WORKLOADS[args.workload]
    decode = spec["T"] < 64
    metric = ("packed-weight HBM GB/s (decode)" if decode else "int8 TOPS (prefill)")

    if args.impl == "reference":
        if rank != 0:
            return 0
        cpu = oracle_sample(args.workload, args.seed, args.cpu_seconds)
        val, u = cpu["value"], cpu["unit"]
        line = {"metric": metric, "value": val, "unit": u, "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "impl": "reference", "dtype": "int8", "data": "synthetic",
                "config": workload_config(args.workload, args.gpus, not args.no_graph),
                "cpu_baseline": cpu,
                "e2e": {"value": val, "unit": u, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    from ternary_bitlinear_quantized_b200 import build as tbuild
    if rank == 0 or world == 1:
        tbuild.build()
    if world > 1:
        torch.distributed.barrier()
    use_graph = not args.no_graph

    main_fields, clocks = measure(args.workload, args, world, use_graph, args.steps)
    prefill = None
    if args.prefill_workload != "none":
        pspec = workloads.WORKLOADS[args.prefill_workload]
        int8_peak = int8_peak_probe() if pspec["T"] >= 64 else None
        pf, pclocks = measure(args.prefill_workload, args, world, use_graph, args.prefill_steps, int8_peak)
        prefill = {"workload": args.prefill_workload, **{k: pf[k] for k in
                   ("metric", "value", "unit", "steps", "ms_per_step", "config", "roofline", "e2e", "gpu_launches")},
                   "clocks": pclocks, "int8_peak_measured_tops": int8_peak}

    attention = measure_attention(args.attention, 200, 20) if args.attention != "none" else None

    cpu = None
    if rank == 0 and world == 1:
        cpu = oracle_sample(args.workload, args.seed, args.cpu_seconds, single_thread_seconds=args.cpu_seconds / 2)
        if prefill is not None:
            prefill["cpu_baseline"] = oracle_sample(args.prefill_workload, args.seed, args.cpu_seconds / 2,
                                                    single_thread_seconds=args.cpu_seconds / 4)

    if rank == 0:
        line = {
            "metric": main_fields["metric"], "value": main_fields["value"], "unit": main_fields["unit"],
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_fields["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": main_fields["config"],
            "roofline": main_fields["roofline"],
            "cpu_baseline": cpu,
            "e2e": main_fields["e2e"],
            "gpu_launches": main_fields["gpu_launches"],
            "clocks": clocks,
        }
        if prefill is not None:
            line["prefill"] = prefill
        if attention is not None:
            line["attention"] = attention
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
