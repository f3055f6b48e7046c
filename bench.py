#!/usr/bin/env python
"""Benchmark of the sparse ternary BitLinear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--tokens T] [--layers L] [--no-rows] [--preroll-s S]

Default workload (the decode GEMV configuration): a 2B LLaMA-alike model
(hidden 2560, FFN 6912, 30 layers) in 2:4 ternary packed form; one step is
one decode pass of a batch of T tokens through every layer: for each of the
four projections (QKV 2560->3840, O 2560->2560, gate|up 2560->13824, down
6912->2560) the per-token int8 quantisation and the sparse ternary GEMV.
The 30 layers hold 521 MB of packed weights, more than 4x the 126 MB L2, so
every step streams its weights from HBM.  value = algorithmic bytes / time
(GB/s).  The same JSON line also carries sub-measurements of the other rows
of the hot path: the tensor-core prefill GEMM (effective TOPS), the per-step
mask + ternarise + pack over a 3B model (GB/s, mask flip rate), the int8
activation quantisation and the STE input gradient.

Under torchrun every rank runs the same workload on its own GPU (the layers
are independent: no data-path collective, weak scaling); the timed region is
bracketed by a barrier and a device synchronisation and the maximum over
ranks is reported.

--impl reference times the CPU oracle (oracle/, plain C) on the host cores on
a bounded sample of the same workload (one layer per step).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse ternary BitLinear effective TOPS (prefill) and decode GEMV HBM GB/s, 1×B200"
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--preroll-s", type=float, default=1.0, help="untimed warm-up seconds before timing")
    ap.add_argument("--tokens", type=int, default=1, help="decode batch (1..8)")
    ap.add_argument("--layers", type=int, default=30)
    ap.add_argument("--decode", choices=["chain_independent", "chain", "fused", "unfused"], default="chain_independent",
                    help="decode step: one persistent launch for all projections, independent of each other "
                         "(chain_independent) or each waiting for the previous one (chain); one fused quant+GEMV "
                         "launch per projection (fused); or quant_act + GEMV per projection (unfused)")
    ap.add_argument("--no-rows", action="store_true", help="skip the sub-measurements of the other rows")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline")
    ap.add_argument("--pack-layers", type=int, default=None, help="layers of the pack workload (default: all 26)")
    ap.add_argument("--flip-steps", type=int, default=100, help="random-walk steps of the mask flip-rate study")
    ap.add_argument("--only", choices=["prefill", "pack", "dgrad", "peaks", "six_eight", "block", "optimizer",
                                       "decode_rows", "oracle"], default=None,
                    help="run one sub-measurement alone and print it (for profiling)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, interval_ms: int = 100):
        self.idx = device_index
        self.interval = interval_ms
        self.proc = None
        self.path = None

    def _bus_id(self):
        try:
            import torch
            p = torch.cuda.get_device_properties(self.idx)
            return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        except Exception:
            return str(self.idx)

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._bus_id(), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={self.interval}"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def stop(self):
        rows = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.out.close()
            with open(self.path) as f:
                for line in f:
                    parts = [x.strip() for x in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        if self.path and os.path.exists(self.path):
            os.unlink(self.path)
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ helpers

def source_sha(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sparse_linear_layers_bitnet_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, src_files):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of the kernel; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel]
        if e.get("source_sha") != source_sha(*src_files):
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


class Timer:
    def __init__(self, torch, stream=None):
        self.torch = torch
        self.stream = stream

    def __enter__(self):
        t = self.torch
        self.e0 = t.cuda.Event(enable_timing=True)
        self.e1 = t.cuda.Event(enable_timing=True)
        self.e0.record(self.stream)
        return self

    def __exit__(self, *a):
        self.e1.record(self.stream)

    def ms(self):
        self.e1.synchronize()
        return self.e0.elapsed_time(self.e1)


class Nvtx:
    """NVTX range around a phase of the run, for timeline profilers (host-side marks only)."""

    def __init__(self, torch, name):
        self.torch, self.name = torch, name

    def __enter__(self):
        self.torch.cuda.nvtx.range_push(self.name)
        return self

    def __exit__(self, *a):
        self.torch.cuda.nvtx.range_pop()


FLUSH_NOTE = "flushed before every timed launch: 256 MB written, then another 256 MB read"


def make_flush(torch, dev):
    """Two 256 MB halves for flush_l2."""
    return torch.empty(2 * 256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)


def flush_l2(torch, buf):
    """Evict the 126 MB L2: write one 256 MB half, then read the other.  The read
    leaves L2 holding clean lines of an unrelated buffer, so the timed kernel
    finds none of its inputs in L2 and does not pay for writing back the
    flush's own dirty lines either."""
    half = buf.numel() // 2
    buf[:half].add_(1)
    buf[half:].amax()


# ------------------------------------------------------------------ decode workload

def decode_shapes():
    from sparse_linear_layers_bitnet_b200 import synth
    return synth.DECODE_2B_MATRICES


def decode_bytes(T, K, N):
    """Algorithmic bytes of one projection: quantisation (bf16 in, int8 + absmax
    out) and GEMV (packed weights 0.25 B each, int8 in, gamma, absmax, bf16 out)."""
    quant = T * K * 2 + T * K + 4 * T
    gemv = N * K // 4 + T * K + 4 * T + 4 + T * N * 2
    return quant, gemv


def decode_bytes_fused(T, K, N):
    """Algorithmic bytes of one fused projection: bf16 activations in, packed
    weights (0.25 B each), gamma, bf16 outputs."""
    return 2 * T * K + N * K // 4 + 4 + 2 * T * N


class Decode:
    def __init__(self, torch, bn, synth, T, layers, seed_base=0, mode="chain"):
        self.torch, self.bn, self.T, self.L, self.mode = torch, bn, T, layers, mode
        fused = mode in ("chain", "chain_independent", "fused")
        self.fused = fused
        dev = torch.device("cuda", torch.cuda.current_device())
        self.mats = decode_shapes()
        self.packed = []
        ws = bn.Workspace(bn.load().bitnet_pack_workspace_size(1, 1), dev)
        for l in range(layers):
            row = []
            for j, (name, K, N) in enumerate(self.mats):
                W = synth.torch_master_weights(N, K, 0.02, seed=seed_base + 1000 * l + j, device=dev)
                pw = bn.PackedWeights(N, K, dev, group_bytes=True, mma=False, dec=True)
                bn.bitnet_pack_nm(W, pw, 1e-5, ws=ws)
                del W
                pw.group_bytes = None   # the GEMV reads the decode layout only
                row.append(pw)
            self.packed.append(row)
        torch.cuda.synchronize()
        # inputs / outputs of every projection of every layer, in flat buffers
        xs = [T * K for _, K, _ in self.mats] * layers
        ys = [T * N for _, _, N in self.mats] * layers
        self.x_flat = synth.torch_activations(1, sum(xs), seed=seed_base + 7, dtype=torch.bfloat16,
                                              device=dev).view(-1)
        self.y_flat = torch.empty(sum(ys), dtype=torch.bfloat16, device=dev)
        self.x_views, self.y_views = [], []
        ox = oy = 0
        for l in range(layers):
            rx, ry = [], []
            for _, K, N in self.mats:
                rx.append(self.x_flat[ox:ox + T * K].view(T, K))
                ry.append(self.y_flat[oy:oy + T * N].view(T, N))
                ox += T * K
                oy += T * N
            self.x_views.append(rx)
            self.y_views.append(ry)
        self.xq = [torch.empty((T, K), dtype=torch.int8, device=dev) for _, K, _ in self.mats]
        self.amax = [torch.empty((T,), dtype=torch.float32, device=dev) for _ in self.mats]
        self.ws = bn.Workspace(max(bn.load().bitnet_linear_workspace_size(),
                                   max(bn.load().bitnet_quant_linear_workspace_size(T, K) for _, K, _ in self.mats)),
                               dev)
        q, g = 0, 0
        for _, K, N in self.mats:
            a, b = decode_bytes(T, K, N)
            q += a
            g += b
        self.quant_bytes_per_layer, self.gemv_bytes_per_layer = q, g
        self.fused_bytes_per_layer = sum(decode_bytes_fused(T, K, N) for _, K, N in self.mats)
        self.step_bytes = (self.fused_bytes_per_layer if fused else q + g) * layers
        self.weight_bytes = sum(N * K // 4 for _, K, N in self.mats) * layers
        self.launches_per_step = (1 if fused else 2) * len(self.mats) * layers
        self.chain = None
        if mode in ("chain", "chain_independent"):
            # chain: the decode pass, every projection waits for the previous one;
            # chain_independent: the same projections without the waits (each has its own input)
            wait = 1 if mode == "chain" else 0
            ops = [dict(X=self.x_views[l][j], W=self.packed[l][j], Y=self.y_views[l][j], wait_prev=wait)
                   for l in range(layers) for j in range(len(self.mats))]
            self.chain = bn.DecodeChain(ops, torch.bfloat16, torch.bfloat16, 1e-5, dev)
            self.launches_per_step = (len(ops) + 127) // 128

    def step(self):
        bn = self.bn
        if self.chain is not None:
            self.chain()
            return
        for l in range(self.L):
            for j in range(len(self.mats)):
                if self.fused:
                    bn.bitnet_quant_linear(self.x_views[l][j], self.packed[l][j], 1e-5, Y=self.y_views[l][j],
                                           ws=self.ws)
                else:
                    bn.bitnet_quant_act(self.x_views[l][j], 1e-5, Xq=self.xq[j], absmax=self.amax[j])
                    bn.bitnet_sparse_linear(self.xq[j], self.amax[j], self.packed[l][j], Y=self.y_views[l][j],
                                            ws=self.ws)

    def gemv_only(self):
        bn = self.bn
        for l in range(self.L):
            for j in range(len(self.mats)):
                bn.bitnet_sparse_linear(self.xq[j], self.amax[j], self.packed[l][j], Y=self.y_views[l][j],
                                        ws=self.ws)

    def capture(self, fn):
        torch = self.torch
        fn()   # first calls outside capture (function attributes, lazy init)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        return g


# ------------------------------------------------------------------ sub-measurements

def measure_prefill(torch, bn, synth, peaks, reps=10):
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = make_flush(torch, dev)
    out = {}
    tot_ops, tot_ms, tot_q_ms = 0.0, 0.0, 0.0
    for name, T, K, N in synth.PREFILL_7B_GEMMS:
        W = synth.torch_master_weights(N, K, 0.02, seed=11, device=dev)
        pw = bn.PackedWeights(N, K, dev, group_bytes=False, mma=True, dec=False)
        bn.bitnet_pack_nm(W, pw, 1e-5)
        del W
        X = synth.torch_activations(T, K, seed=12, outlier_p=0.01, dtype=torch.bfloat16, device=dev)
        Xq = torch.empty((T, K), dtype=torch.int8, device=dev)
        a = torch.empty((T,), dtype=torch.float32, device=dev)
        Y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        ws = bn.Workspace(256, dev)
        for _ in range(3):
            bn.bitnet_quant_act(X, 1e-5, Xq=Xq, absmax=a)
            bn.bitnet_sparse_linear(Xq, a, pw, Y=Y, ws=ws)
        gemm_ms, q_ms = [], []
        for _ in range(reps):
            flush_l2(torch, flush)
            with Timer(torch) as tq:
                bn.bitnet_quant_act(X, 1e-5, Xq=Xq, absmax=a)
            flush_l2(torch, flush)
            with Timer(torch) as tg:
                bn.bitnet_sparse_linear(Xq, a, pw, Y=Y, ws=ws)
            gemm_ms.append(tg.ms())
            q_ms.append(tq.ms())
        ms = statistics.mean(gemm_ms)
        ops = 2.0 * T * K * N
        out[name] = {"T": T, "K": K, "N": N, "gemm_ms": round(ms, 4), "quant_ms": round(statistics.mean(q_ms), 4),
                     "tops": round(ops / ms / 1e9, 1)}
        tot_ops += ops
        tot_ms += ms
        tot_q_ms += statistics.mean(q_ms)
        del pw, X, Xq, Y
    tops = tot_ops / tot_ms / 1e9
    sparse_peak = peaks["bf16"] * 2 * 2   # int8 = 2x bf16 (nominal 4.5 / 2.25 POPS), 2:4 sparse = 2x dense
    out["combined"] = {"tops": round(tops, 1), "tops_incl_quant": round(tot_ops / (tot_ms + tot_q_ms) / 1e9, 1),
                       "frac_of_sparse_int8_peak": round(tops / sparse_peak, 4),
                       "sparse_int8_peak_tops": round(sparse_peak, 1),
                       "frac_of_dense_int8_peak": round(tops / (sparse_peak / 2), 4),
                       "peak_note": f"{peaks['source']} bf16 burst x 2 (int8/bf16 nominal) x 2 (2:4)",
                       "l2": FLUSH_NOTE}
    del flush
    torch.cuda.empty_cache()
    return out


def measure_library_peaks(torch, n=8192, reps=10):
    """Dense int8 (cuBLASLt via torch._int_mm) and bf16 (cuBLAS) GEMM throughput
    on this GPU, run only: the measured denominators for the tensor-core rows
    (MEASURED_PEAKS.json carries no int8 figure)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    out = {}
    a8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
    b8 = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev).t()   # column-major operand
    for _ in range(3):
        torch._int_mm(a8, b8)
    ts = []
    for _ in range(reps):
        with Timer(torch) as t:
            torch._int_mm(a8, b8)
        ts.append(t.ms())
    out["int8_dense_tops"] = round(2.0 * n ** 3 / min(ts) / 1e9, 1)
    del a8, b8
    a = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    b = torch.randn((n, n), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        a @ b
    ts = []
    for _ in range(reps):
        with Timer(torch) as t:
            a @ b
        ts.append(t.ms())
    out["bf16_dense_tflops"] = round(2.0 * n ** 3 / min(ts) / 1e9, 1)
    out["how"] = f"{n}^3, best of {reps}, CUDA events; int8: torch._int_mm (cuBLASLt), bf16: torch.matmul"
    del a, b
    torch.cuda.empty_cache()
    return out


def measure_mma_ceilings(torch, bn, secs=1.0, iters=20000):
    """Ceiling of each tensor-core instruction form the GEMMs issue, on this GPU:
    bitnet_tensor_peak (MMAs back to back on operands resident in shared memory,
    no loads, no epilogue), launches timed with CUDA events for about `secs`,
    SM clocks sampled meanwhile.  Dense-equivalent rates (2 M N K per MMA)."""
    dev_index = torch.cuda.current_device()
    dev = torch.device("cuda", dev_index)
    ws = bn.Workspace(bn.load().bitnet_linear_workspace_size(), dev)
    out = {}
    forms = ((0, "sparse_i8_mma_loop_tops", "tcgen05.mma.sp.cta_group::2.kind::i8 M256 N224 K64"),
             (1, "dense_i8_mma_loop_tops", "tcgen05.mma.cta_group::2.kind::i8 M256 N256 K32"),
             (2, "bf16_mma_loop_tflops", "tcgen05.mma.cta_group::2.kind::f16 (bf16) M256 N256 K16"),
             (3, "sparse_i8_mma_loop_meta_copy_tops", "as the sparse loop, with each stage's metadata copied into "
                                                     "TMEM (tcgen05.cp) right before its two MMAs, two slots"),
             (4, "sparse_i8_mma_loop_meta_ahead_tops", "as the sparse loop, with each metadata copy issued four "
                                                      "stages ahead of its MMAs, eight slots"))
    for kind, name, form in forms:
        for _ in range(3):
            bn.bitnet_tensor_peak(kind, iters, ws)
        torch.cuda.synchronize()
        ck = ClockSampler(dev_index).start()
        ts, ops = [], 0.0
        t_end = time.time() + secs
        while time.time() < t_end:
            with Timer(torch) as t:
                ops = bn.bitnet_tensor_peak(kind, iters, ws)
            ts.append(t.ms())
        c = ck.stop()
        status = bn.bitnet_read_device_status(ws)
        med = ops / (statistics.median(ts) / 1e3) / 1e12
        out[name] = round(ops / (min(ts) / 1e3) / 1e12, 1)
        out[name + "_median"] = round(med, 1)
        out[name + "_per_sm_mhz"] = round(med / c["sm_mhz"], 4) if c.get("sm_mhz") else None
        out[name + "_clocks"] = c
        out[name + "_form"] = f"{form}; {iters} MMAs per CTA pair per launch, {len(ts)} launches, status {status}"
    del ws
    return out


def popcount_u8(torch, x):
    lut = torch.tensor([bin(i).count("1") for i in range(256)], dtype=torch.int64, device=x.device)
    return lut[x.long()].sum().item()


def measure_pack(torch, bn, synth, peaks, steps=3, flip_steps=100, layers=None):
    """Per-step pack over every linear weight of a 3B LLaMA-alike (26 layers)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    layers = layers or synth.LLAMA_3B["layers"]
    mats = synth.LAYER_3B_MATRICES
    Ws, pws = [], []
    for l in range(layers):
        for j, (name, N, K) in enumerate(mats):
            Ws.append(synth.torch_master_weights(N, K, 0.02, seed=50000 + 10 * l + j, device=dev))
            pws.append(bn.PackedWeights(N, K, dev, group_bytes=True, mma=True, dec=False))
    ws = bn.Workspace(max(bn.load().bitnet_pack_update_workspace_size(N, K) for _, N, K in mats), dev)
    n_w = sum(N * K for _, N, K in mats) * layers
    alg_bytes = n_w * (4 + 0.25 + 0.5 + 0.125)   # read fp32, write group bytes, int8 values, metadata
    for W, pw in zip(Ws, pws):
        bn.bitnet_pack_nm(W, pw, 1e-5, ws=ws)
    batch = bn.PackBatch(list(zip(Ws, pws)), 1e-5, dev)
    torch.cuda.synchronize()
    ms, ms_single = [], []
    for s in range(steps):
        for i, W in enumerate(Ws):
            synth.torch_random_walk_(W, 1e-4, seed=s * 1000 + i)
        with Timer(torch) as t:
            batch()
        ms.append(t.ms())
    # the same step with one bitnet_pack_nm_update call per matrix, for comparison
    for s in range(steps):
        for i, W in enumerate(Ws):
            synth.torch_random_walk_(W, 1e-4, seed=(steps + s) * 1000 + i)
        with Timer(torch) as t:
            for W, pw in zip(Ws, pws):
                bn.bitnet_pack_nm_update(W, pw, 1e-5, ws=ws)
        ms_single.append(t.ms())
    # gamma known (as the optimiser step leaves it): every out.gamma is already exact for its W, so the
    # pack reads W once and forms no sum
    for W, pw in zip(Ws, pws):
        bn.bitnet_pack_nm(W, pw, 1e-5, ws=ws)
    batch_k = bn.PackBatch(list(zip(Ws, pws)), 1e-5, dev, gamma_known=True)
    batch_k()
    ms_k = []
    for s_ in range(steps):
        with Timer(torch) as t:
            batch_k()
        ms_k.append(t.ms())
    del batch_k
    # bf16 masters (the method keeps BF16 masters): same matrices rounded to bf16, 2 B/weight read
    Wb = [W.to(torch.bfloat16) for W in Ws]
    # the same output buffers: the gamma of the last fp32 step serves as the first hint
    batch_b = bn.PackBatch(list(zip(Wb, pws)), 1e-5, dev)
    batch_b()
    ms_b = []
    for s in range(steps):
        for i, W in enumerate(Wb):
            W.copy_((W.float() + torch.randn(W.shape, device=dev, generator=torch.Generator(device=dev).manual_seed(
                (2 * steps + s) * 1000 + i)) * 1e-4).to(torch.bfloat16))
        with Timer(torch) as t:
            batch_b()
        ms_b.append(t.ms())
    del batch_b, Wb
    step_ms = statistics.mean(ms)
    gbs = alg_bytes / step_ms / 1e6
    n_mats = len(Ws)
    out = {"weights": n_w, "step_ms": round(step_ms, 3), "gbs": round(gbs, 1),
           "frac_of_hbm": round(gbs / peaks["hbm"], 4),
           "alg_bytes_per_weight": 4.875, "launches_per_step": 2 * ((n_mats + 63) // 64),
           "entry": "bitnet_pack_nm_update_batch over all matrices (each previous gamma as hint; "
                    "bit-identical to bitnet_pack_nm)",
           "gamma_from_optimizer": {"step_ms": round(statistics.mean(ms_k), 3),
                                    "gbs": round(alg_bytes / statistics.mean(ms_k) / 1e6, 1),
                                    "frac_of_hbm": round(alg_bytes / statistics.mean(ms_k) / 1e6 / peaks["hbm"], 4),
                                    "entry": "bitnet_pack_nm_update_batch with gamma_known (one read of W, no sum)"},
           "bf16_masters": {"step_ms": round(statistics.mean(ms_b), 3),
                            "gbs": round(n_w * (2 + 0.875) / statistics.mean(ms_b) / 1e6, 1),
                            "alg_bytes_per_weight": 2.875},
           "per_matrix_calls": {"step_ms": round(statistics.mean(ms_single), 3),
                                "gbs": round(alg_bytes / statistics.mean(ms_single) / 1e6, 1),
                                "entry": "bitnet_pack_nm_update, one call per matrix"}}
    del batch
    if flip_steps <= 0:
        del Ws, pws
        torch.cuda.empty_cache()
        return out
    # mask flip rate over 100 random-walk steps of one layer
    del Ws[len(mats):]
    del pws
    torch.cuda.empty_cache()
    flips = {name: [] for name, _, _ in mats}
    prev = {}
    for s in range(flip_steps + 1):
        for j, (name, N, K) in enumerate(mats):
            W = Ws[j]
            if s > 0:
                synth.torch_random_walk_(W, 1e-4, seed=900000 + 100 * s + j)
            pw = bn.PackedWeights(N, K, dev, group_bytes=False, mma=False, dec=False)
            mask = torch.empty(N * K // 8, dtype=torch.uint8, device=dev)
            bn.bitnet_pack_nm(W, pw, 1e-5, mask_bits=mask, ws=ws)
            if s > 0:
                flips[name].append(popcount_u8(torch, torch.bitwise_xor(mask, prev[name])) / (N * K))
            prev[name] = mask
    fr = {name: statistics.mean(v) for name, v in flips.items()}
    out["mask_flip_rate_per_step"] = {"mean": float(statistics.mean(fr.values())),
                                      **{k: float(v) for k, v in fr.items()}}
    out["flip_rate_sample"] = f"layer 0, {flip_steps} steps of W += N(0, 1e-4)"
    del Ws
    torch.cuda.empty_cache()
    return out


def measure_6of8(torch, bn, synth, reps=10):
    """6:8 weights on the 2:4 tensor cores (window decomposition + activation
    lifting) on the 7B prefill shapes, against cuBLASLt dense int8 on the same
    T x K x N and against the 2:4 layer; plus the per-step 6:8 pack."""
    dev = torch.device("cuda", torch.cuda.current_device())
    flush = make_flush(torch, dev)
    out = {}
    t68 = t24 = tdn = tq = 0.0
    ops_all = 0.0
    for name, T, K, N in synth.PREFILL_7B_GEMMS:
        W = synth.torch_master_weights(N, K, 0.02, seed=21, device=dev)
        pw = bn.packed_6of8(N, K, dev, mma=True, dec=False)
        ws = bn.Workspace(bn.load().bitnet_pack_workspace_size(N, K), dev)
        bn.bitnet_pack_6of8_windows(W, pw, 1e-5, ws=ws)
        pk = []
        for _ in range(3):
            with Timer(torch) as t:
                bn.bitnet_pack_6of8_windows(W, pw, 1e-5, ws=ws)
            pk.append(t.ms())
        p24 = bn.PackedWeights(N, K, dev, group_bytes=False, mma=True, dec=False)
        bn.bitnet_pack_nm(W, p24, 1e-5)
        del W
        X = synth.torch_activations(T, K, seed=22, outlier_p=0.01, dtype=torch.bfloat16, device=dev)
        Xl, a = bn.bitnet_quant_act_lift_6of8(X, 1e-5)
        Xq, a2 = bn.bitnet_quant_act(X, 1e-5)
        Y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        lws = bn.Workspace(256, dev)
        Xi = torch.randint(-127, 128, (T, K), dtype=torch.int8, device=dev)
        Bi = torch.randint(-1, 2, (K, N), dtype=torch.int8, device=dev)
        for _ in range(3):
            bn.bitnet_sparse_linear(Xl, a, pw, Y=Y, ws=lws)
            bn.bitnet_sparse_linear(Xq, a2, p24, Y=Y, ws=lws)
            torch._int_mm(Xi, Bi)
        m68, m24, mdn, mq = [], [], [], []
        for _ in range(reps):
            flush_l2(torch, flush)
            with Timer(torch) as t:
                bn.bitnet_quant_act_lift_6of8(X, 1e-5, Xl=Xl, absmax=a)
            mq.append(t.ms())
            flush_l2(torch, flush)
            with Timer(torch) as t:
                bn.bitnet_sparse_linear(Xl, a, pw, Y=Y, ws=lws)
            m68.append(t.ms())
            flush_l2(torch, flush)
            with Timer(torch) as t:
                bn.bitnet_sparse_linear(Xq, a2, p24, Y=Y, ws=lws)
            m24.append(t.ms())
            flush_l2(torch, flush)
            with Timer(torch) as t:
                torch._int_mm(Xi, Bi)
            mdn.append(t.ms())
        ops = 2.0 * T * K * N
        a68, a24, adn, aq = (statistics.mean(v) for v in (m68, m24, mdn, mq))
        out[name] = {"T": T, "K": K, "N": N, "gemm_6of8_ms": round(a68, 4), "lift_quant_ms": round(aq, 4),
                     "gemm_2of4_ms": round(a24, 4), "cublas_dense_int8_ms": round(adn, 4),
                     "tops_6of8": round(ops / a68 / 1e9, 1), "speedup_vs_dense_int8": round(adn / a68, 3),
                     "pack_6of8_ms": round(statistics.mean(pk), 4),
                     "pack_6of8_gbs": round(N * K * (4 + 3 / 8 + 3 / 4 + 3 / 16) / statistics.mean(pk) / 1e6, 1)}
        t68 += a68
        t24 += a24
        tdn += adn
        tq += aq
        ops_all += ops
        del pw, p24, X, Xl, Xq, Y, Xi, Bi, ws
    out["combined"] = {"tops_6of8": round(ops_all / t68 / 1e9, 1), "speedup_vs_dense_int8": round(tdn / t68, 3),
                       "ratio_6of8_to_2of4_time": round(t68 / t24, 3),
                       "note": "6:8 runs as a 2:4 GEMM over K' = 1.5 K: its ceiling is (2:4 speed-up over dense) / 1.5; "
                               "tops_6of8 counts the 2 T K N dense-equivalent ops of the 6:8 layer",
                       "l2": FLUSH_NOTE}
    del flush
    torch.cuda.empty_cache()
    return out


def measure_dgrad(torch, bn, synth, peaks, reps=5):
    dev = torch.device("cuda", torch.cuda.current_device())
    T = 2048
    h, f = synth.LLAMA_3B["hidden"], synth.LLAMA_3B["ffn"]
    shapes = [("qkv", 3 * h, h), ("o", h, h), ("gate_up", 2 * f, h), ("down", h, f)]
    out, tot_f, tot_ms, tot_ms_c = {}, 0.0, 0.0, 0.0
    for name, N, K in shapes:
        W = synth.torch_master_weights(N, K, 0.02, seed=77, device=dev)
        pw = bn.PackedWeights(N, K, dev, group_bytes=True, mma=False, dec=False)
        bn.bitnet_pack_nm(W, pw, 1e-5)
        del W
        dY = synth.torch_activations(T, N, seed=78, dtype=torch.bfloat16, device=dev)
        dX = torch.empty((T, K), dtype=torch.bfloat16, device=dev)
        ws = bn.Workspace(bn.load().bitnet_dgrad_workspace_size(N, K), dev)
        for _ in range(2):
            bn.bitnet_dgrad(dY, pw, dX=dX, ws=ws)
        ts = []
        for _ in range(reps):
            with Timer(torch) as t:
                bn.bitnet_dgrad(dY, pw, dX=dX, ws=ws)
            ts.append(t.ms())
        ms = statistics.mean(ts)
        flops = 2.0 * T * N * K
        # context: cuBLAS (torch.matmul) bf16 on the same product shape with a dense bf16 B already in memory
        Bd = torch.randn((N, K), dtype=torch.bfloat16, device=dev)
        for _ in range(2):
            torch.matmul(dY, Bd)
        tc = []
        for _ in range(reps):
            with Timer(torch) as t:
                torch.matmul(dY, Bd)
            tc.append(t.ms())
        ms_c = statistics.mean(tc)
        out[name] = {"T": T, "n_out": N, "k": K, "ms": round(ms, 4), "tflops": round(flops / ms / 1e9, 1),
                     "cublas_same_shape_tflops": round(flops / ms_c / 1e9, 1)}
        tot_f += flops
        tot_ms += ms
        tot_ms_c = tot_ms_c + ms_c
        del pw, dY, dX, ws, Bd
    tf = tot_f / tot_ms / 1e9
    out["combined"] = {"tflops": round(tf, 1), "frac_of_bf16_peak": round(tf / peaks["bf16"], 4),
                       "cublas_same_shapes_tflops": round(tot_f / tot_ms_c / 1e9, 1),
                       "note": "includes the bf16 expansion of Wq from group bytes; cuBLAS is given the dense "
                               "bf16 operand ready in memory"}
    torch.cuda.empty_cache()
    return out


def measure_optimizer(torch, bn, synth, peaks, steps=3):
    """The AdamW step with the next gamma over every linear weight of the 3B
    model (26 layers x 7 matrices, 3.22 G fp32 masters): one batched call per
    step against one call per matrix.  28 algorithmic bytes per weight."""
    dev = torch.device("cuda", torch.cuda.current_device())
    layers = synth.LLAMA_3B["layers"]
    mats = synth.LAYER_3B_MATRICES
    Ws, Gs, Ms, Vs = [], [], [], []
    for l in range(layers):
        for j, (name, N, K) in enumerate(mats):
            Ws.append(synth.torch_master_weights(N, K, 0.02, seed=60000 + 10 * l + j, device=dev).reshape(-1))
            Gs.append(synth.torch_master_weights(N, K, 1e-3, seed=70000 + 10 * l + j, device=dev).reshape(-1))
            Ms.append(torch.zeros_like(Ws[-1]))
            Vs.append(torch.zeros_like(Ws[-1]))
    gam = torch.zeros(len(Ws), device=dev)
    n_w = sum(w.numel() for w in Ws)
    batch = bn.AdamWBatch([(Ws[i], Gs[i], Ms[i], Vs[i], gam[i:i + 1]) for i in range(len(Ws))], dev)
    ws1 = bn.Workspace(bn.load().bitnet_adamw_workspace_size(), dev)
    batch(1, lr=1e-4, weight_decay=0.1)
    ms_b, ms_s = [], []
    for st in range(2, 2 + steps):
        with Timer(torch) as t:
            batch(st, lr=1e-4, weight_decay=0.1)
        ms_b.append(t.ms())
    for st in range(2 + steps, 2 + 2 * steps):
        with Timer(torch) as t:
            for i in range(len(Ws)):
                bn.bitnet_adamw_step(Ws[i], Gs[i], Ms[i], Vs[i], st, lr=1e-4, weight_decay=0.1,
                                     gamma_out=gam[i:i + 1], ws=ws1)
        ms_s.append(t.ms())
    mb, msg = statistics.mean(ms_b), statistics.mean(ms_s)
    out = {"weights": n_w, "matrices": len(Ws), "alg_bytes_per_weight": 28,
           "batched": {"step_ms": round(mb, 3), "gbs": round(n_w * 28 / mb / 1e6, 1),
                       "frac_of_hbm": round(n_w * 28 / mb / 1e6 / peaks["hbm"], 4),
                       "entry": "bitnet_adamw_step_batch over all matrices"},
           "per_matrix_calls": {"step_ms": round(msg, 3), "gbs": round(n_w * 28 / msg / 1e6, 1),
                                "entry": "bitnet_adamw_step, one call per matrix"}}
    del batch, Ws, Gs, Ms, Vs
    torch.cuda.empty_cache()
    return out


def _graph(torch, fn):
    fn()   # first call outside capture (function attributes, lazy init)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def _time_graph(torch, g, flush, reps):
    ts = []
    for _ in range(reps):
        flush_l2(torch, flush)
        with Timer(torch) as t:
            g.replay()
        ts.append(t.ms())
    return statistics.median(ts)


def measure_block(torch, bn, synth, peaks, reps=10, T=2048):
    """One training step of a LLaMA-alike block at 3B shapes (hidden 3200, FFN
    8640, 32 heads) over T tokens, every BitLinear on the sparse ternary path:
    pack of the block's four matrices from fp32 masters (gamma known from the
    previous optimiser step: one read of W); forward RMSNorm+quant -> QKV ->
    causal attention -> quant -> O -> residual -> RMSNorm+quant -> gate|up ->
    SwiGLU+quant -> down -> residual; backward: STE dgrad and the dense weight
    gradient of the four matrices; AdamW on the masters, which also forms the
    next gamma.  dY and the weight-gradient inputs are synthetic bf16 tensors of
    the layer shapes.  Attention (torch SDPA) and the residual adds are library
    calls, timed and listed apart.  Each stage is one CUDA graph timed alone
    after an L2 flush; the whole step is one graph.  Context: the same step
    with dense bf16 weights through cuBLAS (torch.matmul), torch elementwise ops
    and torch's fused AdamW, without any pack."""
    F = torch.nn.functional
    dev = torch.device("cuda", torch.cuda.current_device())
    h, f, H = synth.LLAMA_3B["hidden"], synth.LLAMA_3B["ffn"], synth.LLAMA_3B["heads"]
    dh = h // H
    flush = make_flush(torch, dev)
    mats = [("qkv", 3 * h, h), ("o", h, h), ("gate_up", 2 * f, h), ("down", h, f)]
    lib = bn.load()
    masters, pw = {}, {}
    for i, (name, N, K) in enumerate(mats):
        masters[name] = synth.torch_master_weights(N, K, 0.02, seed=300 + i, device=dev)
        pw[name] = bn.PackedWeights(N, K, dev, group_bytes=True, mma=True, dec=False)
        bn.bitnet_pack_nm(masters[name], pw[name], 1e-5)   # first pack sets each gamma hint
    moments = {n: (torch.zeros_like(masters[n]), torch.zeros_like(masters[n])) for n, _, _ in mats}
    ws_wg = bn.Workspace(lib.bitnet_wgrad_workspace_size(), dev)
    # the optimiser leaves the exact gamma of the updated masters in pw.gamma: the pack reads W once
    batch = bn.PackBatch([(masters[n], pw[n]) for n, _, _ in mats], 1e-5, dev, gamma_known=True)
    ws_lin = bn.Workspace(lib.bitnet_linear_workspace_size(), dev)
    ws_dg = bn.Workspace(max(lib.bitnet_dgrad_workspace_size(N, K) for _, N, K in mats), dev)
    norm_w = (1.0 + 0.05 * torch.randn(h, device=dev)).float()
    x = synth.torch_activations(T, h, seed=310, dtype=torch.bfloat16, device=dev)
    bf = torch.bfloat16
    buf = {
        "xq1": torch.empty((T, h), dtype=torch.int8, device=dev), "a1": torch.empty(T, device=dev),
        "qkv": torch.empty((T, 3 * h), dtype=bf, device=dev), "att": torch.empty((T, h), dtype=bf, device=dev),
        "xq2": torch.empty((T, h), dtype=torch.int8, device=dev), "a2": torch.empty(T, device=dev),
        "o": torch.empty((T, h), dtype=bf, device=dev), "x1": torch.empty((T, h), dtype=bf, device=dev),
        "xq3": torch.empty((T, h), dtype=torch.int8, device=dev), "a3": torch.empty(T, device=dev),
        "gu": torch.empty((T, 2 * f), dtype=bf, device=dev),
        "xq4": torch.empty((T, f), dtype=torch.int8, device=dev), "a4": torch.empty(T, device=dev),
        "d": torch.empty((T, h), dtype=bf, device=dev), "x2": torch.empty((T, h), dtype=bf, device=dev),
    }
    dY = {n: synth.torch_activations(T, N, seed=320 + i, dtype=bf, device=dev) for i, (n, N, K) in enumerate(mats)}
    dX = {n: torch.empty((T, K), dtype=bf, device=dev) for n, N, K in mats}
    Xin = {n: synth.torch_activations(T, K, seed=330 + i, dtype=bf, device=dev) for i, (n, N, K) in enumerate(mats)}
    dWs = {n: torch.empty((N, K), dtype=torch.float32, device=dev) for n, N, K in mats}
    step_no = [1]
    b = buf

    def s_pack():
        batch()

    def s_norm1():
        bn.bitnet_rmsnorm_quant(x, norm_w, 1e-6, 1e-5, Xq=b["xq1"], absmax=b["a1"])

    def s_qkv():
        bn.bitnet_sparse_linear(b["xq1"], b["a1"], pw["qkv"], Y=b["qkv"], ws=ws_lin)

    def s_attn():
        q, k, v = b["qkv"].view(1, T, 3, H, dh).permute(2, 0, 3, 1, 4).unbind(0)
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        b["att"].copy_(o.transpose(1, 2).reshape(T, h))

    def s_o():
        bn.bitnet_quant_act(b["att"], 1e-5, Xq=b["xq2"], absmax=b["a2"])
        bn.bitnet_sparse_linear(b["xq2"], b["a2"], pw["o"], Y=b["o"], ws=ws_lin)

    def s_res1():
        torch.add(x, b["o"], out=b["x1"])

    def s_norm2():
        bn.bitnet_rmsnorm_quant(b["x1"], norm_w, 1e-6, 1e-5, Xq=b["xq3"], absmax=b["a3"])

    def s_gate_up():
        bn.bitnet_sparse_linear(b["xq3"], b["a3"], pw["gate_up"], Y=b["gu"], ws=ws_lin)

    def s_swiglu():
        bn.bitnet_swiglu_quant(b["gu"], f, 1e-5, Xq=b["xq4"], absmax=b["a4"])

    def s_down():
        bn.bitnet_sparse_linear(b["xq4"], b["a4"], pw["down"], Y=b["d"], ws=ws_lin)

    def s_res2():
        torch.add(b["x1"], b["d"], out=b["x2"])

    def s_dgrad():
        for n, _, _ in mats:
            bn.bitnet_dgrad(dY[n], pw[n], dX=dX[n], ws=ws_dg)

    def s_wgrad():
        for n, _, _ in mats:
            bn.bitnet_wgrad(dY[n], Xin[n], dW=dWs[n], ws=ws_wg)

    opt_batch = bn.AdamWBatch([(masters[n], dWs[n], moments[n][0], moments[n][1], pw[n].gamma) for n, _, _ in mats],
                              dev)

    def s_adamw():   # one launch for the block's four matrices
        opt_batch(step_no[0], lr=1e-4, weight_decay=0.1)

    s_wgrad()
    s_adamw()   # the first optimiser step sets every gamma the pack then takes as known

    stages = [("pack", s_pack, "ours"), ("rmsnorm_quant_1", s_norm1, "ours"), ("qkv", s_qkv, "ours"),
              ("attention", s_attn, "library"), ("quant_o", s_o, "ours"), ("residual_1", s_res1, "library"),
              ("rmsnorm_quant_2", s_norm2, "ours"), ("gate_up", s_gate_up, "ours"),
              ("swiglu_quant", s_swiglu, "ours"), ("down", s_down, "ours"), ("residual_2", s_res2, "library"),
              ("dgrad_4", s_dgrad, "ours"), ("wgrad_4", s_wgrad, "ours"), ("adamw_4", s_adamw, "ours")]
    out = {"T": T, "hidden": h, "ffn": f, "heads": H, "stages_ms": {}}
    for name, fn, who in stages:
        g = _graph(torch, fn)
        out["stages_ms"][name] = {"ms": round(_time_graph(torch, g, flush, reps), 4), "impl": who}
        del g

    def step():
        for _, fn, _ in stages:
            fn()

    g = _graph(torch, step)
    step_ms = _time_graph(torch, g, flush, reps)
    del g
    st = out["stages_ms"]
    ours_ms = sum(v["ms"] for v in st.values() if v["impl"] == "ours")
    fwd_ops = 2.0 * T * sum(N * K for _, N, K in mats)
    gemm_ms = sum(st[n]["ms"] for n in ("qkv", "gate_up", "down"))
    n_w = sum(N * K for _, N, K in mats)
    out.update({
        "step_ms": round(step_ms, 4),
        "ours_ms": round(ours_ms, 4),
        "library_ms": round(sum(v["ms"] for v in st.values() if v["impl"] == "library"), 4),
        "forward_gemm_ops": fwd_ops,
        "dgrad_tflops": round(fwd_ops / st["dgrad_4"]["ms"] / 1e9, 1),
        "wgrad_tflops": round(fwd_ops / st["wgrad_4"]["ms"] / 1e9, 1),
        "adamw_gbs": round(n_w * 28 / st["adamw_4"]["ms"] / 1e6, 1),   # W, g, m, v read; W, m, v written
        "pack_gbs": round(n_w * 4.875 / st["pack"]["ms"] / 1e6, 1),
        "qkv_gate_up_down_tops": round(2.0 * T * sum(N * K for n, N, K in mats if n != "o") / gemm_ms / 1e9, 1),
        "l2": FLUSH_NOTE,
    })

    # context: the same step with dense bf16 weights (cuBLAS through torch.matmul), torch ops and
    # torch's fused AdamW on fp32 masters
    Wd = {n: masters[n].to(bf) for n, _, _ in mats}
    del batch
    tb = {"x1": torch.empty((T, h), dtype=bf, device=dev)}
    params = [masters[n] for n, _, _ in mats]
    for pm, (n, _, _) in zip(params, mats):
        pm.grad = dWs[n]
    opt = torch.optim.AdamW(params, lr=1e-4, weight_decay=0.1, fused=True, capturable=True)
    opt.step()   # state allocated outside the graph

    def rms(v):
        vf = v.float()
        return (vf * torch.rsqrt(vf.pow(2).mean(-1, keepdim=True) + 1e-6) * norm_w).to(bf)

    def t_step():
        qkv = torch.matmul(rms(x), Wd["qkv"].t())
        q, k, v = qkv.view(1, T, 3, H, dh).permute(2, 0, 3, 1, 4).unbind(0)
        att = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(T, h)
        x1 = x + torch.matmul(att, Wd["o"].t())
        gu = torch.matmul(rms(x1), Wd["gate_up"].t())
        hh = F.silu(gu[:, :f]) * gu[:, f:]
        tb["x1"] = x1 + torch.matmul(hh, Wd["down"].t())
        for n, _, _ in mats:
            torch.matmul(dY[n], Wd[n])
            torch.matmul(dY[n].t(), Xin[n])
        opt.step()

    g = _graph(torch, t_step)
    out["torch_bf16_dense_step_ms"] = round(_time_graph(torch, g, flush, reps), 4)
    del g, Wd, opt, masters
    out["note"] = ("step = pack (known gamma) + forward + STE dgrad + weight gradient + AdamW of one block; the "
                   "bf16 context runs the same step without the pack, on dense bf16 weights already in memory, "
                   "with torch's fused AdamW")
    torch.cuda.empty_cache()
    return out
# ------------------------------------------------------------------ CPU oracle baseline

def oracle_decode_sample(T, target_s):
    """Time the oracle (as it stands) on one decode layer: quantise, integer
    product and dequantise for the four projections; repeat up to target_s."""
    import numpy as np

    import oracle
    from sparse_linear_layers_bitnet_b200 import synth
    mats = decode_shapes()
    prepared = []
    for j, (name, K, N) in enumerate(mats):
        W = synth.master_weights(N, K, 0.02, seed=j)
        g, keep, wq, gb = oracle.pack_weights(W, 1e-5)
        X = synth.bf16_bits_to_f32(synth.to_bf16_bits(synth.activations(T, K, seed=100 + j)))
        prepared.append((g, wq, X))
    bytes_layer = sum(sum(decode_bytes(T, K, N)) for _, K, N in mats)
    reps, t_total = 0, 0.0
    while t_total < target_s or reps == 0:
        t0 = time.perf_counter()
        for g, wq, X in prepared:
            xq, a = oracle.quant_act(X, 1e-5)
            acc = oracle.gemm_i32(xq, wq)
            oracle.dequant(acc, a, g)
        t_total += time.perf_counter() - t0
        reps += 1
    return bytes_layer, reps, t_total, oracle.max_threads(), prepared


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def measure_oracle(target_s=1.5):
    """The CPU oracle, as it stands, on bounded samples of every configuration,
    single-threaded and on all host cores (OpenMP): the reported CPU baseline.
    Units follow the GPU rows: ms per forward (config 1), GB/s of algorithmic
    bytes (configs 2 and 4), dense-equivalent TOPS (config 3), ms per block step
    extrapolated from a token sample (config 5)."""
    import numpy as np

    import oracle
    from sparse_linear_layers_bitnet_b200 import synth

    def timed(fn):
        reps, t = 0, 0.0
        while t < target_s or reps == 0:
            t0 = time.perf_counter()
            fn()
            t += time.perf_counter() - t0
            reps += 1
        return t / reps

    cores = oracle.max_threads()
    out = {"nproc": os.cpu_count(), "cpu_model": _cpu_model(), "omp_threads_all": cores}
    # inputs (built once, outside the timed regions)
    W1, X1 = synth.master_weights(256, 256, 0.02, seed=0), synth.activations(16, 256, seed=0)
    dec = []
    for j, (name, K, N) in enumerate(decode_shapes()):
        g, keep, wq, gb = oracle.pack_weights(synth.master_weights(N, K, 0.02, seed=j), 1e-5)
        dec.append((g, wq, synth.bf16_bits_to_f32(synth.to_bf16_bits(synth.activations(1, K, seed=100 + j)))))
    dec_bytes = sum(decode_bytes_fused(1, K, N) for _, K, N in decode_shapes())
    Ts = 8   # prefill token sample
    pre = []
    for name, T, K, N in synth.PREFILL_7B_GEMMS:
        g, keep, wq, gb = oracle.pack_weights(synth.master_weights(N, K, 0.02, seed=11), 1e-5)
        pre.append((g, wq, synth.activations(Ts, K, seed=12, outlier_p=0.01), K, N))
    Wp = synth.master_weights(3200, 3200, 0.02, seed=21)
    Tb = 4   # block token sample
    blk = []
    for name, K, N in (("qkv", 3200, 9600), ("o", 3200, 3200), ("gate_up", 3200, 17280), ("down", 8640, 3200)):
        g, keep, wq, gb = oracle.pack_weights(synth.master_weights(N, K, 0.02, seed=31), 1e-5)
        blk.append((g, wq, synth.activations(Tb, K, seed=32), synth.activations(Tb, N, seed=33), K, N))

    def c1():
        oracle.forward(W1, X1)

    def c2():
        for g, wq, X in dec:
            xq, a = oracle.quant_act(X, 1e-5)
            oracle.dequant(oracle.gemm_i32(xq, wq), a, g)

    def c3():
        for g, wq, X, K, N in pre:
            xq, a = oracle.quant_act(X, 1e-5)
            oracle.dequant(oracle.gemm_i32(xq, wq), a, g)

    def c4():
        oracle.pack_weights(Wp, 1e-5)

    def c5():
        for g, wq, X, dY, K, N in blk:
            xq, a = oracle.quant_act(X, 1e-5)
            oracle.dequant(oracle.gemm_i32(xq, wq), a, g)
            oracle.dgrad(dY, wq, g)

    pre_ops = sum(2.0 * Ts * K * N for _, _, _, K, N in pre)
    for threads in (1, cores):
        oracle.set_threads(threads)
        key = f"threads_{threads}"
        out[key] = {
            "config1_tiny_ms_per_forward": round(timed(c1) * 1e3, 4),
            "config2_decode_gbs": round(dec_bytes / timed(c2) / 1e9, 4),
            "config3_prefill_tops": round(pre_ops / timed(c3) / 1e12, 5),
            "config4_pack_gbs": round(Wp.size * 4.875 / timed(c4) / 1e9, 4),
            "config5_block_ms_per_step": round(timed(c5) * 2048 / Tb * 1e3, 1),
        }
    oracle.set_threads(cores)
    out["samples"] = ("config 1: one tiny forward (16 x 256 x 256); config 2: one 2B layer (4 projections) at "
                      "T = 1, bf16-valued activations; config 3: both 7B prefill GEMMs (quant, int32 product, "
                      f"dequant) on {Ts} of the 4096 tokens; config 4: pack of one 3200 x 3200 fp32 matrix "
                      f"(4.875 B per weight); config 5: forward and STE dgrad of the 3B block's four "
                      f"projections on {Tb} of 2048 tokens, scaled to 2048")
    return out


def run_reference(args):
    """--impl reference: the CPU oracle on the host cores (rank 0 only)."""
    from sparse_linear_layers_bitnet_b200 import dist
    info = dist.env_info()
    if info.rank != 0:
        return 0
    import oracle
    T = args.tokens
    cores = oracle.max_threads()
    bytes_layer, _, _, _, prepared = oracle_decode_sample(T, 0.0)

    def one_step():
        for g, wq, X in prepared:
            xq, a = oracle.quant_act(X, 1e-5)
            acc = oracle.gemm_i32(xq, wq)
            oracle.dequant(acc, a, g)

    for _ in range(args.warmup):
        one_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_step()
    dt = time.perf_counter() - t0
    value = bytes_layer * args.steps / dt / 1e9
    threads = cores
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": f"decode GEMV, 2B LLaMA-alike (hidden 2560, FFN 6912), {args.layers} layers, batch {T}",
                   "tokens": T, "layers": args.layers,
                   "step": "the CPU oracle (per projection: int8 act quant, int32 product, dequant) on the host "
                           "cores; each timed step is a bounded sample of one layer (QKV, O, gate|up, down), "
                           "GB/s counted on that layer's algorithmic bytes"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"one 2B layer per step, {args.steps} steps, T={T}"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main arm

def run_only(args):
    import torch

    import sparse_linear_layers_bitnet_b200 as bn
    from sparse_linear_layers_bitnet_b200 import synth
    bn.load()
    peaks = load_peaks()
    fn = {"prefill": measure_prefill, "pack": measure_pack, "dgrad": measure_dgrad,
          "peaks": lambda torch, bn, synth, peaks: {**measure_library_peaks(torch), **measure_mma_ceilings(torch, bn)},
          "decode_rows": lambda torch, bn, synth, peaks: measure_decode_rows(torch, bn, synth, args.layers),
          "oracle": lambda torch, bn, synth, peaks: measure_oracle(),
          "six_eight": lambda torch, bn, synth, peaks: measure_6of8(torch, bn, synth),
          "block": measure_block, "optimizer": measure_optimizer}[args.only]
    kw = {"steps": args.steps, "flip_steps": args.flip_steps, "layers": args.pack_layers} if args.only == "pack" else {}
    print(json.dumps({args.only: fn(torch, bn, synth, peaks, **kw)}), flush=True)
    return 0


def measure_decode_rows(torch, bn, synth, layers):
    """The decode step in its other forms: independent and dependent chains at
    T = 1, 4, 8, and the fused and unfused per-projection launches."""
    out = {}
    for t2, mode in ((1, "chain_independent"), (1, "chain"), (1, "unfused"), (1, "fused"), (4, "chain_independent"),
                     (4, "chain"), (4, "unfused"), (8, "chain_independent"), (8, "chain"), (8, "unfused")):
        d2 = Decode(torch, bn, synth, t2, layers, seed_base=31, mode=mode)
        g2 = d2.capture(d2.step)
        for _ in range(3):
            g2.replay()
        with Timer(torch) as t:
            for _ in range(10):
                g2.replay()
        per = t.ms() / 10
        out[f"T{t2}_{mode}"] = {"gbs": round(d2.step_bytes / (per / 1e3) / 1e9, 1), "ms_per_step": round(per, 4),
                                "launches_per_step": d2.launches_per_step}
        del g2, d2
        torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch

    import sparse_linear_layers_bitnet_b200 as bn
    from sparse_linear_layers_bitnet_b200 import dist, synth

    if args.only:
        return run_only(args)
    info = dist.init()
    torch.cuda.set_device(info.local_rank)
    bn.load()
    peaks = load_peaks()
    T = args.tokens
    assert 1 <= T <= 8, "decode batch must be 1..8"
    dev_index = torch.cuda.current_device()

    fused = args.decode in ("chain", "chain_independent", "fused")
    dec = Decode(torch, bn, synth, T, args.layers, seed_base=info.rank * 7919, mode=args.decode)
    g_step = dec.capture(dec.step)

    clocks = ClockSampler(dev_index).start()
    # pre-roll so that clocks settle (untimed, counted as warm-up)
    t_end = time.time() + args.preroll_s
    while time.time() < t_end:
        g_step.replay()
        torch.cuda.synchronize()
    for _ in range(max(args.warmup, 3)):
        g_step.replay()
    dist.barrier()
    torch.cuda.synchronize()
    with Nvtx(torch, "decode timed steps"), Timer(torch) as tm:
        for _ in range(args.steps):
            g_step.replay()
    torch.cuda.synchronize()
    dist.barrier()
    ms_total = tm.ms()
    ck = clocks.stop()
    ms_total = dist.max_over_ranks(ms_total, device=torch.device("cuda", dev_index))
    value = dec.step_bytes * args.steps * info.world / (ms_total / 1e3) / 1e9

    if fused:
        # every kernel launch of the step is the decode chain kernel: its average
        # launch duration is the timed region over the launches in it
        roof_kernel = "k_decode_chain_serial" if args.decode == "chain" else "k_decode_chain"
        gemv_ms_per_launch = ms_total / args.steps / dec.launches_per_step
        gemv_bytes_per_launch = dec.step_bytes / dec.launches_per_step
    else:
        # dominant kernel: the GEMV alone, replayed from a graph of the same
        # launches on the same stream
        roof_kernel = "k_gemv_dec"
        g_gemv = dec.capture(dec.gemv_only)
        for _ in range(3):
            g_gemv.replay()
        reps = max(args.steps, 10)
        with Timer(torch) as tk:
            for _ in range(reps):
                g_gemv.replay()
        gemv_ms_per_launch = tk.ms() / reps / (len(dec.mats) * dec.L)
        gemv_bytes_per_launch = dec.gemv_bytes_per_layer / len(dec.mats)
        del g_gemv
    achieved = gemv_bytes_per_launch / (gemv_ms_per_launch / 1e3) / 1e9
    traffic = ncu_traffic(roof_kernel, {"k_decode_chain": ["chain.cu", "frag.cuh"],
                                        "k_decode_chain_serial": ["chain_serial.cu", "frag.cuh"]}.get(
                                            roof_kernel, ["gemv.cu", "frag.cuh"]))

    # end to end: activations from pinned host memory, outputs back to host
    x_host = torch.empty(dec.x_flat.shape, dtype=dec.x_flat.dtype, pin_memory=True)
    x_host.copy_(dec.x_flat)
    y_host = torch.empty(dec.y_flat.shape, dtype=dec.y_flat.dtype, pin_memory=True)
    for _ in range(3):
        dec.x_flat.copy_(x_host, non_blocking=True)
        g_step.replay()
        y_host.copy_(dec.y_flat, non_blocking=True)
    torch.cuda.synchronize()
    dist.barrier()
    with Nvtx(torch, "decode e2e steps"), Timer(torch) as te:
        for _ in range(args.steps):
            dec.x_flat.copy_(x_host, non_blocking=True)
            g_step.replay()
            y_host.copy_(dec.y_flat, non_blocking=True)
    torch.cuda.synchronize()
    e2e_ms = dist.max_over_ranks(te.ms(), device=torch.device("cuda", dev_index))
    e2e_value = dec.step_bytes * args.steps * info.world / (e2e_ms / 1e3) / 1e9

    rows = {}
    if not args.no_rows and info.world == 1:
        rows["decode_batches"] = measure_decode_rows(torch, bn, synth, args.layers)
        with Nvtx(torch, "row library_peaks"):
            rows["library_peaks"] = measure_library_peaks(torch)
            rows["library_peaks"].update(measure_mma_ceilings(torch, bn))
        with Nvtx(torch, "row prefill_gemm"):
            rows["prefill_gemm"] = measure_prefill(torch, bn, synth, peaks)
        lp = rows["library_peaks"]["int8_dense_tops"]
        pc = rows["prefill_gemm"]["combined"]
        pc["frac_of_2x_measured_int8_dense"] = round(pc["tops"] / (2 * lp), 4)
        pc["frac_of_measured_int8_dense"] = round(pc["tops"] / lp, 4)
        sp = rows["library_peaks"]["sparse_i8_mma_loop_tops_median"]
        pc["frac_of_measured_sparse_i8_mma_loop"] = round(pc["tops"] / sp, 4)
        with Nvtx(torch, "row dgrad"):
            rows["dgrad"] = measure_dgrad(torch, bn, synth, peaks)
        with Nvtx(torch, "row six_eight"):
            rows["six_eight"] = measure_6of8(torch, bn, synth)
        with Nvtx(torch, "row block"):
            rows["block"] = measure_block(torch, bn, synth, peaks)
        with Nvtx(torch, "row pack"):
            rows["pack"] = measure_pack(torch, bn, synth, peaks, flip_steps=args.flip_steps)
        with Nvtx(torch, "row optimizer"):
            rows["optimizer"] = measure_optimizer(torch, bn, synth, peaks)
        rows["oracle"] = measure_oracle()

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": info.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_total / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": f"decode GEMV, 2B LLaMA-alike (hidden 2560, FFN 6912), {args.layers} layers, batch {T}",
                   "tokens": T, "layers": args.layers,
                   "projections": [f"{n} {K}->{N}" for n, K, N in dec.mats],
                   "step": {"chain_independent": "all projections of all layers in one persistent launch "
                                                 "(bitnet_decode_chain, no projection waiting for another: per "
                                                 "projection, int8 act quant + sparse ternary GEMV, each on its own "
                                                 "synthetic activations), CUDA graph",
                            "chain": "all projections of all layers in one persistent launch "
                                     "(bitnet_decode_chain: per projection, int8 act quant + sparse ternary GEMV; "
                                     "each projection waits for the previous one), CUDA graph",
                            "fused": "per layer and projection: one fused launch (bitnet_quant_linear), CUDA graph",
                            "unfused": "per layer and projection: int8 act quant (bitnet_quant_act) + sparse "
                                       "ternary GEMV (bitnet_sparse_linear), programmatic dependent launch, "
                                       "CUDA graph"}[args.decode],
                   "l2": f"inputs larger than L2: {dec.weight_bytes / 1e6:.0f} MB of packed weights per step",
                   "parallelism": f"replicas x{info.world} (independent layers, no collective)"},
        "roofline": {"bound": "hbm", "kernel": roof_kernel, "achieved": round(achieved, 1),
                     "peak": peaks["hbm"], "unit": "GB/s", "frac": round(achieved / peaks["hbm"], 4),
                     "traffic": traffic, "peak_source": peaks["source"],
                     "alg_bytes_per_launch": gemv_bytes_per_launch,
                     "ms_per_launch": round(gemv_ms_per_launch, 5)},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s",
                "h2d_bytes_per_step": int(dec.x_flat.numel() * 2), "d2h_bytes_per_step": int(dec.y_flat.numel() * 2)},
        "gpu_launches": dec.launches_per_step * args.steps,
        "clocks": ck,
    }
    if info.rank == 0 and info.world == 1:
        import oracle
        cores = oracle.max_threads()
        oracle.set_threads(1)
        b1, reps1, secs1, _, _ = oracle_decode_sample(T, args.cpu_seconds / 2)
        oracle.set_threads(cores)
        b, reps, secs, _, _ = oracle_decode_sample(T, args.cpu_seconds / 2)
        line["cpu_baseline"] = {"value": round(b * reps / secs / 1e9, 4), "unit": "GB/s", "cores": cores,
                                "kind": "oracle", "value_1_thread": round(b1 * reps1 / secs1 / 1e9, 4),
                                "cpu_model": _cpu_model(), "nproc": os.cpu_count(),
                                "sample": f"{reps} passes over one 2B layer (4 projections), T={T}, {secs:.1f} s on "
                                          f"{cores} threads (OpenMP over outputs); {reps1} passes, {secs1:.1f} s "
                                          f"on 1 thread"}
    if rows:
        line["rows"] = rows
    if info.rank == 0:
        print(json.dumps(line), flush=True)
    del g_step
    dist.finalize()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
