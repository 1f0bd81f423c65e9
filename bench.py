"""Benchmark of the W4A16 decode path on B200.

Default workload (one "step"): the W4A16 products of a Llama-3-8B decode
step at batch 1 -- q, k, v, o, gate, up, down of 32 distinct decoder layers
(224 packed INT4 matrices, symmetric, group 128, 3.6 GB of codes + scales, so
no step finds its weights in the 126 MB L2).  Weights are random N(0, 0.02^2)
fp16 generated on the device from seeds, quantized with q4_quantize_pack and
the fp16 copies freed; activations are bf16 N(0, 1).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload llama3-8b | llama3-70b-stack [--batch B]]
                    [--layers L] [--no-sweep] [--no-cpu-baseline]

Single operations for profiling: --workload q4-70b-down [--batch B]
[--group-size G] [--asym], w8a16-70b, nvfp4-70b-down, mxfp4-70b-down,
kv8-70b-32k.

A step launches, per layer, q/k/v as one q4_gemv_grouped call, o, gate/up as
one grouped call and down (4 launches; the 7-launch form is reported beside
it as ``ungrouped``).  The default run also reports the INT4/bf16 batch
sweep, act order, the fused layout, W8A16, the KV-cache and FP4 quantizers,
the W4A4 FP4 product against batch, and the Llama-3-70B decode stack (80
layers, asymmetric group 64) at B = 1 and 8.

Prints one JSON line (rank 0).  ``value`` is the aggregate HBM throughput of
the INT4 products (algorithmic bytes / device time, CUDA events, max over
ranks); ``us_per_layer`` the time of one decoder layer's seven products.
With --gpus N > 1 (launched by torchrun) every rank runs its own independent
replica of the workload (weak scaling, no collective in the timed region).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 GEMV µs/layer + HBM GB/s (% of B200 peak) at B=1; INT4/bf16 speedup vs B"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of q4_gemv_sk_kernel per algorithmic byte, from the ncu
# capture of the four launches of one Llama-3-8B layer as the step launches
# them (q/k/v grouped, o, gate/up grouped, down): dram__bytes_read.sum +
# dram__bytes_write.sum = 112.70 MB against 112.62 MB of algorithmic bytes
# (q/k/v, o and down with the cluster fix-up, gate/up on the whole-tile
# grid).  Scaled to the step's average launch; it must be re-taken whenever
# the kernel or its launch plan changes.
GEMV_TRAFFIC_RATIO = 112.698368 / 112.623616
GEMV_TRAFFIC_SOURCE = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum on the 4 "
                       "launches of one B=1 layer "
                       "(profiles/q4_gemv_sk_llama3_8b_layer_grouped_full.txt)")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def algo_bytes(out, inn, g, B, sym=True):
    """Bytes a W4A16 product must move: codes + scales (+ zeros) + x + y."""
    meta = out * (inn // g) * 2 * (1 if sym else 2)
    return out * inn // 2 + meta + B * inn * 2 + B * out * 2


def dense_bytes(out, inn, B):
    return out * inn * 2 + B * inn * 2 + B * out * 2


def fp4_bytes(out, inn, fmt, B):
    """Algorithmic bytes of one W4A4 product: FP4 codes and scale bytes of W
    and x, y in bf16 (the NVFP4 tensor scales are 8 bytes and left out)."""
    blk = 32 if fmt == "mxfp4" else 16
    return (out + B) * (inn // 2 + inn // blk) + B * out * 2


def quant_bytes(out, inn, g, sym=True):
    return out * inn * 2 + out * inn // 2 + out * (inn // g) * 2 * (1 if sym else 2)


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during a region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- workload
def build_llama3_8b(q4, wl, torch, layers, rank, B, device):
    """Quantized weights of `layers` distinct Llama-3-8B layers (sym g128);
    each rank's replica draws its own layers."""
    from post_weight_quantization_group_b200.replicas import replica_layer
    mats = []
    for layer in range(layers):
        seeds = wl.llama3_8b_layer_seeds(replica_layer(layer, rank))
        for name, (out, inn) in wl.LLAMA3_8B.items():
            W = wl.normal_weight(out, inn, seeds[name], device=device)
            mats.append((name, q4.q4_quantize_pack(W, 128, True)))
            del W
    xs = {inn: wl.activations(B, inn, 17 + inn, device=device)
          for inn in sorted({i for _, i in wl.LLAMA3_8B.values()})}
    ys = {name: torch.empty(B, out, dtype=torch.bfloat16, device=device)
          for name, (out, _) in wl.LLAMA3_8B.items()}
    torch.cuda.synchronize()
    return mats, xs, ys


def layer_plan(mats, xs, ys):
    """Launch plan of a decode step over `mats` (7 linears per layer in
    q,k,v,o,gate,up,down order): q/k/v in one grouped call, o, gate/up in one
    grouped call, down -- 4 launches per layer."""
    plan = []
    for l in range(0, len(mats), 7):
        m = dict(mats[l:l + 7])
        for names in (("q_proj", "k_proj", "v_proj"), ("o_proj",), ("gate_proj", "up_proj"),
                      ("down_proj",)):
            ws_ = [m[n] for n in names]
            plan.append((ws_, [ys[n] for n in names], xs[ws_[0].in_features]))
    return plan


def run_plan(q4, plan, wsp):
    for ws_, ys_, x in plan:
        if len(ws_) > 1:
            q4.q4_gemv_grouped(ws_, x, ys=ys_, workspace=wsp)
        else:
            q4.q4_gemm_skinny(ws_[0], x, y=ys_[0], workspace=wsp)


def time_region(torch, fn, steps, warmup, stream):
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)  # ms


def graph_time_us(torch, fn, n, stream):
    """Mean device time of one call of fn(i) over n calls captured in a CUDA
    graph (CUDA events on the launching stream, 2 warm-up replays)."""
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        for i in range(n):
            fn(i)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ms = time_region(torch, g.replay, 3, 1, stream)
    del g
    return ms * 1e3 / (3 * n)


SWEEP_B = (1, 2, 4, 8, 16, 32, 64, 128)


def b_sweep(q4, wl, torch, device, stream):
    """INT4/bf16 speedup vs batch on the Llama-3-70B down_proj shape
    (8192 x 28672, N(0, 0.02^2), sym g128): q4_gemm_skinny against the faster
    of this library's bf16 product (bf16_gemv_ref_bw) and cuBLAS
    (torch.matmul), both reported.  Four INT4 and two bf16 copies rotate so
    no call finds its weights in L2."""
    out, inn = wl.LLAMA3_70B["down_proj"]
    ws = [q4.q4_quantize_pack(wl.normal_weight(out, inn, 30 + i, device=device), 128, True)
          for i in range(4)]
    Wb = [wl.normal_weight(out, inn, 40 + i, device=device).to(torch.bfloat16) for i in range(2)]
    torch.cuda.synchronize()
    rows = {}
    for B in SWEEP_B:
        x = wl.activations(B, inn, 31, device=device)
        y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
        wsp = q4.workspace_for(ws[0], B, device)
        t4 = graph_time_us(torch, lambda i: q4.q4_gemm_skinny(ws[i % 4], x, y=y, workspace=wsp), 16, stream)
        tb = graph_time_us(torch, lambda i: torch.matmul(x, Wb[i % 2].T, out=y), 16, stream)
        tr = graph_time_us(torch, lambda i: q4.bf16_gemv_ref_bw(Wb[i % 2], x, y=y), 16, stream)
        tbest = min(tb, tr)
        rows[B] = {"int4_us": round(t4, 2), "bf16_us": round(tbest, 2),
                   "speedup": round(tbest / t4, 3),
                   "int4_gbs": round(algo_bytes(out, inn, 128, B) / t4 / 1e3, 1),
                   "int4_tflops": round(2 * B * out * inn / t4 / 1e6, 1),
                   "bf16_impl": "bf16_gemv_ref_bw" if tr <= tb else "cublas",
                   "bf16_ref_bw_us": round(tr, 2), "bf16_cublas_us": round(tb, 2),
                   "bf16_ref_bw_gbs": round(dense_bytes(out, inn, B) / tr / 1e3, 1)}
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    # knee of max(t_mem, c B): t_mem the B = 1 time, c the B = 128 slope
    t_mem = rows[1]["int4_us"]
    c = rows[SWEEP_B[-1]]["int4_us"] / SWEEP_B[-1]
    even = next((B for B in SWEEP_B if rows[B]["int4_us"] >= rows[B]["bf16_us"]), None)
    del ws, Wb
    return {"shape": f"{out}x{inn} sym g128", "by_B": rows, "knee_B": round(t_mem / c, 1),
            "B_even": even if even is not None else f"> {SWEEP_B[-1]}"}


def act_order_cost(q4, wl, torch, device, stream):
    """Cost of act order at B = 1 on the 70B down_proj shape (8192 x 28672,
    sym g128, random column order): the gather of x alone, the product alone
    on gathered x, and both (q4_gemm_act_order), graph-timed, two weight
    copies rotating."""
    out, inn = wl.LLAMA3_70B["down_proj"]
    g = torch.Generator().manual_seed(90)
    perm = torch.randperm(inn, generator=g).to(torch.int32).to(device)
    ws = [q4.q4_quantize_pack_perm(wl.normal_weight(out, inn, 91 + i, device=device), perm, 128, True)
          for i in range(2)]
    x = wl.activations(1, inn, 92, device=device)
    xp = torch.empty_like(x)
    y = torch.empty(1, out, dtype=torch.bfloat16, device=device)
    wsp = q4.workspace_for(ws[0], 1, device)
    t_gather = graph_time_us(torch, lambda i: q4.q4_permute_activations(x, perm, xp), 16, stream)
    t_prod = graph_time_us(torch, lambda i: q4.q4_gemv(ws[i % 2], xp, y=y, workspace=wsp), 16, stream)
    t_both = graph_time_us(torch, lambda i: q4.q4_gemm_act_order(ws[i % 2], x, y=y, x_perm=xp,
                                                                  workspace=wsp), 16, stream)
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    del ws
    return {"shape": f"{out}x{inn} sym g128 B=1", "gather_us": round(t_gather, 2),
            "product_us": round(t_prod, 2), "act_order_us": round(t_both, 2),
            "overhead": round(t_both / t_prod - 1.0, 4)}


def fused_layer_cost(q4, wl, torch, device, stream, layers, steps, hbm_peak):
    """The same Llama-3-8B step with q/k/v and gate/up stored as one matrix
    each ([6144, 4096] and [28672, 4096], rows concatenated before
    quantization, as serving engines lay them out): 4 products per layer
    instead of 7, the same weights, codes and bytes (row-wise quantization
    gives the same codes).  Graph-timed like the headline step."""
    mats = []
    for layer in range(layers):
        seeds = wl.llama3_8b_layer_seeds(layer)
        W = {name: wl.normal_weight(out, inn, seeds[name], device=device)
             for name, (out, inn) in wl.LLAMA3_8B.items()}
        for name, parts in (("qkv", ("q_proj", "k_proj", "v_proj")), ("o", ("o_proj",)),
                            ("gate_up", ("gate_proj", "up_proj")), ("down", ("down_proj",))):
            Wc = torch.cat([W[p] for p in parts], dim=0)
            mats.append((name, q4.q4_quantize_pack(Wc, 128, True)))
            del Wc
        del W
    xs = {4096: wl.activations(1, 4096, 17 + 4096, device=device),
          14336: wl.activations(1, 14336, 17 + 14336, device=device)}
    ys = {name: torch.empty(1, w.out, dtype=torch.bfloat16, device=device) for name, w in mats[:4]}
    step_bytes = sum(algo_bytes(w.out, w.in_features, 128, 1) for _, w in mats)

    def step():
        for name, w in mats:
            q4.q4_gemv(w, xs[w.in_features], y=ys[name])

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    n = max(20, steps // 4)
    ms = time_region(torch, graph.replay, n, 3, stream) / n
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    del graph, mats
    gbs = step_bytes / (ms * 1e-3) / 1e9
    return {"layout": "q/k/v and gate/up fused row-wise, 4 products per layer",
            "us_per_layer": round(ms * 1e3 / layers, 3), "gbs": round(gbs, 1),
            "frac_of_measured_hbm": round(gbs / hbm_peak, 4), "bytes_per_step": step_bytes}


def w8a16_cost(q4, wl, torch, device, stream, hbm_peak):
    """Per-channel INT8 W8A16 product (q8_gemv) on the Llama-3-70B down_proj
    and gate_proj shapes at B = 1 and 8, beside the INT4 product (sym g128)
    of the same shape: graph-timed, two weight copies rotating so no call finds
    its weights in L2.  Algorithmic bytes: codes + fp32 row scales + x + y."""
    res = {}
    for name in ("down_proj", "gate_proj"):
        out, inn = wl.LLAMA3_70B[name]
        w8 = [q4.q8_quantize_per_channel(wl.normal_weight(out, inn, 60 + i, device=device).to(torch.bfloat16))
              for i in range(2)]
        w4 = [q4.q4_quantize_pack(wl.normal_weight(out, inn, 60 + i, device=device), 128, True)
              for i in range(2)]
        for B in (1, 8):
            x = wl.activations(B, inn, 61, device=device)
            y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
            wsp = q4.q8_workspace_for(w8[0], B, device)
            t8 = graph_time_us(torch, lambda i: q4.q8_gemv(w8[i % 2], x, y=y, workspace=wsp), 16, stream)
            wsp4 = q4.workspace_for(w4[0], B, device)
            t4 = graph_time_us(torch, lambda i: q4.q4_gemv(w4[i % 2], x, y=y, workspace=wsp4), 16, stream)
            b8 = out * inn + out * 4 + B * inn * 2 + B * out * 2
            res[f"{name}_B{B}"] = {"shape": f"{out}x{inn}", "q8_us": round(t8, 2),
                                   "q8_gbs": round(b8 / t8 / 1e3, 1),
                                   "q8_frac_of_measured_hbm": round(b8 / t8 / 1e3 / hbm_peak, 4),
                                   "q4_g128_us": round(t4, 2)}
        del w8, w4
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    return res


def kv_cache_cost(q4, wl, torch, device, stream, hbm_peak):
    """INT8 and INT4 (group 128) quantization of one Llama-3-70B layer's K
    cache at 32768 tokens ([1, 8, 32768, 128] bf16, 67 MB), and the INT8
    dequantization: graph-timed over four rotating caches (268 MB > L2).
    Algorithmic bytes: cache read + codes + scales written (dequant: the
    reverse)."""
    shape = (1, wl.LLAMA3_70B_KV_HEADS, 32768, wl.LLAMA3_70B_HEAD_DIM)
    caches = [wl.kv_cache(*shape, seed=70 + i, dtype=torch.bfloat16, device=device) for i in range(4)]
    n = caches[0].numel()
    rows = n // shape[-1]
    c8 = [torch.empty(shape, dtype=torch.int8, device=device) for _ in range(4)]
    s8 = [torch.empty(shape[:-1], dtype=torch.bfloat16, device=device) for _ in range(4)]
    p4 = [torch.empty(shape[:-1] + (shape[-1] // 2,), dtype=torch.uint8, device=device) for _ in range(4)]
    s4 = [torch.empty(shape[:-1] + (1,), dtype=torch.float16, device=device) for _ in range(4)]
    d8 = [torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in range(4)]
    t_q8 = graph_time_us(torch, lambda i: q4.kv_quantize_int8(caches[i % 4], c8[i % 4], s8[i % 4]), 16, stream)
    t_q4 = graph_time_us(torch, lambda i: q4.kv_quantize_int4(caches[i % 4], 128, p4[i % 4], s4[i % 4]), 16, stream)
    t_d8 = graph_time_us(torch, lambda i: q4.kv_dequant_int8(c8[i % 4], s8[i % 4], d8[i % 4]), 16, stream)
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    b_q8 = 2 * n + n + 2 * rows
    b_q4 = 2 * n + n // 2 + 2 * rows
    gbs = lambda b, t: round(b / t / 1e3, 1)
    return {"shape": "x".join(map(str, shape)) + " bf16",
            "int8_quantize_us": round(t_q8, 2), "int8_quantize_gbs": gbs(b_q8, t_q8),
            "int8_quantize_frac": round(b_q8 / t_q8 / 1e3 / hbm_peak, 4),
            "int4_g128_quantize_us": round(t_q4, 2), "int4_quantize_gbs": gbs(b_q4, t_q4),
            "int4_quantize_frac": round(b_q4 / t_q4 / 1e3 / hbm_peak, 4),
            "int8_dequant_us": round(t_d8, 2), "int8_dequant_gbs": gbs(b_q8, t_d8),
            "int8_dequant_frac": round(b_q8 / t_d8 / 1e3 / hbm_peak, 4)}


def fp4_cost(q4, wl, torch, device, stream, hbm_peak):
    """MXFP4 and NVFP4 quantization of the Llama-3-70B gate_proj (28672 x 8192
    fp16, 470 MB) and their dequantization to bf16, graph-timed over two
    rotating copies; and the weight MSE of both formats beside symmetric INT4
    at group 32 (the same 4.5 bits per weight as NVFP4) on these N(0, 0.02^2)
    weights.  Algorithmic bytes: fp16 in + codes + scale bytes out (dequant:
    codes + scales in, bf16 out)."""
    out, inn = wl.LLAMA3_70B["gate_proj"]
    Ws = [wl.normal_weight(out, inn, 80 + i, device=device) for i in range(2)]
    mx = [q4.mxfp4_quantize(W) for W in Ws]
    nv = [q4.nvfp4_quantize(W) for W in Ws]
    o16 = torch.empty(out, inn, dtype=torch.bfloat16, device=device)
    lib = q4.load_library()

    def mxq(i):
        w = mx[i % 2]
        lib.mxfp4_quantize(Ws[i % 2].data_ptr(), q4.Q4_F16, out, inn, w.packed.data_ptr(),
                           w.scales.data_ptr(), torch.cuda.current_stream().cuda_stream)

    def nvq(i):
        w = nv[i % 2]
        lib.nvfp4_quantize(Ws[i % 2].data_ptr(), q4.Q4_F16, out, inn, w.packed.data_ptr(),
                           w.scales.data_ptr(), w.tensor_scale.data_ptr(),
                           torch.cuda.current_stream().cuda_stream)

    t_mxq = graph_time_us(torch, mxq, 8, stream)
    t_nvq = graph_time_us(torch, nvq, 8, stream)
    t_mxd = graph_time_us(torch, lambda i: q4.fp4_dequant(mx[i % 2], W_hat=o16), 8, stream)
    t_nvd = graph_time_us(torch, lambda i: q4.fp4_dequant(nv[i % 2], W_hat=o16), 8, stream)
    W = Ws[0]
    mse = lambda What: (What.float() - W.float()).pow(2).mean().item()
    e_mx = mse(q4.fp4_dequant(mx[0]))
    e_nv = mse(q4.fp4_dequant(nv[0]))
    e_i4 = mse(q4.q4_dequant(q4.q4_quantize_pack(W, 32, True)))
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    n = out * inn
    b_mxq, b_nvq = 2 * n + n // 2 + n // 32, 2 * 2 * n + n // 2 + n // 16
    b_mxd, b_nvd = n // 2 + n // 32 + 2 * n, n // 2 + n // 16 + 2 * n
    g = lambda b, t: round(b / t / 1e3, 1)
    del Ws, mx, nv, o16
    return {"shape": f"{out}x{inn} fp16",
            "mxfp4_quantize_us": round(t_mxq, 2), "mxfp4_quantize_gbs": g(b_mxq, t_mxq),
            "nvfp4_quantize_us": round(t_nvq, 2), "nvfp4_quantize_gbs": g(b_nvq, t_nvq),
            "nvfp4_quantize_bytes_note": "two reads of W (tensor amax, then the codes)",
            "mxfp4_dequant_us": round(t_mxd, 2), "mxfp4_dequant_gbs": g(b_mxd, t_mxd),
            "nvfp4_dequant_us": round(t_nvd, 2), "nvfp4_dequant_gbs": g(b_nvd, t_nvd),
            "weight_mse": {"int4_sym_g32": e_i4, "mxfp4": e_mx, "nvfp4": e_nv},
            "frac_of_measured_hbm": {"mxfp4_quantize": round(b_mxq / t_mxq / 1e3 / hbm_peak, 4),
                                     "nvfp4_quantize": round(b_nvq / t_nvq / 1e3 / hbm_peak, 4),
                                     "mxfp4_dequant": round(b_mxd / t_mxd / 1e3 / hbm_peak, 4),
                                     "nvfp4_dequant": round(b_nvd / t_nvd / 1e3 / hbm_peak, 4)}}


FP4_SWEEP_B = (1, 16, 32, 64, 128)


def fp4_w4a4_sweep(q4, wl, torch, device, stream, hbm_peak):
    """W4A4 product (fp4_gemm, block-scaled tcgen05 MMA) against batch on the
    Llama-3-70B down_proj and gate_proj shapes, NVFP4 and MXFP4: seeded FP4
    weight bytes (every code, the formats' scale-byte ranges), activations
    N(0, 1) bf16 quantized by the library (timed separately: the activation
    quantization a W4A4 decode step adds), four weight copies rotating so no
    call finds its weights in L2.  Algorithmic bytes: codes and scale bytes
    of W and x, bf16 y."""
    res = {}
    for name in ("down_proj", "gate_proj"):
        out, inn = wl.LLAMA3_70B[name]
        for fmt in ("nvfp4", "mxfp4"):
            ws = []
            for i in range(4):
                p_, s_ = wl.fp4_operand(out, inn, fmt, 40 + i)
                ts = (torch.tensor([wl.FP4_W_TENSOR_SCALE], dtype=torch.float32, device=device)
                      if fmt == "nvfp4" else None)
                ws.append(q4.FP4Weight(p_.to(device), s_.to(device), out, inn, fmt, ts))
            rows = {}
            for B in FP4_SWEEP_B:
                xb = wl.activations(B, inn, 31, device=device)
                X = q4.fp4_quantize(xb, fmt)
                y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
                wsp = q4.fp4_workspace_for(ws[0], B, device)
                t = graph_time_us(torch, lambda i: q4.fp4_gemm(ws[i % 4], X, y=y, workspace=wsp),
                                  16, stream)
                tq = graph_time_us(torch, lambda i: q4.fp4_quantize(xb, fmt), 16, stream)
                nb = fp4_bytes(out, inn, fmt, B)
                rows[B] = {"us": round(t, 2), "gbs": round(nb / t / 1e3, 1),
                           "frac_of_measured_hbm": round(nb / t / 1e3 / hbm_peak, 4),
                           "tflops": round(2 * B * out * inn / t / 1e6, 1),
                           "x_quantize_us": round(tq, 2)}
            res[f"{name}.{fmt}"] = {"shape": f"{out}x{inn}", "by_B": rows}
            del ws
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    return res


def build_llama3_70b_stack(q4, wl, torch, device):
    """80 distinct Llama-3-70B layers x 7 linears, asymmetric group 64: N(0,
    0.02^2) fp16 weights generated on the device per linear (seed 1000 layer
    + linear index), quantized, fp16 freed (34.2 GB of codes, scales, zeros)."""
    mats = []
    for layer in range(wl.LLAMA3_70B_LAYERS):
        for idx, (name, (out, inn)) in enumerate(wl.LLAMA3_70B.items()):
            W = wl.normal_weight(out, inn, wl.llama3_70b_stack_seed(layer, idx), device=device)
            mats.append((name, q4.q4_quantize_pack(W, 64, False)))
            del W
    torch.cuda.synchronize()
    return mats


def stack_cost(q4, wl, torch, device, stream, B, steps, hbm_peak, mats=None):
    """One Llama-3-70B decode step over the 80-layer stack at batch B, as one
    CUDA graph: grouped launches (q/k/v and gate/up in one call each, 320
    launches) and, beside it, one launch per linear (560)."""
    own = mats is None
    if own:
        mats = build_llama3_70b_stack(q4, wl, torch, device)
    shapes = wl.LLAMA3_70B
    xs = {inn: wl.activations(B, inn, 17 + inn, device=device) for _, (_, inn) in shapes.items()}
    ys = {name: torch.empty(B, out, dtype=torch.bfloat16, device=device)
          for name, (out, _) in shapes.items()}
    wsp = q4.workspace_for(mats[0][1], B, device)
    step_bytes = sum(algo_bytes(*shapes[n], 64, B, sym=False) for n, _ in mats)
    plan = layer_plan(mats, xs, ys)

    def grouped():
        run_plan(q4, plan, wsp)

    def single():
        for name, w in mats:
            q4.q4_gemm_skinny(w, xs[shapes[name][1]], y=ys[name], workspace=wsp)

    res = {"batch": B, "bytes_per_step": step_bytes, "group_size": 64, "symmetric": False}
    for key, fn, nl in (("grouped", grouped, len(plan)), ("per_linear", single, len(mats))):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        st = q4.q4_sync_status()
        assert st == q4.Q4_OK, q4.status_string(st)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        torch.cuda.synchronize()
        with ClockSampler(device.index or 0) as clk:
            ms = time_region(torch, g.replay, steps, 3, stream) / steps
        del g
        gbs = step_bytes / (ms * 1e-3) / 1e9
        res[key] = {"ms_per_step": round(ms, 4), "us_per_layer": round(ms * 1e3 / 80, 2),
                    "gbs": round(gbs, 1), "frac_of_measured_hbm": round(gbs / hbm_peak, 4),
                    "launches_per_step": nl, "steps": steps, "clocks": clk.summary()}
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    if own:
        del mats
        torch.cuda.empty_cache()
    return res


def run_ours(args):
    import torch
    import torch.distributed as dist

    import post_weight_quantization_group_b200 as q4
    from post_weight_quantization_group_b200 import workloads as wl
    from post_weight_quantization_group_b200.replicas import aggregate_throughput, max_over_ranks

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    q4.load_library()
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream()
    B = 1
    layers = args.layers
    mats, xs, ys = build_llama3_8b(q4, wl, torch, layers, rank, B, device)
    shapes = wl.LLAMA3_8B
    step_bytes = sum(algo_bytes(*shapes[n], 128, B) for n, _ in mats)
    wsp = q4.workspace_for(mats[0][1], B, device)
    plan = layer_plan(mats, xs, ys)
    launches_per_step = len(plan)

    def step():
        run_plan(q4, plan, wsp)

    def step_ungrouped():
        for name, w in mats:
            q4.q4_gemv(w, xs[shapes[name][1]], y=ys[name], workspace=wsp)

    # eager warm-up (loads modules, sets kernel attributes), then capture
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    torch.cuda.synchronize()

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = time_region(torch, graph.replay, args.steps, args.warmup, stream)
    if world > 1:
        dist.barrier()
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    ms_eager = time_region(torch, step, max(3, args.steps // 10), 2, stream)
    ms_eager /= max(3, args.steps // 10)
    # the same products launched one per linear (7 per layer)
    for _ in range(3):
        step_ungrouped()
    torch.cuda.synchronize()
    ugraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(ugraph, capture_error_mode="thread_local"):
        step_ungrouped()
    nu = max(20, args.steps // 4)
    ms_ungrouped = time_region(torch, ugraph.replay, nu, 3, stream) / nu
    del ugraph

    ms_max = max_over_ranks(ms, dist, device)
    ms_per_step = ms_max / args.steps
    value = aggregate_throughput(step_bytes * args.steps, ms_max * 1e-3, world) / 1e9

    # ---- bf16 reference on one layer of the same shapes (436 MB > L2)
    bf_mats = []
    for name, (out, inn) in shapes.items():
        bf_mats.append((name, wl.normal_weight(out, inn, 10, device=device).to(torch.bfloat16)))
    bf_bytes = sum(dense_bytes(*shapes[n], B) for n, _ in bf_mats)

    def bf_step():
        for name, Wb in bf_mats:
            q4.bf16_gemv_ref_bw(Wb, xs[shapes[name][1]], y=ys[name])

    for _ in range(3):
        bf_step()
    torch.cuda.synchronize()
    bgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(bgraph, capture_error_mode="thread_local"):
        bf_step()
    nbf = max(20, args.steps // 4)
    ms_bf = time_region(torch, bgraph.replay, nbf, 3, stream) / nbf

    def cublas_step():
        for name, Wb in bf_mats:
            torch.matmul(xs[shapes[name][1]], Wb.T, out=ys[name])

    for _ in range(3):
        cublas_step()
    torch.cuda.synchronize()
    cgraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(cgraph, capture_error_mode="thread_local"):
        cublas_step()
    ms_cublas = time_region(torch, cgraph.replay, nbf, 3, stream) / nbf
    int4_layer_ms = ms_per_step / layers
    del bf_mats, bgraph, cgraph

    # ---- quantize + pack throughput on one layer (fp16 in, codes out)
    qW = [(n, wl.normal_weight(*shapes[n], 11, device=device)) for n in shapes]
    qbytes = sum(quant_bytes(*shapes[n], 128) for n, _ in qW)
    qouts = [(torch.empty(o, i // 2, dtype=torch.uint8, device=device),
              torch.empty(o, i // 128, dtype=torch.float16, device=device)) for o, i in shapes.values()]

    def q_step():
        for (n, W), (qo, so) in zip(qW, qouts):
            q4.q4_quantize_pack(W, 128, True, qweight=qo, scales=so)

    nq = max(10, args.steps // 20)
    ms_q = time_region(torch, q_step, nq, 2, stream) / nq

    # ---- the same with the per-group range (clipping) search over 21 ranges
    def qc_step():
        for (n, W), (qo, so) in zip(qW, qouts):
            q4.q4_quantize_pack_clip(W, 128, 21, qweight=qo, scales=so)

    nqc = max(3, args.steps // 200)
    ms_qc = time_region(torch, qc_step, nqc, 1, stream) / nqc
    Wg = dict(qW)["gate_proj"]
    mse_clip = (q4.q4_dequant(q4.q4_quantize_pack_clip(Wg, 128, 21)) - Wg.float()).pow(2).mean().item()
    mse_rtn = (q4.q4_dequant(q4.q4_quantize_pack(Wg, 128, True)) - Wg.float()).pow(2).mean().item()
    del qW, qouts, Wg

    # ---- end to end through the public API with host buffers
    x_host = {k: v.cpu().pin_memory() for k, v in xs.items()}
    y_host = torch.empty(B, shapes["down_proj"][0], dtype=torch.bfloat16).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in x_host.values())
    d2h = y_host.numel() * y_host.element_size()
    last = ys["down_proj"]

    def e2e_step():
        for k, v in x_host.items():
            xs[k].copy_(v, non_blocking=True)
        graph.replay()
        y_host.copy_(last, non_blocking=True)
        stream.synchronize()

    ne = max(10, args.steps // 10)
    for _ in range(2):
        e2e_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(ne):
        e2e_step()
    e2e_s = max_over_ranks(time.perf_counter() - t0, dist, device)
    e2e_value = aggregate_throughput(step_bytes * ne, e2e_s, world) / 1e9

    clocks = clk.summary()
    peak = peaks["hbm_gbs"]
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02^2) fp16 weights quantized on device; bf16 N(0,1) activations)",
        "config": {"workload": f"Llama-3-8B decode linears q,k,v,o,gate,up,down x {layers} distinct layers per step",
                   "batch": B, "group_size": 128, "symmetric": True, "layers": layers,
                   "linears_per_step": len(mats), "launches_per_step": launches_per_step,
                   "launch_plan": "per layer: q4_gemv_grouped(q,k,v), q4_gemv(o), "
                                  "q4_gemv_grouped(gate,up), q4_gemv(down)",
                   "bytes_per_step": step_bytes, "parallelism": f"replicas x{world}",
                   "l2": f"inputs larger than L2 ({step_bytes / 1e9:.2f} GB of packed weights per step, 126 MB L2)",
                   "timing": "CUDA graph of the step, CUDA events on the launching stream"},
        "us_per_layer": round(int4_layer_ms * 1e3, 3),
        "pct_of_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 2),
        "pct_of_measured_hbm": round(100 * value / world / peak, 2),
        "eager_us_per_layer": round(ms_eager / layers * 1e3, 3),
        "ungrouped": {"us_per_layer": round(ms_ungrouped / layers * 1e3, 3),
                      "gbs": round(step_bytes / (ms_ungrouped * 1e-3) / 1e9, 1),
                      "launches_per_step": len(mats)},
        "bf16": {"us_per_layer": round(min(ms_bf, ms_cublas) * 1e3, 3),
                 "gbs": round(bf_bytes / (min(ms_bf, ms_cublas) * 1e-3) / 1e9, 1),
                 "speedup_int4_vs_bf16_B1": round(min(ms_bf, ms_cublas) / int4_layer_ms, 3),
                 "impl": "fastest of bf16_gemv_ref_bw and cuBLAS",
                 "bf16_gemv_ref_bw_us_per_layer": round(ms_bf * 1e3, 3),
                 "cublas_us_per_layer": round(ms_cublas * 1e3, 3)},
        "quantize_pack": {"gbs": round(qbytes / (ms_q * 1e-3) / 1e9, 1),
                          "us_per_layer": round(ms_q * 1e3, 2)},
        "quantize_pack_clip": {"n_alpha": 21, "gbs": round(qbytes / (ms_qc * 1e-3) / 1e9, 1),
                               "us_per_layer": round(ms_qc * 1e3, 2),
                               "weight_mse_vs_rtn": round(mse_clip / mse_rtn, 4)},
        "roofline": {"bound": "hbm", "achieved": round(value / world, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(value / world / peak, 4),
                     "peak_kind": peak_kind,
                     "traffic": round(GEMV_TRAFFIC_RATIO * step_bytes / launches_per_step),
                     "traffic_unit": "DRAM bytes per launch",
                     "traffic_note": (f"{GEMV_TRAFFIC_RATIO:.4f} x the algorithmic bytes: "
                                      + GEMV_TRAFFIC_SOURCE),
                     "kernel": ("q4_gemv_sk_kernel<bf16,g128,sym,8,1>: cluster fix-up for "
                                "q/k/v, o and down, whole-tile grid for gate/up"),
                     "bytes_per_launch_avg": step_bytes // launches_per_step},
        "clocks": clocks,
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": ne},
        "gpu_launches": args.steps * launches_per_step,
    }
    if rank == 0:
        if world == 1 and not args.no_sweep:
            out["int4_vs_bf16_by_B"] = b_sweep(q4, wl, torch, device, stream)
            out["act_order"] = act_order_cost(q4, wl, torch, device, stream)
            out["fused_qkv_gate_up"] = fused_layer_cost(q4, wl, torch, device, stream, layers,
                                                         args.steps, peak)
            out["w8a16"] = w8a16_cost(q4, wl, torch, device, stream, peak)
            out["kv_cache"] = kv_cache_cost(q4, wl, torch, device, stream, peak)
            out["fp4"] = fp4_cost(q4, wl, torch, device, stream, peak)
            out["fp4_w4a4_by_B"] = fp4_w4a4_sweep(q4, wl, torch, device, stream, peak)
            stack = build_llama3_70b_stack(q4, wl, torch, device)
            out["llama3_70b_stack"] = {
                f"B{b}": stack_cost(q4, wl, torch, device, stream, b, max(10, args.steps // 100),
                                    peak, mats=stack) for b in (1, 8)}
            del stack
            torch.cuda.empty_cache()
        out["cpu_baseline"] = cpu_baseline() if (world == 1 and not args.no_cpu_baseline) else None
        print(json.dumps(out), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()



def run_stack(args):
    """Llama-3-70B decode stack: 80 distinct layers x 7 linears (560 W4A16
    products of 34.2 GB of packed weights), asymmetric group 64, batch B, one
    CUDA graph per step.  Weights N(0, 0.02^2) fp16 generated on the device
    per layer (seed 1000 layer + linear index), quantized, fp16 freed."""
    import torch

    import post_weight_quantization_group_b200 as q4
    from post_weight_quantization_group_b200 import workloads as wl

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    q4.load_library()
    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream()
    B, g = args.batch, 64
    shapes = wl.LLAMA3_70B
    mats = build_llama3_70b_stack(q4, wl, torch, device)
    xs = {inn: wl.activations(B, inn, 17 + inn, device=device) for _, (_, inn) in shapes.items()}
    ys = {name: torch.empty(B, out, dtype=torch.bfloat16, device=device) for name, (out, _) in shapes.items()}
    ws = q4.workspace_for(mats[0][1], B, device)
    for _, w in mats:
        ws = q4.workspace_for(w, B, device)
    step_bytes = sum(algo_bytes(*shapes[n], g, B, sym=False) for n, _ in mats)

    def step():
        for name, w in mats:
            q4.q4_gemm_skinny(w, xs[shapes[name][1]], y=ys[name], workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    assert q4.q4_sync_status() == q4.Q4_OK
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        step()
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        ms = time_region(torch, graph.replay, args.steps, args.warmup, stream)
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    value = step_bytes * args.steps / (ms * 1e-3) / 1e9
    x_host = {k: v.cpu().pin_memory() for k, v in xs.items()}
    y_host = torch.empty(B, shapes["down_proj"][0], dtype=torch.bfloat16).pin_memory()

    def e2e_step():
        for k, v in x_host.items():
            xs[k].copy_(v, non_blocking=True)
        graph.replay()
        y_host.copy_(ys["down_proj"], non_blocking=True)
        stream.synchronize()

    ne = max(3, args.steps // 4)
    e2e_step()
    t0 = time.perf_counter()
    for _ in range(ne):
        e2e_step()
    e2e_value = step_bytes * ne / (time.perf_counter() - t0) / 1e9
    peak = peaks["hbm_gbs"]
    out = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,0.02^2) fp16 weights quantized on device; bf16 N(0,1) activations)",
        "config": {"workload": f"Llama-3-70B decode stack: 80 layers x q,k,v,o,gate,up,down, asym g64, B={B}",
                   "batch": B, "group_size": g, "symmetric": False, "layers": 80,
                   "linears_per_step": len(mats), "bytes_per_step": step_bytes,
                   "l2": f"inputs larger than L2 ({step_bytes / 1e9:.1f} GB per step)",
                   "timing": "CUDA graph of the step, CUDA events on the launching stream"},
        "us_per_layer": round(ms / args.steps / 80 * 1e3, 2),
        "roofline": {"bound": "hbm", "achieved": round(value, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(value / peak, 4), "peak_kind": peak_kind, "traffic": None,
                     "kernel": "q4_gemv_sk_kernel" if B <= 8 else "q4_skinny_tc_kernel"},
        "clocks": clk.summary(),
        "e2e": {"value": round(e2e_value, 1), "unit": UNIT,
                "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in x_host.values()),
                "d2h_bytes_per_step": y_host.numel() * y_host.element_size(), "steps": ne},
        "gpu_launches": args.steps * len(mats),
        "cpu_baseline": None,
    }
    print(json.dumps(out), flush=True)
    del graph

# ------------------------------------------------------- CPU oracle timing
def _oracle_layer():
    """One Llama-3-8B layer (7 linears, sym g128) quantized by the CPU oracle,
    with its B=1 activations.  Preparation is not timed."""
    import numpy as np
    import oracle
    from post_weight_quantization_group_b200 import workloads as wl

    oracle.build()
    prepared = []
    for name, (out, inn) in wl.LLAMA3_8B.items():
        W = wl.normal_weight(out, inn, wl.llama3_8b_layer_seeds(0)[name]).float().numpy()
        q, s, _ = oracle.quantize_pack(W, 128, True)
        x = wl.activations(1, inn, 17 + inn).float().numpy().astype(np.float64)
        prepared.append((out, inn, q, s, x))
    return prepared


def _oracle_pass(prepared, frac=1.0):
    """fp64 oracle product over the first ceil(frac * out) rows of each linear;
    returns algorithmic bytes processed."""
    import numpy as np
    import oracle
    nbytes = 0
    for out, inn, q, s, x in prepared:
        n = max(1, min(out, int(round(out * frac))))
        rows = np.arange(n, dtype=np.int64)
        oracle.gemv(q, s, None, out, inn, 128, True, x, rows=rows)
        nbytes += algo_bytes(n, inn, 128, 1)
    return nbytes


def host_cpu():
    """nproc and the lscpu model name of the host the oracle runs on."""
    model = None
    try:
        txt = subprocess.run(["lscpu"], capture_output=True, text=True, timeout=10).stdout
        for ln in txt.splitlines():
            if ln.startswith("Model name:"):
                model = ln.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError):
        pass
    return {"nproc": os.cpu_count(), "lscpu_model": model, "threads_used": 1}


def _oracle_small_case():
    """The 512 x 1024 parity case (N(0, 0.02^2) fp16, sym g128, B=1, CPU
    generator seed 0), quantized and multiplied whole by the oracle: seconds."""
    import numpy as np
    import torch
    import oracle
    from post_weight_quantization_group_b200 import workloads as wl
    W = wl.normal_weight(512, 1024, 0).float().numpy()
    x = wl.activations(1, 1024, 0, dtype=torch.float16).float().numpy().astype(np.float64)
    t0 = time.perf_counter()
    q, s_, _ = oracle.quantize_pack(W, 128, True)
    oracle.gemv(q, s_, None, 512, 1024, 128, True, x)
    return time.perf_counter() - t0


def _oracle_stack_sample(frac=1.0 / 16):
    """Layer 0 of the Llama-3-70B stack (asym g64, B=1): the first `frac` of
    every linear's rows (weights from the stack's seeds), quantized by the
    oracle (not timed), then its fp64 product (timed).  Returns (seconds,
    algorithmic bytes of the sample)."""
    import numpy as np
    import torch
    import oracle
    from post_weight_quantization_group_b200 import workloads as wl
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    prepared = []
    for idx, (name, (out, inn)) in enumerate(wl.LLAMA3_70B.items()):
        n = max(1, int(out * frac))
        W = wl.normal_weight(out, inn, wl.llama3_70b_stack_seed(0, idx), device=dev)[:n]
        q, s_, z = oracle.quantize_pack(W.float().cpu().numpy(), 64, False)
        x = wl.activations(1, inn, 17 + inn).float().numpy().astype(np.float64)
        prepared.append((n, inn, q, s_, z, x))
        del W
    t0 = time.perf_counter()
    nbytes = 0
    for n, inn, q, s_, z, x in prepared:
        oracle.gemv(q, s_, z, n, inn, 64, False, x)
        nbytes += algo_bytes(n, inn, 64, 1, sym=False)
    return time.perf_counter() - t0, nbytes


def cpu_baseline():
    prepared = _oracle_layer()
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(3):
        nbytes += _oracle_pass(prepared)
    dt = time.perf_counter() - t0
    frac = 1.0 / 16
    t5, b5 = _oracle_stack_sample(frac)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "3 passes over 1 of 32 Llama-3-8B layers (7 linears, sym g128, B=1), "
                      "fp64 product of the CPU oracle, single thread",
            "seconds": round(dt, 2), "host": host_cpu(),
            "small_case_512x1024_seconds": round(_oracle_small_case(), 4),
            "llama3_70b_stack_B1": {
                "sample": "first 1/16 of the rows of each of the 7 linears of layer 0 "
                          "(asym g64, B=1), fp64 product, single thread",
                "seconds": round(t5, 2), "gbs": round(b5 / t5 / 1e9, 4),
                "seconds_per_step_extrapolated": round(t5 / frac * wl_layers_70b(), 1),
                "extrapolation": "x16 (rows) x 80 (layers)"}}


def wl_layers_70b():
    from post_weight_quantization_group_b200 import workloads as wl
    return wl.LLAMA3_70B_LAYERS


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    prepared = _oracle_layer()
    # calibrate, then size each step's row sample so the run takes ~90 s
    t0 = time.perf_counter()
    cb = _oracle_pass(prepared, 0.02)
    rate = cb / (time.perf_counter() - t0)
    layer_bytes = sum(algo_bytes(o, i, 128, 1) for o, i, *_ in prepared)
    frac = min(1.0, max(1e-4, 90.0 * rate / (args.steps + args.warmup) / layer_bytes))
    for _ in range(args.warmup):
        _oracle_pass(prepared, frac)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += _oracle_pass(prepared, frac)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"per step: the first {100 * frac:.3g}% of the rows of each of the 7 linears of "
              f"one Llama-3-8B layer (sym g128, B=1), fp64 product, single thread")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,0.02^2) fp16 weights, bf16 N(0,1) activations)",
        "config": {"workload": "Llama-3-8B decode linears q,k,v,o,gate,up,down, B=1, sym g128 "
                               "(CPU oracle on a row sample)", "batch": 1, "group_size": 128},
        "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_op(args):
    """One operation of the path alone, for profiling and spot timing:
    ``w8a16-70b`` = q8_gemv on the Llama-3-70B down_proj (8192 x 28672, batch
    --batch, two weight copies rotating); ``q4-70b-down`` = q4_gemm_skinny
    (--group-size, symmetric unless --asym) on the same shape and batch (the
    B <= 8 kernel or, above, the tcgen05 kernel); ``nvfp4-70b-down`` / ``mxfp4-70b-down`` = fp4_gemm (W4A4,
    seeded FP4 weight bytes, activations quantized by the library) on the same
    shape and batch; ``kv8-70b-32k`` = kv_quantize_int8
    of one layer's K cache at 32768 tokens ([1, 8, 32768, 128] bf16, four
    caches rotating).  Prints one JSON line (CUDA-event time per call)."""
    import torch
    sys.path.insert(0, ROOT)
    import post_weight_quantization_group_b200 as q4
    from post_weight_quantization_group_b200 import workloads as wl
    q4.load_library()
    device = torch.device("cuda:0")
    stream = torch.cuda.current_stream()
    if args.workload == "w8a16-70b":
        out, inn = wl.LLAMA3_70B["down_proj"]
        B = args.batch
        ws = []
        for i in range(2):
            W = wl.normal_weight(out, inn, 60 + i, device=device).to(torch.bfloat16)
            ws.append(q4.q8_quantize_per_channel(W))
            del W
        torch.cuda.empty_cache()
        x = wl.activations(B, inn, 61, device=device)
        y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
        wsp = q4.q8_workspace_for(ws[0], B, device)
        it = iter(range(1 << 30))
        fn = lambda: q4.q8_gemv(ws[next(it) % 2], x, y=y, workspace=wsp)
        nbytes = out * inn + out * 4 + B * inn * 2 + B * out * 2
        name, cfg = "W8A16 per-channel INT8 GEMV", {"workload": f"Llama-3-70B down_proj {out}x{inn}", "batch": B}
    elif args.workload == "q4-70b-down":
        out, inn = wl.LLAMA3_70B["down_proj"]
        B, g, sym = args.batch, args.group_size, not args.asym
        ws = [q4.q4_quantize_pack(wl.normal_weight(out, inn, 30 + i, device=device), g, sym)
              for i in range(2)]
        torch.cuda.empty_cache()
        x = wl.activations(B, inn, 31, device=device)
        y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
        wsp = q4.workspace_for(ws[0], B, device)
        it = iter(range(1 << 30))
        fn = lambda: q4.q4_gemm_skinny(ws[next(it) % 2], x, y=y, workspace=wsp)
        nbytes = algo_bytes(out, inn, g, B, sym=sym)
        kind = f"{'sym' if sym else 'asym'} g{g}"
        name, cfg = (f"W4A16 INT4 product ({kind})",
                     {"workload": f"Llama-3-70B down_proj {out}x{inn}", "batch": B, "quant": kind})
    elif args.workload in ("nvfp4-70b-down", "mxfp4-70b-down"):
        fmt = args.workload.split("-")[0]
        out, inn = wl.LLAMA3_70B["down_proj"]
        B = args.batch
        ws = []
        for i in range(2):
            p, s = wl.fp4_operand(out, inn, fmt, 40 + i)
            ts = (torch.tensor([wl.FP4_W_TENSOR_SCALE], dtype=torch.float32, device=device)
                  if fmt == "nvfp4" else None)
            ws.append(q4.FP4Weight(p.to(device), s.to(device), out, inn, fmt, ts))
        X = q4.fp4_quantize(wl.activations(B, inn, 31, device=device), fmt)
        y = torch.empty(B, out, dtype=torch.bfloat16, device=device)
        wsp = q4.fp4_workspace_for(ws[0], B, device)
        it = iter(range(1 << 30))
        fn = lambda: q4.fp4_gemm(ws[next(it) % 2], X, y=y, workspace=wsp)
        nbytes = fp4_bytes(out, inn, fmt, B)
        name, cfg = (f"W4A4 {fmt.upper()} product (block-scaled tcgen05)",
                     {"workload": f"Llama-3-70B down_proj {out}x{inn}", "batch": B})
    else:
        shape = (1, wl.LLAMA3_70B_KV_HEADS, 32768, wl.LLAMA3_70B_HEAD_DIM)
        caches = [wl.kv_cache(*shape, seed=70 + i, dtype=torch.bfloat16, device=device) for i in range(4)]
        c8 = [torch.empty(shape, dtype=torch.int8, device=device) for _ in range(4)]
        s8 = [torch.empty(shape[:-1], dtype=torch.bfloat16, device=device) for _ in range(4)]
        it = iter(range(1 << 30))

        def fn():
            i = next(it) % 4
            q4.kv_quantize_int8(caches[i], c8[i], s8[i])
        n = caches[0].numel()
        nbytes = 3 * n + 2 * (n // shape[-1])
        name, cfg = "INT8 KV-cache quantization", {"workload": "Llama-3-70B K cache [1,8,32768,128] bf16"}
    ms = time_region(torch, fn, args.steps, args.warmup, stream) / args.steps
    st = q4.q4_sync_status()
    assert st == q4.Q4_OK, q4.status_string(st)
    print(json.dumps({"metric": name, "value": round(nbytes / (ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                      "us_per_call": round(ms * 1e3, 2), "steps": args.steps, "warmup": args.warmup,
                      "config": cfg, "timing": "CUDA events on the launching stream, eager launches"}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama3-8b",
                    choices=["llama3-8b", "llama3-70b-stack", "w8a16-70b", "q4-70b-down",
                             "kv8-70b-32k", "nvfp4-70b-down", "mxfp4-70b-down"])
    ap.add_argument("--batch", type=int, default=1,
                    help="batch of the llama3-70b-stack and single-op workloads")
    ap.add_argument("--group-size", type=int, default=128, choices=[32, 64, 128],
                    help="INT4 group size of the q4-70b-down workload")
    ap.add_argument("--asym", action="store_true",
                    help="asymmetric (zero-point) INT4 in the q4-70b-down workload")
    ap.add_argument("--layers", type=int, default=32,
                    help="distinct decoder layers per step (32 = the Llama-3-8B depth)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the INT4/bf16 speedup-vs-batch sweep (70B down_proj, B = 1..128)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the CPU oracle (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "llama3-70b-stack":
        run_stack(args)
    elif args.workload in ("w8a16-70b", "q4-70b-down", "kv8-70b-32k", "nvfp4-70b-down",
                           "mxfp4-70b-down"):
        run_op(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
