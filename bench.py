"""Benchmark of the 4-bit MoE expert FFN on B200.

Workload (default, decode_t1): one MoE layer, hidden 2048, expert FFN 512,
128 experts top-8 plus one always-on shared expert, Q4_0 weights and Q8_0
activations; 1000 distinct seeded tokens, each a separate T=1 call of
moe_q4_ffn_forward, issued back to back (captured once as a CUDA graph).  One
step = those 1000 calls.  value = tokens/s over all ranks.

L2: the layer is replicated at 16 distinct device addresses (3.7 GB) and token
i uses replica i mod 16, so the weights a token reads were last touched about
270 MB of traffic earlier (L2 is 126 MB): every step is L2-cold for weights.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the reference arm of this build) on a
bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "decode_t1"
N_TOKENS = 1000
REPLICAS = 16
METRIC = "Q4_0 MoE layer tokens/s (T=1 decode, T=947 prefill); % HBM / int8-TC peak"


def physical_cores() -> int:
    try:
        out = subprocess.run(["lscpu", "-p=CORE,SOCKET"], capture_output=True, text=True).stdout
        pairs = {tuple(line.split(",")) for line in out.splitlines() if line and not line.startswith("#")}
        if pairs:
            return len(pairs)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def oracle_sample(x, lw, seconds=10.0):
    """The oracle as it stands on a bounded token sample (tokens are
    independent): probe, then size the sample to about `seconds` of work."""
    import oracle
    cores = oracle.set_threads(physical_cores())
    t0 = time.perf_counter()
    oracle.moe_forward(lw, x[:16])
    rate = 16 / (time.perf_counter() - t0)
    n = int(min(max(16, rate * seconds), 8000))
    idx = np.arange(n) % x.shape[0]
    xs = np.ascontiguousarray(x[idx])
    t0 = time.perf_counter()
    oracle.moe_forward(lw, xs)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, cores


def simd_sample(x, lw, seconds=5.0):
    """The host SIMD W4A8 decode (the page's own CPU decode method) on a
    bounded token sample, like the oracle's."""
    import cpu_simd
    cores = cpu_simd.set_threads(physical_cores())
    t0 = time.perf_counter()
    cpu_simd.moe_forward(lw, x[:64])
    rate = 64 / (time.perf_counter() - t0)
    n = int(min(max(64, rate * seconds), 20000))
    idx = np.arange(n) % x.shape[0]
    xs = np.ascontiguousarray(x[idx])
    t0 = time.perf_counter()
    cpu_simd.moe_forward(lw, xs)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, cores


def rank_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(value: float, device) -> float:
    """The slowest rank's value (every rank calls this in the same order); the
    value itself on one rank or without a process group."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units every rank processed, over the slowest rank's time (weak scaling)."""
    return world * units_per_rank / (ms / 1000.0)


def rank_tokens(x0: np.ndarray, rank: int) -> np.ndarray:
    """The decode tokens of one replica: rank 0 the workload's own, rank r > 0
    its own seeded draw of the same shape (the layer weights are the same on
    every rank)."""
    if rank == 0:
        return x0
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([17, rank])))
    return rng.standard_normal(x0.shape, dtype=np.float32)


def run_reference(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return 0
    import synth
    x, lw = synth.workload_inputs(WORKLOAD, seed=0, T=N_TOKENS)
    for _ in range(args.warmup):
        oracle_sample(x, lw, seconds=1.0)
    vals, total_tokens, total_s = [], 0, 0.0
    for _ in range(args.steps):
        v, n, dt, cores = oracle_sample(x, lw, seconds=max(1.0, 60.0 / max(1, args.steps)))
        vals.append(v)
        total_tokens += n
        total_s += dt
    value = total_tokens / total_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * total_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "tokens_per_step": N_TOKENS},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{total_tokens} tokens of the {N_TOKENS}-token decode workload over "
                                   f"{args.steps} steps, OpenMP over tokens on {cores} physical cores "
                                   f"({cpu_model()})"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        import tempfile
        self.gpu = gpu_index
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"moe_q4_clocks_gpu{gpu_index}_", suffix=".csv")
        os.close(fd)

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [s.strip() for s in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def graph_kernel_nodes(graph) -> int:
    """Kernel nodes in a captured torch CUDA graph (cudaGraphNodeTypeKernel == 0)."""
    import torch
    lib = None
    for cand in ("libcudart.so.12", "libcudart.so"):
        try:
            lib = ctypes.CDLL(cand)
            break
        except OSError:
            continue
    if lib is None:
        import glob
        for c in glob.glob(os.path.join(os.path.dirname(torch.__file__), "..", "nvidia", "cuda_runtime", "lib",
                                        "libcudart.so*")):
            lib = ctypes.CDLL(c)
            break
    g = ctypes.c_void_p(graph.raw_cuda_graph())
    n = ctypes.c_size_t(0)
    assert lib.cudaGraphGetNodes(g, None, ctypes.byref(n)) == 0
    nodes = (ctypes.c_void_p * n.value)()
    assert lib.cudaGraphGetNodes(g, nodes, ctypes.byref(n)) == 0
    kernels = 0
    for i in range(n.value):
        t = ctypes.c_int(-1)
        assert lib.cudaGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) == 0
        kernels += int(t.value == 0)
    return kernels


def source_digest(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str):
    """dram bytes per launch from the committed ncu summary, if the kernel's
    source has not changed since it was captured (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(kernel)
    if not rec:
        return None
    if source_digest(rec["sources"]) != rec["digest"]:
        return None
    return rec["bytes_per_launch"]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def int8_peak_tops():
    """Dense int8 tensor peak: the measured bf16 GEMM peak x the nominal
    int8/bf16 ratio (4.5 / 2.25 PFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["bf16_tflops"]) * 2.0, "measured bf16 x nominal int8/bf16 ratio 2"
    return 1590.0 * 2.0, "fallback bf16 x nominal int8/bf16 ratio 2"


def rescale_ceiling(m, torch, stream, peak):
    """The tensor-core epilogue's per-block rescale alone (moe_q4_rescale_ceiling):
    accumulator elements per second for binary16 and int8 operands, and the
    int8 rate that bounds (64 ops an element: 32 multiply-adds)."""
    sink = torch.zeros(1, dtype=torch.float32, device="cuda")
    out = {}
    for name, i8 in (("binary16_operands", False), ("int8_operands", True)):
        times = []
        n = 0
        for rep in range(7):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            n = m.moe_q4_rescale_ceiling(i8, 4096, sink, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
        eps = n / (ms * 1e-3)
        out[name] = {"ms": ms, "elements_per_s": eps, "int8_tops_bound": eps * 64 / 1e12,
                     "frac_of_int8_peak": eps * 64 / 1e12 / peak}
    out["how"] = ("one CTA per SM, 16 warps, 4096 operand stages of the epilogue's inner loop over all of TMEM "
                  "(4 blocks x 32 columns a thread a stage), no other role")
    return out


def prefill_lines(m, torch, stream, names=("prefill_t947", "zipf_t16384")):
    """Single-pass prefill of the two prefill workloads on the automatic path
    (tensor cores at these sizes): tokens/s over whole forwards and the int8
    ops/s of the gate/up kernel, L2 flushed (256 MB written) before each rep;
    the gate/up rate also as a fraction of the epilogue-rescale ceiling of its
    operand type (binary16 on 64- and 128-slot tiles, the automatic choice at
    these sizes; int8 on 32-slot ones)."""
    import synth
    out = {}
    peak, peak_src = int8_peak_tops()
    ceil = rescale_ceiling(m, torch, stream, peak)
    out["rescale_ceiling"] = ceil
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    variants = (("auto", m.PATH_AUTO), ("tc_n32", m.PATH_TENSOR_CORE_N32), ("tc_n64", m.PATH_TENSOR_CORE_N64),
                ("tc_n128", m.PATH_TENSOR_CORE_N128))
    for name in names:
        x_np, lw = synth.workload_inputs(name, seed=0)
        L = m.Layer.from_host(lw)
        x = torch.from_numpy(x_np).cuda()
        T = x.shape[0]
        y = torch.empty_like(x)
        ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, T))
        pairs = T * (lw.top_k + 1)
        gu_ops = 2.0 * pairs * 2 * lw.ffn * lw.hidden
        all_ops = 2.0 * pairs * 3 * lw.ffn * lw.hidden
        for vname, path in variants:
            tot, gu = [], []
            for rep in range(8):
                flush.zero_()
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
                for e in evs[2:]:
                    e.record(stream)  # torch creates the CUDA event on first record
                evs[0].record(stream)
                m.moe_q4_ffn_forward_debug(L, x, y, ws, path=path, ev_start=evs[2], ev_stop=evs[3], stream=stream)
                evs[1].record(stream)
                torch.cuda.synchronize()
                if rep >= 3:
                    tot.append(evs[0].elapsed_time(evs[1]))
                    gu.append(evs[2].elapsed_time(evs[3]))
            ms, gu_ms = float(np.median(tot)), float(np.median(gu))
            rec = {"tokens_per_s": T / (ms * 1e-3), "ms": ms, "gateup_ms": gu_ms,
                   "gateup_int8_tops": gu_ops / (gu_ms * 1e-3) / 1e12,
                   "gateup_frac_of_int8_peak": gu_ops / (gu_ms * 1e-3) / 1e12 / peak,
                   "gateup_frac_of_rescale_ceiling": gu_ops / (gu_ms * 1e-3) / 1e12 / ceil[
                       "int8_operands" if vname == "tc_n32" else "binary16_operands"]["int8_tops_bound"],
                   "layer_int8_tops": all_ops / (ms * 1e-3) / 1e12,
                   "layer_frac_of_int8_peak": all_ops / (ms * 1e-3) / 1e12 / peak}
            if vname == "auto":
                rec.update({"int8_peak_tops": peak, "peak_source": peak_src, "l2": "256 MB flush before each rep"})
                out[name] = rec
            else:
                out[name][vname] = rec
        # the router (logits + top-k: the same kernels the forward launches)
        # alone, and its share of the automatic forward
        idx = torch.empty((T, lw.top_k), dtype=torch.int32, device="cuda")
        wts = torch.empty((T, lw.top_k), dtype=torch.float32, device="cuda")
        lg = torch.empty((T, lw.n_experts), dtype=torch.float32, device="cuda")
        rt = []
        for rep in range(8):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            m.moe_q4_route(L, x, idx, wts, lg, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 3:
                rt.append(e0.elapsed_time(e1))
        r_ms = float(np.median(rt))
        out[name]["router_ms"] = r_ms
        out[name]["router_share"] = r_ms / out[name]["ms"]
        out[name]["router_fp32_tflops"] = 2.0 * T * lw.hidden * lw.n_experts / (r_ms * 1e-3) / 1e12
        del L, x, y, ws, idx, wts, lg
    del flush
    return out


def chunked_lines(m, torch, stream):
    """Single pass against chunked prefill (the page's Methodologie 4 claim):
    the 947- and 16384-token prompts through moe_q4_ffn_forward in chunks of
    C tokens (ceil(T/C) calls back to back), tokens/s per C; 256 MB written
    between reps to flush L2."""
    import synth
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for name, sizes in (("prefill_t947", (64, 128, 256, 512, 947)),
                        ("zipf_t16384", (256, 1024, 4096, 16384))):
        x_np, lw = synth.workload_inputs(name, seed=0)
        L = m.Layer.from_host(lw)
        x = torch.from_numpy(x_np).cuda()
        T = x.shape[0]
        y = torch.empty_like(x)
        rec = {}
        for C in sizes:
            ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(L, C))
            times = []
            for rep in range(5):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                for t0 in range(0, T, C):
                    m.moe_q4_ffn_forward(L, x[t0:t0 + C], y[t0:t0 + C], ws, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
                if rep >= 2:
                    times.append(e0.elapsed_time(e1))
            ms = float(np.median(times))
            rec[str(C)] = {"ms": ms, "tokens_per_s": T / (ms * 1e-3), "calls": -(-T // C)}
            del ws
        out[name] = rec
        del L, x, y
    del flush
    return out


def batch64_lines(m, torch, stream):
    """One layer on batches of 8 to 512 tokens, on the automatic path, the
    streaming dp4a kernels and the 32- and 64-slot tensor-core kernels: tokens/s,
    and HBM GB/s over the experts the batch activates + Wr + x/y; the layer
    rotates over 4 device copies (912 MB) so every rep is L2-cold."""
    import synth
    hbm, src = measured_peaks()
    x_np, lw = synth.workload_inputs("prefill_t947", seed=0)
    base = m.Layer.from_host(lw)
    layers = [base] + [base.replica() for _ in range(3)]
    out = {"peak_source": src}
    for T in (8, 16, 32, 64, 96, 128, 192, 256, 384, 512):
        x = torch.from_numpy(x_np[:T].copy()).cuda()
        y = torch.empty_like(x)
        ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(base, T))
        rec = {}
        for vname, path in (("auto", m.PATH_AUTO), ("dp4a", m.PATH_GROUPED_DP4A), ("tc_n32", m.PATH_TENSOR_CORE_N32),
                            ("tc_n64", m.PATH_TENSOR_CORE_N64)):
            times = []
            for rep in range(12):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                m.moe_q4_ffn_forward_debug(layers[rep % 4], x, y, ws, path=path, stream=stream)
                e1.record(stream)
                torch.cuda.synchronize()
                if rep >= 4:
                    times.append(e0.elapsed_time(e1))
            us = float(np.median(times)) * 1000.0
            cnt = m.workspace_views(base, T, ws)["cnt"][:lw.n_experts].cpu().numpy()
            active = int(np.count_nonzero(cnt)) + 1
            nbytes = (active * 3 * lw.ffn * (lw.hidden // 32) * 18 + lw.n_experts * lw.hidden * 4 +
                      2 * T * lw.hidden * 4)
            rec[vname] = {"us": us, "tokens_per_s": T / (us * 1e-6), "active_experts": active,
                          "algorithmic_bytes": nbytes, "hbm_gbs": nbytes / (us * 1e-6) / 1e9,
                          "hbm_frac": nbytes / (us * 1e-6) / 1e9 / hbm}
        out[f"T{T}"] = rec
        del ws
    del layers
    return out


def gemv_lines(m, torch, stream):
    """The W4A8 LM-head GEMV: one 131072 x 2048 Q4_0 matrix (151 MB, beyond
    the 126 MB L2; two copies alternate so every rep is L2-cold) against
    1..8 tokens; HBM GB/s over the matrix + x + y bytes."""
    import synth
    hbm, src = measured_peaks()
    N, H = 131072, 2048
    rng = np.random.Generator(np.random.PCG64(7))
    W = torch.from_numpy(synth._q4_0_matrix(rng, N, H // 32)).cuda()
    Ws = [W, W.clone()]
    out = {"rows": N, "hidden": H, "peak_source": src}
    for T in (1, 4, 8):
        x = torch.from_numpy(np.random.default_rng(T).standard_normal((T, H)).astype(np.float32)).cuda()
        y = torch.empty((T, N), dtype=torch.float32, device="cuda")
        ws = m.alloc_workspace(m.moe_q4_gemv_workspace_bytes(T, H))
        times = []
        for rep in range(12):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            m.moe_q4_gemv(Ws[rep % 2], x, y, ws, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 4:
                times.append(e0.elapsed_time(e1))
        us = float(np.median(times)) * 1000.0
        nbytes = N * (H // 32) * 18 + T * H * 4 + T * N * 4
        out[f"T{T}"] = {"us": us, "hbm_gbs": nbytes / (us * 1e-6) / 1e9, "hbm_frac": nbytes / (us * 1e-6) / 1e9 / hbm}
    del W, Ws
    return out


def streamed_lines(m, torch, stream):
    """Host-streamed experts (expert matrices in page-locked host memory,
    the selected experts copied per call): decode T = 1 and the 947-token
    prefill; link GB/s over the expert bytes that cross per call, beside a
    plain page-locked host-to-device copy of the same bytes (the link's
    rate for one large copy)."""
    import synth
    out = {}
    ref_bytes = 129 * 3 * 512 * (2048 // 32) * 18
    src = torch.empty(ref_bytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(ref_bytes, dtype=torch.uint8, device="cuda")
    times = []
    for rep in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            dst.copy_(src, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if rep >= 1:
            times.append(e0.elapsed_time(e1))
    out["link_copy"] = {"bytes": ref_bytes, "ms": float(np.median(times)),
                        "gbs": ref_bytes / (float(np.median(times)) * 1e-3) / 1e9}
    del src, dst
    for name, T in (("decode_t1", 1), ("prefill_t947", 947)):
        x_np, lw = synth.workload_inputs(name, seed=0, T=T if name == "decode_t1" else None)
        Lh = m.Layer.from_host_pinned(lw)
        x = torch.from_numpy(x_np[:T].copy()).cuda()
        y = torch.empty_like(x)
        ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(Lh, T))
        st = m.alloc_workspace(m.moe_q4_staging_bytes(Lh))
        times = []
        for rep in range(6):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            m.moe_q4_ffn_forward_streamed(Lh, x, y, ws, st, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
        cnt = m.workspace_views(Lh, T, ws)["cnt"][:lw.n_experts].cpu().numpy()
        staged = (int(np.count_nonzero(cnt)) + 1) * 3 * lw.ffn * (lw.hidden // 32) * 18
        out[name] = {"T": T, "ms": ms, "tokens_per_s": T / (ms * 1e-3), "expert_bytes_staged": staged,
                     "link_gbs": staged / (ms * 1e-3) / 1e9}
        del Lh, x, y, ws, st
    return out


def stack_lines(m, torch, stream):
    """The 40-layer stack (x <- x + MoE_l(RMSNorm(x)), independently seeded
    layers, 9.1 GB of weights: every step is L2-cold) through the one-call
    entry, captured as one CUDA graph: a batched decode step of 64 tokens and
    a 4096-token prefill.  Decode reports HBM bandwidth over the algorithmic
    bytes (the experts each layer's routing activates, router weights, x in
    and y out); prefill reports int8 ops/s against the int8 tensor peak."""
    import synth
    c = synth.WORKLOADS["stack40"]
    H, F, E, k, NL = c["H"], c["F"], c["E"], c["k"], c["layers"]
    layers = [m.Layer.from_host(synth.stack_layer(l, H, F, E, k, c["shared"], 0)) for l in range(NL)]
    hbm, hbm_src = measured_peaks()
    peak, peak_src = int8_peak_tops()
    expert_bytes = 3 * F * (H // 32) * 18
    out = {}
    for T, key in ((c["T"], "stack40_decode_t64"), (c["T_prefill"], "stack40_prefill_t4096")):
        x0 = torch.from_numpy(synth.stack_inputs(T, H, 0)).cuda()
        ws = m.alloc_workspace(m.moe_q4_stack_workspace_bytes(layers[0], T))
        # experts each layer activates (layer by layer, outside the timed region)
        active = 0
        if T == c["T"]:
            x = x0.clone()
            y = torch.zeros_like(x)
            lws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(layers[0], T))
            for l, L in enumerate(layers):
                xn = m.moe_q4_residual_rmsnorm(x, y if l else None, stream=stream)
                m.moe_q4_ffn_forward(L, xn, y, lws, stream=stream)
                torch.cuda.synchronize()
                cnt = m.workspace_views(L, T, lws)["cnt"][:E].cpu().numpy()
                active += int(np.count_nonzero(cnt)) + 1          # + the shared expert
            del lws
        x = x0.clone()
        m.moe_q4_stack_forward(layers, x, stream=stream, workspace=ws)      # eager warm-up
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            m.moe_q4_stack_forward(layers, x, stream=stream, workspace=ws)
        times = []
        for rep in range(6):
            x.copy_(x0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            if rep >= 2:
                times.append(e0.elapsed_time(e1))
        ms = float(np.median(times))
        rec = {"T": T, "layers": NL, "ms": ms, "tokens_per_s": T / (ms * 1e-3),
               "l2": "9.1 GB of weights per step, far beyond the 126 MB L2"}
        if active:
            nbytes = active * expert_bytes + NL * (E * H * 4 + 2 * T * H * 4)
            rec.update({"algorithmic_bytes": nbytes, "active_experts_per_layer": active / NL - 1,
                        "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm,
                        "peak_source": hbm_src})
        else:
            ops = NL * 2.0 * T * (k + 1) * 3 * F * H
            rec.update({"int8_tops": ops / (ms * 1e-3) / 1e12, "frac_of_int8_peak": ops / (ms * 1e-3) / 1e12 / peak,
                        "peak_source": peak_src})
        out[key] = rec
        del g, x, x0, ws
    del layers
    torch.cuda.empty_cache()
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = rank_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))

    import quantized_moe_q4_b200 as m
    import synth

    x0_np, lw = synth.workload_inputs(WORKLOAD, seed=0, T=N_TOKENS)
    x_np = rank_tokens(x0_np, rank)          # each replica decodes its own tokens
    base = m.Layer.from_host(lw)
    replicas = args.replicas
    layers = [base] + [base.replica() for _ in range(replicas - 1)]
    H, F, E, k = lw.hidden, lw.ffn, lw.n_experts, lw.top_k
    x = torch.from_numpy(x_np).cuda()
    y = torch.empty_like(x)
    ws = m.alloc_workspace(m.moe_q4_ffn_workspace_bytes(base, 1))
    stream = torch.cuda.Stream()
    # every launch, graph replay and event of the run goes to this one stream
    # (CUDAGraph.replay launches on the current stream)
    torch.cuda.set_stream(stream)

    def step_calls(timer=None):
        for i in range(N_TOKENS):
            L = layers[i % replicas]
            if timer is None:
                m.moe_q4_ffn_forward(L, x[i:i + 1], y[i:i + 1], ws, stream=stream)
            else:
                m.moe_q4_ffn_forward_debug(L, x[i:i + 1], y[i:i + 1], ws, decode_kernel_ns=timer, stream=stream)

    # eager run once (also checks the calls succeed), then capture
    with torch.cuda.stream(stream):
        step_calls()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(graph, stream=stream):
        step_calls()
    graph.instantiate()
    kernels_per_step = graph_kernel_nodes(graph)

    for _ in range(max(3, args.warmup)):
        graph.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = ev0.elapsed_time(ev1)
    clk = clocks.stop()
    ms = max_over_ranks(ms, "cuda")
    ms_per_step = ms / args.steps
    value = whole_job_rate(N_TOKENS * args.steps, world, ms)

    # dominant kernel (the fused T=1 FFN kernel) timed inside the same
    # programmatic-launch chain: the same 1000 calls, captured again with the
    # kernel's own %globaltimer spans (its first CTA) accumulated on the device
    # -- no event node between the router and FFN kernels.  The launch overlaps
    # the router kernel (it starts early and waits for the logits), so its
    # duration is taken from that wait returning to its end; the span from its
    # start is reported beside it
    timer = torch.zeros(3, dtype=torch.int64, device="cuda")
    g2 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        step_calls(timer=timer)
    torch.cuda.synchronize()
    with torch.cuda.graph(g2, stream=stream):
        step_calls(timer=timer)
    for _ in range(max(3, args.warmup)):
        g2.replay()
    torch.cuda.synchronize()
    timer.zero_()
    e0t, e1t = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0t.record(stream)
    for _ in range(args.steps):
        g2.replay()
    e1t.record(stream)
    torch.cuda.synchronize()
    t_ns, t_n, t_resident_ns = (int(v) for v in timer.cpu().tolist())
    dom_us = t_ns / max(1, t_n) / 1e3
    resident_us = t_resident_ns / max(1, t_n) / 1e3
    timed_graph_ms_per_step = e0t.elapsed_time(e1t) / args.steps
    del g2

    # algorithmic bytes of one launch of the dominant kernel (the fused T=1 FFN
    # kernel: top-k, Q8_0 of x, gate/up, SwiGLU, requant, down, combine): the
    # three Q4_0 matrices of the k routed experts and the shared expert, the
    # router logits and x read, y written
    nb, nbF = H // 32, F // 32
    experts = k + 1
    ffn_bytes = experts * 3 * F * nb * 18 + E * 4 + H * 4 + H * 4
    peak, peak_src = measured_peaks()
    achieved = ffn_bytes / (dom_us * 1e-6) / 1e9
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": committed_traffic("decode_ffn"), "kernel": "decode_ffn_kernel (T=1)",
                "algorithmic_bytes_per_launch": ffn_bytes, "avg_launch_us": dom_us,
                "avg_resident_us": resident_us, "launches_timed": t_n,
                "how": "mean %globaltimer span of the kernel's first CTA from its wait on the router kernel "
                       "returning to its end (avg_resident_us: from its start, which overlaps the router kernel), "
                       "accumulated on the device inside the same graph of 1000 PDL-chained calls (no event "
                       f"between kernels); that graph ran at {timed_graph_ms_per_step:.3f} ms per step",
                "peak_source": f"{peak_src} hbm_gbs"}
    # whole token against the roofline too
    tok_bytes = experts * 3 * F * nb * 18 + E * H * 4 + H * 4 * 2
    tok_frac = (tok_bytes * value / world) / 1e9 / peak

    # end to end through the host entry point: per token H2D copy of x, forward,
    # D2H copy of y, all captured once and replayed; pinned host buffers
    xh = torch.from_numpy(x_np).pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    wsh = m.alloc_workspace(m.moe_q4_ffn_host_workspace_bytes(base, 1))
    g3 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for i in range(N_TOKENS):
            m.moe_q4_ffn_forward_host(layers[i % replicas], xh[i:i + 1], yh[i:i + 1], wsh, stream=stream)
    torch.cuda.synchronize()
    with torch.cuda.graph(g3, stream=stream):
        for i in range(N_TOKENS):
            m.moe_q4_ffn_forward_host(layers[i % replicas], xh[i:i + 1], yh[i:i + 1], wsh, stream=stream)
    for _ in range(3):
        g3.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev0.record(stream)
    for _ in range(args.steps):
        g3.replay()
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ev0.elapsed_time(ev1)
    e2e_ms = max_over_ranks(e2e_ms, "cuda")
    e2e_value = whole_job_rate(N_TOKENS * args.steps, world, e2e_ms)
    del g3

    extras = set(args.extras.split(",")) if args.extras != "none" else set()
    prefill = None
    if rank == 0 and "prefill" in extras:
        prefill = prefill_lines(m, torch, stream)
    elif rank == 0 and "prefill947" in extras:   # the 947-token line alone (small profiling runs)
        prefill = prefill_lines(m, torch, stream, names=("prefill_t947",))
    stack = stack_lines(m, torch, stream) if rank == 0 and "stack" in extras else None
    chunked = chunked_lines(m, torch, stream) if rank == 0 and "chunked" in extras else None
    gemv = gemv_lines(m, torch, stream) if rank == 0 and "gemv" in extras else None
    batch64 = batch64_lines(m, torch, stream) if rank == 0 and "batch64" in extras else None
    streamed = streamed_lines(m, torch, stream) if rank == 0 and "streamed" in extras else None

    cpu = None
    simd = None
    if rank == 0 and world == 1 and "cpu" in extras:
        v2, n2, dt2, cores2 = simd_sample(x_np, lw, seconds=5.0)
        simd = {"value": v2, "unit": "tokens/s", "cores": cores2, "kind": "simd_w4a8",
                "sample": f"{n2} tokens of the decode workload, {dt2:.1f} s, AVX2/VNNI integer W4A8 "
                          f"(cpu_simd/, the page's CPU decode method) on {cores2} physical cores"}
        v, n, dt, cores = oracle_sample(x_np, lw, seconds=10.0)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{n} tokens of the decode workload (T=1 each, independent), {dt:.1f} s, "
                         f"OpenMP over tokens on {cores} physical cores ({cpu_model()})"}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": WORKLOAD, "tokens_per_step": N_TOKENS, "T_per_call": 1, "hidden": H, "ffn": F,
                   "experts": E, "top_k": k, "shared_expert": True, "weights": "Q4_0", "activations": "Q8_0",
                   "l2": f"weights rotate over {replicas} replicas ({replicas * 228} MB) -> L2-cold",
                   "parallelism": f"replicas x{world} (tokens independent, no collective)",
                   "graph": "1000 calls captured as one CUDA graph"},
        "roofline": roofline,
        "token_hbm_frac": tok_frac,
        "cpu_baseline": cpu,
        "cpu_simd_baseline": simd,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": N_TOKENS * H * 4,
                "d2h_bytes_per_step": N_TOKENS * H * 4, "how": "moe_q4_ffn_forward_host per token (pinned "
                                                              "host x/y), graph-captured"},
        "gpu_launches": kernels_per_step * args.steps,
        "clocks": clk,
        "prefill": prefill,
        "stack": stack,
        "chunked_prefill": chunked,
        "lm_head_gemv": gemv,
        "decode_batches": batch64,
        "host_streamed_experts": streamed,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--replicas", type=int, default=REPLICAS,
                    help="device copies of the decode layer the tokens rotate over (16: L2-cold)")
    ap.add_argument("--extras", default="prefill,stack,chunked,gemv,batch64,streamed,cpu",
                    help="comma list of the extra lines (prefill, prefill947, stack, chunked, gemv, batch64, "
                         "streamed, cpu) or 'none'")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
