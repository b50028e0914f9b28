"""Benchmark of the FP8 W8A8 row-wise linear path on B200.

One step is one pass of the whole path over one batch of synthetic input. For
the default workload (the large dense layer K=5376, N=21504, the only one that
spans the metric's M = 1..65536) a step is:

  1. the QAT q4_0 -> per-channel E4M3 repack of the 21504x5376 weight,
  2. the load-time conversion of an E4M3FNUZ-stored copy of that weight,
  3. the per-token activation quantization and the row-wise FP8 GEMM at
     M = 65536 (64 requests x 1,024 tokens), M = 1 and M = 64,

with every input resident in HBM. Decode GEMMs rotate over weight copies that
together exceed L2 several times, and before each op that would otherwise hit
in L2 the step flushes it (256 MiB written, then 256 MiB read); the flushes
are timed separately and not counted in the step time. Other workloads:
``decode`` (K=2048, N=8192, M = 1/8/64), ``prefill`` (K=4096, N=14336,
M = 128/1024/8192 with the FNUZ load conversion), ``moe`` (8192 tokens,
top-8 of 128 experts, hidden 2048, intermediate 704: routing, quantization,
gather, grouped gate/up GEMM, GeGLU + quantization, grouped down GEMM,
combine), ``tiny`` (K=256, N=128, M=4) and ``large8k`` (the large layer at
M=8192, for profiling). Prefill GEMMs (M > 128, FP8 and int8) go through the
workspace entry points (``fp8_rowwise_linear_ws`` / ``int8_rowwise_linear_ws``,
one zero-filled workspace per workload), so that a partial last wave of CTA
pair tiles is split by k-blocks; at M = 65536 and 8192 there are too many waves
for the split and the GEMM is the plain one.

Timing: the step is one CUDA graph replayed K times after W warm-up steps,
with CUDA events on the launching stream; ops of at least 200 us are timed
inside the step, shorter ones as the median of 5 replays of a graph of
back-to-back launches of that op alone. SM clocks and throttle reasons are
sampled with nvidia-smi during the timed region.

Output: one JSON line (rank 0). ``value`` is GEMM TFLOP/s of the whole step
(all ranks' FLOPs / max-over-ranks device time); ``kernels`` breaks the step
into ops with their own time, TFLOP/s, GB/s of algorithmic bytes and roofline
fractions - against the measured denominators (the HBM copy; FP8 dense = 2 x
the bf16 cuBLAS figure, the burst one for timed regions under 2 s, else the
sustained one) and against the spec (8 TB/s, 4.5 PF), and for tensor-bound ops
against the FP8 ceiling torch._scaled_mm reaches on the box; ``roofline`` is
the dominant kernel's; ``e2e`` repeats the step through the public API from
pinned host buffers with the copies in the timed region; ``cpu_baseline`` times
the CPU oracle on a bounded sample. A default single-GPU run of ``large`` also
times the ops of ``decode``, ``prefill`` and ``moe`` (each in its own step
graph) and appends them to ``kernels``, so one line covers every
configuration; ``value`` and ``roofline`` stay those of ``large``.

``--impl reference`` times the CPU oracle itself (rank 0 only) on a bounded
sample of the same workload and prints the same JSON line with
``"impl": "reference"``.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 W8A8 row-wise linear TFLOP/s and GB/s, % of roofline, M=1..65536"
UNIT = "TFLOP/s"

# Fallback denominators (used only if MEASURED_PEAKS.json is absent).
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
FP8_PER_BF16 = 2.0  # nominal dense ratio, 4.5 PF fp8 / 2.25 PF bf16
SPEC_FP8_TFLOPS = 4500.0  # B200 dense FP8, vendor spec
SPEC_HBM_GBS = 8000.0     # B200 HBM3e, about 8 TB/s
SPEC_BF16_TFLOPS = 2250.0  # B200 dense bf16, vendor spec


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS,
            "bf16_sustained": FALLBACK_BF16_TFLOPS_SUSTAINED, "source": "fallback"}


# --------------------------------------------------------------------- workloads
WORKLOADS = {
    "large": dict(K=5376, N=21504, Ms=(65536, 1, 64), seed=3, outl=0.01, repack=True, fnuz=True,
                  desc="large dense layer K=5376 N=21504, M in {65536,1,64}, QAT repack + FNUZ load conversion"),
    "large8k": dict(K=5376, N=21504, Ms=(8192, 1, 64), seed=3, outl=0.01, repack=True, fnuz=True,
                    desc="large dense layer K=5376 N=21504 at M in {8192,1,64} (profiling size), repack + FNUZ"),
    "decode": dict(K=2048, N=8192, Ms=(1, 8, 64), seed=1, outl=0.01, repack=False, fnuz=False,
                   builds=True, siblings=3,
                   desc="decode GEMM sweep K=2048 N=8192, M in {1,8,64}; int8 W8A8 and W4A16 builds; "
                        "three sibling linears sharing one quantized x"),
    "prefill": dict(K=4096, N=14336, Ms=(8192, 1024, 128), seed=2, outl=0.01, repack=False, fnuz=True,
                    builds=True,
                    desc="prefill GEMM K=4096 N=14336, M in {8192,1024,128}, FNUZ load conversion; "
                         "int8 W8A8 and W4A16 builds"),
    "tiny": dict(K=256, N=128, Ms=(4,), seed=0, outl=0.0, repack=True, fnuz=False,
                 desc="tiny W8A8 linear M=4 K=256 N=128"),
    "moe": dict(moe=True, tokens=8192, hidden=2048, inter=704, experts=128, top_k=8, seed=4, outl=0.01,
                desc="MoE layer: 128 experts (gate/up/down, hidden 2048, inter 704), 8192 tokens top-8"),
}


def gemm_flops(M, N, K):
    return 2.0 * M * N * K


def linear_bytes(M, N, K):
    """Algorithmic HBM bytes of quantize + GEMM (quantizer separate, so x8 and
    s_tok are written and read back once)."""
    quant = 2 * M * K + M * K + 4 * M
    gemm = M * K + N * K + 4 * M + 4 * N + 2 * M * N
    return quant, gemm


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------------- our arm
def _pinned(torch, a):
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a)
    return t.pin_memory()


def setup_dense(torch, f, wl, seed, dev, flushable):
    """Inputs and ops of a dense-layer workload. Returns (ops, h, D, outs)."""
    from workloads import activations_bf16, q4_weights

    K, N, Ms = wl["K"], wl["N"], wl["Ms"]
    q4, d = q4_weights(N, K, seed=seed)
    h = {"q4": _pinned(torch, q4), "d": _pinned(torch, d)}
    for M in Ms:
        h[f"x{M}"] = _pinned(torch, activations_bf16(M, K, seed=seed + M, outlier_frac=wl["outl"]))
    D = {k: v.to(dev) for k, v in h.items()}
    for M in Ms:
        D[f"x{M}"] = D[f"x{M}"].view(torch.bfloat16)
    w8, s_ch = f.repack_qat(D["q4"], D["d"])
    if wl["fnuz"]:
        # The E4M3FNUZ-stored copy of the same weights: identical bytes, doubled
        # scales (every E4M3 code the repack emits means half as much in FNUZ).
        D["wf"] = w8.clone()
        D["sf"] = s_ch * 2
        h["wf"] = D["wf"].cpu().pin_memory()
        h["sf"] = D["sf"].cpu().pin_memory()
    w8c = torch.empty_like(w8)
    s_c = torch.empty_like(s_ch)
    bufs = {}
    for M in Ms:
        bufs[M] = (torch.empty((M, K), dtype=torch.uint8, device=dev),
                   torch.empty((M,), dtype=torch.float32, device=dev),
                   torch.empty((M, N), dtype=torch.bfloat16, device=dev))
    # Decode-sized GEMMs stream their weights from HBM: in the step each one
    # follows an L2 flush; timed alone, they rotate over weight copies that
    # together exceed 2.5x the L2.
    wsrc = (w8c, s_c) if wl["fnuz"] else (w8, s_ch)
    ncopies = max(2, -(-int(2.5 * 126e6) // (N * K)))
    wcopies = [wsrc[0]] + [wsrc[0].clone() for _ in range(ncopies - 1)]

    # the GEMM workspace that lets a partial last wave of pair tiles be split
    # by k-blocks (zero-filled once; every call leaves its flags zero)
    gws = f.linear_workspace(dev)
    L = []  # (name, fn(rotation), flops, bytes, bound, flushed_before, launches)
    if wl["repack"]:
        L.append(("repack_qat", lambda i: f.repack_qat(D["q4"], D["d"], w8, s_ch), 0.0,
                  N * K * 1.625 + 4 * N, "hbm", False, 1))
    if wl["fnuz"]:
        L.append(("convert_fnuz", lambda i: f.convert_fnuz(D["wf"], D["sf"], w8c, s_c), 0.0,
                  2.0 * N * K + 8 * N, "hbm", False, 1))
    for M in Ms:
        x8, st, y = bufs[M]
        qb, gb = linear_bytes(M, N, K)
        fl = gemm_flops(M, N, K)
        if M > 128:
            L.append((f"quant_act[M={M}]", lambda i, x=D[f"x{M}"], x8=x8, st=st: f.quant_act(x, x8, st),
                      0.0, qb, "hbm", False, 1))
            L.append((f"gemm_prefill[M={M}]",
                      lambda i, x8=x8, st=st, y=y: f.rowwise_linear_ws(x8, st, wsrc[0], wsrc[1], gws, y),
                      fl, gb, "tensor", False, 1))
        else:
            L.append((f"linear_decode[M={M}]",
                      lambda i, x=D[f"x{M}"], x8=x8, st=st, y=y: f.linear(
                          x, wcopies[i % ncopies], wsrc[1], y, x8, st),
                      fl, qb + gb, "hbm", flushable, 2))
    if wl.get("siblings"):
        # q/k/v-like siblings of one activation at M = 1: x quantized once, then
        # the GEMMs as a chain of dependents (fp8_linear_bf16_siblings)
        ns = wl["siblings"]
        M = 1
        x8, st, _ = bufs[M]
        sib_y = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in range(ns)]
        qb, gb = linear_bytes(M, N, K)
        L.append((f"linear_siblings_x{ns}[M={M}]",
                  lambda i, x=D[f"x{M}"], x8=x8, st=st: f.linear_siblings(
                      x, [(wcopies[(i * ns + j) % ncopies], wsrc[1]) for j in range(ns)], sib_y, x8, st),
                  ns * gemm_flops(M, N, K), qb + ns * gb - (ns - 1) * (M * K + 4 * M), "hbm", flushable,
                  1 + ns))
    if wl.get("builds"):
        # the int8 W8A8 build (int8 weights per channel, int8 activations per
        # token) and the W4A16 build (the QAT int4 weights, bf16 activations)
        # of the same layer, at every M
        w8i, s8i = f.int8_repack_qat(D["q4"], D["d"])
        i8copies = [w8i] + [w8i.clone() for _ in range(ncopies - 1)]
        ncq = max(2, -(-int(2.5 * 126e6) // int(N * K * 0.625)))
        q4copies = [(D["q4"], D["d"])] + [(D["q4"].clone(), D["d"].clone()) for _ in range(ncq - 1)]
        ws = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
        for M in Ms:
            x8, st, y = bufs[M]
            x8i = torch.empty((M, K), dtype=torch.int8, device=dev)
            qb, gb = linear_bytes(M, N, K)
            fl = gemm_flops(M, N, K)
            if M > 128:
                L.append((f"int8_quant_act[M={M}]", lambda i, x=D[f"x{M}"], x8i=x8i, st=st: f.int8_quant_act(x, x8i, st),
                          0.0, qb, "hbm", False, 1))
                L.append((f"int8_gemm[M={M}]",
                          lambda i, x8i=x8i, st=st, y=y: f.int8_rowwise_linear_ws(x8i, st, w8i, s8i, gws, y),
                          fl, gb, "tensor", False, 1))
                # unpack to the workspace (0.625 B in, 2 B out per weight), then the bf16 GEMM
                L.append((f"w4a16_unpack[N={N}]", lambda i: f.w4a16_dequant(D["q4"], D["d"], ws), 0.0,
                          N * K * 2.625, "hbm", False, 1))
                L.append((f"w4a16_bf16_gemm[M={M}]", lambda i, x=D[f"x{M}"], y=y: f.bf16_linear(x, ws, y),
                          fl, 2.0 * M * K + 2.0 * N * K + 2.0 * M * N, "tensor_bf16", False, 1))
            else:
                L.append((f"int8_linear_decode[M={M}]",
                          lambda i, x=D[f"x{M}"], x8i=x8i, st=st, y=y: f.int8_linear(
                              x, i8copies[i % ncopies], s8i, y, x8i, st),
                          fl, qb + gb, "hbm", flushable, 2))
                wsb = None if f.w4a16_workspace_bytes(M, N, K) == 0 else ws
                L.append((f"w4a16_linear_decode[M={M}]",
                          lambda i, x=D[f"x{M}"], y=y, wsb=wsb: f.w4a16_linear(
                              x, q4copies[i % ncq][0], q4copies[i % ncq][1], y, wsb),
                          fl, N * K * 0.625 + 2.0 * M * K + 2.0 * M * N, "hbm", flushable, 1))
    outs = [bufs[M][2] for M in Ms]
    cfg = {"K": K, "N": N, "M": list(Ms)}
    return L, h, D, outs, cfg


def setup_moe(torch, f, wl, seed, dev):
    """The MoE layer: route, quantize, gather, gate/up GEMM with the GeGLU
    unit in its epilogue, quantization of h, down GEMM, combine. Expert
    weights are resident (repacked, and the gate/up rows interleaved, at
    setup)."""
    from workloads import activations_bf16, f32_to_bf16_bits, moe_routing, q4_weights

    T, Hd, I, E, k = wl["tokens"], wl["hidden"], wl["inter"], wl["experts"], wl["top_k"]
    R = T * k
    h = {"x": _pinned(torch, activations_bf16(T, Hd, seed=seed, outlier_frac=wl["outl"])),
         "ids": _pinned(torch, moe_routing(T, E, k, seed=seed))}
    D = {key: v.to(dev) for key, v in h.items()}
    D["x"] = D["x"].view(torch.bfloat16)
    wgu, sgu = f.repack_qat(*[torch.from_numpy(a).to(dev) for a in q4_weights(E * 2 * I, Hd, seed=seed + 1)])
    wgu, sgu = f.moe_interleave_gate_up(wgu, sgu, E, I)  # load-time layout of the fused GeGLU
    wdn, sdn = f.repack_qat(*[torch.from_numpy(a).to(dev) for a in q4_weights(E * Hd, I, seed=seed + 2)])
    perm = torch.empty(R, dtype=torch.int32, device=dev)
    inv = torch.empty(R, dtype=torch.int32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    x8 = torch.empty((T, Hd), dtype=torch.uint8, device=dev)
    st = torch.empty((T,), dtype=torch.float32, device=dev)
    xr = torch.empty((R, Hd), dtype=torch.uint8, device=dev)
    sr = torch.empty((R,), dtype=torch.float32, device=dev)
    hb = torch.empty((R, I), dtype=torch.bfloat16, device=dev)
    h8 = torch.empty((R, I), dtype=torch.uint8, device=dev)
    sh = torch.empty((R,), dtype=torch.float32, device=dev)
    dn = torch.empty((R, Hd), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, Hd), dtype=torch.bfloat16, device=dev)
    ids = D["ids"]

    # the bf16 router (router.proj stays bf16 in every build) and its top-k
    # choice with softmax weights: computed as the layer does; the expert path
    # below routes by the workload's seeded uniform ids, so that every expert
    # gets its binomial share of the 65,536 rows as the configuration fixes
    w_router = torch.from_numpy(f32_to_bf16_bits(
        (np.random.default_rng(seed + 3).standard_normal((E, Hd)) * Hd ** -0.5).astype(np.float32)).view(np.int16)
    ).to(dev).view(torch.bfloat16)
    logits = torch.empty((T, E), dtype=torch.bfloat16, device=dev)
    r_ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    r_w = torch.empty((T, k), dtype=torch.float32, device=dev)

    def route(i):
        f.raw.fp8_moe_route(ids.data_ptr(), T, k, E, perm.data_ptr(), inv.data_ptr(), off.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)

    fl_gu = gemm_flops(R, 2 * I, Hd)
    fl_dn = gemm_flops(R, Hd, I)
    L = [
        ("router_bf16_gemm", lambda i: f.bf16_linear(D["x"], w_router, logits), gemm_flops(T, E, Hd),
         2.0 * T * Hd + 2.0 * E * Hd + 2.0 * T * E, "hbm", False, 1),
        ("router_topk", lambda i: f.moe_topk(logits, k, r_ids, r_w), 0.0, 2.0 * T * E + 8.0 * T * k,
         "hbm", False, 1),
        ("moe_route", route, 0.0, 4.0 * R * 3 + 4 * (E + 1), "latency", False, 3),
        ("quant_act", lambda i: f.quant_act(D["x"], x8, st), 0.0, 3.0 * T * Hd + 4 * T, "hbm", False, 1),
        ("moe_gather", lambda i: f.moe_gather(x8, st, perm, k, xr, sr), 0.0,
         1.0 * T * Hd + 1.0 * R * Hd + 8 * R, "hbm", False, 1),
        ("grouped_gate_up_geglu", lambda i: f.grouped_linear_geglu(xr, sr, off, wgu, sgu, I, hb), fl_gu,
         1.0 * R * Hd + E * 2 * I * Hd + 2.0 * R * I, "tensor", False, 1),
        ("quant_h", lambda i: f.quant_act(hb, h8, sh), 0.0, 3.0 * R * I + 4 * R, "hbm", False, 1),
        ("grouped_down", lambda i: f.grouped_linear(h8, sh, off, wdn, sdn, dn), fl_dn,
         1.0 * R * I + E * Hd * I + 2.0 * R * Hd, "tensor", False, 1),
        ("moe_combine", lambda i: f.moe_combine(dn, inv, T, k, out=out), 0.0,
         2.0 * R * Hd + 2.0 * T * Hd + 4 * R, "hbm", False, 1),
    ]
    cfg = {"tokens": T, "hidden": Hd, "inter": I, "experts": E, "top_k": k}
    return L, h, D, [out], cfg


def max_over_ranks(vals, world, device):
    """Element-wise maximum of per-rank float values over all ranks (a
    float64 all-reduce on ``device``; the identity for one rank)."""
    if world <= 1:
        return [float(v) for v in vals]
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(v) for v in vals], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_tflops(world, flops_per_rank_step, steps, ms):
    """Whole-job throughput: every rank does ``flops_per_rank_step`` per step
    (weak scaling), timed by the slowest rank's ``ms`` for ``steps`` steps."""
    return world * flops_per_rank_step * steps / (ms * 1e-3) / 1e12


def time_ops(torch, step_ops, steps, warmup, flush_l2, stream, on_timed=None):
    """Times one workload's ops. Each op alone: R back-to-back launches in one
    CUDA graph, one event pair around each replay (per-op event nodes would
    add several us to us-scale kernels), the median of 5 replays and their
    spread. Then `steps` steps replayed from one CUDA graph with an event pair
    per step, one per L2 flush (subtracted) and one around every op that runs
    >= 200 us alone (too long for the pair to matter). `on_timed(replay)` is
    called to run the timed replay (it may bracket it with barriers and the
    clock sampler). Returns a dict of per-op and per-step times in ms."""
    for _ in range(warmup):
        for name, fn, *_rest in step_ops:
            fn(0)
    torch.cuda.synchronize()

    def time_alone(fn, reps, trials=5):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(reps):
                fn(r)
        g.replay()
        torch.cuda.synchronize()
        per = []
        for _ in range(trials):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            per.append(a.elapsed_time(b) / reps)
        del g
        return statistics.median(per), (min(per), max(per))

    alone_ms, alone_spread = [], []
    for name, fn, fl, by, bound, flushed, nl in step_ops:
        reps = 40 if flushed else 5
        # a pause first, so that the power state a long preceding op left
        # behind (clocks lowered under the power cap) has recovered
        torch.cuda.synchronize()
        time.sleep(0.3)
        med, spread = time_alone(fn, reps)
        alone_ms.append(med)
        alone_spread.append(spread)

    long_op = [ms >= 0.2 for ms in alone_ms]

    def ev():
        return torch.cuda.Event(enable_timing=True, external=True)

    graph = torch.cuda.CUDAGraph()
    steps_ev, flush_ev, op_ev = [], [], []
    with torch.cuda.graph(graph):
        for _ in range(steps):
            e0, e1 = ev(), ev()
            fl_pairs, op_pairs = [], {}
            e0.record()
            for i, (name, fn, fl, by, bound, flushed, nl) in enumerate(step_ops):
                if flushed:
                    a, b = ev(), ev()
                    a.record()
                    flush_l2()
                    b.record()
                    fl_pairs.append((a, b))
                if long_op[i]:
                    a, b = ev(), ev()
                    a.record()
                    fn(0)
                    b.record()
                    op_pairs[i] = (a, b)
                else:
                    fn(0)
            e1.record()
            steps_ev.append((e0, e1))
            flush_ev.append(fl_pairs)
            op_ev.append(op_pairs)
    graph.replay()  # untimed graph warm-up
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)

    def replay():
        t0.record(stream)
        graph.replay()
        t1.record(stream)
        torch.cuda.synchronize()

    (on_timed or (lambda r: r()))(replay)
    step_ms_list = []
    for (e0, e1), fls in zip(steps_ev, flush_ev):
        step_ms_list.append(e0.elapsed_time(e1) - sum(a.elapsed_time(b) for a, b in fls))
    in_step_ms = {i: float(np.mean([op_ev[s_i][i][0].elapsed_time(op_ev[s_i][i][1])
                                    for s_i in range(steps)]))
                  for i in range(len(step_ops)) if long_op[i]}
    graph_ms = t0.elapsed_time(t1)
    del graph
    op_ms = [in_step_ms.get(i, alone_ms[i]) for i in range(len(step_ops))]
    return {"op_ms": op_ms, "alone_spread": alone_spread, "long_op": long_op,
            "total_ms": float(np.sum(step_ms_list)), "graph_ms": graph_ms}


def roofline_peaks(peaks, timed_s, scaled_mm):
    """Denominators for one timed region. The measured bf16 cuBLAS figure is
    taken as a burst for regions under 2 s (the part stays near its boost
    clock) and as sustained for longer ones; FP8 dense = 2 x bf16 (the nominal
    ratio, 4.5 / 2.25 PF). Spec denominators beside them: 4.5 PF FP8 dense and
    8 TB/s HBM3e."""
    burst = timed_s < 2.0
    bf16 = peaks["bf16"] if burst else peaks["bf16_sustained"]
    return {
        "fp8": bf16 * FP8_PER_BF16, "bf16": bf16,
        "fp8_note": (f"fp8 dense = 2 x {peaks['source']} {'burst' if burst else 'sustained'} bf16 cuBLAS "
                     f"({bf16}); timed region {timed_s:.2f} s"),
        "hbm": peaks["hbm_gbs"], "hbm_note": f"{peaks['source']} HBM copy",
        "fp8_spec": SPEC_FP8_TFLOPS, "hbm_spec": SPEC_HBM_GBS,
        "fp8_scaled_mm": scaled_mm,
    }


def kernel_rows(step_ops, t, pk, workload):
    rows = []
    for i, ((name, fn, fl, by, bound, pre, nl), ms) in enumerate(zip(step_ops, t["op_ms"])):
        k = {"workload": workload, "op": name, "us": round(ms * 1e3, 2),
             "gbs": round(by / (ms * 1e-3) / 1e9, 1), "tflops": round(fl / (ms * 1e-3) / 1e12, 1),
             "bound": bound, "timed": "in step" if t["long_op"][i] else "alone, back to back (median of 5)"}
        if not t["long_op"][i]:
            k["us_range"] = [round(t["alone_spread"][i][0] * 1e3, 2), round(t["alone_spread"][i][1] * 1e3, 2)]
        if bound == "tensor":
            k["frac"] = round(k["tflops"] / pk["fp8"], 3)
            k["frac_spec"] = round(k["tflops"] / pk["fp8_spec"], 3)
            if pk["fp8_scaled_mm"]:
                k["frac_scaled_mm"] = round(k["tflops"] / pk["fp8_scaled_mm"], 3)
        elif bound == "tensor_bf16":  # bf16 MMAs: the measured bf16 cuBLAS figure, 2.25 PF spec
            k["frac"] = round(k["tflops"] / pk["bf16"], 3)
            k["frac_spec"] = round(k["tflops"] / SPEC_BF16_TFLOPS, 3)
        elif bound == "hbm":
            k["frac"] = round(k["gbs"] / pk["hbm"], 3)
            k["frac_spec"] = round(k["gbs"] / pk["hbm_spec"], 3)
        rows.append(k)
    return rows


def scaled_mm_ceiling(torch, dev):
    """The box's FP8 GEMM ceiling through the library route: torch._scaled_mm
    (e4m3 x e4m3 -> bf16 with row-wise fp32 scales) at 8192^3, best of 10
    after warm-up. A timing-only measurement beside the product path; None
    where the build has no row-wise FP8 scaled mm."""
    n = 8192
    try:
        g = torch.Generator(device=dev).manual_seed(0)
        a = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev, generator=g).to(torch.float8_e4m3fn).t()
        sa = torch.ones((n, 1), device=dev, dtype=torch.float32)
        sb = torch.ones((1, n), device=dev, dtype=torch.float32)
        out = torch.empty((n, n), device=dev, dtype=torch.bfloat16)

        def mm():
            torch._scaled_mm(a, b, scale_a=sa, scale_b=sb, out_dtype=torch.bfloat16, out=out)

        for _ in range(5):
            mm()
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b, out
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:
        return None


# The other workloads whose ops the default run also measures (rank 0 of a
# single-GPU run), so that one bench line covers every configuration.
EXTRA_WORKLOADS = ("decode", "prefill", "moe")


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import fp8_w8a8_linear_b200 as f

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MiB
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # Write 256 MiB (evicts the cache), then read another 256 MiB so the
        # write-back of those dirty lines happens here, not inside the next op.
        flush.zero_()
        torch.sum(flush_rd, dim=0, out=flush_sum)

    def setup(name):
        wl = WORKLOADS[name]
        seed = wl["seed"] + 1000 * rank  # each rank has its own batch (weak scaling)
        if wl.get("moe"):
            return setup_moe(torch, f, wl, seed, dev)
        return setup_dense(torch, f, wl, seed, dev, True)

    wl = WORKLOADS[args.workload]
    step_ops, h, D, outs, cfg = setup(args.workload)
    n_launch_per_step = sum(o[6] for o in step_ops)

    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    sampler = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    clocks = {}

    def timed(replay):
        sampler.start()
        time.sleep(0.25)
        replay()  # under the clock sampler only
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        replay()
        if world > 1:
            dist.barrier()
        clocks.update(sampler.stop())

    t = time_ops(torch, step_ops, args.steps, args.warmup, flush_l2, stream, on_timed=timed)
    assert f.device_status() == 0, "device status set while timing"
    status = 0
    total_ms = t["total_ms"]
    step_ms = total_ms / args.steps
    if world > 1:
        total_ms = max_over_ranks([total_ms], world, dev)[0]
        step_ms = total_ms / args.steps
    flops_step = sum(o[2] for o in step_ops)
    value = job_tflops(world, flops_step, args.steps, total_ms)
    op_ms = t["op_ms"]

    peaks = load_peaks()
    smm = scaled_mm_ceiling(torch, dev) if (rank == 0 and world == 1) else None
    pk = roofline_peaks(peaks, t["graph_ms"] * 1e-3, smm)
    kernels = kernel_rows(step_ops, t, pk, args.workload)
    dom = max(range(len(step_ops)), key=lambda i: op_ms[i])  # the longest op of the step
    dname, _, dfl, dby, dbound, _, _ = step_ops[dom]
    dms = op_ms[dom]
    if dbound == "tensor":
        ach = round(dfl / (dms * 1e-3) / 1e12, 1)
        roof = {"kernel": dname, "bound": "tensor", "achieved": ach, "peak": round(pk["fp8"], 1),
                "unit": "TFLOP/s", "peak_note": pk["fp8_note"],
                "peak_spec": pk["fp8_spec"], "frac_spec": round(ach / pk["fp8_spec"], 3)}
        if smm:
            roof["peak_scaled_mm"] = round(smm, 1)
            roof["frac_scaled_mm"] = round(ach / smm, 3)
    else:
        ach = round(dby / (dms * 1e-3) / 1e9, 1)
        roof = {"kernel": dname, "bound": "hbm", "achieved": ach, "peak": pk["hbm"], "unit": "GB/s",
                "peak_note": pk["hbm_note"], "peak_spec": pk["hbm_spec"],
                "frac_spec": round(ach / pk["hbm_spec"], 3)}
    roof["frac"] = round(roof["achieved"] / roof["peak"], 3)
    roof["traffic"] = TRAFFIC.get((args.workload, dname))

    # ---- end to end through the public API, from pinned host buffers: the
    # step's inputs are copied in and its results read back every step.
    e2e_steps = max(1, min(args.steps, 3))
    outs_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    h2d = sum(v.numel() * v.element_size() for v in h.values())
    d2h = sum(o.numel() * o.element_size() for o in outs_host)

    def e2e_step():
        for key in h:
            D[key].view(h[key].dtype).copy_(h[key], non_blocking=True)
        for name, fn, *_ in step_ops:
            fn(0)
        for oh, od in zip(outs_host, outs):
            oh.copy_(od, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ea.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    eb.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ea.elapsed_time(eb)
    if world > 1:
        e2e_ms = max_over_ranks([e2e_ms], world, dev)[0]
    e2e_val = job_tflops(world, flops_step, e2e_steps, e2e_ms)
    status |= f.device_status()
    del step_ops, h, D, outs

    # ---- the other configurations' ops (single-GPU runs of the default
    # workload): each workload's own step graph, ops timed as above.
    others = {}
    if world == 1 and args.workload == "large" and not args.no_extra:
        for name in EXTRA_WORKLOADS:
            ops_x, _, _, _, cfg_x = setup(name)
            clk = {}

            def timed_x(replay, clk=clk):
                sampler.start()
                time.sleep(0.25)
                replay()
                clk.update(sampler.stop())

            steps_x = min(args.steps, 10)
            tx = time_ops(torch, ops_x, steps_x, args.warmup, flush_l2, stream, on_timed=timed_x)
            pkx = roofline_peaks(peaks, tx["graph_ms"] * 1e-3, smm)
            kernels += kernel_rows(ops_x, tx, pkx, name)
            fl_x = sum(o[2] for o in ops_x)
            others[name] = {"config": cfg_x, "desc": WORKLOADS[name]["desc"], "steps": steps_x,
                            "ms_per_step": round(tx["total_ms"] / steps_x, 4),
                            "tflops": round(job_tflops(1, fl_x, steps_x, tx["total_ms"]), 2),
                            "peak_note": pkx["fp8_note"], "clocks": clk}
            status |= f.device_status()
            del ops_x
            torch.cuda.empty_cache()

    out = None
    if rank == 0:
        config = {"workload": args.workload, "desc": wl["desc"], **cfg,
                  "parallelism": f"replicas x{world} (independent batches, no collective on the data path)",
                  "l2": ("inputs > L2 for the long ops; before each decode GEMM a 256 MiB write then a "
                         "256 MiB read flush L2 (not timed)")}
        out = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "timing": {"method": "CUDA graph of all timed steps; event pair per step with the L2 flushes' "
                                 "own pairs subtracted; per-op times in step for ops >= 200 us, else "
                                 "from a back-to-back graph of that op alone",
                       "graph_ms_incl_flushes": round(t["graph_ms"], 3)},
            "data": "synthetic (seeded q4_0-grid weights, bf16 N(0,1) activations with 1% x20 outlier channels)",
            "config": config,
            "kernels": kernels,
            "roofline": roof,
            "denominators": {"fp8_tflops_measured": round(pk["fp8"], 1), "fp8_note": pk["fp8_note"],
                             "fp8_tflops_spec": SPEC_FP8_TFLOPS,
                             "fp8_tflops_scaled_mm": None if smm is None else round(smm, 1),
                             "scaled_mm_how": "torch._scaled_mm e4m3, row-wise fp32 scales, bf16 out, "
                                              "8192^3, best of 10 (library GEMM, off the product path)",
                             "hbm_gbs_measured": pk["hbm"], "hbm_gbs_spec": SPEC_HBM_GBS},
            "other_workloads": others,
            "gpu_launches": n_launch_per_step * args.steps,
            "clocks": clocks,
            "device_status": status,
            "e2e": {"value": round(e2e_val, 3), "unit": UNIT, "steps": e2e_steps,
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        }
    return out


# Measured DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum)
# of the dominant kernel, from the ncu summaries under profiles/, keyed by
# (workload, op); reset to absent whenever that kernel changes. The M=65536
# figure is the M=8192 capture of the same K and N scaled by 8 (x8, y and
# the number of weight re-reads all grow in proportion to M).
TRAFFIC = {
    ("large8k", "gemm_prefill[M=8192]"): 614.62e6,
    ("large", "gemm_prefill[M=65536]"): 8 * 614.62e6,
}


# --------------------------------------------------------------------- oracle arm
def oracle_sample_moe(wl, rank: int = 0):
    """The CPU oracle on a bounded sample of one MoE step: the routing sort of
    all tokens, the activation quant of all tokens, and for the first two
    experts the repack of their weights, the gather, gate/up GEMM, GeGLU,
    quant and down GEMM of their rows."""
    import oracle
    from oracle import moe
    from workloads import activations_bf16, moe_routing, q4_weights

    T, Hd, I, E, k = wl["tokens"], wl["hidden"], wl["inter"], wl["experts"], wl["top_k"]
    seed = wl["seed"] + 1000 * rank
    xb = activations_bf16(T, Hd, seed=seed, outlier_frac=wl["outl"])
    ids = moe_routing(T, E, k, seed=seed)
    ne = 2
    q_gu = q4_weights(E * 2 * I, Hd, seed=seed + 1, rows=slice(0, ne * 2 * I))
    q_dn = q4_weights(E * Hd, I, seed=seed + 2, rows=slice(0, ne * Hd))
    t0 = time.perf_counter()
    perm, inv, off = moe.route_sort(ids, E)
    a = oracle.quant_act(xb)
    xs, ss = moe.gather_rows(a.codes, a.scales, perm[:off[ne]], k)
    wgu = oracle.repack_qat(*q_gu)
    wdn = oracle.repack_qat(*q_dn)
    off_s = off[:ne + 1]
    gu = moe.grouped_linear_ref(xs, ss, off_s, wgu.codes.reshape(ne, 2 * I, Hd), wgu.scales.reshape(ne, 2 * I))
    gu_b = (np.asarray(gu, np.float32).view(np.uint32) >> 16).astype(np.uint16)
    h = moe.geglu_bf16(gu_b, I)
    hq = oracle.quant_act(h)
    moe.grouped_linear_ref(hq.codes, hq.scales, off_s, wdn.codes.reshape(ne, Hd, I), wdn.scales.reshape(ne, Hd))
    dt = time.perf_counter() - t0
    rows = int(off[ne])
    flops = gemm_flops(rows, 2 * I, Hd) + gemm_flops(rows, Hd, I)
    desc = (f"routing sort and activation quant of all {T} tokens; weights repack, gather, gate/up GEMM, "
            f"GeGLU, quant and down GEMM for experts 0..{ne - 1} ({rows} rows)")
    return dt, flops, desc


def oracle_sample(workload: str, rank: int = 0):
    """The CPU oracle on a bounded sample of one step: the repack and FNUZ
    conversion of 2048 weight rows, the activation quant of min(M, 2048) token
    rows per M, and the exact GEMM of those tokens against those 2048 weight
    rows. Returns (seconds, GEMM FLOPs, description)."""
    import oracle
    from workloads import activations_bf16, q4_weights

    wl = WORKLOADS[workload]
    if wl.get("moe"):
        return oracle_sample_moe(wl, rank)
    K, N = wl["K"], wl["N"]
    ns = min(N, 2048)
    seed = wl["seed"] + 1000 * rank
    q4, d = q4_weights(N, K, seed=seed, rows=slice(0, ns))
    xs = {M: activations_bf16(M, K, seed=seed + M, outlier_frac=wl["outl"], rows=slice(0, min(M, 2048)))
          for M in wl["Ms"]}
    t0 = time.perf_counter()
    w = oracle.repack_qat(q4, d)
    if wl["fnuz"]:
        cn, sn = oracle.fnuz_copy_of_e4m3(w.codes, w.scales)
        oracle.convert_fnuz_to_e4m3(cn, sn)
    flops = 0.0
    for M, xb in xs.items():
        a = oracle.quant_act(xb)
        oracle.rowwise_linear_ref(a.codes, a.scales, w.codes, w.scales)
        flops += gemm_flops(xb.shape[0], ns, K)
    dt = time.perf_counter() - t0
    desc = (f"{ns} of {N} weight rows (repack{', FNUZ conversion' if wl['fnuz'] else ''}), "
            f"min(M,2048) token rows per M in {list(wl['Ms'])} (quant + exact fp64 GEMM vs those rows), K={K}")
    return dt, flops, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info()]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def run_reference(args):
    steps = []
    for i in range(args.warmup + args.steps):
        dt, fl, desc = oracle_sample(args.workload)
        if i >= args.warmup:
            steps.append((dt, fl))
    tot = sum(s[0] for s in steps)
    value = sum(s[1] for s in steps) / tot / 1e12
    wl = WORKLOADS[args.workload]
    cores = blas_threads()
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * tot / len(steps), 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "desc": wl["desc"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="large", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations' ops in a default single-GPU run")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                dt, fl, desc = oracle_sample(args.workload)
                out["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": blas_threads(),
                                       "kind": "oracle", "sample": desc, "seconds": round(dt, 2)}
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
