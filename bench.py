"""Benchmark of the weight-only quantization hot path on B200 GPUs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of every hot-path row over the 7B-class decode layer set
(N, K) = (4096, 4096), (11008, 4096), (4096, 11008):
  quantize_pack int4 asymmetric group-128   (3 launches)
  quantize_pack int8 symmetric per-channel  (3 launches)
  dequantize int4                           (3 launches)
  W4A16 decode GEMV, M = 1                  (3 launches)
  W8A16 decode GEMV, M = 1                  (3 launches)
  W4A16 prefill GEMM, M = 2048 tokens       (3 launches)
plus the 70B-class decode layers (N, K) = (28672, 8192), (8192, 28672):
  W4A16 decode GEMV, M = 1                  (2 launches)
  W8A16 decode GEMV, M = 1                  (2 launches)
Every input is resident in HBM and rotates over ROT copies (ROT x the packed
layer set is far larger than the 126 MB L2), so each part reads cold weights.
Each step is one captured CUDA graph (all parts, one rotation) with external
CUDA event nodes between the parts, so the GPU runs a step without host gaps
and each part's time is the device time between its two event nodes.  `value` is the headline of the metric:
W4A16 decode GEMV GB/s (algorithmic bytes / GEMV time), aggregated over all
ranks.  The other parts, the roofline of every kernel, the configurations
that are not part of the step (70B decode shapes at M = 4, 8, 16, the
2048 x 8192 x 8192 prefill GEMM, the 7.8e9-parameter bulk quantization), an end-to-end number
through the public Python API with host buffers, and the CPU oracle baseline
are reported in the same JSON line.

With --impl reference the CPU oracle is the reference arm: it runs the same
decode step (dequantize + fp64 matmul) on a row sample of the same layers.

Multi-GPU: the path does not shard (one GPU per problem); N ranks run N
independent replicas, launched by torchrun; times are the max over ranks.
"""
import argparse
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

import synthetic  # noqa: E402

METRIC = "W4A16 decode GEMV GB/s (% of HBM peak); prefill GEMM TFLOP/s; quantize GB/s"
LAYERS = synthetic.DECODE_7B
LAYERS_70B = synthetic.DECODE_70B
PREFILL_M = synthetic.PREFILL["M"]
ROT = 8
GEMV_LAUNCH_OVERLAP = 1      # static weights: see qz_set_launch_overlap in qz.h
GROUP = 128
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------------------
# algorithmic work per launch
# ---------------------------------------------------------------------------

def w4_gemv_bytes(M, N, K, g=GROUP):
    return N * K // 2 + N * (K // g) * 3 + 2 * M * K + 2 * M * N


def w8_gemv_bytes(M, N, K):
    return N * K + 2 * N + 2 * M * K + 2 * M * N


def quant_int4_bytes(N, K, g=GROUP):
    return 2 * N * K + N * K // 2 + N * (K // g) * 3


def quant_int8_bytes(N, K):
    return 2 * N * K + N * K + 2 * N


def dequant_int4_bytes(N, K, g=GROUP):
    return quant_int4_bytes(N, K, g)


def gemm_flops(M, N, K):
    return 2 * M * N * K


FP4_BLOCK = {0: 32, 1: 16}     # MXFP4, NVFP4 values per block scale


def fp4_gemv_bytes(M, N, K, kind):
    return N * K // 2 + N * K // FP4_BLOCK[kind] + (4 if kind == 1 else 0) + 2 * M * K + 2 * M * N


def fp4_quant_bytes(N, K, kind):
    return 2 * N * K + N * K // 2 + N * K // FP4_BLOCK[kind]


def gptq_flops(N, K, n):
    """Algorithmic fp64 flops of one GPTQ call (2 per multiply-add): the
    symmetric H = 2 X X^T, one triangle of K^2 / 2 entries over n samples
    (n K^2); the Cholesky of the damped H (K^3 / 3); the triangular inverse
    (K^3 / 3); the weight updates, where quantizing column j moves every later
    column k > j of every row once (K^2 / 2 pairs per row, N K^2 in all,
    whether applied inside a block or by the lazy batch update)."""
    return n * K * K + (2 * K ** 3) // 3 + N * K * K


# fp64 peak of a B200 derived from its unit counts and clock (the pages and
# the measured-peaks file give none): 148 SMs x 64 fp64 FMA lanes x 2 flops
# x 1.965 GHz.
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12
# Dense FP4 tensor-core peak: the measured bf16 peak times the nominal ratio
# of the two (9 PFLOP/s FP4 to 2.25 PFLOP/s bf16, dense).
FP4_TO_BF16_NOMINAL = 4.0


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def ncu_traffic():
    """Per-launch-set DRAM traffic from the committed ncu summary, keyed by
    part, valid only while every source file of the kernel is unchanged since
    the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    import hashlib
    with open(path) as f:
        data = json.load(f)
    out = {}
    for part, rec in data.get("kernels", {}).items():
        srcs = [os.path.join(ROOT, f) for f in rec.get("sources", [])]
        if not srcs or not all(os.path.exists(f) for f in srcs):
            continue
        h = hashlib.sha256()
        for f in srcs:
            with open(f, "rb") as fh:
                h.update(fh.read())
        if h.hexdigest()[:16] == rec.get("sources_sha256_16"):
            out[part] = rec
    return out


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self):
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self, device_index):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r.split(",") for r in self.tmp.read().strip().splitlines() if r.strip()]
        os.unlink(self.tmp.name)
        rows = [[c.strip() for c in r] for r in rows if len(r) >= 9]
        mine = [r for r in rows if r[0] == str(device_index)] or rows
        if not mine:
            return None
        sm = [float(r[1]) for r in mine if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in mine if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in mine for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(mine)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

class LayerSet:
    """Resident inputs/outputs of one step, ROT rotating copies of every input."""

    def __init__(self, qz, dev):
        self.qz, self.dev = qz, dev
        self.w, self.c4, self.s4, self.z4, self.c8, self.s8 = ([] for _ in range(6))
        for p in range(ROT):
            w_p, c4_p, s4_p, z4_p, c8_p, s8_p = [], [], [], [], [], []
            for li, (N, K) in enumerate(LAYERS):
                if p == 0:
                    w = synthetic.weights(N, K, sigma=0.02, seed=1 + li, device=dev)
                else:
                    w = self.w[0][li].clone()
                c4, s4, z4 = qz.qz_quantize_pack(w, 4, False, GROUP)
                c8, s8, _ = qz.qz_quantize_pack(w, 8, True, K)
                w_p.append(w); c4_p.append(c4); s4_p.append(s4); z4_p.append(z4)
                c8_p.append(c8); s8_p.append(s8)
            self.w.append(w_p); self.c4.append(c4_p); self.s4.append(s4_p)
            self.z4.append(z4_p); self.c8.append(c8_p); self.s8.append(s8_p)
        # outputs (written every step) and activations
        self.q4 = [qz.qz_quantize_pack(self.w[0][li], 4, False, GROUP) for li in range(len(LAYERS))]
        self.q8 = [qz.qz_quantize_pack(self.w[0][li], 8, True, K)
                   for li, (N, K) in enumerate(LAYERS)]
        self.deq = [torch.empty((N, K), dtype=torch.bfloat16, device=dev) for N, K in LAYERS]
        self.a1 = [synthetic.activations(1, K, seed=50 + li, device=dev)
                   for li, (N, K) in enumerate(LAYERS)]
        self.ap = [synthetic.activations(PREFILL_M, K, seed=60 + li, device=dev)
                   for li, (N, K) in enumerate(LAYERS)]
        # 70B-class decode layers (W4A16 and W8A16 at M = 1): packed weights
        # only, ROT copies each (ROT x 246 MB int4, ROT x 470 MB int8)
        self.c4_70, self.s4_70, self.z4_70, self.c8_70, self.s8_70 = ([] for _ in range(5))
        for li, (N, K) in enumerate(LAYERS_70B):
            w = synthetic.weights(N, K, sigma=0.015, seed=4 + li, device=dev)
            c4, s4, z4 = qz.qz_quantize_pack(w, 4, False, GROUP)
            c8, s8, _ = qz.qz_quantize_pack(w, 8, True, K)
            del w
            self.c4_70.append([c4] + [c4.clone() for _ in range(ROT - 1)])
            self.s4_70.append([s4] + [s4.clone() for _ in range(ROT - 1)])
            self.z4_70.append([z4] + [z4.clone() for _ in range(ROT - 1)])
            self.c8_70.append([c8] + [c8.clone() for _ in range(ROT - 1)])
            self.s8_70.append([s8] + [s8.clone() for _ in range(ROT - 1)])
        self.a1_70 = [synthetic.activations(1, K, seed=70 + li, device=dev)
                      for li, (N, K) in enumerate(LAYERS_70B)]
        self.y4_70 = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for N, K in LAYERS_70B]
        self.y8_70 = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for N, K in LAYERS_70B]
        self.y4 = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for N, K in LAYERS]
        self.y8 = [torch.empty((1, N), dtype=torch.bfloat16, device=dev) for N, K in LAYERS]
        self.yg = [torch.empty((PREFILL_M, N), dtype=torch.bfloat16, device=dev) for N, K in LAYERS]
        ws = 256
        for N, K in LAYERS:
            ws = max(ws, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 1, N, K, GROUP),
                     qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMV, 1, N, K, K),
                     qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, PREFILL_M, N, K, GROUP))
        for N, K in LAYERS_70B:
            ws = max(ws, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 1, N, K, GROUP),
                     qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMV, 1, N, K, K))
        self.ws = torch.zeros(ws, dtype=torch.uint8, device=dev)

    # each part issues its launches for rotation p on the current stream
    def quant4(self, p):
        for li, (N, K) in enumerate(LAYERS):
            c, s, z = self.q4[li]
            self.qz.qz_quantize_pack(self.w[p][li], 4, False, GROUP, codes=c, scales=s, zeros=z)

    def quant8(self, p):
        for li, (N, K) in enumerate(LAYERS):
            c, s, _ = self.q8[li]
            self.qz.qz_quantize_pack(self.w[p][li], 8, True, K, codes=c, scales=s)

    def dequant(self, p):
        for li, (N, K) in enumerate(LAYERS):
            self.qz.qz_dequantize(self.c4[p][li], self.s4[p][li], self.z4[p][li], N, K, 4, False,
                                  GROUP, out=self.deq[li])

    def gemv4(self, p):
        for li, (N, K) in enumerate(LAYERS):
            self.qz.qz_w4a16_gemv(self.a1[li], self.c4[p][li], self.s4[p][li], self.z4[p][li], N,
                                  K, GROUP, y=self.y4[li], workspace=self.ws)

    def gemv8(self, p):
        for li, (N, K) in enumerate(LAYERS):
            self.qz.qz_w8a16_gemv(self.a1[li], self.c8[p][li], self.s8[p][li], N, K,
                                  y=self.y8[li], workspace=self.ws)

    def gemv4_70b(self, p):
        for li, (N, K) in enumerate(LAYERS_70B):
            self.qz.qz_w4a16_gemv(self.a1_70[li], self.c4_70[li][p], self.s4_70[li][p],
                                  self.z4_70[li][p], N, K, GROUP, y=self.y4_70[li],
                                  workspace=self.ws)

    def gemv8_70b(self, p):
        for li, (N, K) in enumerate(LAYERS_70B):
            self.qz.qz_w8a16_gemv(self.a1_70[li], self.c8_70[li][p], self.s8_70[li][p], N, K,
                                  y=self.y8_70[li], workspace=self.ws)

    def gemm(self, p):
        for li, (N, K) in enumerate(LAYERS):
            self.qz.qz_w4a16_gemm(self.ap[li], self.c4[p][li], self.s4[p][li], self.z4[p][li], N,
                                  K, GROUP, y=self.yg[li], workspace=self.ws)


PARTS = [  # name, method, unit, work per step, bound, launches per step
    ("quantize_pack_int4_g128", "quant4", "GB/s",
     sum(quant_int4_bytes(N, K) for N, K in LAYERS), "hbm", len(LAYERS)),
    ("quantize_pack_int8_per_channel", "quant8", "GB/s",
     sum(quant_int8_bytes(N, K) for N, K in LAYERS), "hbm", len(LAYERS)),
    ("dequantize_int4", "dequant", "GB/s",
     sum(dequant_int4_bytes(N, K) for N, K in LAYERS), "hbm", len(LAYERS)),
    ("w4a16_gemv_m1", "gemv4", "GB/s", sum(w4_gemv_bytes(1, N, K) for N, K in LAYERS), "hbm",
     len(LAYERS)),
    ("w8a16_gemv_m1", "gemv8", "GB/s", sum(w8_gemv_bytes(1, N, K) for N, K in LAYERS), "hbm",
     len(LAYERS)),
    ("w4a16_gemv_70b_m1", "gemv4_70b", "GB/s",
     sum(w4_gemv_bytes(1, N, K) for N, K in LAYERS_70B), "hbm", len(LAYERS_70B)),
    ("w8a16_gemv_70b_m1", "gemv8_70b", "GB/s",
     sum(w8_gemv_bytes(1, N, K) for N, K in LAYERS_70B), "hbm", len(LAYERS_70B)),
    ("w4a16_gemm_prefill_m2048", "gemm", "TFLOP/s",
     sum(gemm_flops(PREFILL_M, N, K) for N, K in LAYERS), "tensor", len(LAYERS)),
]
LAUNCHES_PER_STEP = sum(p[5] for p in PARTS)


def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise max over ranks of per-rank times (the replicas' timing
    rule: a multi-GPU number is as slow as its slowest rank)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def replica_rate(work_per_rank, seconds, world):
    """Whole-job throughput of `world` independent replicas that each did
    `work_per_rank` in at most `seconds` (max over ranks)."""
    return work_per_rank * world / seconds


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def rate(work, ms, unit):
    if unit == "TFLOP/s":
        return work / (ms * 1e-3) / 1e12
    return work / (ms * 1e-3) / 1e9


def roofline_obj(part, work, ms_per_launch_set, launches, bound, pk, traffic, sustained):
    achieved = rate(work, ms_per_launch_set, "TFLOP/s" if bound == "tensor" else "GB/s")
    if bound == "tensor":
        peak = pk["bf16_tflops_sustained"] if sustained else pk["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        peak, unit = pk["hbm_gbs"], "GB/s"
    t = traffic.get(part)
    return {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4),
            "peak_kind": ("sustained" if (bound == "tensor" and sustained) else "burst")
            + (" of measured" if pk["source"] == "measured" else " of fallback"),
            "traffic": (t["dram_bytes_per_launch_set"] if t else None),
            "algorithmic": work, "launches": launches}


def qz_gemm_kernel_for(M):
    """Which kernel qz_w4a16_gemm / qz_w8a16_gemm run for M tokens."""
    return "decode GEMV" if M <= GEMM_ROUTES_TO_GEMV_UP_TO else "tcgen05 GEMM"


GEMM_ROUTES_TO_GEMV_UP_TO = 32


def read_floor(ls, stream, pk, parts):
    """The floor of the decode GEMV parts: a plain streaming read (cuBLAS
    matrix-vector products over the same packed codes, scales and zeros as
    fp32 words) of
    each step's layers, in the same harness as the step (one CUDA graph per
    rotation of the same resident copies, replayed back to back, timed with
    events).  For the short 7B layers it is a latency floor, not HBM."""
    ones = torch.ones(1 << 15, dtype=torch.float32, device=ls.dev)
    sinks = {}

    def as_matrix(t):
        # each weight row's bytes as fp32 words (codes: N x K/8); a row whose
        # bytes are not a multiple of 4 reads the tensor as a flat matrix
        if t.dim() == 2 and t.shape[1] * t.element_size() % 4 == 0:
            return t.view(torch.float32)
        v = t.reshape(-1).view(torch.float32)
        return v.view(-1, 16 if v.numel() % 16 == 0 else 1)

    def reads(tensors):
        def f(p):
            for i, t in enumerate(tensors(p)):
                # the matrix times a ones vector (the values are irrelevant):
                # cuBLAS's matrix-vector product reads each byte once and
                # writes one word per row
                m = as_matrix(t)
                out = sinks.setdefault((i, m.shape[0]), torch.empty(m.shape[0], dtype=torch.float32,
                                                                    device=ls.dev))
                torch.mv(m, ones[:m.shape[1]], out=out)
        return f

    # every byte the GEMV reads (three reads per layer), and the codes alone
    # (one read per layer, as the GEMV launches once per layer)
    sets = {
        "w4a16_gemv_m1": (reads(lambda p: [x for li in range(len(LAYERS))
                                           for x in (ls.c4[p][li], ls.s4[p][li], ls.z4[p][li])]),
                          sum(w4_gemv_bytes(1, N, K) for N, K in LAYERS)),
        "w4a16_gemv_m1/codes_only": (reads(lambda p: [ls.c4[p][li] for li in range(len(LAYERS))]),
                                     sum(N * K // 2 for N, K in LAYERS)),
        "w4a16_gemv_70b_m1": (reads(lambda p: [x for li in range(len(LAYERS_70B))
                                               for x in (ls.c4_70[li][p], ls.s4_70[li][p],
                                                         ls.z4_70[li][p])]),
                              sum(w4_gemv_bytes(1, N, K) for N, K in LAYERS_70B)),
        "w4a16_gemv_70b_m1/codes_only": (reads(lambda p: [ls.c4_70[li][p]
                                                          for li in range(len(LAYERS_70B))]),
                                         sum(N * K // 2 for N, K in LAYERS_70B)),
    }
    out = {"method": "cuBLAS matrix-vector product (torch.mv) of the packed codes (N x K/8 fp32 "
                     "words), scales and zeros of each layer with a ones vector; one graph per "
                     "rotation, 40 replays"}
    with torch.cuda.stream(stream):
        for name, (f, nbytes) in sets.items():
            graphs = []
            for p in range(ROT):
                f(p)
                graphs.append(capture(lambda p=p: f(p), stream))
            for g in graphs[:3]:
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for i in range(40):
                graphs[i % ROT].replay()
            e1.record(stream)
            e1.synchronize()
            us = e0.elapsed_time(e1) / 40 * 1e3
            part_us = parts[name.split("/")[0]]["ms"] * 1e3
            out[name] = {"floor_us": round(us, 2), "floor_GB/s": round(nbytes / us / 1e3, 1),
                         "floor_frac_hbm": round(nbytes / us / 1e3 / pk["hbm_gbs"], 4),
                         "gemv_us": round(part_us, 2), "gemv_over_floor": round(part_us / us, 3)}
            del graphs
    torch.cuda.synchronize()
    return out


def run_extras(qz, dev, pk, stream):
    """Configurations outside the step, each timed with CUDA events on graphs."""
    out = {}

    def time_graph(g, reps=20, warm=3):
        for _ in range(warm):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / reps

    with torch.cuda.stream(stream):
        # prefill GEMM, M = 2048, N = K = 8192
        cfg = synthetic.PREFILL
        M, N, K = cfg["M"], cfg["N"], cfg["K"]
        w = synthetic.weights(N, K, sigma=cfg["sigma"], seed=cfg["seed"], device=dev)
        a = synthetic.activations(M, K, seed=cfg["seed"] + 1000, device=dev)
        c, s, z = qz.qz_quantize_pack(w, 4, False, GROUP)
        y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        wsp = torch.zeros(max(256, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, M, N, K, GROUP),
                              qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMM, M, N, K, K)),
                          dtype=torch.uint8, device=dev)
        qz.qz_w4a16_gemm(a, c, s, z, N, K, GROUP, y=y, workspace=wsp)
        g = capture(lambda: qz.qz_w4a16_gemm(a, c, s, z, N, K, GROUP, y=y, workspace=wsp), stream)
        ms = time_graph(g)
        tf = gemm_flops(M, N, K) / (ms * 1e-3) / 1e12
        out["prefill_gemm_2048x8192x8192"] = {
            "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
            "frac_of_burst": round(tf / pk["bf16_tflops"], 4),
            "frac_of_sustained": round(tf / pk["bf16_tflops_sustained"], 4)}
        # cuBLAS bf16 GEMM of the same shape, as the practical ceiling
        wb = qz.qz_dequantize(c, s, z, N, K, 4, False, GROUP)
        yb = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        torch.matmul(a, wb.t(), out=yb)
        gb = capture(lambda: torch.matmul(a, wb.t(), out=yb), stream)
        msb = time_graph(gb)
        out["prefill_gemm_2048x8192x8192"]["cublas_bf16_same_shape_TFLOP/s"] = round(
            gemm_flops(M, N, K) / (msb * 1e-3) / 1e12, 1)
        del wb, yb, g, gb, c, s, z
        # W8A16 prefill GEMM, same shape, int8 symmetric per-channel
        c8, s8, _ = qz.qz_quantize_pack(w, 8, True, K)
        qz.qz_w8a16_gemm(a, c8, s8, N, K, y=y, workspace=wsp)
        ms = time_graph(capture(lambda: qz.qz_w8a16_gemm(a, c8, s8, N, K, y=y, workspace=wsp),
                                stream))
        tf = gemm_flops(M, N, K) / (ms * 1e-3) / 1e12
        out["prefill_w8a16_gemm_2048x8192x8192"] = {
            "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
            "frac_of_burst": round(tf / pk["bf16_tflops"], 4),
            "frac_of_sustained": round(tf / pk["bf16_tflops_sustained"], 4)}
        del c8, s8
        # W4A4 prefill (FP4 weights and activations, the activations quantized
        # inside the call), same shape; the FP4 peak is the measured bf16 burst
        # peak times the nominal FP4 : bf16 ratio
        fp4_peak = pk["bf16_tflops"] * FP4_TO_BF16_NOMINAL
        for kind, name in ((1, "nvfp4"), (0, "mxfp4")):
            fc, fs, fts = qz.qz_fp4_quantize(w, kind)
            fsm = qz.qz_fp4_scales_to_mma(fs, N, K, kind)
            wsa = torch.empty(qz.qz_workspace_bytes(qz.QZ_OP_FP4A4_GEMM, M, N, K, 0),
                              dtype=torch.uint8, device=dev)
            qz.qz_fp4a4_gemm(a, fc, fsm, fts, N, K, kind, y=y, workspace=wsa)
            ms = time_graph(capture(
                lambda: qz.qz_fp4a4_gemm(a, fc, fsm, fts, N, K, kind, y=y, workspace=wsa), stream))
            # the activation quantization alone (row-major scales, same work)
            aq = qz.qz_fp4_quantize(a, kind)
            msq = time_graph(capture(lambda: qz.qz_fp4_quantize(
                a, kind, codes=aq[0], scales=aq[1], tensor_scale=aq[2]), stream))
            tf = gemm_flops(M, N, K) / (ms * 1e-3) / 1e12
            out[f"prefill_w4a4_{name}_2048x8192x8192"] = {
                "ms": round(ms, 4), "TFLOP/s": round(tf, 1),
                "fp4_peak_TFLOP/s_derived": round(fp4_peak, 1),
                "frac_of_fp4_peak": round(tf / fp4_peak, 4),
                "activation_quantize_ms": round(msq, 4),
                "note": "ms covers the whole call: activation amax and quantization, then the "
                        "block-scaled tcgen05 GEMM"}
            del fc, fs, fts, fsm, wsa, aq
        del a, y

        # Small-M crossover on the same layer: M <= 32 runs the decode kernel,
        # larger M the tcgen05 GEMM.  Weights rotate over copies larger than L2.
        packs4 = [qz.qz_quantize_pack(w if r == 0 else w.clone(), 4, False, GROUP) for r in range(4)]
        packs8 = [qz.qz_quantize_pack(w if r == 0 else w.clone(), 8, True, K) for r in range(2)]
        sweep = {}
        for Ms in (16, 32, 64, 128, 256, 512):
            a = synthetic.activations(Ms, K, seed=Ms, device=dev)
            y = torch.empty((Ms, N), dtype=torch.bfloat16, device=dev)
            ws = torch.zeros(max(256, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, Ms, N, K, GROUP),
                                 qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMM, Ms, N, K, K)),
                             dtype=torch.uint8, device=dev)

            def f4():
                for c, s, z in packs4:
                    qz.qz_w4a16_gemm(a, c, s, z, N, K, GROUP, y=y, workspace=ws)

            def f8():
                for c, s, _ in packs8:
                    qz.qz_w8a16_gemm(a, c, s, N, K, y=y, workspace=ws)

            f4(); f8()
            ms4 = time_graph(capture(f4, stream)) / len(packs4)
            ms8 = time_graph(capture(f8, stream)) / len(packs8)
            b4, b8 = w4_gemv_bytes(Ms, N, K), w8_gemv_bytes(Ms, N, K)
            if GEMM_ROUTES_TO_GEMV_UP_TO < Ms <= 64:
                # the same tokens through the decode GEMV (up to 64 tokens)
                wsg = torch.zeros(max(256, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, Ms, N, K,
                                                                 GROUP),
                                      qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMV, Ms, N, K, K)),
                                  dtype=torch.uint8, device=dev)

                def g4():
                    for c, s, z in packs4:
                        qz.qz_w4a16_gemv(a, c, s, z, N, K, GROUP, y=y, workspace=wsg)

                def g8():
                    for c, s, _ in packs8:
                        qz.qz_w8a16_gemv(a, c, s, N, K, y=y, workspace=wsg)

                g4(); g8()
                gm4 = time_graph(capture(g4, stream)) / len(packs4)
                gm8 = time_graph(capture(g8, stream)) / len(packs8)
                sweep[f"M{Ms}_decode_gemv"] = {
                    "w4_us": round(gm4 * 1e3, 2), "w4_frac_hbm": round(b4 / gm4 / 1e6 / pk["hbm_gbs"], 4),
                    "w8_us": round(gm8 * 1e3, 2), "w8_frac_hbm": round(b8 / gm8 / 1e6 / pk["hbm_gbs"], 4)}
                del wsg
            sweep[f"M{Ms}"] = {
                "kernel": qz_gemm_kernel_for(Ms),
                "w4_us": round(ms4 * 1e3, 2), "w4_GB/s": round(b4 / ms4 / 1e6, 1),
                "w4_frac_hbm": round(b4 / ms4 / 1e6 / pk["hbm_gbs"], 4),
                "w4_TFLOP/s": round(gemm_flops(Ms, N, K) / (ms4 * 1e-3) / 1e12, 1),
                "w8_us": round(ms8 * 1e3, 2), "w8_GB/s": round(b8 / ms8 / 1e6, 1),
                "w8_frac_hbm": round(b8 / ms8 / 1e6 / pk["hbm_gbs"], 4),
                "w8_TFLOP/s": round(gemm_flops(Ms, N, K) / (ms8 * 1e-3) / 1e12, 1)}
        out["small_m_crossover_8192x8192"] = sweep
        del w, a, y, ws, packs4, packs8

        # 70B decode shapes, W4 and W8, M in {1, 4, 8, 16}
        d70 = {}
        for li, (N, K) in enumerate(synthetic.DECODE_70B):
            w = synthetic.weights(N, K, sigma=0.015, seed=4 + li, device=dev)
            packs4 = [qz.qz_quantize_pack(w if r == 0 else w.clone(), 4, False, GROUP) for r in range(2)]
            packs8 = [qz.qz_quantize_pack(w if r == 0 else w.clone(), 8, True, K) for r in range(2)]
            del w
            for M in synthetic.DECODE_70B_M:
                a = synthetic.activations(M, K, seed=M, device=dev)
                y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                ws = torch.zeros(max(256, qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, N, K, GROUP)),
                                 dtype=torch.uint8, device=dev)

                def f4():
                    for c, s, z in packs4:
                        qz.qz_w4a16_gemv(a, c, s, z, N, K, GROUP, y=y, workspace=ws)

                def f8():
                    for c, s, _ in packs8:
                        qz.qz_w8a16_gemv(a, c, s, N, K, y=y, workspace=ws)

                f4(); f8()
                ms4 = time_graph(capture(f4, stream)) / 2
                ms8 = time_graph(capture(f8, stream)) / 2
                b4, b8 = w4_gemv_bytes(M, N, K), w8_gemv_bytes(M, N, K)
                d70[f"N{N}_K{K}_M{M}"] = {
                    "w4_us": round(ms4 * 1e3, 2), "w4_GB/s": round(b4 / ms4 / 1e6, 1),
                    "w4_frac_hbm": round(b4 / ms4 / 1e6 / pk["hbm_gbs"], 4),
                    "w8_us": round(ms8 * 1e3, 2), "w8_GB/s": round(b8 / ms8 / 1e6, 1),
                    "w8_frac_hbm": round(b8 / ms8 / 1e6 / pk["hbm_gbs"], 4)}
            del packs4, packs8
        out["decode_70b"] = d70

        # FP4 with block scales (MXFP4, NVFP4) on the 70B decode layers, M = 1
        # and 16, weights rotating over two copies; the quantizer on the same
        # layers
        fp4 = {}
        for li, (N, K) in enumerate(synthetic.DECODE_70B):
            w = synthetic.weights(N, K, sigma=0.015, seed=4 + li, device=dev)
            for kind, name in ((0, "mxfp4"), (1, "nvfp4")):
                packs = [qz.qz_fp4_quantize(w if r == 0 else w.clone(), kind) for r in range(2)]
                c0, s0, t0 = packs[0]

                def fq():
                    qz.qz_fp4_quantize(w, kind, codes=c0, scales=s0, tensor_scale=t0)

                fq()
                msq = time_graph(capture(fq, stream))
                qb = fp4_quant_bytes(N, K, kind)
                fp4[f"{name}_quantize_N{N}_K{K}"] = {
                    "us": round(msq * 1e3, 2), "GB/s": round(qb / msq / 1e6, 1),
                    "frac_hbm": round(qb / msq / 1e6 / pk["hbm_gbs"], 4)}
                for M in (1, 16):
                    a = synthetic.activations(M, K, seed=M, device=dev)
                    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
                    ws = torch.zeros(max(256, qz.qz_workspace_bytes(qz.QZ_OP_FP4A16_GEMV, M, N, K,
                                                                    0)),
                                     dtype=torch.uint8, device=dev)

                    def fg():
                        for c, sc, ts in packs:
                            qz.qz_fp4a16_gemv(a, c, sc, ts, N, K, kind, y=y, workspace=ws)

                    fg()
                    ms = time_graph(capture(fg, stream)) / len(packs)
                    b = fp4_gemv_bytes(M, N, K, kind)
                    fp4[f"{name}_gemv_N{N}_K{K}_M{M}"] = {
                        "us": round(ms * 1e3, 2), "GB/s": round(b / ms / 1e6, 1),
                        "frac_hbm": round(b / ms / 1e6 / pk["hbm_gbs"], 4)}
                del packs, c0, s0, t0
            del w
        out["fp4_decode_70b"] = fp4

        # GPTQ of one 7B-class layer (4096 x 4096), 128 calibration samples
        N, K, n = 4096, 4096, 128
        w = synthetic.weights(N, K, sigma=0.02, seed=1, device=dev)
        x = synthetic.activations(n, K, seed=77, device=dev)
        gws = torch.empty(qz.qz_workspace_bytes(qz.QZ_OP_GPTQ, 1, N, K, GROUP), dtype=torch.uint8,
                          device=dev)
        gc, gsc, gz = qz.qz_gptq_quantize(w, x, 4, False, GROUP, workspace=gws)

        def fgptq():
            qz.qz_gptq_quantize(w, x, 4, False, GROUP, codes=gc, scales=gsc, zeros=gz,
                                workspace=gws)

        fgptq()
        ms = time_graph(capture(fgptq, stream), reps=5, warm=1)
        fl = gptq_flops(N, K, n)
        out["gptq_4096x4096"] = {
            "ms": round(ms, 3), "fp64_GFLOP/s": round(fl / (ms * 1e-3) / 1e9, 1),
            "frac_fp64_peak": round(fl / (ms * 1e-3) / 1e12 / FP64_PEAK_TFLOPS, 4),
            "fp64_peak_TFLOP/s_derived": round(FP64_PEAK_TFLOPS, 2),
            "calibration_samples": n}
        del w, x, gws, gc, gsc, gz

        # bulk quantization: 32 layer sets, 7.785e9 parameters
        total_params, b4, b8 = 0, 0, 0
        for N, K in synthetic.BULK_LAYER_SET:
            total_params += N * K
            b4 += quant_int4_bytes(N, K)
            b8 += quant_int8_bytes(N, K)
        sets = synthetic.BULK_SETS
        layers = []
        for si in range(sets):
            for li, (N, K) in enumerate(synthetic.BULK_LAYER_SET):
                layers.append((N, K, synthetic.weights(N, K, sigma=0.02, seed=100 + si * 16 + li,
                                                       device=dev)))
        outs4, outs8 = {}, {}
        for N, K in set(synthetic.BULK_LAYER_SET):
            outs4[(N, K)] = (torch.empty((N, K // 2), dtype=torch.uint8, device=dev),
                             torch.empty((N, K // GROUP), dtype=torch.bfloat16, device=dev),
                             torch.empty((N, K // GROUP), dtype=torch.uint8, device=dev))
            outs8[(N, K)] = (torch.empty((N, K), dtype=torch.uint8, device=dev),
                             torch.empty((N, 1), dtype=torch.bfloat16, device=dev), None)

        def bulk4():
            for N, K, w in layers:
                c, s, z = outs4[(N, K)]
                qz.qz_quantize_pack(w, 4, False, GROUP, codes=c, scales=s, zeros=z)

        def bulk8():
            for N, K, w in layers:
                c, s, _ = outs8[(N, K)]
                qz.qz_quantize_pack(w, 8, True, K, codes=c, scales=s)

        bulk4(); bulk8()
        ms4 = time_graph(capture(bulk4, stream), reps=3, warm=1)
        ms8 = time_graph(capture(bulk8, stream), reps=3, warm=1)
        out["bulk_quantize"] = {
            "params": total_params * sets,
            "int4_g128_ms": round(ms4, 3), "int4_g128_GB/s": round(b4 * sets / ms4 / 1e6, 1),
            "int4_frac_hbm": round(b4 * sets / ms4 / 1e6 / pk["hbm_gbs"], 4),
            "int8_pc_ms": round(ms8, 3), "int8_pc_GB/s": round(b8 * sets / ms8 / 1e6, 1),
            "int8_frac_hbm": round(b8 * sets / ms8 / 1e6 / pk["hbm_gbs"], 4)}
        del layers, outs4, outs8
    torch.cuda.synchronize()
    # a bounded device-side wait that ran out makes every figure above void
    assert qz.qz_device_status() == 0, "a bounded device-side wait ran out in the extras"
    torch.cuda.empty_cache()
    return out


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def _timed_passes(fn, target_s):
    passes, t0 = 0, time.perf_counter()
    while True:
        fn()
        passes += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            return passes, el


def cpu_baseline(decode_s=6.0, quant_s=3.0):
    """The oracle, as it stands, on this host's cores, with all threads and
    with one: the decode step (dequantize + fp64 matmul, M = 1) over the
    7B-class layer set, and quantize_pack int4 group-128 of the same layers.
    Bounded: about 2 x (decode_s + quant_s) seconds of CPU work."""
    import oracle
    threads = oracle.max_threads()
    prepared = []
    for li, (N, K) in enumerate(LAYERS):
        wb = synthetic.bf16_bits(synthetic.weights(N, K, sigma=0.02, seed=1 + li))
        ab = synthetic.bf16_bits(synthetic.activations(1, K, seed=50 + li))
        prepared.append((N, K, wb, oracle.quantize_pack(wb, 4, False, GROUP), ab))
    dec_bytes = sum(w4_gemv_bytes(1, N, K) for N, K in LAYERS)
    q_bytes = sum(quant_int4_bytes(N, K) for N, K in LAYERS)

    def decode():
        for N, K, _, (c, s, z), ab in prepared:
            oracle.matmul_f64(ab, oracle.dequantize(c, s, z, N, K, 4, False, GROUP))

    def quantize():
        for N, K, wb, _, _ in prepared:
            oracle.quantize_pack(wb, 4, False, GROUP)

    out = {}
    for label, n in (("all", threads), ("1thread", 1)):
        oracle.set_threads(n)
        dp, de = _timed_passes(decode, decode_s)
        qp, qe = _timed_passes(quantize, quant_s)
        out[label] = (dec_bytes * dp / de / 1e9, dp, de, q_bytes * qp / qe / 1e9, qp, qe)
    oracle.set_threads(threads)
    d_all, dp, de, q_all, qp, qe = out["all"]
    d_one, dp1, de1, q_one, qp1, qe1 = out["1thread"]
    return {"value": round(d_all, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(),
            "value_1thread": round(d_one, 4),
            "quantize_pack_int4_g128_GB/s": round(q_all, 4),
            "quantize_pack_int4_g128_GB/s_1thread": round(q_one, 4),
            "sample": f"decode (dequantize + fp64 matmul, M=1) over the three 7B-class layers: "
                      f"{dp} passes in {de:.1f} s on {threads} threads, {dp1} in {de1:.1f} s on "
                      f"1; quantize_pack int4 g128 of the same layers: {qp} passes in "
                      f"{qe:.1f} s on {threads} threads, {qp1} in {qe1:.1f} s on 1"}


def run_reference(args):
    """CPU oracle as the reference arm: each step is the oracle's decode pass
    over a row sample (1/16 of the rows) of the three 7B-class layers."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    threads = oracle.max_threads()
    oracle.set_threads(threads)
    sample = []
    nbytes = 0
    for li, (N, K) in enumerate(LAYERS):
        n = N // 16
        wb = synthetic.bf16_bits(synthetic.weights(N, K, sigma=0.02, seed=1 + li))[:n]
        ab = synthetic.bf16_bits(synthetic.activations(1, K, seed=50 + li))
        sample.append((n, K, oracle.quantize_pack(wb, 4, False, GROUP), ab))
        nbytes += w4_gemv_bytes(1, n, K)

    def step():
        for n, K, (c, s, z), ab in sample:
            oracle.matmul_f64(ab, oracle.dequantize(c, s, z, n, K, 4, False, GROUP))

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = nbytes * args.steps / el / 1e9
    line = {"metric": METRIC, "value": round(v, 4), "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_obj(),
            "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": threads,
                             "kind": "oracle", "cpu_model": cpu_model(),
                             "sample": "rows 0..N/16 of each of the three 7B-class layers per step"},
            "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_obj():
    return {"workload": "7B-class decode layer set (N,K)=(4096,4096),(11008,4096),(4096,11008): "
                        "int4 asym group-128 + int8 sym per-channel quantize_pack, int4 dequantize, "
                        "W4A16/W8A16 decode GEMV at M=1, W4A16 prefill GEMM at M=2048; plus "
                        "the 70B-class decode layers' W4A16/W8A16 GEMV at M=1",
            "weights": "bf16 ~N(0,0.02) + 0.1% x20 outliers, seeds 1..3",
            "activations": "bf16 ~N(0,1)",
            "l2": f"inputs rotate over {ROT} resident copies (packed W4 set {ROT} x 56 MB > L2)",
            "decode_70b": "W4A16 and W8A16 GEMV at M=1 on (28672,8192),(8192,28672), weights "
                          "bf16 ~N(0,0.015) + 0.1% x20, rotating over the same number of copies",
            "value_is": "w4a16_gemv_m1 part (algorithmic bytes / event-timed GEMV time)",
            "gemv_launch_overlap": (
                f"qz_set_launch_overlap({GEMV_LAUNCH_OVERLAP}): each decode GEMV may start while "
                "the previous kernel finishes and fetch its first weight blocks early; weights "
                "are static across the step"),
            "parallelism": "replicas"}


PROFILE_CASES = {
    # name: (kind, M, N, K)
    "gemv_w4_70b": ("gemv4", 1, 28672, 8192),
    "gemv_w4_70b_m16": ("gemv4", 16, 28672, 8192),
    "gemv_w4_7b": ("gemv4", 1, 4096, 4096),
    "gemv_w8_70b": ("gemv8", 1, 28672, 8192),
    "gemm_prefill": ("gemm", 2048, 8192, 8192),
    "gemm8_prefill": ("gemm8", 2048, 8192, 8192),
    "gemm_m32": ("gemm", 32, 8192, 8192),
    "gemm_m64": ("gemm", 64, 8192, 8192),
    "gemm_m128": ("gemm", 128, 8192, 8192),
    "quant_int4": ("quant4", 0, 28672, 8192),
    "gemv_nvfp4_70b": ("gemv_nv", 1, 28672, 8192),
    "gemv_mxfp4_70b": ("gemv_mx", 1, 28672, 8192),
    "gptq_4096": ("gptq", 128, 4096, 4096),
    "gemm_w4a4_nv": ("w4a4_nv", 2048, 8192, 8192),
    "gemm_w4a4_mx": ("w4a4_mx", 2048, 8192, 8192),
    "quant_int8": ("quant8", 0, 28672, 8192),
    "quant_nvfp4": ("quant_nv", 0, 28672, 8192),
    "quant_mxfp4": ("quant_mx", 0, 28672, 8192),
    "dequant_int4": ("dequant", 0, 28672, 8192),
}


def run_kernel_case(name, reps):
    """One kernel on one configuration, launched `reps` times after its
    inputs are prepared (used for ncu captures: small, deterministic)."""
    import weight_only_quantization_wise_b200 as qz
    kind, M, N, K = PROFILE_CASES[name]
    dev = torch.device("cuda", 0)
    w = synthetic.weights(N, K, sigma=0.015, seed=4, device=dev)
    op = {"gemv4": qz.QZ_OP_W4A16_GEMV, "gemv8": qz.QZ_OP_W8A16_GEMV, "gemm": qz.QZ_OP_W4A16_GEMM,
          "gemm8": qz.QZ_OP_W8A16_GEMM, "gemv_nv": qz.QZ_OP_FP4A16_GEMV,
          "gemv_mx": qz.QZ_OP_FP4A16_GEMV}.get(kind)
    g = K if kind in ("gemv8", "gemm8") else GROUP
    ws = torch.zeros(max(256, qz.qz_workspace_bytes(op, max(M, 1), N, K, g) if op is not None else 0),
                     dtype=torch.uint8, device=dev)
    if kind in ("gemv4", "gemm", "dequant"):
        c, s, z = qz.qz_quantize_pack(w, 4, False, GROUP)
    if kind in ("gemv8", "gemm8"):
        c, s, _ = qz.qz_quantize_pack(w, 8, True, K)
    if kind in ("gemv_nv", "gemv_mx", "w4a4_nv", "w4a4_mx"):
        fk = qz.QZ_FP4_NV if kind in ("gemv_nv", "w4a4_nv") else qz.QZ_FP4_MX
        c, s, ts = qz.qz_fp4_quantize(w, fk)
        if kind.startswith("w4a4"):
            s = qz.qz_fp4_scales_to_mma(s, N, K, fk)
            ws = torch.empty(qz.qz_workspace_bytes(qz.QZ_OP_FP4A4_GEMM, M, N, K, 0),
                             dtype=torch.uint8, device=dev)
    a = synthetic.activations(max(M, 1), K, seed=5, device=dev)
    torch.cuda.synchronize()
    for _ in range(reps):
        if kind == "gemv4":
            qz.qz_w4a16_gemv(a, c, s, z, N, K, GROUP, workspace=ws)
        elif kind == "gemv8":
            qz.qz_w8a16_gemv(a, c, s, N, K, workspace=ws)
        elif kind == "gemm":
            qz.qz_w4a16_gemm(a, c, s, z, N, K, GROUP, workspace=ws)
        elif kind == "gemm8":
            qz.qz_w8a16_gemm(a, c, s, N, K, workspace=ws)
        elif kind == "quant4":
            qz.qz_quantize_pack(w, 4, False, GROUP)
        elif kind == "quant8":
            qz.qz_quantize_pack(w, 8, True, K)
        elif kind in ("quant_nv", "quant_mx"):
            qz.qz_fp4_quantize(w, qz.QZ_FP4_NV if kind == "quant_nv" else qz.QZ_FP4_MX)
        elif kind == "dequant":
            qz.qz_dequantize(c, s, z, N, K, 4, False, GROUP)
        elif kind in ("gemv_nv", "gemv_mx"):
            qz.qz_fp4a16_gemv(a, c, s, ts, N, K, fk, workspace=ws)
        elif kind in ("w4a4_nv", "w4a4_mx"):
            qz.qz_fp4a4_gemm(a, c, s, ts, N, K, fk, workspace=ws)
        elif kind == "gptq":
            x = synthetic.activations(M, K, seed=77, device=dev)
            qz.qz_gptq_quantize(w, x, 4, False, GROUP)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    print(f"{name}: {reps} launches ok")


def run_layer_sets():
    """Every part of the step on the 7B layer set, one input copy, each part's
    three launches issued twice in a row (for ncu: the second set of each part
    is the measured one)."""
    import weight_only_quantization_wise_b200 as qz
    global ROT
    ROT = 1
    dev = torch.device("cuda", 0)
    ls = LayerSet(qz, dev)
    torch.cuda.synchronize()
    for name, method, *_ in PARTS:
        for _ in range(2):
            getattr(ls, method)(0)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0
    print("layer sets: " + ", ".join(p[0] for p in PARTS) + " (x2 each) ok")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--kernel", choices=sorted(PROFILE_CASES) + ["layer_sets"],
                    help="run one kernel case a few times, or every part once on the 7B "
                         "layer set (layer_sets), for profiling, and exit")
    ap.add_argument("--reps", type=int, default=3)
    args = ap.parse_args()
    if args.kernel == "layer_sets":
        run_layer_sets()
        return
    if args.kernel:
        run_kernel_case(args.kernel, args.reps)
        return
    if args.impl == "reference":
        run_reference(args)
        return
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    import weight_only_quantization_wise_b200 as qz
    pk = peaks()
    stream = torch.cuda.Stream(device=dev)
    ls = LayerSet(qz, dev)
    # the decode GEMVs overlap the previous kernel's tail: the step's weights
    # are quantized once here and never written again (qz_set_launch_overlap)
    qz.qz_set_launch_overlap(GEMV_LAUNCH_OVERLAP)
    torch.cuda.synchronize()

    # Every part runs once eagerly, then each step (all parts, one rotation)
    # becomes one CUDA graph with external timing events recorded between the
    # parts inside it, so a step runs without host gaps and each part's time
    # is the device time between its two event nodes.
    with torch.cuda.stream(stream):
        for name, meth, *_ in PARTS:
            getattr(ls, meth)(0)
    torch.cuda.synchronize()
    assert qz.qz_device_status() == 0

    npart = len(PARTS)

    def new_events():
        return [(torch.cuda.Event(enable_timing=True, external=True),
                 torch.cuda.Event(enable_timing=True, external=True)) for _ in range(npart)]

    def capture_step(p, evs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for j, (name, meth, *_r) in enumerate(PARTS):
                evs[j][0].record(stream)
                getattr(ls, meth)(p)
                evs[j][1].record(stream)
        return g

    # the events must outlive the graphs that record them
    warm_ev = [new_events() for _ in range(args.warmup)]
    warm = [capture_step(i % ROT, warm_ev[i]) for i in range(args.warmup)]
    ev = [new_events() for _ in range(args.steps)]
    timed = [capture_step((args.warmup + i) % ROT, ev[i]) for i in range(args.steps)]
    torch.cuda.synchronize()

    with torch.cuda.stream(stream):
        for g in warm:
            g.replay()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()

    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler()
    sampler.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.nvtx.range_push("timed")
    with torch.cuda.stream(stream):
        e_start.record(stream)
        for g in timed:
            g.replay()
        e_end.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop(local)
    total_ms = e_start.elapsed_time(e_end)
    part_ms = [sum(ev[i][j][0].elapsed_time(ev[i][j][1]) for i in range(args.steps)) / args.steps
               for j in range(npart)]
    assert qz.qz_device_status() == 0

    # max over ranks
    agg = max_over_ranks([total_ms] + part_ms, dist, dev)
    total_ms, part_ms = agg[0], agg[1:]

    traffic = ncu_traffic()
    parts, roofs = {}, {}
    # every kernel is timed inside a step of about a millisecond, far short
    # of the seconds it takes to reach the power cap: burst peaks apply
    for (name, meth, unit, work, bound, nl), ms in zip(PARTS, part_ms):
        parts[name] = {"ms": round(ms, 5), "value": round(rate(work, ms, unit), 2), "unit": unit,
                       "launches": nl}
        roofs[name] = roofline_obj(name, work, ms, nl, bound, pk, traffic, sustained=False)
    dominant = max(zip(PARTS, part_ms), key=lambda x: x[1])[0][0]
    gemv_idx = [p[0] for p in PARTS].index("w4a16_gemv_m1")
    gemv_bytes = PARTS[gemv_idx][3]
    value = replica_rate(gemv_bytes, part_ms[gemv_idx] * 1e-3, world) / 1e9

    # end to end through the public API, host buffers, per decode step
    e2e = None
    # one pinned host buffer holds the step's three activation vectors, one
    # its three outputs: one copy in, one copy out per step
    ks, ns = [K for N, K in LAYERS], [N for N, K in LAYERS]
    host_a_all = torch.cat([x.reshape(-1).cpu() for x in ls.a1]).pin_memory()
    host_y_all = torch.empty(sum(ns), dtype=torch.bfloat16).pin_memory()
    dev_a_all = torch.empty_like(host_a_all, device=dev)
    dev_y_all = torch.empty(sum(ns), dtype=torch.bfloat16, device=dev)
    dev_a = [v.view(1, -1) for v in torch.split(dev_a_all, ks)]
    dev_y = [v.view(1, -1) for v in torch.split(dev_y_all, ns)]
    h2d = host_a_all.numel() * 2
    d2h = host_y_all.numel() * 2

    def e2e_body(p):
        dev_a_all.copy_(host_a_all, non_blocking=True)
        for li, (N, K) in enumerate(LAYERS):
            qz.qz_w4a16_gemv(dev_a[li], ls.c4[p][li], ls.s4[p][li], ls.z4[p][li], N, K, GROUP,
                             y=dev_y[li], workspace=ls.ws)
        host_y_all.copy_(dev_y_all, non_blocking=True)

    # each decode step (copy in, the three GEMVs through the public API, copy
    # out) is one captured CUDA graph, replayed and waited for on the host
    with torch.cuda.stream(stream):
        e2e_body(0)
    stream.synchronize()
    e2e_graphs = [capture(lambda p=p: e2e_body(p), stream) for p in range(ROT)]

    def e2e_step(p):
        with torch.cuda.stream(stream):
            e2e_graphs[p].replay()
        stream.synchronize()

    for i in range(args.warmup):
        e2e_step(i % ROT)
    if dist:
        dist.barrier()
    t0 = time.perf_counter()
    for i in range(args.steps):
        e2e_step(i % ROT)
    el = max_over_ranks([time.perf_counter() - t0], dist, dev)[0]
    del e2e_graphs
    e2e = {"value": round(replica_rate(gemv_bytes * args.steps, el, world) / 1e9, 3), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "note": "decode step through qz_w4a16_gemv: the three activation vectors copied in "
                   "from one pinned host buffer, the three outputs copied out to one, captured "
                   "with the three public-API calls as one CUDA graph per step, replayed and "
                   "synchronized on the host every step; weights resident"}

    extras = None
    if rank == 0 and not args.no_extras:
        del warm, timed                      # the graphs first, then their events
        del warm_ev, ev
        extras = run_extras(qz, dev, pk, stream)
        extras["decode_read_floor"] = read_floor(ls, stream, pk, parts)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "weights_dtype": "int4 (int8 for the W8A16 part)", "data": "synthetic",
            "config": config_obj(),
            "roofline": roofs[dominant] | {"kernel": dominant},
            "rooflines": roofs, "parts": parts,
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clocks, "peaks": pk, "extra": extras,
        }
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
