"""Benchmark of the HLWQ Q5 hot path on B200.

Headline (one JSON line on rank 0): fused dequant-GEMV weight GB/s on the dense
decode layer 5120 x 5120 (M = 1, bf16 activation, fp32 output).  One "step" is
a decode pass over L = 64 distinct 5120 x 5120 Q5 layers (64 x 16.8 MB = 1.07
GB of codes and norms, > 8x the 126 MB L2, so every byte comes from HBM), each
layer one launch of the fused kernel, replayed from a CUDA graph.  ``value`` =
weight bytes (packed codes + fp16 norms) of all ranks / device time (max over
ranks).  At N = 1 the same run also measures the other parts of the metric
("components"): quantizer Gweights/s on the 128-expert layer (128 x (1408 x 2816
+ 2816 x 704) weights), GEMM TFLOP/s on 27648 x 5120 at M = 16/64/256, MoE GB/s
on the 256(+1)-expert layer at T = 1/8/64 and the 128-expert layer at T = 1/16,
the Q5 -> INT4 re-encoder on 27648 x 5120 and the Q3 KV-cache encoding (131072
vectors of 256: quantize, decode, scores for 6 queries).

``--impl reference`` times the CPU oracle (oracle/, fp64 numpy) on the host
cores on a bounded sample of the same GEMV workload and prints the same line.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "HLWQ-Q5 fused GEMV weight GB/s (% of HBM peak); quantize Gweights/s; GEMM TFLOP/s"
O_DIM, I_DIM = 5120, 5120
NB = (I_DIM + 127) // 128
WEIGHT_BYTES = O_DIM * NB * 80 + O_DIM * NB * 2           # packed + norms per layer
GEMV_ALGO_BYTES = WEIGHT_BYTES + I_DIM * 2 + O_DIM * 4     # + x (bf16) + y (fp32)
LAYERS = 64
NVML_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
                0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
                0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_traffic():
    """Per-launch DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) from
    the committed ncu summaries (profiles/traffic.json).  An entry counts only
    while the kernel sources it was measured on are unchanged (sha1 of the
    listed files); otherwise its traffic is reported as null."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return {}
    with open(p) as f:
        entries = json.load(f)
    out = {}
    for key, e in entries.items():
        m = hashlib.sha1()
        try:
            for name in e["sources"]:
                with open(os.path.join(ROOT, "dequant_matmul_b200", "csrc", name), "rb") as src:
                    m.update(src.read())
        except OSError:
            continue
        if m.hexdigest() == e.get("source_sha1"):
            out[key] = e["dram_bytes_per_launch"]
    return out


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch_dev: int, period_s: float = 0.001):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        self.period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_dev).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(torch_dev)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nv = pynvml
        except Exception as e:  # pragma: no cover - best effort
            self.error = repr(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.reasons |= int(r)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml_unavailable"]}
        names = [v for k, v in NVML_REASONS.items() if self.reasons & k and k != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ---------------------------------------------------------------- helpers
def time_graph(fn, reps: int, warmup: int, stream):
    """Captures fn() in a CUDA graph and times `reps` replays with CUDA events."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):          # replay() launches on the current stream
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    e.synchronize()
    return s.elapsed_time(e) / reps, g


def frac(a, p):
    return round(a / p, 4) if (a is not None and p) else None


# ---------------------------------------------------------------- ranks (N > 1: independent replicas)
def max_over_ranks(value: float, world: int, device="cpu") -> float:
    """The largest of the ranks' values (every rank gets it); the timed region
    of a multi-GPU run is the slowest rank's."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank_step: int, steps: int, ms_total_max: float) -> float:
    """Whole-job throughput: the bytes all ranks processed / the slowest rank's time."""
    return world * bytes_per_rank_step * steps / (ms_total_max * 1e6)


# ---------------------------------------------------------------- components (N = 1)
def components(hl, cb, peaks, stream, parts=("quantize", "gemm", "moe", "int4", "kv", "codes", "tq3")):
    import torch
    from dequant_matmul_b200 import synth
    out = {}
    torch.cuda.synchronize()

    if "quantize" in parts:
        out.update(bench_quantize(hl, cb, peaks, stream))
    if "gemm" in parts:
        out.update(bench_gemm(hl, cb, peaks, stream))
    if "moe" in parts:
        out.update(bench_moe(hl, cb, peaks, stream))
    if "int4" in parts:
        out.update(bench_int4(hl, cb, peaks, stream))
    if "kv" in parts:
        out.update(bench_kv(hl, peaks, stream))
    if "codes" in parts:
        out.update(bench_codes(hl, cb, peaks, stream))
    if "tq3" in parts:
        out.update(bench_tq3(hl, peaks, stream))
    return out


def bench_quantize(hl, cb, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    out = {}
    # Quantizer: the 128-expert layer, gate_up 1408 x 2816 and down 2816 x 704 per expert.
    E, GU, DN = 128, (1408, 2816), (2816, 704)
    w_gu = synth.student_t_device((E,) + GU, seed=50)
    w_dn = synth.student_t_device((E,) + DN, seed=51)
    p_gu = torch.empty(E, GU[0], 22, 80, dtype=torch.uint8, device="cuda")
    n_gu = torch.empty(E, GU[0], 22, dtype=torch.uint16, device="cuda")
    p_dn = torch.empty(E, DN[0], 6, 80, dtype=torch.uint8, device="cuda")
    n_dn = torch.empty(E, DN[0], 6, dtype=torch.uint16, device="cuda")

    def quant_layer():
        hl.quantize(w_gu, cb, p_gu, n_gu, stream=stream)
        hl.quantize(w_dn, cb, p_dn, n_dn, stream=stream)

    ms, _ = time_graph(quant_layer, reps=10, warmup=3, stream=stream)
    ms_gu, _ = time_graph(lambda: hl.quantize(w_gu, cb, p_gu, n_gu, stream=stream), reps=10, warmup=2, stream=stream)
    ms_dn, _ = time_graph(lambda: hl.quantize(w_dn, cb, p_dn, n_dn, stream=stream), reps=10, warmup=2, stream=stream)
    n_w = E * (GU[0] * GU[1] + DN[0] * DN[1])
    qbytes = 2 * n_w + (p_gu.numel() + p_dn.numel()) + 2 * (n_gu.numel() + n_dn.numel())
    out["quantize"] = {"workload": "128 experts x (1408x2816 + 2816x704) bf16 -> Q5", "ms": round(ms, 4),
                       "ms_gate_up": round(ms_gu, 4), "ms_down": round(ms_dn, 4),
                       "gweights_per_s": round(n_w / ms / 1e6, 2),
                       "roofline": {"bound": "hbm", "achieved": round(qbytes / ms / 1e6, 1), "peak": peaks["hbm_gbs"],
                                    "unit": "GB/s", "frac": frac(qbytes / ms / 1e6, peaks["hbm_gbs"]),
                                    "algo_bytes": qbytes}}
    del w_gu, w_dn, p_gu, n_gu, p_dn, n_dn
    return out


def bench_gemm(hl, cb, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    out = {}
    # GEMM 27648 x 5120 at M = 16, 64, 256 (bf16 out); two weight copies alternate (> L2).
    O3, I3 = 27648, 5120
    copies = []
    for c in range(2):
        w = synth.student_t_device((O3, I3), seed=60 + c)
        copies.append(hl.quantize(w, cb, stream=stream))
        del w
    gemm = {}
    for M in (1, 4, 16, 64, 256):
        X = synth.activations_device(M, I3, seed=M)
        Y = torch.empty(M, O3, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(max(1, hl.workspace_bytes(hl.HLWQ_OP_GEMM, O3, I3, M)), dtype=torch.uint8, device="cuda")

        def run_gemm():
            for p, n in copies:
                hl.gemm(p, n, cb, X, Y=Y, workspace=ws, stream=stream)

        reps = 5 if M >= 16 else 20
        ms, _ = time_graph(run_gemm, reps=reps, warmup=3, stream=stream)
        ms /= len(copies)
        flops = 2.0 * M * O3 * I3
        byts = O3 * 40 * 82 + M * I3 * 2 + M * O3 * 2
        tf = flops / ms / 1e9
        gb = byts / ms / 1e6
        gemm[f"M{M}"] = {"ms": round(ms, 4), "tflops": round(tf, 2), "gbs": round(gb, 1),
                         "tensor_frac": frac(tf, peaks["bf16_tflops"]), "hbm_frac": frac(gb, peaks["hbm_gbs"])}
    out["gemm_27648x5120"] = gemm
    del copies
    return out


def bench_int4(hl, cb, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    # Q5 -> INT4 re-encoding of the 27648 x 5120 layer; two copies alternate (> L2).
    O3, I3 = 27648, 5120
    nb = I3 // 128
    copies = []
    for c in range(2):
        w = synth.student_t_device((O3, I3), seed=90 + c)
        copies.append(hl.quantize(w, cb, stream=stream))
        del w
    q4 = torch.empty(O3, nb, 64, dtype=torch.uint8, device="cuda")
    sc = torch.empty(O3, nb, dtype=torch.uint16, device="cuda")
    zr = torch.empty(O3, nb, dtype=torch.uint16, device="cuda")

    def run():
        for p, n in copies:
            hl.requantize_int4(p, n, cb, I3, q4, sc, zr, stream=stream)

    ms, _ = time_graph(run, reps=10, warmup=3, stream=stream)
    ms /= len(copies)
    byts = O3 * nb * (80 + 2 + 64 + 2 + 2)   # Q5 codes + norm in, INT4 codes + scale + zero out
    gbs = byts / ms / 1e6
    del copies, q4, sc, zr
    return {"requantize_int4_27648x5120": {"ms": round(ms, 4), "gweights_per_s": round(O3 * I3 / ms / 1e6, 2),
                                           "gbs": round(gbs, 1), "hbm_frac": frac(gbs, peaks["hbm_gbs"]),
                                           "algo_bytes": byts}}


def bench_codes(hl, cb, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    # One-code-per-byte layout of the 27648 x 5120 layer, both directions.
    O3, I3 = 27648, 5120
    nb = I3 // 128
    w = synth.student_t_device((O3, I3), seed=97)
    packed, _ = hl.quantize(w, cb, stream=stream)
    del w
    codes = torch.empty(O3, nb, 128, dtype=torch.uint8, device="cuda")
    back = torch.empty_like(packed)
    res = {}
    byts = O3 * nb * (80 + 128)
    ms, _ = time_graph(lambda: hl.codes_unpack(packed, codes, stream=stream), reps=10, warmup=3, stream=stream)
    res["unpack"] = {"ms": round(ms, 4), "gbs": round(byts / ms / 1e6, 1), "hbm_frac": frac(byts / ms / 1e6, peaks["hbm_gbs"])}
    ms, _ = time_graph(lambda: hl.codes_pack(codes, back, stream=stream), reps=10, warmup=3, stream=stream)
    res["pack"] = {"ms": round(ms, 4), "gbs": round(byts / ms / 1e6, 1), "hbm_frac": frac(byts / ms / 1e6, peaks["hbm_gbs"])}
    torch.cuda.synchronize()
    res["round_trip_equal"] = bool(torch.equal(back, packed))
    del packed, codes, back
    return {"codes_int8_27648x5120": res}


def bench_tq3(hl, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    # TQ3 (3-bit HIGGS) weights: quantize the 27648 x 5120 layer; decode GEMV at
    # 5120 x 5120 and 27648 x 5120 over enough weight copies to exceed L2.
    cb8 = hl.kv_codebook("cuda")
    signs = synth.sign_vectors(42).cuda()
    res = {}
    O3, I3 = 27648, 5120
    nb = I3 // 128
    w = synth.student_t_device((O3, I3), seed=98)
    packed = torch.empty(O3, nb, 48, dtype=torch.uint8, device="cuda")
    norms = torch.empty(O3, nb, dtype=torch.float32, device="cuda")
    ms, _ = time_graph(lambda: hl.tq3_quantize(w, signs, cb8, packed, norms, stream=stream), reps=5, warmup=3,
                       stream=stream)
    b = O3 * I3 * 2 + O3 * nb * (48 + 4)
    res["quantize_27648x5120"] = {"ms": round(ms, 4), "gweights_per_s": round(O3 * I3 / ms / 1e6, 2),
                                  "gbs": round(b / ms / 1e6, 1), "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
    out16 = torch.empty(O3, I3, dtype=torch.bfloat16, device="cuda")
    ms, _ = time_graph(lambda: hl.tq3_dequantize(packed, norms, signs, cb8, I3, out=out16, stream=stream), reps=5,
                       warmup=3, stream=stream)
    b = O3 * nb * (48 + 4) + O3 * I3 * 2
    res["dequantize_bf16_27648x5120"] = {"ms": round(ms, 4), "gbs": round(b / ms / 1e6, 1),
                                         "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
    del out16
    for (Og, Ig) in ((27648, 5120), (5120, 5120)):
        nbg = Ig // 128
        wbytes = Og * nbg * (48 + 4)
        ncopy = max(2, -(-(320 << 20) // wbytes))
        copies = []
        for c in range(ncopy):
            if Og == O3 and c == 0:
                copies.append((packed, norms))
                continue
            wc = synth.student_t_device((Og, Ig), seed=100 + c) if c < 2 else None
            if wc is not None:
                copies.append(hl.tq3_quantize(wc, signs, cb8, stream=stream))
                del wc
            else:  # further copies: same codes at other addresses
                copies.append((copies[c % 2][0].clone(), copies[c % 2][1].clone()))
        x = synth.activations_device(1, Ig, seed=101)[0]
        y = torch.empty(Og, dtype=torch.float32, device="cuda")

        def run():
            for p, n in copies:
                hl.tq3_gemv(p, n, signs, cb8, x, y=y, stream=stream)

        ms, _ = time_graph(run, reps=20, warmup=3, stream=stream)
        ms /= len(copies)
        b = wbytes + Ig * 2 + Og * 4
        res[f"gemv_{Og}x{Ig}"] = {"ms": round(ms, 5), "us": round(ms * 1e3, 2), "gbs": round(b / ms / 1e6, 1),
                                  "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"]), "copies": len(copies),
                                  "algo_bytes": b}
        if Og == O3:
            # small-M GEMM on the tensor cores (bf16 out), the same weight copies
            for M in (16, 64):
                X = synth.activations_device(M, Ig, seed=102 + M)
                Y = torch.empty(M, Og, dtype=torch.bfloat16, device="cuda")
                ws = torch.empty(max(1, hl.workspace_bytes(hl.HLWQ_OP_TQ3_GEMM, Og, Ig, M)), dtype=torch.uint8,
                                 device="cuda")

                def run_gemm():
                    for p, n in copies:
                        hl.tq3_gemm(p, n, signs, cb8, X, Y=Y, workspace=ws, stream=stream)

                ms, _ = time_graph(run_gemm, reps=5, warmup=3, stream=stream)
                ms /= len(copies)
                b = wbytes + M * Ig * 2 + M * Og * 2
                tf = 2.0 * M * Og * Ig / ms / 1e9
                res[f"gemm_{Og}x{Ig}_M{M}"] = {"ms": round(ms, 4), "tflops": round(tf, 2),
                                               "gbs": round(b / ms / 1e6, 1),
                                               "tensor_frac": frac(tf, peaks["bf16_tflops"]),
                                               "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
        del copies
    del w, packed, norms
    return {"tq3": res}


def bench_kv(hl, peaks, stream):
    import torch
    from dequant_matmul_b200 import synth
    # Q3 KV cache: 4 KV heads x 32768 tokens = 131072 vectors of 256 (a long
    # context of the head_dim-256 GQA model); scores for one GQA group of 6
    # query heads against one head's 32768 keys, and against all 131072.
    N = 4 * 32768
    cb8 = hl.kv_codebook("cuda")
    X = synth.activations_device(N, 256, seed=95)
    packed = torch.empty(N, 96, dtype=torch.uint8, device="cuda")
    norms = torch.empty(N, dtype=torch.uint16, device="cuda")
    out16 = torch.empty(N, 256, dtype=torch.bfloat16, device="cuda")
    Q = synth.activations_device(6, 256, seed=96)
    S = torch.empty(6, N, dtype=torch.float32, device="cuda")
    res = {}
    ms, _ = time_graph(lambda: hl.kv_quantize(X, cb8, packed, norms, stream=stream), reps=10, warmup=3, stream=stream)
    b = N * (512 + 96 + 2)
    res["quantize"] = {"ms": round(ms, 4), "vectors_per_s_M": round(N / ms / 1e3, 2), "gbs": round(b / ms / 1e6, 1),
                       "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
    ms, _ = time_graph(lambda: hl.kv_dequantize(packed, norms, cb8, out=out16, stream=stream), reps=10, warmup=3,
                       stream=stream)
    b = N * (96 + 2 + 512)
    res["dequantize_bf16"] = {"ms": round(ms, 4), "gbs": round(b / ms / 1e6, 1),
                              "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
    ms, _ = time_graph(lambda: hl.kv_scores(Q, packed, norms, cb8, S=S, stream=stream), reps=10, warmup=3,
                       stream=stream)
    b = N * (96 + 2 + 6 * 4)
    res["scores_6q"] = {"ms": round(ms, 4), "keys_per_s_G": round(N / ms / 1e6, 2), "gbs": round(b / ms / 1e6, 1),
                        "hbm_frac": frac(b / ms / 1e6, peaks["hbm_gbs"])}
    # the residual window: one head's 32768 tokens, the last 128 kept exact
    # (scores of the GQA group over encoded + window keys in one launch), and
    # a decode step's append of one token (which encodes the token leaving
    # the window)
    T1 = 32768
    cache = hl.KVWindowCache(capacity=T1, R=128, cb8=cb8)
    cache.append(X[:T1 - 1])
    Sw = torch.empty(6, T1 - 1, dtype=torch.float32, device="cuda")
    ms, _ = time_graph(lambda: cache.scores(Q, S=Sw, stream=stream), reps=10, warmup=3, stream=stream)
    b = cache.n_enc * (96 + 2) + 128 * 512 + (T1 - 1) * 6 * 4
    res["window_scores_6q_32767tok"] = {"ms": round(ms, 4), "keys_per_s_G": round((T1 - 1) / ms / 1e6, 2),
                                        "gbs": round(b / ms / 1e6, 1), "encoded": cache.n_enc, "window": 128}
    x1 = X[T1 - 1:T1]
    st = (cache.n_enc, cache.n_total)
    win0 = cache.window.clone()

    def append_one():
        # restore the state each replay so every step appends the same token
        cache.n_enc, cache.n_total = st
        cache.append(x1, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(3):
            append_one()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(20):
            append_one()
        e1.record(stream)
        e1.synchronize()
    cache.window.copy_(win0)
    res["window_append_1tok"] = {"us": round(e0.elapsed_time(e1) * 1e3 / 20, 2),
                                 "note": "eager calls (host bookkeeping between launches): encodes 1 token, copies 1"}
    del X, packed, norms, out16, Q, S, cache, Sw
    return {"kv_q3_131072x256": res}


def bench_moe(hl, cb, peaks, stream):
    """MoE layers.  Each timed call routes its own tokens: a graph replays R
    calls with R different routings (logits and activations), R chosen so
    that the experts the calls read add up to more than twice the L2, so
    every call reads its experts from HBM without an L2 scrub.  GB/s counts
    each call's distinct experts once."""
    import torch
    from dequant_matmul_b200 import synth
    out = {}

    def layer(gu, dn, shared, E, H, F, T, per_expert, seed, flags=0):
        n_sh = 1 if shared is not None else 0
        est = min(E, T * 8) + n_sh                                   # distinct experts, upper estimate
        R = max(2, min(32, -(-2 * 126 * 2 ** 20 // (est * per_expert))))
        sets = []
        for r in range(R):
            g = torch.Generator(device="cuda").manual_seed(seed + 1000 * r + T)
            sets.append((torch.randn(T, E, generator=g, device="cuda"),
                         synth.activations_device(T, H, seed=seed + 7 * r + T),
                         torch.empty(T, H, dtype=torch.float32, device="cuda"),
                         torch.empty(T, 8, dtype=torch.int32, device="cuda"),
                         torch.empty(T, 8, dtype=torch.float32, device="cuda")))
        ws = torch.empty(hl.workspace_bytes(hl.HLWQ_OP_MOE, H, F, T, E, 8), dtype=torch.uint8, device="cuda")

        def run():
            for lg, X, Y, ids, wts in sets:
                hl.moe_gemv(gu, dn, cb, lg, X, 8, shared=shared, Y=Y, ids=ids, weights=wts, workspace=ws,
                            stream=stream, flags=flags)

        ms, _ = time_graph(run, reps=10, warmup=3, stream=stream)
        ms /= R
        distinct = sum(int(torch.unique(st[3]).numel()) + n_sh for st in sets) / R
        byts = distinct * per_expert
        return {"ms": round(ms, 4), "distinct_experts": round(distinct, 1), "routings": R,
                "gbs": round(byts / ms / 1e6, 1), "hbm_frac": frac(byts / ms / 1e6, peaks["hbm_gbs"])}

    # 256 experts + shared, hidden 2048, intermediate 512, top-8.
    E4, H4, F4 = 256, 2048, 512
    gu_w = synth.student_t_device((E4, 2 * F4, H4), seed=70)
    dn_w = synth.student_t_device((E4, H4, F4), seed=71)
    gu = hl.quantize(gu_w, cb, stream=stream)
    dn = hl.quantize(dn_w, cb, stream=stream)
    del gu_w, dn_w
    sh = (hl.quantize(synth.student_t_device((2 * F4, H4), seed=72), cb, stream=stream),
          hl.quantize(synth.student_t_device((H4, F4), seed=73), cb, stream=stream))
    per_expert = (2 * F4 * 16 + H4 * 4) * 82
    moe4 = {f"T{T}": layer(gu, dn, sh, E4, H4, F4, T, per_expert, 80) for T in (1, 8, 64)}
    # the default takes the fused path at T = 1 and 8 and the grouped path
    # (each active expert read once for all its tokens) at T = 64; the grouped
    # path forced at T = 8 for comparison
    moe4["T8_grouped"] = layer(gu, dn, sh, E4, H4, F4, 8, per_expert, 80, flags=hl.HLWQ_FLAG_MOE_GROUPED)
    out["moe_256x(1024x2048+2048x512)_top8_shared"] = moe4
    del gu, dn, sh
    # the 128-expert layer, hidden 2816, intermediate 704 (tail block
    # zero-padded), top-8, no shared expert, T = 1 and 16.
    E5, H5, F5 = 128, 2816, 704
    gu5 = hl.quantize(synth.student_t_device((E5, 2 * F5, H5), seed=90), cb, stream=stream)
    dn5 = hl.quantize(synth.student_t_device((E5, H5, F5), seed=91), cb, stream=stream)
    per_expert5 = (2 * F5 * 22 + H5 * 6) * 82
    moe5 = {f"T{T}": layer(gu5, dn5, None, E5, H5, F5, T, per_expert5, 110) for T in (1, 16)}
    out["moe_128x(1408x2816+2816x704)_top8"] = moe5
    return out


# ---------------------------------------------------------------- CPU oracle
def cpu_oracle_gemv(seconds: float, rows_per_step: int = 64, steps=None):
    """Times the oracle's GEMV (dequantize + fp64 dot) on row slices of the
    5120 x 5120 layer on the host cores.  Returns (GB/s of weight bytes, sample
    description, threads, per-step ms list)."""
    import numpy as np
    import torch

    import oracle as O
    from dequant_matmul_b200 import synth
    W = synth.student_t((rows_per_step, I_DIM), df4_seed=0)
    q = O.quantize(W)
    x = synth.activations(1, I_DIM, seed=1)
    per_bytes = rows_per_step * NB * 82
    done, t0, times = 0, time.perf_counter(), []
    while True:
        s = time.perf_counter()
        O.matmul(q["packed"], q["norms"], I_DIM, x)
        times.append((time.perf_counter() - s) * 1e3)
        done += 1
        if steps is not None and done >= steps:
            break
        if steps is None and time.perf_counter() - t0 >= seconds:
            break
    el = sum(times) / 1e3
    threads = torch.get_num_threads()
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        pass
    return done * per_bytes / el / 1e9, f"oracle GEMV on {rows_per_step} rows x {I_DIM} (of 5120x5120), {done} reps", \
        threads, times


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--layers", type=int, default=LAYERS,
                    help="distinct 5120x5120 layers per step (fewer only for small profiling captures; "
                         "keep their bytes above the L2)")
    ap.add_argument("--only", choices=["components", "quantize", "gemm", "moe", "int4", "kv", "codes", "tq3"], default=None,
                    help="run only the component measurements (used for profiling captures)")
    args = ap.parse_args()
    nl = max(1, args.layers)
    warmup = max(3, args.warmup)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        # warm-up steps, then exactly `steps` timed oracle steps (each a 64-row slice)
        cpu_oracle_gemv(0, steps=warmup)
        gbs, sample, threads, times = cpu_oracle_gemv(0, steps=args.steps)
        ms = sum(times) / len(times)
        line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": "dense decode GEMV 5120x5120 HLWQ-Q5, M=1 (64-row slice per step)"},
                "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from dequant_matmul_b200 import hlwq as hl
    from dequant_matmul_b200 import synth

    peaks = load_peaks()
    stream = torch.cuda.Stream()
    cb = hl.codebook("cuda")
    if args.only is not None:
        parts = ("quantize", "gemm", "moe", "int4", "kv", "codes", "tq3") if args.only == "components" else (args.only,)
        print(json.dumps({"components": components(hl, cb, peaks, stream, parts)}), flush=True)
        return
    # nl (default 64) distinct layers (quantized on the device from seeded synthetic weights)
    layers = []
    with torch.cuda.stream(stream):
        for l in range(nl):
            w = synth.student_t_device((O_DIM, I_DIM), seed=1000 + 7 * rank + l)
            layers.append(hl.quantize(w, cb, stream=stream))
            del w
        xs = synth.activations_device(nl, I_DIM, seed=2)
        ys = torch.empty(nl, O_DIM, dtype=torch.float32, device="cuda")
    torch.cuda.synchronize()

    flags = hl.HLWQ_FLAG_WEIGHTS_STATIC   # weights are static across the decode pass

    def step():
        for l, (p, n) in enumerate(layers):
            hl.gemv(p, n, cb, xs[l], y=ys[l], stream=stream, flags=flags)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        step()
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            g.replay()
    torch.cuda.synchronize()

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk, torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(args.steps):
            g.replay()
        end.record(stream)
        end.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms_total = max_over_ranks(start.elapsed_time(end), world, "cuda")
    ms_step = ms_total / args.steps
    value = whole_job_gbs(world, nl * WEIGHT_BYTES, args.steps, ms_total)
    launch_ms = ms_step / nl
    achieved = GEMV_ALGO_BYTES / launch_ms / 1e6

    # end-to-end through the public API with host buffers (pinned), no graph
    x_host = xs.cpu().pin_memory()
    y_host = torch.empty(nl, O_DIM, dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step():
        xs.copy_(x_host, non_blocking=True)
        for l, (p, n) in enumerate(layers):
            hl.gemv(p, n, cb, xs[l], y=ys[l], stream=stream, flags=flags)
        y_host.copy_(ys, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(2):
            e2e_step()
        stream.synchronize()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e2.record(stream)
        e2.synchronize()
    e2e_val = whole_job_gbs(world, nl * WEIGHT_BYTES, e2e_steps, max_over_ranks(s2.elapsed_time(e2), world, "cuda"))

    comp = None
    if world == 1 and not args.no_components:
        comp = components(hl, cb, peaks, stream)

    if rank == 0:
        traffic = load_traffic().get("gemv_5120x5120_m1")
        cpu = None
        if world == 1:
            gbs, sample, threads, _ = cpu_oracle_gemv(args.cpu_seconds)
            cpu = {"value": round(gbs, 5), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample}
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16*f16->f32", "data": "synthetic",
            "config": {"workload": "dense decode GEMV 5120x5120 HLWQ-Q5 (bf16 Student-t(4) std 0.02 weights, "
                                   f"x bf16 N(0,1)), M=1, {nl} distinct layers per step",
                       "global_batch": 1, "bytes_per_step_per_gpu": nl * WEIGHT_BYTES,
                       "launch": "hlwq_gemv_ex(HLWQ_FLAG_WEIGHTS_STATIC): programmatic dependent launch, "
                                 "x read after the previous kernel completes",
                       "l2": f"inputs larger than L2 ({nl} layers x 16.8 MB = {nl * 16.8e-3:.2f} GB)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": frac(achieved, peaks["hbm_gbs"]), "traffic": traffic,
                         "peak_source": peaks["source"], "algo_bytes_per_launch": GEMV_ALGO_BYTES,
                         "launch_us": round(launch_ms * 1e3, 3)},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 2), "unit": "GB/s", "h2d_bytes_per_step": nl * I_DIM * 2,
                    "d2h_bytes_per_step": nl * O_DIM * 4},
            "gpu_launches": nl * args.steps,
            "clocks": clk.summary(),
        }
        if comp is not None:
            line["components"] = comp
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        del g
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
