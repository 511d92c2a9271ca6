"""Throughput of the rotated W4A4 linear layer on B200.

One step = the whole online hot path on one batch of tokens:
  K1  rq_rotate_quantize_act  (PCA projection + RPBH rotate + normalise + INT4/LM/NVFP4 quantize + pack)
  K2  rq_w4a4_linear          (4-bit x 4-bit tcgen05 GEMM + fused rank-r low-rank add, BF16 out)
Weights are folded and quantized once, offline, before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config all|c1..c5] [--impl ours|reference]

Prints one JSON line (rank 0).  The headline (top-level ``value``, ``roofline``,
``e2e``, ``cpu_baseline``) is the largest single-GPU layer, the Wan-2.1-like
W2A4 MLP with CFG (65520 tokens x 1536 -> 8960); with ``--config all`` (the
default) the other four layers, and the PixArt-like fc1 layer with the full PCA
rotation in place of RPBH (``c2p``: K1 is then rq_pca_rotate_quantize_act, a
BF16 tensor-core product x V plus the split/quantize pass), are timed in the
same run and reported under ``configs``.  Multi-GPU (torchrun): every rank runs the same layers on its own
token batches (weak scaling, no collective on the data path); times are the
max over ranks.  ``--impl reference`` times the CPU oracle on the host cores on
a bounded sample of the headline workload.  ``--measure-peaks`` times
torch._scaled_mm (FP8 e4m3, and block-scaled FP4 where this torch supports it)
at 8192^3 and prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from rotated_bit_post_b200 import inputs, multirank  # noqa: E402

METRIC = "W4A4 rotated-linear tokens/s & effective TFLOPS (% FP4/FP8 peak) on 1 B200"
HEADLINE = "c5"
ORDER = ["c1", "c2", "c3", "c4", "c5", "c2p"]
L2_FLUSH_BYTES = 256 << 20

# Dense tensor-core work per SM per clock (FLOP), from the instruction rates:
# kind::f8f6f4 and kind::i8 retire a 128 x 256 x 32 MMA every 128 cycles
# (measured back to back on one CTA per SM), the block-scaled FP4 kind twice
# that (its nominal dense rate is 2x FP8), kind::f16 half of it.
MMA_FLOP_PER_CLK_SM = {"fp8": 2 * 128 * 256 * 32 / 128, "s8": 2 * 128 * 256 * 32 / 128,
                       "fp4": 2 * 128 * 256 * 64 / 128, "bf16": 2 * 128 * 256 * 16 / 128}
NOMINAL_RATIO_TO_BF16 = {"fp8": 2, "s8": 2, "fp4": 4}

# DRAM bytes (read + write) per launch of each kernel from a 1-pass ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the current kernels at the
# full sizes, L2 flushed before each step as in the timed run; None where the
# kernel changed after the last capture.  Outputs still dirty in L2 when a
# kernel ends are written back later and not counted here.  The capture command
# and per-kernel figures are kept with the other ncu summaries under profiles/.
TRAFFIC = {
    "k2": {"c1": 0.9e6, "c2": 5.8e6, "c3": None, "c4": 53.5e6, "c5": 1170.8e6, "c2p": 5.8e6},
    "k1": {"c1": 0.6e6, "c2": 9.6e6, "c3": 28.4e6, "c4": 122.9e6, "c5": 232.4e6, "c2p": 31.0e6},
}


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="all", choices=["all"] + ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bf16-linear", action="store_true", help="skip the cuBLAS BF16 linear on the same shapes")
    ap.add_argument("--tokens", type=int, default=0,
                    help="token rows per rank (default: the workload's own); smaller cases for profiler captures")
    ap.add_argument("--measure-peaks", action="store_true")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: CPU seconds for warm-up plus timed steps together")
    return ap.parse_args(argv)


def measured_peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
         "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        p.update({k: d[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained", "sm_max_mhz") if k in d})
        p["source"] = "measured"
    return p


def tensor_peak(kind: str, sms: int, run_mhz=None):
    """The denominator for a tensor-core kernel of `kind` ("fp8", "s8", "fp4"):
    the highest of (a) the measured BF16 matmul burst x the nominal ratio, and
    (b) the MMA issue rate x SM count x the maximum SM clock.  Both are returned
    with (c) the issue rate at the clock sampled during the run, for context."""
    pk = measured_peaks()
    from_bf16 = pk["bf16_tflops"] * NOMINAL_RATIO_TO_BF16[kind]
    issue_max = MMA_FLOP_PER_CLK_SM[kind] * sms * pk["sm_max_mhz"] * 1e6 / 1e12
    peak = max(from_bf16, issue_max)
    out = {"peak": peak,
           "peak_source": ("tcgen05 MMA issue rate x %d SMs x %.0f MHz (max clock)" % (sms, pk["sm_max_mhz"])
                           if issue_max >= from_bf16 else
                           "%s bf16 burst x nominal ratio %d" % (pk["source"], NOMINAL_RATIO_TO_BF16[kind])),
           "alt_peaks": {"bf16_burst_x_ratio": from_bf16, "mma_issue_rate_at_max_clock": issue_max}}
    if run_mhz:
        out["alt_peaks"]["mma_issue_rate_at_run_clock"] = MMA_FLOP_PER_CLK_SM[kind] * sms * run_mhz * 1e6 / 1e12
    return out


def mma_kind(w):
    from rotated_bit_post_b200 import rq
    return "fp4" if w.a_fmt == rq.NVFP4 else "s8" if w.a_fmt == rq.INT4 else "fp8"


DTYPE = {"fp4": "e2m1", "s8": "s8", "fp8": "e4m3"}
DTYPE_NOTE = {"fp4": "e2m1 x e2m1 with UE4M3 block scales, FP32 accumulate",
              "s8": "INT4 codes as s8 (16 v), S32 accumulate per 128-wide group, FP32 epilogue",
              "fp8": "codebook codes expanded to e4m3, FP32 accumulate"}


def workload_config(w, extra=None):
    fmt = inputs.FORMAT_NAMES
    cfg = {"workload": f"{w.name}: {w.description}", "M": w.M, "K": w.K, "N": w.N, "block": w.block,
           "formats": f"{fmt[w.a_fmt]}/{fmt[w.w_fmt]}", "rank": w.rank, "out": "bf16",
           "l2": "flushed before every step (256 MiB write, untimed)"}
    if extra:
        cfg.update(extra)
    return cfg


def flops_per_step(w):
    return 2.0 * w.M * w.N * w.K + 2.0 * w.M * w.N * w.rank


def pca_flops(w):
    """The rotation product y = x V of the full PCA rotation: 2 M K^2."""
    return 2.0 * w.M * w.K * w.K


def pca_rotation_bits(w):
    """V^T (K x K BF16 bits, row n = eigenvector n): all eigenvectors of the
    calibration tokens' second moment X^T X / n, dominant first.  A calibrated
    input of the layer, prepared once on the host like the weights."""
    cal = inputs.bf16_to_f32(inputs.calibration_tokens(w, n=max(inputs.CALIB_TOKENS, w.K))).astype(np.float64)
    ev, V = np.linalg.eigh(cal.T @ cal / cal.shape[0])
    V = V[:, np.argsort(ev)[::-1]]
    return inputs.bf16_bits(np.ascontiguousarray(V.T).astype(np.float32))


def k1_bytes(w):
    """Algorithmic bytes of one activation pass: BF16 read, packed codes, the
    per-token scale, NVFP4 block scales and the BF16 PCA coefficients (the full
    PCA rotation adds the FP32 rotated rows, written once and read once, and
    V once)."""
    from rotated_bit_post_b200 import rq
    per_tok = 2 * w.K + w.K // 2 + 4 + (w.K // 16 if w.a_fmt == rq.NVFP4 else 0) + 2 * w.rank
    if w.rotation == "pca":
        return w.M * (per_tok + 8 * w.K) + 2 * w.K * w.K
    return w.M * per_tok


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else None
    except Exception:
        return None


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}
    PERIOD_S = 0.001

    def __init__(self, index):
        self.samples, self.reasons, self.ok = [], set(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.PERIOD_S)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml, %d ms period, during the timed steps" % int(self.PERIOD_S * 1e3)}


# ----------------------------------------------------------------- CPU oracle
def oracle_step(w, X_bits, W_prep, tables):
    """The oracle's hot path on a sample of rows: rotate/quantize + FP64 GEMM."""
    from oracle import rq_oracle as orc
    if w.rotation == "pca":
        oa = orc.quantize_pca(orc.rotate_pca(inputs.bf16_to_f32(X_bits), tables), w.rank)
        return orc.reference_gemm(orc.INT4, orc.INT4, oa["q"], oa["scale"], W_prep["q"], W_prep["scale"],
                                  c_bf16=oa["coef"], L_bf16=W_prep["coef"])
    sign, perm, ab, ac, wc, U_f32 = tables
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X_bits), w.a_fmt, w.block, sign, perm, ab, U_f32)
    return orc.reference_gemm(w.a_fmt, w.w_fmt, oa["q"], oa["scale"], W_prep["q"], W_prep["scale"],
                              oa["block_scale"], W_prep["block_scale"], ac, wc, oa["coef"], W_prep["coef"])


def oracle_setup(w):
    from oracle import rq_oracle as orc
    if w.rotation == "pca":
        V = inputs.bf16_to_f32(np.ascontiguousarray(pca_rotation_bits(w).T))
        W_prep = orc.quantize_pca(orc.rotate_pca(inputs.bf16_to_f32(inputs.weights(w)), V), w.rank, weight_rows=True)
        return W_prep, V
    sign, perm = orc.make_rotation(w.K, w.block, 0)
    ab = ac = wb = wc = None
    if w.a_fmt == orc.LM16:
        ab, ac = orc.codebook_tables(w.K, 16)
    if w.w_fmt == orc.LM16:
        wb, wc = ab, ac
    elif w.w_fmt == orc.LM4:
        wb, wc = orc.codebook_tables(w.K, 4)
    U_f32 = None
    if w.rank:
        U64, _ = orc.pca_basis(inputs.bf16_to_f32(inputs.calibration_tokens(w)), w.rank)
        U_f32 = inputs.bf16_to_f32(inputs.bf16_bits(U64.astype(np.float32)))
    Wb = inputs.weights(w)
    W_prep = orc.rotate_quantize(inputs.bf16_to_f32(Wb), w.w_fmt, w.block, sign, perm, wb, U_f32, weight_rows=True)
    return W_prep, (sign, perm, ab, ac, wc, U_f32)


def cpu_baseline(w, target_s):
    """Time the oracle (as it stands) on a bounded sample of tokens; tokens/s.
    The sample is sized from a doubling probe so that it takes about
    `target_s` seconds."""
    W_prep, tables = oracle_setup(w)
    oracle_step(w, inputs.activations(w, M=32), W_prep, tables)  # warm (imports, BLAS threads)
    def timed(n):
        X = inputs.activations(w, M=n)
        t0 = time.perf_counter()
        oracle_step(w, X, W_prep, tables)
        return time.perf_counter() - t0

    # doubling probes until one takes an eighth of the target (or covers the
    # layer); the last two separate the per-call cost from the per-token cost
    n, t_prev = 32, timed(32)
    while n < w.M:
        n2 = min(w.M, 2 * n)
        t2 = timed(n2)
        per_tok = max((t2 - t_prev) / (n2 - n), t2 / n2 * 1e-3)
        n, t_prev = n2, t2
        if t2 >= target_s / 8:
            break
    else:
        per_tok = t_prev / n
    fixed = max(t_prev - n * per_tok, 0.0)
    rows = int(min(w.M, max(32, (target_s - fixed) / per_tok)))
    # a layer smaller than the target is run several times over
    reps = max(1, int((target_s - fixed) / max(rows * per_tok + fixed, 1e-6))) if rows == w.M else 1
    X = inputs.activations(w, M=rows)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle_step(w, X, W_prep, tables)
    dt = time.perf_counter() - t0
    return {"value": rows * reps / dt, "unit": "tokens/s", "cores": host_cores(), "blas_threads": blas_threads(),
            "kind": "oracle",
            "sample": f"{reps} x {rows} of {w.M} tokens of {w.name} (rotate/quantize + FP64 GEMM over all {w.N} "
                      f"outputs), {dt:.1f} s, weights prepared untimed; numpy element-wise steps single-threaded, "
                      f"FP64 matmul on the BLAS pool"}


def run_reference(args, w, rank, world):
    """The oracle as the reference arm: each step is a bounded sample of tokens,
    sized so that warm-up plus timed steps take about two minutes."""
    W_prep, tables = oracle_setup(w)
    probe = 16
    X = inputs.activations(w, M=probe)
    oracle_step(w, X, W_prep, tables)
    t0 = time.perf_counter()
    oracle_step(w, X, W_prep, tables)
    per_row = (time.perf_counter() - t0) / probe
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = int(max(8, min(w.M, budget / max(per_row, 1e-9))))
    X = inputs.activations(w, M=rows)
    for _ in range(args.warmup):
        oracle_step(w, X, W_prep, tables)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, X, W_prep, tables)
    dt = time.perf_counter() - t0
    tok_s = rows * args.steps / dt
    out = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": workload_config(w, {"sample_tokens_per_step": rows}),
           "effective_tflops": flops_per_step(w) * rows / w.M * args.steps / dt / 1e12,
           "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": host_cores(),
                            "blas_threads": blas_threads(), "kind": "oracle",
                            "sample": f"{rows} of {w.M} tokens of {w.name} per step (rotate/quantize + FP64 GEMM "
                                      f"over all {w.N} outputs), weights prepared untimed"},
           "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------- GPU arm
class Layer:
    """One layer on the device: tables, prepared weights, activation buffers and
    the two hot-path calls through the C ABI."""

    def __init__(self, w, dev, rank, stream):
        import torch
        from rotated_bit_post_b200 import rq
        self.w, self.dev, self.stream, self.rq = w, dev, stream, rq
        sign, perm, rot = rq.rq_make_rotation(w.K, w.block, 0)
        self.rot = torch.from_numpy(rot).to(dev)
        cb_a = rq.rq_make_codebook(w.K, 16) if w.a_fmt == rq.LM16 else None
        cb_w = cb_a if w.w_fmt == rq.LM16 else (rq.rq_make_codebook(w.K, 4) if w.w_fmt == rq.LM4 else None)
        self.U = None
        if w.rank:
            U_bits, _ = rq.rq_pca_basis(inputs.calibration_tokens(w), w.rank)
            self.U = torch.from_numpy(U_bits.view(np.int16)).to(dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        Wt = torch.from_numpy(inputs.weights(w).view(np.int16)).to(dev)
        self.wb = rq.weight_buffers(w.w_fmt, w.N, w.K, w.rank)
        rq.rq_quantize_weights(w.w_fmt, Wt, w.block, self.rot, None if cb_w is None else cb_w["boundaries_f32"],
                               self.U, self.wb["L"], self.wb["codes"], self.wb["scale"], self.wb["block_scale"],
                               self.status)
        del Wt
        self.X_np = multirank.rank_activations(w, rank)   # rank r draws its own tokens
        self.X = torch.from_numpy(self.X_np.view(np.int16)).to(dev)
        self.ab = rq.act_buffers(w.a_fmt, w.M, w.K, w.rank)
        self.Y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
        self.a_bnd = None if cb_a is None else cb_a["boundaries_f32"]
        self.a_lut = None if cb_a is None else cb_a["centroids_e4m3"]
        self.w_lut = None if cb_w is None else cb_w["centroids_e4m3"]
        self.check()

    def k1(self, x=None):
        w, ab = self.w, self.ab
        self.rq.rq_rotate_quantize_act(w.a_fmt, self.X if x is None else x, w.block, self.rot, self.a_bnd, self.U,
                                       ab["c"], ab["codes"], ab["scale"], ab["block_scale"], self.status,
                                       self.stream)

    def k2(self, y=None):
        w, ab, wb = self.w, self.ab, self.wb
        self.rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, w.M, w.N, w.K, ab["codes"], ab["scale"], ab["block_scale"],
                               wb["codes"], wb["scale"], wb["block_scale"], self.a_lut, self.w_lut, ab["c"],
                               wb["L"], self.Y if y is None else y, 0, self.status, self.stream)

    def check(self):
        import torch
        torch.cuda.synchronize()
        rc, code = self.rq.rq_read_status(self.status)
        if rc != 0:
            raise RuntimeError(f"kernel status {code:#x}")


class PcaLayer(Layer):
    """The same layer with the full PCA rotation: K1 is
    rq_pca_rotate_quantize_act (y = x V into an FP32 workspace, then the first
    r coordinates to BF16 and the rest to INT4); K2 is the INT4 GEMM with the
    rank-r BF16 term, as for the RPBH layer with the projection branch."""

    def __init__(self, w, dev, rank, stream):
        import torch
        from rotated_bit_post_b200 import rq
        self.w, self.dev, self.stream, self.rq = w, dev, stream, rq
        self.Vt = torch.from_numpy(pca_rotation_bits(w).view(np.int16)).to(dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        Wt = torch.from_numpy(inputs.weights(w).view(np.int16)).to(dev)
        ws = torch.empty((w.N, w.K), dtype=torch.float32, device=dev)
        self.wb = {"codes": torch.empty((w.N, w.K // 2), dtype=torch.uint8, device=dev),
                   "scale": torch.empty((w.K // 128, w.N), dtype=torch.float32, device=dev),
                   "L": torch.empty((w.N, w.rank), dtype=torch.int16, device=dev), "block_scale": None}
        rq.rq_pca_quantize_weights(Wt, self.Vt, w.rank, ws, self.wb["L"], self.wb["codes"], self.wb["scale"],
                                   self.status)
        del Wt, ws
        self.X_np = multirank.rank_activations(w, rank)
        self.X = torch.from_numpy(self.X_np.view(np.int16)).to(dev)
        self.ab = {"codes": torch.empty((w.M, w.K // 2), dtype=torch.uint8, device=dev),
                   "scale": torch.empty(w.M, dtype=torch.float32, device=dev),
                   "c": torch.empty((w.M, w.rank), dtype=torch.int16, device=dev), "block_scale": None}
        self.ws = torch.empty((w.M, w.K), dtype=torch.float32, device=dev)
        self.Y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
        self.a_bnd = self.a_lut = self.w_lut = None
        self.check()

    def k1(self, x=None):
        w, ab = self.w, self.ab
        self.rq.rq_pca_rotate_quantize_act(self.X if x is None else x, self.Vt, w.rank, self.ws, ab["c"],
                                           ab["codes"], ab["scale"], self.status, self.stream)


def make_layer(w, dev, rank, stream):
    return (PcaLayer if w.rotation == "pca" else Layer)(w, dev, rank, stream)


def time_layer(L, args, flush, dist):
    """Warm-up, then exactly `steps` timed steps (L2 flushed between them,
    outside the events), each bracketed by CUDA events on the launching stream
    and nothing in between, so that the GEMM's prologue overlaps the tail of
    the activation kernel (programmatic dependent launch).  Then a second run
    of the same steps with an event between the two kernels gives each
    kernel's own duration.  Returns (step ms list, k1 ms list, k2 ms list,
    clock summary)."""
    import torch
    stream = L.stream
    for _ in range(args.warmup):
        flush.zero_()
        L.k1()
        L.k2()
    L.check()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(L.dev.index) as clocks:
        for i in range(args.steps):
            flush.zero_()               # untimed: between the events of consecutive steps
            ev[i][0].record(stream)
            L.k1()
            L.k2()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    L.check()
    t_step = [e[0].elapsed_time(e[1]) for e in ev]
    n_split = max(5, min(50, args.steps))
    ev3 = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_split)]
    for i in range(n_split):
        flush.zero_()
        ev3[i][0].record(stream)
        L.k1()
        ev3[i][1].record(stream)
        L.k2()
        ev3[i][2].record(stream)
    torch.cuda.synchronize()
    L.check()
    t_k1 = [e[0].elapsed_time(e[1]) for e in ev3]
    t_k2 = [e[1].elapsed_time(e[2]) for e in ev3]
    return t_step, t_k1, t_k2, clocks.summary()


def time_bf16_linear(L, args, flush):
    """The same layer as a plain BF16 linear (cuBLAS via torch), for context."""
    import torch
    w = L.w
    Wb = torch.from_numpy(inputs.weights(w).view(np.int16)).to(L.dev).view(torch.bfloat16)
    Xb = L.X.view(torch.bfloat16)
    Yb = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=L.dev)
    for _ in range(3):
        torch.matmul(Xb, Wb.t(), out=Yb)
    n_lin = max(5, min(50, args.steps))
    evl = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_lin)]
    for a, b in evl:
        flush.zero_()
        a.record(L.stream)
        torch.matmul(Xb, Wb.t(), out=Yb)
        b.record(L.stream)
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in evl)
    return {"ms": ms, "tflops": 2.0 * w.M * w.N * w.K / (ms * 1e-3) / 1e12, "tokens_per_s": w.M / (ms * 1e-3),
            "what": "torch.matmul BF16 x BF16^T (cuBLAS), same M, N, K, L2 flushed before each call, median of "
                    f"{n_lin}; no rotation or quantization"}


def time_e2e(L, args, dist, world):
    """End to end through the public API with host buffers.  Every step copies
    its token batch from pinned host memory to the device, runs K1 and K2, and
    copies its BF16 output back to pinned host memory.  The copies run on their
    own streams, double-buffered, so that step i+1's upload and step i-1's
    download overlap step i's kernels (PCIe is full duplex); the timed region
    spans the first upload to the last download."""
    import torch
    w, dev, stream = L.w, L.dev, L.stream
    X_host = torch.from_numpy(L.X_np.view(np.int16)).pin_memory()
    Y_host = torch.empty((w.M, w.N), dtype=torch.bfloat16).pin_memory()
    Xd = [torch.empty_like(L.X), torch.empty_like(L.X)]
    Yd = [L.Y, torch.empty_like(L.Y)]
    s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    n_e2e = max(5, min(30, args.steps))

    def run_steps(n, e_first=None, e_last=None):
        up_done = [torch.cuda.Event() for _ in range(n)]
        x_free = [torch.cuda.Event() for _ in range(n)]
        comp_done = [torch.cuda.Event() for _ in range(n)]
        down_done = [torch.cuda.Event() for _ in range(n)]
        if e_first is not None:
            e_first.record(s_up)
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(s_up):
                if i >= 2:
                    s_up.wait_event(x_free[i - 2])
                Xd[b].copy_(X_host, non_blocking=True)
                up_done[i].record(s_up)
            stream.wait_event(up_done[i])
            if i >= 2:
                stream.wait_event(down_done[i - 2])
            L.k1(Xd[b])
            x_free[i].record(stream)
            L.k2(Yd[b])
            comp_done[i].record(stream)
            with torch.cuda.stream(s_down):
                s_down.wait_event(comp_done[i])
                Y_host.copy_(Yd[b], non_blocking=True)
                down_done[i].record(s_down)
        if e_last is not None:
            e_last.record(s_down)

    run_steps(3)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    run_steps(n_e2e, e0, e1)
    torch.cuda.synchronize()
    ms = multirank.max_over_ranks(dist, e0.elapsed_time(e1) / n_e2e, dev)
    L.check()
    return {"value": multirank.aggregate_tokens_per_s(w.M, world, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": L.X.numel() * 2, "d2h_bytes_per_step": L.Y.numel() * 2, "ms_per_step": ms,
            "steps": n_e2e,
            "note": "per step: pinned host X -> device, K1, K2, device Y -> pinned host; uploads and downloads "
                    "on their own streams overlap the neighbouring steps' kernels"}


def layer_result(L, args, t_step, t_k1, t_k2, clocks, dist, world, sms):
    """Per-layer figures: step time (sum over exactly `steps` steps, max over
    ranks), per-kernel medians, and the roofline of the dominant kernel."""
    w = L.w
    step_ms_total = multirank.max_over_ranks(dist, sum(t_step), L.dev)
    ms_per_step = step_ms_total / args.steps
    med_step = statistics.median(t_step)
    k1_ms, k2_ms = statistics.median(t_k1), statistics.median(t_k2)
    fl = flops_per_step(w)
    kind = mma_kind(w)
    tp = tensor_peak(kind, sms, clocks.get("sm_mhz"))
    pk = measured_peaks()
    k2_tflops = fl / (k2_ms * 1e-3) / 1e12
    kb = k1_bytes(w)
    k1_gbs = kb / (k1_ms * 1e-3) / 1e9
    k1_roof = {"kernel": "k1_rotate_quantize (rq_rotate_quantize_act)", "bound": "hbm", "achieved": k1_gbs,
               "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": k1_gbs / pk["hbm_gbs"],
               "frac_of_8tbs": k1_gbs / 8000.0,
               "peak_source": pk["source"] + " copy (MEASURED_PEAKS hbm_gbs)",
               "algorithmic_per_launch": f"{kb} B (2K + K/2 + 4 [+ K/16] [+ 2r] per token)",
               "traffic": None if args.tokens else TRAFFIC["k1"].get(w.name)}
    if w.rotation == "pca":
        # the rotation product bounds it: a BF16 contraction of 2 M K^2 FLOP
        # (the split/quantize pass that follows is in the same time)
        pf = pca_flops(w)
        k1_tf = pf / (k1_ms * 1e-3) / 1e12
        k1_roof = {"kernel": "dense_gemm_kernel<BF16> + pca_quant_kernel (rq_pca_rotate_quantize_act)", "bound": "tensor",
                   "achieved": k1_tf, "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": k1_tf / pk["bf16_tflops"],
                   "peak_source": pk["source"] + " bf16 burst (MEASURED_PEAKS bf16_tflops)",
                   "algorithmic_per_launch": f"{pf:.4g} FLOP (2MK^2); HBM {kb} B at {k1_gbs:.0f} GB/s "
                                             f"(2K + 8K + K/2 + 4 + 2r per token, + 2K^2 for V)",
                   "traffic": None if args.tokens else TRAFFIC["k1"].get(w.name)}
    k2_roof = {"kernel": "gemm kernel of rq_w4a4_linear", "bound": "tensor", "achieved": k2_tflops,
               "peak": tp["peak"], "unit": "TFLOP/s", "frac": k2_tflops / tp["peak"],
               "peak_source": tp["peak_source"], "alt_peaks": tp["alt_peaks"],
               "algorithmic_per_launch": f"{fl:.4g} FLOP (2MNK + 2MNr)",
               "traffic": None if args.tokens else TRAFFIC["k2"].get(w.name)}
    dominant = k2_roof if k2_ms >= k1_ms else k1_roof
    return {
        "config": workload_config(w),
        "dtype": DTYPE[kind], "dtype_note": DTYPE_NOTE[kind],
        "tokens_per_s": multirank.aggregate_tokens_per_s(w.M, world, ms_per_step),
        "ms_per_step": ms_per_step, "median_ms_per_step": med_step,
        "effective_tflops": fl * world / (ms_per_step * 1e-3) / 1e12,
        "effective_frac_of_peak": fl / (med_step * 1e-3) / 1e12 / tp["peak"],
        "kernels": {"k1_rotate_quantize_us": 1e3 * k1_ms, "k1_gbs": k1_gbs, "k1_frac_hbm": k1_gbs / pk["hbm_gbs"],
                    "k2_gemm_us": 1e3 * k2_ms, "k2_tflops": k2_tflops, "k2_frac_peak": k2_tflops / tp["peak"],
                    "timing": "medians over steps timed with an event between the two kernels (the timed "
                              "steps themselves have none, so the GEMM prologue overlaps the activation "
                              "kernel's tail)"},
        "roofline": dominant, "roofline_k1": k1_roof, "roofline_k2": k2_roof,
        "clocks": clocks,
    }


def run_ours(args, names, rank, world, dist):
    import torch

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    results = {}
    for name in names:
        w = inputs.workload(name)
        if args.tokens:
            w = dataclasses.replace(w, M=args.tokens)
        L = make_layer(w, dev, rank, stream)
        t_step, t_k1, t_k2, clocks = time_layer(L, args, flush, dist)
        res = layer_result(L, args, t_step, t_k1, t_k2, clocks, dist, world, sms)
        if not args.no_bf16_linear:
            res["bf16_linear"] = time_bf16_linear(L, args, flush)
            res["speedup_vs_bf16_linear"] = res["bf16_linear"]["ms"] / res["median_ms_per_step"]
        if not args.no_e2e:
            res["e2e"] = time_e2e(L, args, dist, world)
        results[name] = res
        del L
        torch.cuda.empty_cache()

    if rank != 0:
        return
    head = results[HEADLINE] if HEADLINE in results else results[names[-1]]
    hw = inputs.workload(HEADLINE if HEADLINE in results else names[-1])
    out = {"metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
           "median_ms_per_step": head["median_ms_per_step"], "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": head["dtype"], "dtype_note": head["dtype_note"],
           "data": "synthetic (seeded DiT-shaped activations, N(0,0.02) weights)",
           "config": dict(head["config"], parallelism=f"token-parallel x{world} (independent batches)"),
           "effective_tflops": head["effective_tflops"], "effective_frac_of_peak": head["effective_frac_of_peak"],
           "kernels": head["kernels"], "roofline": head["roofline"], "clocks": head["clocks"],
           "e2e": head.get("e2e"), "bf16_linear": head.get("bf16_linear"),
           "speedup_vs_bf16_linear": head.get("speedup_vs_bf16_linear"),
           "gpu_launches": 2 * args.steps,
           "gpu_launches_note": "per timed step of the headline layer: one K1 and one K2 launch"}
    if len(names) > 1:
        out["configs"] = {n: results[n] for n in names}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(hw, 15.0)
        if len(names) > 1:
            for n in names:
                if n != HEADLINE:
                    out["configs"][n]["cpu_baseline"] = cpu_baseline(inputs.workload(n), 3.0)
            out["configs"][HEADLINE]["cpu_baseline"] = out["cpu_baseline"]
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------- peaks
def measure_peaks():
    """torch._scaled_mm at 8192^3: FP8 e4m3 (per-tensor scales) and, where this
    torch supports it, NVFP4 (e2m1 with e4m3 scales per 16 elements); best of
    10 calls (burst) and back to back for 4 s (sustained)."""
    import torch
    dev = torch.device("cuda", 0)
    n = 8192
    out = {"what": "torch._scaled_mm %d^3" % n, "torch": torch.__version__}

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        best = 1e9
        for _ in range(10):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            best = min(best, a.elapsed_time(b))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cnt = 0
        t0 = time.time()
        with ClockSampler(0) as clk:
            a.record()
            while time.time() - t0 < 4.0:
                for _ in range(20):
                    fn()
                cnt += 20
                torch.cuda.synchronize()
            b.record()
            torch.cuda.synchronize()
        sus = a.elapsed_time(b) / cnt
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12, 2.0 * n ** 3 / (sus * 1e-3) / 1e12, clk.summary()

    a = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device=dev).to(torch.float8_e4m3fn).t()
    one = torch.ones((), device=dev)
    burst, sus, clk = timed(lambda: torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16))
    out["fp8_e4m3"] = {"burst_tflops": burst, "sustained_tflops": sus, "clocks": clk}
    try:
        fp4 = getattr(torch, "float4_e2m1fn_x2")
        a4 = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(fp4)
        b4 = torch.randint(0, 256, (n, n // 2), dtype=torch.uint8, device=dev).view(fp4)
        # block scales: one e4m3 per 16 elements, in the swizzled 128x4 layout cuBLAS expects
        sa = torch.full((n * n // 16,), 1.0, device=dev).to(torch.float8_e4m3fn)
        sb = torch.full((n * n // 16,), 1.0, device=dev).to(torch.float8_e4m3fn)
        burst, sus, clk = timed(lambda: torch._scaled_mm(a4, b4.t(), sa, sb, out_dtype=torch.bfloat16))
        out["fp4_nvfp4"] = {"burst_tflops": burst, "sustained_tflops": sus, "clocks": clk}
    except Exception as e:  # not every torch build routes block-scaled FP4 through _scaled_mm
        out["fp4_nvfp4"] = {"unavailable": f"{type(e).__name__}: {str(e)[:200]}"}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.measure_peaks:
        measure_peaks()
        return
    names = ORDER if args.config == "all" else [args.config]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle runs once, on rank 0, on the headline layer; other ranks have nothing to do
        if rank == 0:
            w = inputs.workload(HEADLINE if args.config == "all" else args.config)
            if args.tokens:
                w = dataclasses.replace(w, M=args.tokens)
            run_reference(args, w, rank, world)
        return
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, names, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
