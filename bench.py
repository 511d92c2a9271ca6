"""Throughput of the rotated W4A4 linear layer on B200.

One step = the whole online hot path on one batch of tokens:
  K1  rq_rotate_quantize_act  (PCA projection + RPBH rotate + normalise + INT4/LM/NVFP4 quantize + pack)
  K2  rq_w4a4_linear          (4-bit x 4-bit tcgen05 GEMM + fused rank-r low-rank add, BF16 out)
Weights are folded and quantized once, offline, before timing.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs the same
layer on its own token batch (weak scaling, no collective on the data path);
the time is the max over ranks.  ``--impl reference`` times the CPU oracle on
the host cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
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
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="c2", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-bf16-linear", action="store_true", help="skip the cuBLAS BF16 linear on the same shapes")
    ap.add_argument("--tokens", type=int, default=0,
                    help="token rows per rank (default: the workload's own); smaller cases for profiler captures")
    return ap.parse_args()


def peaks():
    p = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        p.update({k: d[k] for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained") if k in d})
        p["source"] = "measured"
    return p


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


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

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
            time.sleep(0.005)

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
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, 5 ms period"}


# ----------------------------------------------------------------- CPU oracle
def oracle_step(w, X_bits, W_prep, tables):
    """The oracle's hot path on a sample of rows: rotate/quantize + FP64 GEMM."""
    from oracle import rq_oracle as orc
    sign, perm, ab, ac, wc, U_f32 = tables
    oa = orc.rotate_quantize(inputs.bf16_to_f32(X_bits), w.a_fmt, w.block, sign, perm, ab, U_f32)
    return orc.reference_gemm(w.a_fmt, w.w_fmt, oa["q"], oa["scale"], W_prep["q"], W_prep["scale"],
                              oa["block_scale"], W_prep["block_scale"], ac, wc, oa["coef"], W_prep["coef"])


def oracle_setup(w, n_weight_rows=None):
    from oracle import rq_oracle as orc
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


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [p.get("num_threads") for p in threadpool_info() if p.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(w, target_s=12.0):
    """Time the oracle (as it stands) on a bounded sample of tokens; tokens/s."""
    W_prep, tables = oracle_setup(w)
    rows = 64
    X = inputs.activations(w, M=rows)
    oracle_step(w, X, W_prep, tables)  # warm (imports, BLAS threads)
    t0 = time.perf_counter()
    oracle_step(w, X, W_prep, tables)
    dt = time.perf_counter() - t0
    rows = int(min(w.M, max(64, rows * target_s / max(dt, 1e-3) / 2)))
    X = inputs.activations(w, M=rows)
    t0 = time.perf_counter()
    oracle_step(w, X, W_prep, tables)
    dt = time.perf_counter() - t0
    return {"value": rows / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{rows} of {w.M} tokens of {w.name} (rotate/quantize + FP64 GEMM over all {w.N} outputs), "
                      f"{dt:.1f} s, weights prepared untimed"}


def run_reference(args, w, rank, world):
    """The oracle as the reference arm: each step is a bounded sample of tokens,
    sized so that warm-up plus timed steps take about two minutes."""
    W_prep, tables = oracle_setup(w)
    probe = 32
    X = inputs.activations(w, M=probe)
    oracle_step(w, X, W_prep, tables)
    t0 = time.perf_counter()
    oracle_step(w, X, W_prep, tables)
    per_row = (time.perf_counter() - t0) / probe
    budget = 120.0 / max(1, args.steps + args.warmup)
    rows = int(max(16, min(w.M, budget / max(per_row, 1e-9))))
    X = inputs.activations(w, M=rows)
    for _ in range(args.warmup):
        oracle_step(w, X, W_prep, tables)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(w, X, W_prep, tables)
    dt = time.perf_counter() - t0
    tok_s = rows * args.steps / dt
    cores = blas_threads()
    out = {"impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": workload_config(w, {"sample_tokens_per_step": rows}),
           "effective_tflops": flops_per_step(w) * rows / w.M * args.steps / dt / 1e12,
           "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                            "sample": f"{rows} of {w.M} tokens of {w.name} per step (rotate/quantize + FP64 GEMM "
                                      f"over all {w.N} outputs), weights prepared untimed"},
           "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
           "gpu_launches": 0}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------- GPU arm
def run_ours(args, w, rank, world, dist):
    import torch
    from rotated_bit_post_b200 import rq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()

    # ---------------- offline preparation (untimed)
    sign, perm, rot = rq.rq_make_rotation(w.K, w.block, 0)
    rot_t = torch.from_numpy(rot).to(dev)
    cb_a = rq.rq_make_codebook(w.K, 16) if w.a_fmt == rq.LM16 else None
    cb_w = cb_a if w.w_fmt == rq.LM16 else (rq.rq_make_codebook(w.K, 4) if w.w_fmt == rq.LM4 else None)
    U_t = None
    if w.rank:
        U_bits, _ = rq.rq_pca_basis(inputs.calibration_tokens(w), w.rank)
        U_t = torch.from_numpy(U_bits.view(np.int16)).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    Wt = torch.from_numpy(inputs.weights(w).view(np.int16)).to(dev)
    wb = rq.weight_buffers(w.w_fmt, w.N, w.K, w.rank)
    rq.rq_quantize_weights(w.w_fmt, Wt, w.block, rot_t, None if cb_w is None else cb_w["boundaries_f32"], U_t,
                           wb["L"], wb["codes"], wb["scale"], wb["block_scale"], status)
    del Wt
    # this rank's token batch (rank r draws its own tokens)
    X_np = multirank.rank_activations(w, rank)
    X = torch.from_numpy(X_np.view(np.int16)).to(dev)
    ab = rq.act_buffers(w.a_fmt, w.M, w.K, w.rank)
    Y = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
    a_bnd = None if cb_a is None else cb_a["boundaries_f32"]
    a_lut = None if cb_a is None else cb_a["centroids_e4m3"]
    w_lut = None if cb_w is None else cb_w["centroids_e4m3"]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def k1(x):
        rq.rq_rotate_quantize_act(w.a_fmt, x, w.block, rot_t, a_bnd, U_t, ab["c"], ab["codes"], ab["scale"],
                                  ab["block_scale"], status, stream)

    def k2(y=None):
        rq.rq_w4a4_linear(w.a_fmt, w.w_fmt, w.M, w.N, w.K, ab["codes"], ab["scale"], ab["block_scale"],
                          wb["codes"], wb["scale"], wb["block_scale"], a_lut, w_lut, ab["c"], wb["L"],
                          Y if y is None else y, 0, status, stream)

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        flush.zero_()
        k1(X)
        k2()
    torch.cuda.synchronize()
    rc, code = rq.rq_read_status(status)
    if rc != 0:
        raise RuntimeError(f"kernel status {code:#x}")

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        for i in range(args.steps):
            flush.zero_()               # untimed: between the events of consecutive steps
            ev[i][0].record(stream)
            k1(X)
            ev[i][1].record(stream)
            k2()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    barrier()
    t_k1 = [e[0].elapsed_time(e[1]) for e in ev]
    t_k2 = [e[1].elapsed_time(e[2]) for e in ev]
    step_ms = sum(a + b for a, b in zip(t_k1, t_k2))
    step_ms = multirank.max_over_ranks(dist, step_ms, dev)
    rc, code = rq.rq_read_status(status)
    if rc != 0:
        raise RuntimeError(f"kernel status {code:#x}")

    # ---------------- the same layer as a plain BF16 linear (cuBLAS via torch), for context
    bf16_linear = None
    if not args.no_bf16_linear:
        Wb = torch.from_numpy(inputs.weights(w).view(np.int16)).to(dev).view(torch.bfloat16)
        Xb = X.view(torch.bfloat16)
        Yb = torch.empty((w.M, w.N), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            torch.matmul(Xb, Wb.t(), out=Yb)
        n_lin = max(5, min(50, args.steps))
        evl = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_lin)]
        for a, b in evl:
            flush.zero_()
            a.record(stream)
            torch.matmul(Xb, Wb.t(), out=Yb)
            b.record(stream)
        torch.cuda.synchronize()
        lin_ms = statistics.mean(a.elapsed_time(b) for a, b in evl)
        bf16_linear = {"ms": lin_ms, "tflops": 2.0 * w.M * w.N * w.K / (lin_ms * 1e-3) / 1e12,
                       "tokens_per_s": w.M / (lin_ms * 1e-3), "what": "torch.matmul BF16 x BF16^T (cuBLAS), "
                       "same M, N, K, L2 flushed before each call, no rotation or quantization"}
        del Wb, Yb

    # ---------------- end to end through the public API with host buffers
    # Every step copies its token batch from pinned host memory to the device,
    # runs K1 and K2, and copies its BF16 output back to pinned host memory.
    # The copies run on their own streams, double-buffered, so that step i+1's
    # upload and step i-1's download overlap step i's kernels (PCIe is full
    # duplex); the timed region spans the first upload to the last download.
    e2e = None
    if not args.no_e2e:
        X_host = torch.from_numpy(X_np.view(np.int16)).pin_memory()
        Y_host = torch.empty((w.M, w.N), dtype=torch.bfloat16).pin_memory()
        Xd = [torch.empty_like(X), torch.empty_like(X)]
        Yd = [Y, torch.empty_like(Y)]
        s_up, s_down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        n_e2e = max(5, min(50, args.steps))

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
                k1(Xd[b])
                x_free[i].record(stream)
                k2(Yd[b])
                comp_done[i].record(stream)
                with torch.cuda.stream(s_down):
                    s_down.wait_event(comp_done[i])
                    Y_host.copy_(Yd[b], non_blocking=True)
                    down_done[i].record(s_down)
            if e_last is not None:
                e_last.record(s_down)

        run_steps(3)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run_steps(n_e2e, e0, e1)
        torch.cuda.synchronize()
        e2e_ms = e0.elapsed_time(e1) / n_e2e
        e2e_ms = multirank.max_over_ranks(dist, e2e_ms, dev)
        rc, code = rq.rq_read_status(status)
        if rc != 0:
            raise RuntimeError(f"kernel status {code:#x}")
        e2e = {"value": multirank.aggregate_tokens_per_s(w.M, world, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": X.numel() * 2,
               "d2h_bytes_per_step": Y.numel() * 2, "ms_per_step": e2e_ms,
               "note": "per step: pinned host X -> device, K1, K2, device Y -> pinned host; uploads and "
                       "downloads on their own streams overlap the neighbouring steps' kernels"}
        del Xd, Yd

    if rank != 0:
        return

    ms_per_step = step_ms / args.steps
    k1_ms = statistics.mean(t_k1)
    k2_ms = statistics.mean(t_k2)
    tok_s = multirank.aggregate_tokens_per_s(w.M, world, ms_per_step)
    fl = flops_per_step(w)
    pk = peaks()
    mma_ratio = 4 if w.a_fmt == rq.NVFP4 else 2          # nominal FP4 / FP8 vs BF16 dense ratio
    tensor_peak = pk["bf16_tflops"] * mma_ratio
    k2_tflops = fl / (k2_ms * 1e-3) / 1e12
    k1_bytes = w.M * (2 * w.K + w.K // 2 + 4 + (w.K // 16 if w.a_fmt == rq.NVFP4 else 0) + 2 * w.rank)
    k1_gbs = k1_bytes / (k1_ms * 1e-3) / 1e9
    dominant_is_k2 = k2_ms >= k1_ms
    if dominant_is_k2:
        roof = {"kernel": "rq_w4a4_linear (gemm_fp8/nvf4)", "bound": "tensor", "achieved": k2_tflops,
                "peak": tensor_peak, "unit": "TFLOP/s", "frac": k2_tflops / tensor_peak,
                "peak_source": f"{pk['source']} bf16 burst {pk['bf16_tflops']} x nominal ratio {mma_ratio} "
                               f"({'fp4' if mma_ratio == 4 else 'fp8'}/bf16)",
                "algorithmic_per_launch": f"{fl:.4g} FLOP (2MNK + 2MNr)", "traffic": None if args.tokens else TRAFFIC.get(w.name)}
    else:
        roof = {"kernel": "rq_rotate_quantize_act", "bound": "hbm", "achieved": k1_gbs, "peak": pk["hbm_gbs"],
                "unit": "GB/s", "frac": k1_gbs / pk["hbm_gbs"], "peak_source": pk["source"] + " copy",
                "algorithmic_per_launch": f"{k1_bytes} B", "traffic": None}
    out = {"metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "e4m3" if w.a_fmt != rq.NVFP4 else "e2m1",
           "data": "synthetic (seeded DiT-shaped activations, N(0,0.02) weights)",
           "config": workload_config(w, {"parallelism": f"token-parallel x{world} (independent batches)"}),
           "effective_tflops": fl * world / (ms_per_step * 1e-3) / 1e12,
           "effective_frac_of_peak": fl / (ms_per_step * 1e-3) / 1e12 / tensor_peak,
           "kernels": {"k1_rotate_quantize_us": 1e3 * k1_ms, "k1_gbs": k1_gbs,
                       "k1_frac_hbm": k1_gbs / pk["hbm_gbs"], "k2_gemm_us": 1e3 * k2_ms,
                       "k2_tflops": k2_tflops, "k2_frac_peak": k2_tflops / tensor_peak},
           "roofline": roof, "clocks": clocks.summary(), "e2e": e2e,
           "bf16_linear": bf16_linear,
           "speedup_vs_bf16_linear": None if bf16_linear is None else bf16_linear["ms"] / ms_per_step,
           "gpu_launches": 2 * args.steps}
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(out), flush=True)


# DRAM bytes per launch of the GEMM (read + write) from a 1-pass ncu capture of
# the current kernels at the full sizes, keyed by workload (the DRAM-traffic
# summary under profiles/ gives the command and the per-kernel figures).
# (None: the kernel changed after the last capture)
TRAFFIC = {"c2": 5_847_552, "c3": None, "c4": 56_036_096, "c5": None}


def main():
    args = parse()
    w = inputs.WORKLOADS[args.config]
    if args.tokens:
        w = dataclasses.replace(w, M=args.tokens)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle runs once, on rank 0; other ranks have nothing to do
        if rank == 0:
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
        run_ours(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
