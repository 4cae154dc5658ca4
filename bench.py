#!/usr/bin/env python
"""Throughput of the GPTQ layer solver on B200: quantized weights/s per layer, split by phase.

One step = the whole hot path on one synthetic layer: H = 2 X^T X over the calibration tokens,
dampening + U = chol(H^-1), the column loop with lazy block updates, and packing.  Inputs (X, W)
are resident in HBM before timing; X (0.40 GB for the default layer) is larger than the 126 MB L2,
so every step streams it from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--layer NAME] [--impl ours|reference]

N > 1 runs under torchrun, one rank per GPU; each rank quantizes its own copy of the layer
(independent problems, no collective on the data path), so the job's value is N layers per step.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ quantized weights/sec & per-layer solve ms (1×B200), % of phase roofline"
DEFAULT_LAYER = "opt125m_768x768"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--layer", default=DEFAULT_LAYER)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=10)
    return p.parse_args()


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def slowest_rank_ms(ms: float, device) -> float:
    """The largest of the ranks' device-timed values (a multi-GPU time is the slowest rank's)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def layer_for_rank(L, rank: int):
    """Rank r quantizes its own layer of the same shape (inputs seeded seed + r): weak scaling, no
    data-path collective."""
    import dataclasses
    return dataclasses.replace(L, seed=L.seed + rank)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# fp32 FMA peak of the part: 148 SMs x 128 FMA lanes x 2 flops x clock (nominal max 1965 MHz)
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 / bf16 tensor throughput of the B200


def fp32_peak_tflops(sm_mhz: float) -> float:
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu, self.proc, self.path = gpu_index, None, None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def kernel_traffic(name: str, sources: list[str]):
    """DRAM bytes per launch recorded from an ncu capture, if the kernel source is unchanged since."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(name)
    if not rec:
        return None
    h = hashlib.sha256()
    for s in sources:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return rec["bytes_per_launch"] if rec.get("source_sha256") == h.hexdigest() else None


def cores_info():
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        blas = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=cores)
    except Exception:
        blas = cores
    return cores, blas


def oracle_step(L, W64, X):
    """One step of the oracle on the layer: the fp64 statement of the whole path (test infrastructure)."""
    import numpy as np
    import oracle
    H = np.zeros((L.d, L.d))
    for t0 in range(0, L.n_tokens, 16384):
        oracle.hessian_accumulate(H, X[t0:t0 + 16384].double().numpy())
    res = oracle.gptq_layer(W64, None, L.bits, L.group_size, L.block_size, L.damp, H=H)
    return res


def run_reference(args, L):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from post_weight_quantization_21_b200 import workloads as wl
    W64 = wl.make_w(L).double().numpy()
    X = wl.make_x(L)
    for _ in range(args.warmup):
        oracle_step(L, W64, X)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(L, W64, X)
    dt = (time.perf_counter() - t0) / args.steps
    value = L.m * L.d / dt
    cores, blas = cores_info()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(L),
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": blas, "kind": "oracle",
                             "sample": f"the full {L.name} layer per step: fp64 H over all {L.n_tokens} tokens, "
                                       "U, column loop, pack (numpy/BLAS on the host cores)"},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(L):
    xb = L.n_tokens * L.d * (2 if str(L.x_dtype).endswith("16") else 4)
    return {"workload": L.name, "m": L.m, "d": L.d, "n_tokens": L.n_tokens, "bits": L.bits,
            "group_size": L.group_size, "block_size": L.block_size, "damp": L.damp,
            "w_dtype": str(L.w_dtype).replace("torch.", ""), "x_dtype": str(L.x_dtype).replace("torch.", ""),
            "l2": f"inputs larger than L2: X = {xb / 1e9:.2f} GB streamed from HBM every step"}


def main():
    args = parse()
    from post_weight_quantization_21_b200 import workloads as wl
    L = wl.LAYERS[args.layer]
    if args.impl == "reference":
        return run_reference(args, L)

    import torch
    import torch.distributed as dist
    import post_weight_quantization_21_b200 as g

    rank, world, local = dist_env()
    L = layer_for_rank(L, rank)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    pk = peaks()

    solver = g.LayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, L.x_dtype,
                           L.w_dtype, device=dev)
    # seeded inputs made on the device (the large layers' X is tens of GB); host copies below
    solver.W.copy_(wl.make_w(L, device=dev))
    wl.make_x(L, device=dev, out=solver.X)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        solver.hessian(stream)
        if ev is not None:
            ev[1].record(stream)
        solver.prepare(stream)
        if ev is not None:
            ev[2].record(stream)
        solver.quantize(stream)
        if ev is not None:
            ev[3].record(stream)
        solver.pack(stream)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    solver.check_status(stream)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = g.gptq_kernel_launches()
    start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    end.record(stream)
    torch.cuda.synchronize(dev)
    launches = g.gptq_kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    solver.check_status(stream)

    total_ms = start.elapsed_time(end)
    phase_ms = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(4)]
    total_ms = slowest_rank_ms(total_ms, dev)
    ms_per_step = total_ms / args.steps
    value = world * L.m * L.d / (ms_per_step * 1e-3)

    # end to end through the host: pinned inputs in, packed codes + grids out, every step
    W_h = torch.empty(solver.W.shape, dtype=solver.W.dtype).pin_memory()
    X_h = torch.empty(solver.X.shape, dtype=solver.X.dtype).pin_memory()
    W_h.copy_(solver.W)
    X_h.copy_(solver.X)
    n_groups = 1 if L.group_size == 0 else L.d // L.group_size
    out_p = torch.empty(L.m, L.d * L.bits // 32, dtype=torch.int32).pin_memory()
    out_s = torch.empty(L.m, n_groups, dtype=torch.float32).pin_memory()
    out_z = torch.empty(L.m, n_groups, dtype=torch.int32).pin_memory()
    solver.run_host(W_h, X_h, out_p, out_s, out_z, stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(args.e2e_steps):
        solver.run_host(W_h, X_h, out_p, out_s, out_z, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = slowest_rank_ms(e2e_ms, dev)
    h2d = W_h.numel() * W_h.element_size() + X_h.numel() * X_h.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (out_p, out_s, out_z))

    # roofline of each phase (algorithmic work per launch / measured time), against the pipe the
    # library runs it on for this shape: bf16 tensor cores (Hessian), 3xTF32 tensor cores (block
    # products of the blocked prepare, lazy block updates), or fp32 FMA units
    sm_mhz = clk["sm_mhz"] if clk else 1965.0
    long_region = total_ms > 1000.0
    bf16_peak = pk["bf16_tflops_sustained"] if long_region else pk["bf16_tflops"]
    fp32_peak = fp32_peak_tflops(1965.0)
    tf32x3_peak = bf16_peak * TF32_PER_BF16 / 3.0   # three tf32 MMAs per fp32-accurate product
    tc = g.gptq_tensor_core_phases(L.m, L.d, L.n_tokens, L.x_dtype, L.bits, L.group_size, L.block_size)
    h_flops = L.n_tokens * L.d * (L.d + 1)                 # symmetric half of 2 N d^2
    p_flops = 2.0 / 3.0 * L.d ** 3                          # Cholesky + triangular inverse
    q_flops = float(L.m) * L.d * L.d                        # column loop + lazy updates
    k_bytes = L.m * L.d * (1 + L.bits / 8)                  # pack: codes in, words out
    p_peak, p_pipe = (tf32x3_peak, "tensor(3xtf32)") if tc & g.GPTQ_TC_PREPARE else (fp32_peak, "fp32 FMA")
    q_peak, q_pipe = (tf32x3_peak, "tensor(3xtf32)") if tc & g.GPTQ_TC_LAZY else (fp32_peak, "fp32 FMA")
    phases = {
        "hessian": {"ms": phase_ms[0], "tflops": h_flops / phase_ms[0] / 1e9,
                    "frac": h_flops / phase_ms[0] / 1e9 / bf16_peak, "pipe": "tensor(bf16)"},
        "prepare": {"ms": phase_ms[1], "tflops": p_flops / phase_ms[1] / 1e9,
                    "frac": p_flops / phase_ms[1] / 1e9 / p_peak, "pipe": p_pipe},
        "quantize": {"ms": phase_ms[2], "tflops": q_flops / phase_ms[2] / 1e9,
                     "frac": q_flops / phase_ms[2] / 1e9 / q_peak, "pipe": q_pipe},
        "pack": {"ms": phase_ms[3], "gbs": k_bytes / phase_ms[3] / 1e6,
                 "frac": k_bytes / phase_ms[3] / 1e6 / pk["hbm_gbs"], "pipe": "hbm"},
    }
    roof_ms = (h_flops / bf16_peak / 1e9 + p_flops / p_peak / 1e9 + q_flops / q_peak / 1e9
               + k_bytes / pk["hbm_gbs"] / 1e6)
    # the same sum with prepare and quantize bounded by the fp32 FMA units (their roofline before
    # the block products moved to the tensor cores)
    roof_fp32_ms = (h_flops / bf16_peak / 1e9 + p_flops / fp32_peak / 1e9 + q_flops / fp32_peak / 1e9
                    + k_bytes / pk["hbm_gbs"] / 1e6)
    h_tflops = h_flops / phase_ms[0] / 1e9
    roofline = {"bound": "tensor", "kernel": "hessian (A1)", "achieved": h_tflops, "peak": bf16_peak,
                "unit": "TFLOP/s", "frac": h_tflops / bf16_peak,
                "peak_source": f"{pk['source']} bf16 {'sustained' if long_region else 'burst'}",
                "algorithmic": f"N*d*(d+1) = {h_flops:.4g} flop per launch (N={L.n_tokens}, d={L.d})",
                "traffic": kernel_traffic("hessian_" + L.name, hessian_sources())}

    line = {"metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": config_of(L),
            "e2e": {"value": world * L.m * L.d / (e2e_ms * 1e-3), "unit": "weights/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches), "roofline": roofline, "phases": phases,
            "phase_roofline_ms": roof_ms, "end_to_end_roofline_frac": roof_ms / ms_per_step,
            "peaks": {"bf16_tflops": bf16_peak, "tf32x3_tflops": tf32x3_peak, "fp32_fma_tflops": fp32_peak,
                      "hbm_gbs": pk["hbm_gbs"],
                      "note": "bf16 and HBM measured; tf32 = bf16 x 1.1/2.25 (nominal ratio) / 3 MMAs; fp32 FMA = "
                              "148 SMs x 128 lanes x 2 x 1965 MHz"},
            "end_to_end_roofline_frac_fp32_pipes": roof_fp32_ms / ms_per_step,
            "clocks": clk}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        W64 = W_h.double().numpy()
        X = X_h
        cores, blas = cores_info()
        t0 = time.perf_counter()
        n = 0
        while True:
            oracle_step(L, W64, X)
            n += 1
            if time.perf_counter() - t0 > 10.0 or n >= 20:
                break
        dt = (time.perf_counter() - t0) / n
        line["cpu_baseline"] = {"value": L.m * L.d / dt, "unit": "weights/s", "cores": blas, "kind": "oracle",
                                "sample": f"{n} full oracle step(s) of the {L.name} layer (fp64, all "
                                          f"{L.n_tokens} tokens), {dt:.2f} s each"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def hessian_sources():
    return ["post_weight_quantization_21_b200/csrc/hessian.cu", "post_weight_quantization_21_b200/csrc/hessian_tc.cu",
            "post_weight_quantization_21_b200/csrc/tc_common.cuh"]


if __name__ == "__main__":
    main()
