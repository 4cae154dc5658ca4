#!/usr/bin/env python
"""Throughput of the GPTQ layer solver on B200: quantized weights/s per layer, split by phase.

One step = the whole hot path on one synthetic layer: H = 2 X^T X over the calibration tokens,
dampening + U = chol(H^-1), the column loop with lazy block updates, and packing.  The default layer
is the largest that fits one GPU: the OPT-175B-like fc2 projection, W [12288, 49152], 262,144
calibration tokens (X 25.8 GB, H and U 9.7 GB each).  Inputs (X, W) are resident in HBM before
timing; X is larger than the 126 MB L2, so every step streams it from HBM.

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
DEFAULT_LAYER = "opt175b_fc2_12288x49152"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--layer", default=DEFAULT_LAYER)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--mode", default="layers", choices=["layers", "sharded"],
                   help="N > 1: 'layers' = each rank solves its own layer (weak scaling); 'sharded' = one layer "
                        "split across the ranks (tokens for H + all-reduce, rows for the solve; strong scaling)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--pipeline", action="store_true",
                   help="time the sequential block pipeline instead (OPT-125M-like synthetic blocks, 128 x 2048 "
                        "calibration tokens): one JSON line of its own")
    p.add_argument("--e2e-steps", type=int, default=None,
                   help="end-to-end steps (default: 10, or 3 on layers whose step takes over 0.5 s)")
    p.add_argument("--probe", choices=["hessian", "gemv"], default=None,
                   help="profiling target, no JSON line: run only the layer's Hessian (gptq_hessian_accumulate) or "
                        "its dequantizing product (gptq_dequant_matmul, one fp16 row, uniform random codes) "
                        "--steps times and print the CUDA-event time of each call")
    p.add_argument("--tokens", type=int, default=None, help="calibration tokens (default: the layer's own)")
    return p.parse_args()


def run_probe(args, L):
    """One kernel of the layer, alone: the command ncu captures are taken on (a few GB on the device)."""
    import torch
    import post_weight_quantization_21_b200 as g
    from post_weight_quantization_21_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    st = torch.zeros(2, dtype=torch.int32, device=dev)
    if args.probe == "hessian":
        X = wl.make_x(L, device=dev)
        H = torch.empty(L.d, L.d, device=dev)
        ws = torch.empty(max(g.gptq_hessian_workspace_size(L.n_tokens, L.d, X.dtype), 256), dtype=torch.uint8,
                         device=dev)

        def call():
            g.gptq_hessian_accumulate(X, H, st, ws, 2.0, False)
    else:
        gen = torch.Generator(device="cpu").manual_seed(0)
        ng = 1 if L.group_size == 0 else L.d // L.group_size
        packed = torch.randint(-2 ** 31, 2 ** 31 - 1, (L.m, L.d * L.bits // 32), generator=gen,
                               dtype=torch.int32).to(dev)
        scales = (torch.rand(L.m, ng, generator=gen) * 0.01).to(dev)
        zeros = torch.randint(0, 2 ** L.bits, (L.m, ng), generator=gen, dtype=torch.int32).to(dev)
        x = torch.randn(1, L.d, generator=gen).to(torch.float16).to(dev)
        y = torch.empty(1, L.m, device=dev)
        ws = torch.empty(g.gptq_dequant_matmul_workspace_size(L.m, L.d, 1), dtype=torch.uint8, device=dev)

        def call():
            g.gptq_dequant_matmul(packed, scales, zeros, L.bits, L.group_size, x, y, st, ws)
    for i in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize(dev)
        code, detail = g.gptq_read_status(st)
        print(f"{args.probe} {L.name} tokens={L.n_tokens}: {e0.elapsed_time(e1):.3f} ms, status {code}")
        if code != g.GPTQ_OK:
            raise g.GPTQError(code, args.probe, detail)


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


class ShardedRunner:
    """One layer split across the ranks (ShardedLayerSolver) behind the calls the timing loop makes."""

    def __init__(self, L, dev):
        from post_weight_quantization_21_b200.sharded import ShardedLayerSolver
        from post_weight_quantization_21_b200 import workloads as wl
        self.s = ShardedLayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, L.x_dtype,
                                    L.w_dtype, dev, token_align=wl.CHUNK_TOKENS)
        self.W, self.X = self.s.W_local, self.s.X_local
        (t0, t1), (r0, r1) = self.s.tokens, self.s.rows
        self.n_local, self.m_local = t1 - t0, r1 - r0
        for c in range(t0 // wl.CHUNK_TOKENS, (t1 + wl.CHUNK_TOKENS - 1) // wl.CHUNK_TOKENS):
            chunk = wl.make_x_chunk(L, c, dev)
            a = c * wl.CHUNK_TOKENS - t0
            self.X[a:a + chunk.shape[0]].copy_(chunk)
        self.W.copy_(wl.make_w(L, device=dev)[r0:r1])
        self.packed, self.scales, self.zeros = self.s.packed, self.s.scales, self.s.zeros

    def hessian(self, stream):
        self.s.hessian()

    def prepare(self, stream):
        self.s.prepare()

    def quantize(self, stream):
        self.s.quantize()

    def pack(self, stream):
        self.s.pack()

    def check_status(self, stream):
        self.s.check_status()

    def run_host(self, W_h, X_h, out_p, out_s, out_z, stream):
        self.s.run_host(W_h, X_h, out_p, out_s, out_z)


def dequant_gemv_figures(g, solver, L, dev, pk, reps: int = 20):
    """The inference product with this layer's packed weights, one fp16 input row (the step after the
    path): gptq_dequant_matmul against torch's fp16 matrix-vector product with W, both timed by CUDA
    events over ``reps`` launches (the packed words and W are larger than L2)."""
    import torch
    x = torch.randn(1, L.d, device=dev, dtype=torch.float16)
    y = torch.empty(1, L.m, device=dev)
    ws = torch.empty(g.gptq_dequant_matmul_workspace_size(L.m, L.d, 1), dtype=torch.uint8, device=dev)
    st = torch.zeros(2, dtype=torch.int32, device=dev)
    W16 = solver.W.to(torch.float16)
    xt = x.t().contiguous()

    def ours():
        g.gptq_dequant_matmul(solver.packed, solver.scales, solver.zeros, L.bits, L.group_size, x, y, st, ws)

    def fp16():
        torch.matmul(W16, xt)

    out = {}
    for name, fn in (("ours", ours), ("fp16", fp16)):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize(dev)
        out[name] = e0.elapsed_time(e1) / reps
    del W16
    n_groups = 1 if L.group_size == 0 else L.d // L.group_size
    nbytes = L.m * L.d * L.bits // 8 + 8 * L.m * n_groups + 2 * L.d + 4 * L.m
    gbs = nbytes / (out["ours"] * 1e-3) / 1e9
    return {"kernel": "dequant_matmul_staged_kernel + dequant_reduce_kernel", "batch": 1, "x_dtype": "float16",
            "ms": out["ours"], "algorithmic_bytes": nbytes, "gbs": gbs, "bound": "hbm",
            "frac": gbs / pk["hbm_gbs"], "peak_source": f"of {pk['source']} HBM copy",
            "fp16_gemv_ms": out["fp16"], "fp16_gemv": "torch.matmul(W fp16, x) (cuBLAS)",
            "speedup_vs_fp16": out["fp16"] / out["ours"]}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 / bf16 tensor throughput of the B200


def fp32_spec_tflops(sm_mhz: float) -> float:
    """fp32 FMA peak from the part's unit counts: 148 SMs x 128 FMA lanes x 2 flops x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def measure_fp32_fma_tflops(device, n: int = 8192, reps: int = 10) -> float:
    """Measured fp32 FMA throughput: a cuBLAS fp32 GEMM (TF32 off, so it runs on the FMA units)
    n^3, best of ``reps`` by CUDA events, in the way the bf16 tensor peak is measured."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        a = torch.randn(n, n, device=device)
        b = torch.randn(n, n, device=device)
        c = torch.empty(n, n, device=device)
        for _ in range(3):
            torch.matmul(a, b, out=c)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


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


FULL_ORACLE_MAX_D = 1024  # layers up to this width: the oracle runs the whole layer every step


def oracle_full_step(L, W64, X):
    """One step of the oracle on the whole layer: the fp64 statement of the path (test infrastructure)."""
    import numpy as np
    import oracle
    H = np.zeros((L.d, L.d))
    for t0 in range(0, L.n_tokens, 16384):
        oracle.hessian_accumulate(H, X[t0:t0 + 16384].double().numpy())
    return oracle.gptq_layer(W64, None, L.bits, L.group_size, L.block_size, L.damp, H=H)


class StagedOracle:
    """The oracle on a bounded sample of a layer too large for it, extrapolated to the whole layer.

    A step runs the oracle's phases, one at a time, on two sub-problems of the same layer: the first
    n_s tokens, the first d1 and d2 channels and the first m_s rows.  Each phase's time is then scaled
    to the full layer with a cost model:
        Hessian   t = h N d^2                     (from the d2 run)
        prepare   t = p d^3                       (from the d2 run)
        quantize  t = q2 m d^2 + q1 m d           (two-point fit; lazy updates + column loop)
        pack      t = k m d                       (from the d2 run)
    Negative fitted coefficients (timing noise) are taken as 0.
    """

    def __init__(self, L, W, X_sample, d1=1024, d2=4096, m_s=512):
        import numpy as np
        self.L, self.d1, self.d2 = L, d1, d2
        self.m_s = min(m_s, L.m)
        self.n_s = X_sample.shape[0]
        self.W = {dd: np.ascontiguousarray(W[:self.m_s, :dd].double().numpy()) for dd in (d1, d2)}
        self.X = {dd: np.ascontiguousarray(X_sample[:, :dd].double().numpy()) for dd in (d1, d2)}
        g = L.group_size
        if g and (d1 % g or d2 % g):
            raise ValueError("sample widths must hold whole groups")

    def _phases(self, dd):
        import oracle
        L = self.L
        t0 = time.perf_counter()
        H = oracle.hessian(self.X[dd])
        t1 = time.perf_counter()
        U = oracle.inverse_upper_cholesky(oracle.dampen(H, L.damp))
        t2 = time.perf_counter()
        res = oracle.gptq_quantize(self.W[dd], U, L.bits, L.group_size, L.block_size)
        t3 = time.perf_counter()
        oracle.pack_codes(res["codes"], L.bits)
        t4 = time.perf_counter()
        return t1 - t0, t2 - t1, t3 - t2, t4 - t3

    def step(self) -> float:
        """Runs one sample; returns the extrapolated seconds of one full-layer oracle step."""
        L, d1, d2, m_s = self.L, self.d1, self.d2, self.m_s
        h1, p1, q1, k1 = self._phases(d1)
        h2, p2, q2, k2 = self._phases(d2)

        def fit(t_a, t_b, fa, fb, ga, gb):  # t = A f + B g through two points, A, B >= 0
            det = fa * gb - fb * ga
            A = max((t_a * gb - t_b * ga) / det, 0.0)
            B = max((fa * t_b - fb * t_a) / det, 0.0)
            return A, B

        t_h = h2 * (L.n_tokens / self.n_s) * (L.d / d2) ** 2
        t_p = p2 * (L.d / d2) ** 3
        Q2, Q1 = fit(q1, q2, m_s * d1 ** 2, m_s * d2 ** 2, m_s * d1, m_s * d2)
        t_q = Q2 * L.m * L.d ** 2 + Q1 * L.m * L.d
        t_k = k2 * (L.m * L.d) / (m_s * d2)
        self.last = {"hessian_s": t_h, "prepare_s": t_p, "quantize_s": t_q, "pack_s": t_k}
        return t_h + t_p + t_q + t_k

    def describe(self) -> str:
        return (f"extrapolated: oracle phases timed on sub-problems of the {self.L.name} layer (first "
                f"{self.n_s} tokens, first {self.d1} and {self.d2} channels, first {self.m_s} rows), scaled "
                "to the full layer by per-phase cost models (Hessian N d^2, prepare d^3, pack m d from the wider "
                "run; quantize m d^2 + m d fitted to both widths)")


def oracle_sample_inputs(L, device="cpu"):
    """The first chunk of X (2048 tokens) for the staged oracle."""
    from post_weight_quantization_21_b200 import workloads as wl
    return wl.make_x_chunk(L, 0, device).cpu()


def run_reference(args, L):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from post_weight_quantization_21_b200 import workloads as wl
    cores, blas = cores_info()
    if L.d <= FULL_ORACLE_MAX_D:
        W64 = wl.make_w(L).double().numpy()
        X = wl.make_x(L)
        for _ in range(args.warmup):
            oracle_full_step(L, W64, X)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            oracle_full_step(L, W64, X)
        dt = (time.perf_counter() - t0) / args.steps
        sample = (f"the full {L.name} layer per step: fp64 H over all {L.n_tokens} tokens, U, column loop, "
                  "pack (numpy/BLAS on the host cores)")
    else:
        st = StagedOracle(L, wl.make_w(L), oracle_sample_inputs(L))
        for _ in range(args.warmup):
            st.step()
        dt = statistics.mean(st.step() for _ in range(args.steps))
        sample = st.describe() + f"; one sample per step, mean of {args.steps}"
    value = L.m * L.d / dt
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(L),
            "cpu_baseline": {"value": value, "unit": "weights/s", "cores": blas, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "weights/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_of(L):
    xb = L.n_tokens * L.d * (2 if str(L.x_dtype).endswith("16") else 4)
    return {"workload": L.name, "m": L.m, "d": L.d, "n_tokens": L.n_tokens, "bits": L.bits,
            "group_size": L.group_size, "block_size": L.block_size, "damp": L.damp,
            "w_dtype": str(L.w_dtype).replace("torch.", ""), "x_dtype": str(L.x_dtype).replace("torch.", ""),
            "l2": f"inputs larger than L2: X = {xb / 1e9:.2f} GB streamed from HBM every step"}


def run_pipeline(args):
    """Sequential quantization of synthetic OPT-125M-like blocks (d 768, 12 heads, ffn 3072) on 128 x 2048
    calibration tokens: per block, the full-precision forward with the Hessians of its four linear
    inputs, the six layer solves, and the forward with the dequantized weights."""
    import torch
    from post_weight_quantization_21_b200 import pipeline as P
    cfg = P.BlockConfig(d_model=768, n_heads=12, d_ffn=3072, seq_len=2048, bits=4, group_size=0, block_size=128)
    dev = torch.device("cuda", 0)
    X = torch.randn(128 * cfg.seq_len, cfg.d_model, device=dev, generator=torch.Generator(device=dev).manual_seed(0))
    X = X.to(torch.bfloat16)
    bq = P.BlockQuantizer(cfg, device=dev, chunk_seqs=16)
    x = X
    for b in range(args.warmup):
        _, x = bq.quantize_block(P.make_block(cfg, seed=b, device=dev), x)
    times = []
    for b in range(args.steps):
        _, x = bq.quantize_block(P.make_block(cfg, seed=1000 + b, device=dev), x)
        times.append(dict(bq.timing))
    ms = {k: statistics.mean(t[k] for t in times) for k in times[0]}
    total = sum(ms.values())
    weights = sum(cfg.shape(n)[0] * cfg.shape(n)[1] for n in P.LINEARS)
    print(json.dumps({"metric": "sequential block pipeline: ms per block", "value": total, "unit": "ms",
                      "higher_is_better": False, "steps": args.steps, "warmup": args.warmup,
                      "split_ms": ms, "weights_per_s": weights / (total * 1e-3),
                      "config": {"workload": "synthetic OPT-125M-like decoder block", "d_model": 768, "n_heads": 12,
                                 "d_ffn": 3072, "tokens": 128 * 2048, "bits": 4, "group_size": 0}}), flush=True)


def main():
    args = parse()
    from post_weight_quantization_21_b200 import workloads as wl
    L = wl.LAYERS[args.layer]
    if args.tokens is not None:
        L = L.with_tokens(args.tokens)
    if args.probe:
        return run_probe(args, L)
    if args.impl == "reference":
        return run_reference(args, L)
    if args.pipeline:
        return run_pipeline(args)

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

    # seeded inputs made on the device (the large layers' X is tens of GB); host copies below
    if args.mode == "sharded":
        L = wl.LAYERS[args.layer]                     # one layer shared by all ranks
        solver = ShardedRunner(L, dev)
        n_eff, m_eff, job_weights = solver.n_local, solver.m_local, L.m * L.d
    else:
        solver = g.LayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, L.x_dtype,
                               L.w_dtype, device=dev)
        solver.W.copy_(wl.make_w(L, device=dev))
        wl.make_x(L, device=dev, out=solver.X)
        n_eff, m_eff, job_weights = L.n_tokens, L.m, world * L.m * L.d
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
    value = job_weights / (ms_per_step * 1e-3)

    # end to end through the host: pinned inputs in, packed codes + grids out, every step
    W_h = torch.empty(solver.W.shape, dtype=solver.W.dtype, pin_memory=True)
    X_h = torch.empty(solver.X.shape, dtype=solver.X.dtype, pin_memory=True)
    W_h.copy_(solver.W)
    X_h.copy_(solver.X)
    n_groups = 1 if L.group_size == 0 else L.d // L.group_size
    out_p = torch.empty(m_eff, L.d * L.bits // 32, dtype=torch.int32, pin_memory=True)
    out_s = torch.empty(m_eff, n_groups, dtype=torch.float32, pin_memory=True)
    out_z = torch.empty(m_eff, n_groups, dtype=torch.int32, pin_memory=True)
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else (3 if ms_per_step > 500.0 else 10)
    solver.run_host(W_h, X_h, out_p, out_s, out_z, stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(stream)
    for _ in range(e2e_steps):
        solver.run_host(W_h, X_h, out_p, out_s, out_z, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    solver.check_status(stream)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = slowest_rank_ms(e2e_ms, dev)
    h2d = W_h.numel() * W_h.element_size() + X_h.numel() * X_h.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (out_p, out_s, out_z))

    gemv = dequant_gemv_figures(g, solver, L, dev, pk) if args.mode == "layers" else None

    # denominators: bf16 and HBM measured (MEASURED_PEAKS.json); fp32 FMA measured here by a cuBLAS
    # fp32 GEMM; 3xTF32 derived from the measured bf16 figure and the nominal tf32/bf16 ratio
    fp32_meas = measure_fp32_fma_tflops(dev)
    long_region = total_ms > 1000.0
    bf16_peak = pk["bf16_tflops_sustained"] if long_region else pk["bf16_tflops"]
    fp32_peak = fp32_meas
    tf32x3_peak = bf16_peak * TF32_PER_BF16 / 3.0   # three tf32 MMAs per fp32-accurate product
    tc = g.gptq_tensor_core_phases(L.m, L.d, L.n_tokens, L.x_dtype, L.bits, L.group_size, L.block_size)
    # this rank's algorithmic work (sharded mode: its tokens and rows; the prepare step is replicated)
    h_flops = n_eff * L.d * (L.d + 1)                      # symmetric half of 2 N d^2
    p_flops = 2.0 / 3.0 * L.d ** 3                          # Cholesky + triangular inverse
    q_flops = float(m_eff) * L.d * L.d                      # column loop + lazy updates
    k_bytes = m_eff * L.d * (1 + L.bits / 8)                # pack: codes in, words out
    p_peak, p_pipe = (tf32x3_peak, "tensor(3xtf32)") if tc & g.GPTQ_TC_PREPARE else (fp32_peak, "fp32 FMA")
    q_peak, q_pipe = (tf32x3_peak, "tensor(3xtf32)") if tc & g.GPTQ_TC_LAZY else (fp32_peak, "fp32 FMA")
    bf16_src = f"{pk['source']} bf16 {'sustained' if long_region else 'burst'}"
    peak_src = {"tensor(bf16)": f"of {bf16_src}", "tensor(3xtf32)": f"derived: {bf16_src} x 1.1/2.25 / 3",
                "fp32 FMA": "of measured fp32 GEMM", "hbm": f"of {pk['source']} HBM copy"}
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
    for ph in phases.values():
        ph["peak_source"] = peak_src[ph["pipe"]]
    roof_ms = (h_flops / bf16_peak / 1e9 + p_flops / p_peak / 1e9 + q_flops / q_peak / 1e9
               + k_bytes / pk["hbm_gbs"] / 1e6)
    # the same sum with prepare and quantize bounded by the fp32 FMA units (their roofline before
    # the block products moved to the tensor cores)
    roof_fp32_ms = (h_flops / bf16_peak / 1e9 + p_flops / fp32_peak / 1e9 + q_flops / fp32_peak / 1e9
                    + k_bytes / pk["hbm_gbs"] / 1e6)
    h_tflops = h_flops / phase_ms[0] / 1e9
    roof_hessian = {"bound": "tensor", "kernel": "hessian_tc_kernel (A1, one launch per step)",
                    "achieved": h_tflops, "peak": bf16_peak, "unit": "TFLOP/s", "frac": h_tflops / bf16_peak,
                    "peak_source": bf16_src,
                    "algorithmic": f"N*d*(d+1) = {h_flops:.4g} flop per launch (N={n_eff}, d={L.d})",
                    "traffic": kernel_traffic("hessian_" + L.name, hessian_sources())}
    # the phase that takes the largest share of the step
    work = {"hessian": (h_flops, "N*d*(d+1) flop"), "prepare": (p_flops, "2/3 d^3 flop"),
            "quantize": (q_flops, "m*d^2 flop"), "pack": (k_bytes, "m*d*(1+b/8) byte")}
    top = max(phases, key=lambda k: phases[k]["ms"])
    if top == "hessian":
        roofline = roof_hessian
    else:
        ph = phases[top]
        hbm = ph["pipe"] == "hbm"
        achieved = ph["gbs"] if hbm else ph["tflops"]
        peak = pk["hbm_gbs"] if hbm else {"tensor(3xtf32)": tf32x3_peak, "fp32 FMA": fp32_peak}[ph["pipe"]]
        kernels = {"prepare": "prepare phase (A2+A3): factor_kernel, tf32x3_gemm_kernel (trsm/syrk/trtri), "
                              "diag_mean, reverse_damp, leaf_copy, rotate" if tc & g.GPTQ_TC_PREPARE
                              else "prepare phase (A2+A3): prepare_kernel (one cooperative launch)",
                   "quantize": "quantize phase (A4-A6): column loop + lazy block updates",
                   "pack": "pack_kernel (A7)"}[top]
        roofline = {"bound": "hbm" if hbm else "tensor" if ph["pipe"].startswith("tensor") else "alu",
                    "kernel": kernels, "achieved": achieved, "peak": peak, "unit": "GB/s" if hbm else "TFLOP/s",
                    "frac": achieved / peak, "peak_source": ph["peak_source"],
                    "algorithmic": f"{work[top][1]} = {work[top][0]:.4g} per step (one phase = one unit)",
                    "traffic": None}

    cfg = config_of(L)
    cfg["parallelism"] = (f"{world} ranks, one layer: tokens sharded for H + all-reduce, U replicated, rows "
                          "sharded" if args.mode == "sharded" else f"{world} independent layer(s), one per rank")
    line = {"metric": METRIC, "value": value, "unit": "weights/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong" if args.mode == "sharded" else "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic", "config": cfg,
            "e2e": {"value": job_weights / (e2e_ms * 1e-3), "unit": "weights/s", "ms_per_step": e2e_ms,
                    "steps": e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches), "roofline": roofline, "roofline_hessian": roof_hessian,
            "phases": phases, "phase_roofline_ms": roof_ms, "end_to_end_roofline_frac": roof_ms / ms_per_step,
            "peaks": {"bf16_tflops": bf16_peak, "tf32x3_tflops": tf32x3_peak, "fp32_fma_tflops": fp32_peak,
                      "fp32_fma_spec_tflops_at_max_clock": fp32_spec_tflops(1965.0), "hbm_gbs": pk["hbm_gbs"],
                      "note": "bf16 and HBM measured (MEASURED_PEAKS.json); fp32 FMA measured in this run "
                              "(cuBLAS fp32 GEMM 8192^3, TF32 off, best of 10); tf32 = bf16 x 1.1/2.25 "
                              "(nominal ratio) / 3 MMAs"},
            "end_to_end_roofline_frac_fp32_pipes": roof_fp32_ms / ms_per_step,
            "clocks": clk}
    if gemv is not None:
        line["dequant_gemv"] = gemv
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores, blas = cores_info()
        t0 = time.perf_counter()
        n, times = 0, []
        if L.d <= FULL_ORACLE_MAX_D:
            W64 = W_h.double().numpy()
            while True:
                oracle_full_step(L, W64, X_h)
                n += 1
                if time.perf_counter() - t0 > 10.0 or n >= 20:
                    break
            dt = (time.perf_counter() - t0) / n
            sample = f"{n} full oracle step(s) of the {L.name} layer (fp64, all {L.n_tokens} tokens), {dt:.2f} s each"
        else:
            st = StagedOracle(L, W_h, X_h[:2048])
            while True:
                times.append(st.step())
                n += 1
                if time.perf_counter() - t0 > 10.0 or n >= 20:
                    break
            dt = statistics.mean(times)
            sample = st.describe() + f"; {n} sample(s) in {time.perf_counter() - t0:.1f} s"
        line["cpu_baseline"] = {"value": L.m * L.d / dt, "unit": "weights/s", "cores": blas, "kind": "oracle",
                                "sample": sample, "seconds_per_layer": dt}
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
