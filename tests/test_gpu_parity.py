"""GPU parity: every stage of the CUDA path against the fp64 oracle on the same seeded inputs.

Each test calls the library through its C ABI (ctypes binding) and compares element by element with
the oracle at sizes the oracle finishes in seconds (several tiles and a ragged tail), plus the
bench's full-size layer (opt125m 768x768, 262,144 tokens) end to end.
"""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_21_b200 as g
from post_weight_quantization_21_b200 import workloads as wl

import gpu_support as S

pytestmark = pytest.mark.gpu


def _x(n, d, dtype, seed, corr=True):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=gen, dtype=torch.float64)
    if corr:
        A = torch.randn(d, d, generator=gen, dtype=torch.float64) / d ** 0.5
        x = x @ A + 0.3 * torch.randn(n, d, generator=gen, dtype=torch.float64)
    return x.to(dtype)


# ------------------------------------------------------------------------------------------ A1
@pytest.mark.parametrize("n,d,dtype", [
    (256, 128, torch.float32),       # the tiny layer
    (1000, 200, torch.float32),      # ragged tile tail, ragged token tail
    (5000, 200, torch.bfloat16),
    (3000, 136, torch.float16),
    (2048 * 9 + 17, 520, torch.bfloat16),  # tensor-core path from here on: ragged 128/256 tiles
    (4096, 256, torch.bfloat16),
    (20000, 392, torch.float16),
    (6144, 1024, torch.bfloat16),
    (64, 384, torch.bfloat16),           # a single 64-token stage
    (100, 512, torch.float16),           # one stage plus a ragged token tail
])
def test_hessian_matches_oracle(n, d, dtype):
    X = _x(n, d, dtype, seed=n + d)
    H = S.hessian(X.to(S.dev())).cpu().numpy()
    Href = oracle.hessian(X.double().numpy())
    assert S.upper_rel_fro(H, Href) <= S.H_REL_FRO


def test_hessian_accumulates_and_handles_empty_input():
    X = _x(4096, 64, torch.bfloat16, seed=5).to(S.dev())
    H = S.hessian(X[:1000])
    S.hessian(X[1000:], accumulate_into=H)
    Href = oracle.hessian(X.cpu().double().numpy())
    assert S.upper_rel_fro(H.cpu().numpy(), Href) <= S.H_REL_FRO
    H0 = S.hessian(X[:0])                          # 0 tokens, overwrite mode: H = 0
    assert torch.count_nonzero(torch.triu(H0)) == 0
    S.hessian(X[:0], accumulate_into=H)            # 0 tokens, accumulate mode: unchanged
    assert S.upper_rel_fro(H.cpu().numpy(), Href) <= S.H_REL_FRO


def test_hessian_tensor_core_accumulate_mode():
    X = _x(9000, 512, torch.bfloat16, seed=9).to(S.dev())
    H = S.hessian(X[:5000])
    S.hessian(X[5000:], accumulate_into=H)
    Href = oracle.hessian(X.cpu().double().numpy())
    assert S.upper_rel_fro(H.cpu().numpy(), Href) <= S.H_REL_FRO


def test_hessian_timeout_is_reported_and_the_context_stays_usable():
    """Failure detection without a fault: the test hook makes the tensor-core Hessian's MMA issuer give
    up a bounded wait (about 0.5 ms at the base clock) on a barrier nothing arrives on.  The call's
    status word reports GPTQ_ERR_TIMEOUT at wait 5; the next call on the same stream runs normally."""
    X = _x(8192, 512, torch.bfloat16, seed=17).to(S.dev())
    n, d = X.shape
    assert g.gptq_tensor_core_phases(64, d, n, X.dtype, 4) & g.GPTQ_TC_HESSIAN
    H = torch.empty(d, d, device=S.dev())
    ws = torch.empty(max(g.gptq_hessian_workspace_size(n, d, X.dtype), 256), dtype=torch.uint8, device=S.dev())
    st = torch.zeros(2, dtype=torch.int32, device=S.dev())
    g.lib().gptq_test_hessian_timeout(1_000_000)
    g.gptq_hessian_accumulate(X, H, st, ws, 2.0, False)
    code, detail = g.gptq_read_status(st)
    assert (code, detail) == (g.GPTQ_ERR_TIMEOUT, 5)
    g.gptq_hessian_accumulate(X, H, st, ws, 2.0, False)      # a fresh sum clears the status word
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_OK, (code, detail)
    assert S.upper_rel_fro(H.cpu().numpy(), oracle.hessian(X.cpu().double().numpy())) <= S.H_REL_FRO


def test_hessian_full_size_opt125m_layer():
    L = wl.LAYERS["opt125m_768x768"]
    X = wl.make_x(L)
    H = S.hessian(X.to(S.dev())).cpu().numpy()
    Href = oracle.hessian(X.double().numpy())
    assert S.upper_rel_fro(H, Href) <= S.H_REL_FRO


# ------------------------------------------------------------------------------------------ A2 + A3
# above 1024 the blocked path: tensor-core tiles when d % 4 == 0 (1100, 1500, 2048, 4224), fp32 tiles else (1102)
@pytest.mark.parametrize("d", [1, 5, 31, 33, 64, 128, 200, 768, 1000, 1100, 1102, 1500, 2048, 4224])
def test_prepare_matches_oracle(d):
    n = max(4 * d, 64)
    X = _x(n, d, torch.float64, seed=d)
    H = oracle.hessian(X.numpy())
    Hd = oracle.dampen(H, 0.01)
    Uref = oracle.inverse_upper_cholesky(Hd)
    U = S.prepare(torch.from_numpy(H).float().to(S.dev())).cpu().numpy().astype(np.float64)
    assert np.all(np.tril(U, -1) == 0.0)
    rel = np.linalg.norm(U - Uref) / np.linalg.norm(Uref)
    res = np.linalg.norm(U @ Hd @ U.T - np.eye(d)) / np.sqrt(d)
    kappa = np.linalg.cond(Hd)
    # fp32 factorisation: forward error ~ kappa * eps32; residual ~ d * eps32
    assert rel <= max(1e-5, 10 * kappa * 6e-8), (rel, kappa)
    assert res <= 1e-4, res


def test_prepare_reports_indefinite_matrix():
    d = 96
    H = torch.eye(d) * 2.0
    H[37, 37] = -50.0  # damping 0.01 * mean(diag) cannot lift this pivot
    U, code, detail = S.prepare(H.to(S.dev()), expect_ok=False)
    assert code == 3  # GPTQ_ERR_NOT_PD
    assert detail == 37


# ------------------------------------------------------------------------------------------ A4 - A6
QUANT_CASES = [
    # m, d, bits, group, block
    (64, 128, 4, 0, 32),
    (100, 256, 3, 0, 128),
    (37, 512, 2, 0, 64),
    (64, 512, 3, 128, 128),
    (64, 512, 4, 32, 128),
    (64, 512, 4, 256, 128),
    (48, 384, 4, 64, 32),
    (1, 128, 4, 0, 128),
]

# many rows or wider than 4096: per-block launches (column loop, then the all-rows lazy GEMM)
PER_BLOCK_CASES = [
    (2100, 256, 4, 0, 128),
    (2500, 512, 3, 128, 128),
    (2049, 256, 4, 0, 32),
    (6200, 256, 3, 0, 128),    # past 6144 rows: four lanes per row in the column loop
    (40, 4224, 3, 128, 128),
    (24, 4352, 4, 0, 64),
]


@pytest.mark.parametrize("m,d,bits,gs,B", QUANT_CASES)
def test_quantize_matches_oracle_given_U(m, d, bits, gs, B):
    X = _x(4 * d, d, torch.float64, seed=m * d + bits)
    H = oracle.hessian(X.numpy())
    U = oracle.inverse_upper_cholesky(oracle.dampen(H, 0.01))
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    W = (torch.randn(m, d, generator=torch.Generator().manual_seed(d + m)) * 0.02).half()
    ref = oracle.gptq_quantize(W.double().numpy(), U32.astype(np.float64), bits, gs, B)
    gpu = S.quantize(W.to(S.dev()), torch.from_numpy(U32).to(S.dev()), bits, gs, B)
    S.compare_quantization(gpu, ref, gs, W.double().numpy(), H, label=f"{m}x{d} b{bits} g{gs} B{B}")


@pytest.mark.parametrize("flags", [0, g.GPTQ_FLAG_FP32_FMA], ids=["tf32x3", "fp32fma"])
@pytest.mark.parametrize("m,d,bits,gs,B", PER_BLOCK_CASES)
def test_quantize_per_block_paths(m, d, bits, gs, B, flags):
    X = _x(4 * d, d, torch.float64, seed=m * d + bits)
    H = oracle.hessian(X.numpy())
    U = oracle.inverse_upper_cholesky(oracle.dampen(H, 0.01))
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    W = (torch.randn(m, d, generator=torch.Generator().manual_seed(d + m)) * 0.02).half()
    ref = oracle.gptq_quantize(W.double().numpy(), U32.astype(np.float64), bits, gs, B)
    gpu = S.quantize(W.to(S.dev()), torch.from_numpy(U32).to(S.dev()), bits, gs, B, flags=flags)
    S.compare_quantization(gpu, ref, gs, W.double().numpy(), H, label=f"{m}x{d} b{bits} g{gs} B{B} f{flags}")


# Edge cases of the method on both quantize paths: a zero row of W (flat range, grid [-1, 1]), a zero
# group, an all-positive row (range widened to 0), outlier weights (x10) under group grids, dead input
# channels (H_ii = 0: only the damping keeps Hd positive definite), 2-bit groups, a group of 128
# spanning several blocks of 32 or 64.
EDGE_CASES = [
    # m, d, bits, group, block
    (64, 512, 2, 128, 128),     # fused path
    (64, 512, 4, 128, 32),
    (2100, 512, 2, 128, 128),   # per-block path (many rows)
    (2100, 512, 4, 128, 32),
    (40, 4352, 3, 128, 64),     # per-block path (wide)
]


def _edge_inputs(m, d, seed):
    gen = torch.Generator().manual_seed(seed)
    X = _x(4 * d, d, torch.float64, seed=seed)
    dead = [3, 77, d // 2, d - 1]
    X[:, dead] = 0.0
    W = torch.randn(m, d, generator=gen) * 0.02
    k = max(1, (m * d) // 200)                    # 0.5 % of the entries x10
    idx = torch.randperm(m * d, generator=gen)[:k]
    W.view(-1)[idx] *= 10.0
    W[5] = 0.0                                    # zero row
    W[7, 128:256] = 0.0                           # zero group (and a zero stretch of a per-row grid)
    W[9] = W[9].abs()                             # all-positive row
    return X, W.half(), dead


@pytest.mark.parametrize("m,d,bits,gs,B", EDGE_CASES)
def test_quantize_edge_cases(m, d, bits, gs, B):
    X, W, dead = _edge_inputs(m, d, seed=m + d + bits + B)
    H = oracle.hessian(X.numpy())
    assert np.all(np.diag(H)[dead] == 0.0)
    U = oracle.inverse_upper_cholesky(oracle.dampen(H, 0.01))
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    ref = oracle.gptq_quantize(W.double().numpy(), U32.astype(np.float64), bits, gs, B)
    gpu = S.quantize(W.to(S.dev()), torch.from_numpy(U32).to(S.dev()), bits, gs, B)
    S.compare_quantization(gpu, ref, gs, W.double().numpy(), H, label=f"edge {m}x{d} b{bits} g{gs} B{B}")
    # the zero row: every code is the zero point, the grid is [-1, 1]
    assert np.all(gpu[0][5] == gpu[2][5][0]) and np.all(gpu[2][5] == ref["zeros"][5])
    np.testing.assert_allclose(gpu[1][5], np.float32(2.0) / np.float32(2 ** bits - 1), rtol=1e-7)


@pytest.mark.parametrize("d", [768, 2048])
def test_prepare_dead_channels(d):
    X, _, dead = _edge_inputs(16, d, seed=d)
    H = oracle.hessian(X.numpy())
    Hd = oracle.dampen(H, 0.01)
    Uref = oracle.inverse_upper_cholesky(Hd)
    U = S.prepare(torch.from_numpy(H).float().to(S.dev())).cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(U - Uref) / np.linalg.norm(Uref)
    kappa = np.linalg.cond(Hd)
    assert rel <= max(1e-5, 10 * kappa * 6e-8), (rel, kappa)
    # the last channel is dead: its row and column of Hd are lambda e_(d-1), so U_(d-1,d-1) = lambda^-1/2
    lam = 0.01 * np.mean(np.diag(H))
    np.testing.assert_allclose(U[d - 1, d - 1], lam ** -0.5, rtol=1e-5)


def test_quantize_fp32_and_bf16_weights():
    d, m = 256, 32
    X = _x(4 * d, d, torch.float64, seed=3)
    H = oracle.hessian(X.numpy())
    U32 = np.ascontiguousarray(oracle.inverse_upper_cholesky(oracle.dampen(H, 0.01)), dtype=np.float32)
    for dt in (torch.float32, torch.bfloat16):
        W = (torch.randn(m, d, generator=torch.Generator().manual_seed(1)) * 0.02).to(dt)
        ref = oracle.gptq_quantize(W.double().numpy(), U32.astype(np.float64), 4, 0, 128)
        gpu = S.quantize(W.to(S.dev()), torch.from_numpy(U32).to(S.dev()), 4, 0, 128)
        S.compare_quantization(gpu, ref, 0, W.double().numpy(), H, label=str(dt))


# ------------------------------------------------------------------------------------------ A7
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("m,d", [(1, 32), (7, 96), (33, 768)])
def test_pack_bit_exact(bits, m, d):
    codes = torch.randint(0, 2 ** bits, (m, d), generator=torch.Generator().manual_seed(m + d + bits),
                          dtype=torch.uint8)
    got = S.pack(codes.to(S.dev()), bits)
    np.testing.assert_array_equal(got, oracle.pack_codes(codes.numpy().astype(np.int64), bits))


@pytest.mark.parametrize("offset", [1, 4, 8])
def test_pack_codes_at_any_alignment(offset):
    """The kernel reads a unit's 32 code bytes as 16-, 4- or 1-byte loads by the codes' alignment; the
    words are the same whichever it takes (codes that carry bits above b are masked)."""
    m, d, bits = 5, 160, 3
    codes = torch.randint(0, 256, (m, d), generator=torch.Generator().manual_seed(offset), dtype=torch.uint8)
    buf = torch.zeros(m * d + 64, dtype=torch.uint8, device=S.dev())
    view = buf[offset:offset + m * d].view(m, d)
    view.copy_(codes.to(S.dev()))
    got = S.pack(view, bits)
    np.testing.assert_array_equal(got, oracle.pack_codes(codes.numpy().astype(np.int64) & 7, bits))


# ------------------------------------------------------------------------------------------ end to end
def _layer_end_to_end(L, check_h=True):
    W = wl.make_w(L)
    X = wl.make_x(L)
    from post_weight_quantization_21_b200 import LayerSolver
    s = LayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, X.dtype, W.dtype)
    s.X.copy_(X)
    s.W.copy_(W)
    s.run()
    s.check_status()
    torch.cuda.synchronize()
    ref = oracle.gptq_layer(W.double().numpy(), X.double().numpy(), L.bits, L.group_size, L.block_size, L.damp)
    if check_h:
        assert S.upper_rel_fro(s.H.cpu().numpy(), ref["H"]) <= S.H_REL_FRO
    gpu = (s.codes.cpu().numpy().astype(np.int64), s.scales.cpu().numpy(), s.zeros.cpu().numpy().astype(np.int64))
    stats = S.compare_quantization(gpu, ref, L.group_size, W.double().numpy(), ref["H"], ref["E"], label=L.name)
    np.testing.assert_array_equal(s.packed.cpu().numpy(), oracle.pack_codes(gpu[0], L.bits))
    return stats


def test_end_to_end_tiny_layer():
    _layer_end_to_end(wl.LAYERS["tiny_64x128"])


def test_end_to_end_opt125m_layer():
    st = _layer_end_to_end(wl.LAYERS["opt125m_768x768"])
    print("opt125m end-to-end", st)


def test_end_to_end_reduced_llama_q_layer():
    """The 3-bit group-128 setting on a 1024-wide slice of the q_proj layer (all stages chained)."""
    L = wl.LAYERS["llama7b_q_4096x4096"]
    import dataclasses
    L = dataclasses.replace(L, m=512, d=1024, n_tokens=16 * 2048)
    _layer_end_to_end(L)


def test_run_host_streams_x_in_chunks():
    """LayerSolver.run_host: X crosses in HOST_CHUNK_TOKENS chunks whose Hessians accumulate as they land
    (a ragged last chunk of 40 tokens takes the fp32 Hessian path); results match the oracle."""
    m, d, bits, gs = 256, 512, 4, 128
    n = 2 * g.LayerSolver.HOST_CHUNK_TOKENS + 40
    gen = torch.Generator().manual_seed(9)
    X = (torch.randn(n, d, generator=gen) @ (torch.randn(d, d, generator=gen) / d ** 0.5)).to(torch.bfloat16)
    W = (torch.randn(m, d, generator=gen) * 0.02).half()
    s = g.LayerSolver(m, d, n, bits, gs, 128, 0.01, X.dtype, W.dtype, device=S.dev())
    n_groups = d // gs
    out_p = torch.empty(m, d * bits // 32, dtype=torch.int32).pin_memory()
    out_s = torch.empty(m, n_groups, dtype=torch.float32).pin_memory()
    out_z = torch.empty(m, n_groups, dtype=torch.int32).pin_memory()
    s.run_host(W.pin_memory(), X.pin_memory(), out_p, out_s, out_z)
    torch.cuda.synchronize()
    s.check_status()
    H = oracle.hessian(X.double().numpy())
    assert S.upper_rel_fro(s.H.double().cpu().numpy(), H) <= S.H_REL_FRO
    U = oracle.inverse_upper_cholesky(oracle.dampen(H, 0.01))
    ref = oracle.gptq_quantize(W.double().numpy(), U, bits, gs, 128)
    codes = oracle.unpack_codes(out_p.numpy(), bits, d).astype(np.int64)
    S.compare_quantization((codes, out_s.numpy(), out_z.numpy().astype(np.int64)), ref, gs, W.double().numpy(), H,
                           label="run_host")
