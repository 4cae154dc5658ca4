"""GPU parity of act-order ("desc_act"): the permutation, the permuted Hessian and the column loop in
that order, through the C ABI, against the oracle on the same seeded inputs.

The permutation is integer work decided by comparisons of the same fp32 diagonal on both sides, so it
and the gathered Hessian must be bit-exact; the quantization follows the usual code rules.
"""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_21_b200 as g
from post_weight_quantization_21_b200 import workloads as wl

import gpu_support as S

pytestmark = pytest.mark.gpu


def _x(n, d, seed, scale_spread=True):
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn(n, d, generator=gen, dtype=torch.float64)
    x = x @ (torch.randn(d, d, generator=gen, dtype=torch.float64) / d ** 0.5) + 0.3 * torch.randn(
        n, d, generator=gen, dtype=torch.float64)
    if scale_spread:  # distinct channel scales, so the order is far from ties
        x = x * (0.2 + 3.0 * torch.rand(d, generator=gen, dtype=torch.float64))
    return x


def _act_order(H32: torch.Tensor):
    d = H32.shape[0]
    perm = torch.full((d,), -7, dtype=torch.int32, device=S.dev())
    Hp = torch.full((d, d), float("nan"), device=S.dev())
    st = torch.zeros(2, dtype=torch.int32, device=S.dev())
    g.gptq_act_order(H32, perm, Hp, st)
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_OK, (code, detail)
    return perm.cpu().numpy().astype(np.int64), Hp.cpu().numpy()


@pytest.mark.parametrize("d", [1, 33, 256, 1000, 4100])
def test_act_order_permutation_and_permuted_hessian(d):
    X = _x(max(4 * d, 64), d, seed=d)
    H32 = oracle.hessian(X.numpy()).astype(np.float32)
    H32 = np.triu(H32) + np.triu(H32, 1).T                    # exactly symmetric fp32
    perm, Hp = _act_order(torch.from_numpy(H32).to(S.dev()))
    ref = oracle.act_order_permutation(H32.astype(np.float64))
    np.testing.assert_array_equal(perm, ref)
    iu = np.triu_indices(d)
    np.testing.assert_array_equal(Hp[iu], H32[np.ix_(ref, ref)][iu])


def test_act_order_ties_keep_column_order():
    """Exactly equal diagonal entries (including zeros of dead channels) keep their column order."""
    d = 300
    rng = np.random.default_rng(3)
    vals = rng.choice([0.0, 1.0, 2.5, 7.0], size=d).astype(np.float32)
    H32 = np.diag(vals).astype(np.float32)
    H32[0, 5] = H32[5, 0] = 0.25
    perm, _ = _act_order(torch.from_numpy(H32).to(S.dev()))
    np.testing.assert_array_equal(perm, oracle.act_order_permutation(H32.astype(np.float64)))


ACT_CASES = [
    # m, d, bits, group, block
    (64, 512, 3, 128, 128),     # fused path
    (48, 384, 4, 0, 32),
    (2100, 512, 4, 128, 128),   # per-block path
    (40, 4352, 3, 128, 64),
]


@pytest.mark.parametrize("m,d,bits,gs,B", ACT_CASES)
def test_quantize_act_order_matches_oracle(m, d, bits, gs, B):
    X = _x(4 * d, d, seed=m + d)
    H = oracle.hessian(X.numpy())
    perm = oracle.act_order_permutation(H)
    U = oracle.inverse_upper_cholesky(oracle.dampen(H[np.ix_(perm, perm)], 0.01))
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    W = (torch.randn(m, d, generator=torch.Generator().manual_seed(d)) * 0.02).half()
    ref = oracle.gptq_quantize_act_order(W.double().numpy(), H, bits, gs, B, perm=perm)
    ref_u32 = oracle.gptq_quantize(W.double().numpy()[:, perm], U32.astype(np.float64), bits, gs, B)
    n_groups = 1 if gs == 0 else d // gs
    codes = torch.empty(m, d, dtype=torch.uint8, device=S.dev())
    scales = torch.empty(m, n_groups, device=S.dev())
    zeros = torch.empty(m, n_groups, dtype=torch.int32, device=S.dev())
    st = torch.zeros(2, dtype=torch.int32, device=S.dev())
    ws = torch.empty(g.gptq_quantize_act_order_workspace_size(m, d, bits, gs, B), dtype=torch.uint8, device=S.dev())
    g.gptq_quantize_layer_act_order(W.to(S.dev()), torch.from_numpy(U32).to(S.dev()),
                                    torch.from_numpy(perm.astype(np.int32)).to(S.dev()), codes, scales, zeros, st,
                                    ws, bits, gs, B)
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_OK, (code, detail)
    inv = np.argsort(perm)
    # the oracle run on the same fp32 U, codes back in the original order
    want = {"codes": ref_u32["codes"][:, inv], "scales": ref_u32["scales"], "zeros": ref_u32["zeros"],
            "Wq": ref_u32["Wq"][:, inv]}
    got_codes = codes.cpu().numpy().astype(np.int64)
    # the code comparison walks each row in quantization order (a row's first mismatch is the
    # near-tie; later ones follow its trajectory)
    S.compare_quantization((got_codes[:, perm], scales.cpu().numpy(), zeros.cpu().numpy().astype(np.int64)),
                           {k: (v[:, perm] if k in ("codes", "Wq") else v) for k, v in want.items()}, gs,
                           label=f"act-order {m}x{d} b{bits} g{gs} B{B}")
    # and in the original order: the layer's reconstruction error against the oracle's
    deq = S.dequant(got_codes[:, perm], scales.cpu().numpy(), zeros.cpu().numpy().astype(np.int64), gs)[:, inv]
    E_gpu = oracle.reconstruction_error(W.double().numpy(), deq, H)
    E_ref = oracle.reconstruction_error(W.double().numpy(), ref["Wq"], H)
    assert abs(E_gpu - E_ref) / E_ref <= S.E_REL


def test_quantize_act_order_reports_a_bad_permutation():
    """A repeated entry in perm is reported on the device as GPTQ_ERR_ARG; nothing is read out of
    bounds (the kernels check every index) and the call still completes."""
    m, d = 16, 128
    perm = np.arange(d, dtype=np.int32)
    perm[10] = 3                                               # column 3 twice, column 10 never
    U = torch.eye(d, device=S.dev())
    W = (torch.randn(m, d) * 0.02).half().to(S.dev())
    codes = torch.empty(m, d, dtype=torch.uint8, device=S.dev())
    scales = torch.empty(m, 1, device=S.dev())
    zeros = torch.empty(m, 1, dtype=torch.int32, device=S.dev())
    st = torch.zeros(2, dtype=torch.int32, device=S.dev())
    ws = torch.empty(g.gptq_quantize_act_order_workspace_size(m, d, 4, 0, 128), dtype=torch.uint8, device=S.dev())
    g.gptq_quantize_layer_act_order(W, U, torch.from_numpy(perm).to(S.dev()), codes, scales, zeros, st, ws, 4, 0, 128)
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_ERR_ARG and detail in (3, 10)


def test_end_to_end_act_order_layer():
    """LayerSolver with act-order on a 512 x 1024 slice of the 3-bit group-128 q_proj layer (Student-t
    inputs with outlier channels): every stage chained on the GPU against the oracle."""
    import dataclasses
    L = dataclasses.replace(wl.LAYERS["llama7b_q_4096x4096"], m=512, d=1024, n_tokens=16 * 2048)
    W, X = wl.make_w(L), wl.make_x(L)
    s = g.LayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, X.dtype, W.dtype,
                      act_order=True)
    s.X.copy_(X)
    s.W.copy_(W)
    s.run()
    s.check_status()
    torch.cuda.synchronize()
    H = oracle.hessian(X.double().numpy())
    ref = oracle.gptq_quantize_act_order(W.double().numpy(), H, L.bits, L.group_size, L.block_size, L.damp)
    perm = s.perm.cpu().numpy().astype(np.int64)
    dg = np.sort(np.diag(H))[::-1]
    gaps = np.abs(np.diff(dg)) / dg[1:]
    if gaps.min() > 1e-4:  # no near-ties in this seeded layer: the fp32 and fp64 orders agree
        np.testing.assert_array_equal(perm, ref["perm"])
    Hp = H[np.ix_(perm, perm)]
    U = oracle.inverse_upper_cholesky(oracle.dampen(Hp, L.damp))
    ref_in_order = oracle.gptq_quantize(W.double().numpy()[:, perm], U, L.bits, L.group_size, L.block_size)
    codes = s.codes.cpu().numpy().astype(np.int64)
    st = S.compare_quantization((codes[:, perm], s.scales.cpu().numpy(), s.zeros.cpu().numpy().astype(np.int64)),
                                ref_in_order, L.group_size, W.double().numpy()[:, perm], Hp,
                                label="act-order 512x1024 chained")
    np.testing.assert_array_equal(s.packed.cpu().numpy(), oracle.pack_codes(codes, L.bits))
    print("act-order chained", st)
