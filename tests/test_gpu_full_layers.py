"""GPU parity at the full sizes of the large layers (the launch configurations bench.py times).

The oracle cannot afford an fp64 H of every large layer end to end, so each stage is checked on
what it can compute exactly, and no stage takes an input from the CUDA path:

* H: the full GPU Hessian against fp64 on sampled 128x128 blocks (diagonal, off-diagonal and
  outlier-channel blocks), all 262,144 tokens; only the sampled channels leave the device.
* U: the trailing k x k principal block of U depends only on the trailing k x k block of the
  dampened Hessian (write Hd = R R^T with R upper: U = R^-1 and U_22 = R_22^-1).  The oracle builds
  that block (and the damping from all column norms) from X in fp64 and factors it.
* Column loop: the full m x d layer quantized on the GPU with an oracle U (from a token subsample
  of the same inputs) against the oracle's quantization of the same rows with the same U.  At
  d = 49152 the oracle cannot factor a Hessian, so the column loop there takes a seeded dense
  upper-triangular U (an input of the quantize call like any other) on both sides.
* U over its whole range at d = 49152: on 64 sampled rows spread over [0, d), the identity
  U Hd U^T = I (Hd = 2 X^T X + lambda I applied to vectors by streaming X through the host in fp64),
  and on 64 sampled columns the residual Hd U^T (U e_j) - e_j.
* End to end on the 4096- and 11008-wide layers: all stages chained on the GPU against the fp64
  oracle (H, U, the quantization of sampled rows, packing).
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_21_b200 import workloads as wl

import gpu_support as S

pytestmark = pytest.mark.gpu

LARGE = ["llama7b_q_4096x4096", "llama7b_up_11008x4096", "llama7b_down_4096x11008"]
WIDEST = "opt175b_fc2_12288x49152"


def _blocks(d, oc, rng):
    starts = sorted({0, d - 128, (d // 2) // 128 * 128} | {int(c) // 128 * 128 for c in oc[:3]})
    pairs = [(a, a) for a in starts] + [(starts[0], starts[-1]), (starts[1], starts[-1])]
    pairs += [(int(rng.integers(0, d // 128)) * 128, int(rng.integers(0, d // 128)) * 128) for _ in range(4)]
    return [(min(a, b), max(a, b)) for a, b in pairs]


def _x_cpu_chunks(X, step=16384, cols=None):
    idx = None if cols is None else torch.as_tensor(cols, device=X.device)
    for t0 in range(0, X.shape[0], step):
        Xc = X[t0:t0 + step]
        if idx is not None:
            Xc = Xc.index_select(1, idx)
        yield Xc.cpu().double().numpy()


@pytest.mark.parametrize("name", ["llama7b_q_4096x4096", "llama7b_down_4096x11008", WIDEST])
def test_hessian_sampled_blocks(name):
    L = wl.LAYERS[name]
    X = wl.make_x(L, device="cuda")
    H = S.hessian(X)
    rng = np.random.default_rng(0)
    blocks = _blocks(L.d, wl.outlier_channels(L).numpy(), rng)
    got = {(a, b): H[a:a + 128, b:b + 128].double().cpu().numpy() for a, b in blocks}
    del H
    starts = sorted({s for pair in blocks for s in pair})
    pos = {s0: 128 * k for k, s0 in enumerate(starts)}
    cols = np.concatenate([np.arange(s0, s0 + 128) for s0 in starts])
    ref = {p: np.zeros((128, 128)) for p in blocks}
    for Xc in _x_cpu_chunks(X, cols=cols):
        for (a, b) in blocks:
            ref[(a, b)] += 2.0 * Xc[:, pos[a]:pos[a] + 128].T @ Xc[:, pos[b]:pos[b] + 128]
    num = den = 0.0
    for (a, b), R in ref.items():
        G = got[(a, b)]
        if a == b:
            iu = np.triu_indices(128)
            G, R = G[iu], R[iu]
        num += np.sum((G - R) ** 2)
        den += np.sum(R ** 2)
    assert np.sqrt(num / den) <= S.H_REL_FRO


@pytest.mark.parametrize("name,k", [("llama7b_q_4096x4096", 512), ("llama7b_down_4096x11008", 512),
                                    (WIDEST, 2048)])
def test_prepare_trailing_block(name, k):
    L = wl.LAYERS[name]
    X = wl.make_x(L, device="cuda")
    H = S.hessian(X)
    U = S.prepare(H, L.damp)[-k:, -k:].double().cpu().numpy()
    del H
    torch.cuda.empty_cache()
    colsq = np.zeros(L.d)
    Hk = np.zeros((k, k))
    for Xc in _x_cpu_chunks(X, step=16384 if L.d <= 16384 else 2048):
        colsq += np.einsum("ij,ij->j", Xc, Xc)
        Hk += 2.0 * Xc[:, -k:].T @ Xc[:, -k:]
    lam = L.damp * np.mean(2.0 * colsq)
    Hd_k = Hk + lam * np.eye(k)
    Uref = oracle.inverse_upper_cholesky(Hd_k)
    rel = np.linalg.norm(U - Uref) / np.linalg.norm(Uref)
    kappa = np.linalg.cond(Hd_k)
    assert rel <= max(1e-5, 10 * kappa * 6e-8), (rel, kappa)
    assert np.all(U[np.tril_indices(k, -1)] == 0.0)


def _sampled_rows_and_columns(d, k, rng):
    """k indices spread over [0, d): both ends, the first 2048 (the last panels of the reversed
    factorisation) and the rest at random."""
    fixed = {0, 1, 127, 128, 2047, d // 2, d - 129, d - 1}
    low = set(rng.choice(2048, size=k // 4, replace=False).tolist())
    rest = rng.choice(d, size=k, replace=False).tolist()
    idx = sorted(fixed | low)
    for r in rest:
        if len(idx) >= k:
            break
        if r not in idx:
            idx.append(r)
    return np.array(sorted(idx[:k]))


def test_prepare_widest_layer_sampled_rows_and_columns():
    """U of the 49152-wide layer over its whole range, against what fp64 fixes without factoring:
    on sampled rows u_i of the GPU's U, G = U_S Hd U_S^T must be the identity; on sampled columns,
    Hd U^T (U e_j) = e_j.  Hd v = 2 X^T (X v) + lambda v is applied in fp64 on the host, streaming X
    in chunks of 2048 tokens; lambda comes from the same pass (0.01 * mean of 2 * column norms)."""
    L = wl.LAYERS[WIDEST]
    X = wl.make_x(L, device="cuda")
    H = S.hessian(X)
    U = S.prepare(H, L.damp)
    del H
    torch.cuda.empty_cache()
    rng = np.random.default_rng(5)
    rows = _sampled_rows_and_columns(L.d, 64, rng)
    cols = _sampled_rows_and_columns(L.d, 64, np.random.default_rng(6))
    idx_r = torch.as_tensor(rows, device=U.device)
    idx_c = torch.as_tensor(cols, device=U.device)
    US = U.index_select(0, idx_r).double().cpu().numpy()          # [64, d] sampled rows
    C = U.index_select(1, idx_c).double().cpu().numpy()           # [d, 64] sampled columns
    Y = np.zeros((L.d, len(cols)))                                # U^T (U e_j), rows of U streamed
    for r0 in range(0, L.d, 2048):
        Ub = U[r0:r0 + 2048].double().cpu().numpy()
        Y += Ub.T @ C[r0:r0 + 2048]
    for k, i in enumerate(rows):                                  # strictly lower part of sampled rows is zero
        assert np.all(US[k, :i] == 0.0)
    del U
    torch.cuda.empty_cache()
    V = np.concatenate([US.T, Y], axis=1)                         # [d, 128]
    HV = np.zeros_like(V)
    colsq = np.zeros(L.d)
    for Xc in _x_cpu_chunks(X, step=2048):
        colsq += np.einsum("ij,ij->j", Xc, Xc)
        HV += Xc.T @ (Xc @ V)
    del X
    lam = L.damp * np.mean(2.0 * colsq)
    HV = 2.0 * HV + lam * V
    nr = len(rows)
    G = US @ HV[:, :nr]
    g_err = np.abs(G - np.eye(nr)).max()
    R = HV[:, nr:]
    R[cols, np.arange(len(cols))] -= 1.0
    c_err = np.linalg.norm(R, axis=0).max()
    S.NOTES.append((WIDEST + " U", f"sampled rows max |U Hd U^T - I| = {g_err:.3e} (bound {L.d * 6e-8:.3e}); "
                                   f"sampled columns max ||Hd U^T U e_j - e_j|| = {c_err:.3e}"))
    # fp32 factorisation and inversion of a d x d matrix: the identity's entries carry sums of d
    # rounded products each; d * eps32 bounds their linear growth
    assert g_err <= L.d * 6e-8, g_err
    assert c_err <= 1.0, c_err


@pytest.mark.parametrize("name", LARGE)
def test_quantize_full_layer_with_oracle_u(name):
    L = wl.LAYERS[name]
    Lsub = L.with_tokens(8 * 2048)
    Xs = wl.make_x(Lsub).double().numpy()
    Hs = oracle.hessian(Xs)
    U = oracle.inverse_upper_cholesky(oracle.dampen(Hs, L.damp))
    U32 = np.ascontiguousarray(U, dtype=np.float32)
    W = wl.make_w(L)
    gpu = S.quantize(W.cuda(), torch.from_numpy(U32).cuda(), L.bits, L.group_size, L.block_size)
    rows = np.sort(np.random.default_rng(1).choice(L.m, size=min(L.m, 512), replace=False))
    ref = oracle.gptq_quantize(W[rows].double().numpy(), U32.astype(np.float64), L.bits, L.group_size,
                               L.block_size)
    Wr = W[rows].double().numpy()
    st = S.compare_quantization((gpu[0][rows], gpu[1][rows], gpu[2][rows]), ref, L.group_size, Wr, Hs,
                                label=name)
    print(name, st)


def test_quantize_widest_layer_with_seeded_u():
    L = wl.LAYERS[WIDEST]
    rows = np.sort(np.random.default_rng(3).choice(L.m, size=256, replace=False))
    U = wl.make_upper(L.d, seed=11, device="cuda")
    W = wl.make_w(L, device="cuda")
    gpu = S.quantize(W, U, L.bits, L.group_size, L.block_size, rows=rows)
    Wr = W[torch.as_tensor(rows, device=W.device)].double().cpu().numpy()
    del W
    U64 = U.cpu().double().numpy()
    del U
    ref = oracle.gptq_quantize(Wr, U64, L.bits, L.group_size, L.block_size)
    st = S.compare_quantization(gpu, ref, L.group_size, label=WIDEST)
    print(WIDEST, st)


# The chained layers: every stage on the GPU from the layer's own X and W, against the fp64 oracle
# from the same X (H over all tokens streamed to the host, its U, the quantization of sampled rows).
# The 11008-wide layer takes 32,768 of its tokens (16 chunks of 2,048), which keeps the host's fp64
# Hessian to a minute; its Hessian over all 262,144 tokens is checked on sampled blocks above.
CHAINED = [("llama7b_q_4096x4096", None), ("llama7b_up_11008x4096", None),
           ("llama7b_down_4096x11008", 16 * 2048)]


@pytest.mark.parametrize("name,n_tokens", CHAINED)
def test_end_to_end_chained_layer(name, n_tokens):
    L = wl.LAYERS[name]
    if n_tokens is not None:
        L = L.with_tokens(n_tokens)
    X = wl.make_x(L, device="cuda")
    W = wl.make_w(L)
    from post_weight_quantization_21_b200 import LayerSolver
    s = LayerSolver(L.m, L.d, L.n_tokens, L.bits, L.group_size, L.block_size, L.damp, X.dtype, W.dtype)
    s.X.copy_(X)
    s.W.copy_(W)
    s.run()
    s.check_status()
    torch.cuda.synchronize()
    H = np.zeros((L.d, L.d))
    for Xc in _x_cpu_chunks(X):
        oracle.hessian_accumulate(H, Xc)
    del X
    assert S.upper_rel_fro(s.H.cpu().numpy(), H) <= S.H_REL_FRO
    Hd = oracle.dampen(H, L.damp)
    U = oracle.inverse_upper_cholesky(Hd)
    # the GPU's U from its own H against the oracle's U from the fp64 H (the prepare tests' bound)
    Ug = s.U.double().cpu().numpy()
    rel = np.linalg.norm(Ug - U) / np.linalg.norm(U)
    ev = np.linalg.eigvalsh(Hd)
    kappa = ev[-1] / ev[0]
    S.NOTES.append((f"{name} chained U", f"rel err {rel:.3e}, kappa {kappa:.3e}"))
    assert rel <= max(1e-5, 10 * kappa * 6e-8), (rel, kappa)
    del Ug
    rows = np.sort(np.random.default_rng(2).choice(L.m, size=1024, replace=False))
    Wr = W[rows].double().numpy()
    ref = oracle.gptq_quantize(Wr, U, L.bits, L.group_size, L.block_size)
    ref["E"] = oracle.reconstruction_error(Wr, ref["Wq"], H)
    gpu = (s.codes.cpu().numpy().astype(np.int64)[rows], s.scales.cpu().numpy()[rows],
           s.zeros.cpu().numpy().astype(np.int64)[rows])
    st = S.compare_quantization(gpu, ref, L.group_size, Wr, H, ref["E"], label=f"{L.name} chained")
    packed = s.packed.cpu().numpy()[rows]
    np.testing.assert_array_equal(packed, oracle.pack_codes(gpu[0], L.bits))
    print(name, "chained", st)
