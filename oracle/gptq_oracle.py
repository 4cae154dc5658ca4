"""GPTQ layer-wise solver: the oracle.

TEST INFRASTRUCTURE ONLY.  This is a plain, slow, fp64 CPU statement of what the GPTQ solver
computes.  Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import it.  It shares no code with the CUDA library and must never serve as a fallback for it.

Sources (web pages about GPTQ, Frantar, Ashkboos, Hoefler, Alistarh, ICLR 2023):

[FDE]  "GPTQ: Accurate Post-Training Quantization for Generative Pre-trained Transformers",
       fdeinterviews.com breakdown: section 01 "The paper in one minute" and the figure
       "THE IDEA, VISUALLY" (steps 1-4 of "quantize a column, correct the rest").
[ZLY]  "GPTQ：用于生成式预训练 Transformer 的准确训练后量化", blog.zhiliyouxian.com: sections
       数学基础 (problem statement), 算法流程 (layer routine), 关键优化 (128-column blocks),
       实践指南 (damp_percent = 0.01, group_size = 128, desc_act = False).
[NUB]  "[Paper Review] GPTQ ...", nubint.ai: "Proposed method" (OBQ lineage, lazy batch updates,
       Cholesky reformulation and dampening).
[CSDN] "GPTQ量化参数搜索工具", agent.csdn.net: 关键参数说明 table (bits, group_size, zero point).

Precision.  Every floating-point step is fp64, except the two places where a floating-point value
decides an integer (the zero point and the code of each weight).  There the decision is taken in
fp32, the precision of the CUDA kernels: the quotient x / scale is the IEEE round-to-nearest fp32
quotient of the fp32 operands, then rounded half-to-even.

Readings of the pages (they are silent or garbled here; the plainest reading is used):
* Grid: asymmetric min/max uniform grid on {0..2^b-1}; the range is widened to contain 0; an all-zero
  range becomes [-1, 1]; zero = rint(-xmin/scale); q = clamp(rint(x/scale) + zero, 0, maxq), the
  quotients taken in fp32 (see Precision).
* Per-row grids come from the original row before the column loop; per-group grids come from the
  current (already compensated) values of the group's columns when the loop reaches the group.
* The column loop quantizes the current, compensated value of each column ([FDE] figure, step 1),
  not the original value ([ZLY]'s listing is garbled on this point).
* Packing: per row, a little-endian bit stream of b-bit codes in int32 words (no layout on the pages).

Pins (tests/test_oracle_pins.py): H proportional to I reduces to round-to-nearest; the Cholesky form
equals the explicit OBS recursion; brute force on d <= 6; the expected statistic against RTN;
invariances; hand-worked golden files.  The grid convention and the pack layout are not fixed by the
pages ("parity unpinned" by the pages); they are pinned by textbook properties of a uniform
quantizer and by a hand-worked packing example.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "hessian", "hessian_accumulate", "dampen", "inverse_upper_cholesky",
    "inverse_upper_cholesky_reversed", "grid_params", "quantize_codes", "dequantize",
    "gptq_quantize", "rtn_quantize", "obs_quantize", "conditional_ls_values",
    "bruteforce_best_codes", "reconstruction_error", "pack_codes", "unpack_codes", "gptq_layer",
    "act_order_permutation", "gptq_quantize_act_order", "act_order_group_index", "dequant_matmul",
]


# --------------------------------------------------------------------------------------------
# A1  Hessian.  [FDE] section 01: "a least-squares problem whose curvature is the matrix
#     H = 2XX^T, computed from the calibration inputs" (X there is [in, tokens]; here X is
#     [tokens, in], so H = 2 X^T X).  [ZLY] 算法流程 step 1 writes X.T @ X / len(X): the same matrix
#     up to a positive factor, which changes no code (pinned by the scale-invariance test).
# --------------------------------------------------------------------------------------------
def hessian(X, scale: float = 2.0) -> np.ndarray:
    X = np.asarray(X, dtype=np.float64)
    return scale * (X.T @ X)


def hessian_accumulate(H: np.ndarray, X_chunk, scale: float = 2.0) -> np.ndarray:
    """H += scale * Xc^T Xc for one chunk of tokens (the sum over tokens is additive)."""
    Xc = np.asarray(X_chunk, dtype=np.float64)
    H += scale * (Xc.T @ Xc)
    return H


# --------------------------------------------------------------------------------------------
# A2  Dampening.  [ZLY] 算法流程 "H = H + lambda * I  # 正则化" and 实践指南 damp_percent = 0.01;
#     [NUB] "Uses a Cholesky reformulation and dampening to maintain numerical stability".
#     lambda = damp * mean(diag H).
# --------------------------------------------------------------------------------------------
def dampen(H, damp: float = 0.01) -> np.ndarray:
    H = np.asarray(H, dtype=np.float64)
    lam = damp * float(np.mean(np.diag(H)))
    return H + lam * np.eye(H.shape[0])


# --------------------------------------------------------------------------------------------
# A3  U = chol(H^-1), upper.  [FDE] figure step 2 "U = chol(H^-1)", section 01 "the needed rows of
#     the inverse Hessian are taken from a Cholesky decomposition".  Written as the definition:
#     invert Hd through its Cholesky factor, then take the upper Cholesky factor of the inverse.
# --------------------------------------------------------------------------------------------
def _lower_inverse(L: np.ndarray) -> np.ndarray:
    """L^{-1} for lower-triangular L by forward substitution, column by column of the identity."""
    n = L.shape[0]
    X = np.zeros_like(L)
    for j in range(n):
        e = np.zeros(n)
        e[j] = 1.0
        x = np.zeros(n)
        for i in range(j, n):
            x[i] = (e[i] - L[i, j:i] @ x[j:i]) / L[i, i]
        X[:, j] = x
    return X


def inverse_upper_cholesky(Hd) -> np.ndarray:
    """Route of the pages: L = chol(Hd); Hinv = L^-T L^-1; U = upper Cholesky factor of Hinv."""
    Hd = np.asarray(Hd, dtype=np.float64)
    L = np.linalg.cholesky(Hd)
    n = Hd.shape[0]
    if n <= 64:
        Linv = _lower_inverse(L)
    else:
        import scipy.linalg
        Linv = scipy.linalg.solve_triangular(L, np.eye(n), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T  # upper: U^T U = Hinv


def inverse_upper_cholesky_reversed(Hd) -> np.ndarray:
    """Cross-check route: write Hd = R R^T with R upper (Cholesky of the index-reversed matrix);
    then U = R^-1 is upper with U^T U = Hd^-1, so by uniqueness it is the same factor."""
    Hd = np.asarray(Hd, dtype=np.float64)
    n = Hd.shape[0]
    J = np.eye(n)[::-1]
    Lr = np.linalg.cholesky(J @ Hd @ J)
    R = J @ Lr @ J
    import scipy.linalg
    return scipy.linalg.solve_triangular(R, np.eye(n), lower=False)


# --------------------------------------------------------------------------------------------
# A4  Grid.  [FDE] figure step 1 "round column i to the 3/4-bit grid"; [CSDN] 关键参数说明 lists
#     bits and a zero point; [ZLY] 实践指南 group_size = 128.  The grid formula is not printed on the
#     pages; see the module docstring for the reading.  Decisions are taken in fp32.
# --------------------------------------------------------------------------------------------
def grid_params(xmin, xmax, bits: int):
    """Per-entry fp32 scale and int zero point from range endpoints (arrays of equal shape)."""
    maxq = np.float32(2 ** bits - 1)
    lo = np.minimum(np.asarray(xmin, dtype=np.float64), 0.0).astype(np.float32)
    hi = np.maximum(np.asarray(xmax, dtype=np.float64), 0.0).astype(np.float32)
    flat = lo == hi
    lo = np.where(flat, np.float32(-1.0), lo)
    hi = np.where(flat, np.float32(1.0), hi)
    scale = ((hi - lo) / maxq).astype(np.float32)
    zero = np.rint(((-lo) / scale).astype(np.float32))
    return scale, zero.astype(np.int64)


def quantize_codes(x, scale, zero, bits: int) -> np.ndarray:
    """q = clamp(rint(x / scale) + zero, 0, 2^b - 1), the quotient an IEEE fp32 division."""
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    r = np.rint((x32 / np.asarray(scale, dtype=np.float32)).astype(np.float32)).astype(np.int64)
    return np.clip(r + np.asarray(zero, dtype=np.int64), 0, 2 ** bits - 1)


def dequantize(q, scale, zero) -> np.ndarray:
    return np.asarray(scale, dtype=np.float64) * (np.asarray(q, dtype=np.float64)
                                                  - np.asarray(zero, dtype=np.float64))


# --------------------------------------------------------------------------------------------
# A5 + A6  Column loop with error compensation and lazy 128-column block updates.
#     [FDE] figure: (1) round column i; (2) err = (w_i - q_i) / U_ii; (3) W[:, i+1:] -= err x
#     U[i, i+1:]; (4) apply in blocks of 128 columns.  Section 01: same column order for every row.
#     [ZLY] 关键优化 1: BLOCK_SIZE = 128.  block_size = 0 runs the plain unblocked definition; a
#     positive block size applies step 3 inside the block at once and the rest of the update once
#     per block (identical in exact arithmetic when each group lies in one block or each block in
#     one group).
# --------------------------------------------------------------------------------------------
def _check_groups(d: int, group_size: int, block_size: int):
    if group_size:
        if d % group_size:
            raise ValueError("group_size must divide d")
        if block_size and (group_size % block_size) and (block_size % group_size):
            raise ValueError("group_size and block_size must divide one another")


def gptq_quantize(W, U, bits: int, group_size: int = 0, block_size: int = 0):
    """Quantize all rows of W given the upper factor U.  Returns dict(codes, scales, zeros, Wq, Err)."""
    Wc = np.array(W, dtype=np.float64)  # current (compensated) values
    U = np.asarray(U, dtype=np.float64)
    m, d = Wc.shape
    _check_groups(d, group_size, block_size)
    n_groups = 1 if group_size == 0 else d // group_size
    scales = np.zeros((m, n_groups), dtype=np.float32)
    zeros = np.zeros((m, n_groups), dtype=np.int64)
    codes = np.zeros((m, d), dtype=np.int64)
    Wq = np.zeros((m, d), dtype=np.float64)
    Err = np.zeros((m, d), dtype=np.float64)
    if group_size == 0:
        s, z = grid_params(Wc.min(axis=1), Wc.max(axis=1), bits)
        scales[:, 0], zeros[:, 0] = s, z
    B = block_size if block_size else d
    for i1 in range(0, d, B):
        i2 = min(i1 + B, d)
        for i in range(i1, i2):
            if group_size and i % group_size == 0:
                cols = Wc[:, i:i + group_size]
                s, z = grid_params(cols.min(axis=1), cols.max(axis=1), bits)
                scales[:, i // group_size], zeros[:, i // group_size] = s, z
            g = i // group_size if group_size else 0
            q = quantize_codes(Wc[:, i], scales[:, g], zeros[:, g], bits)
            wq = dequantize(q, scales[:, g], zeros[:, g])
            err = (Wc[:, i] - wq) / U[i, i]
            Wc[:, i + 1:i2] -= np.outer(err, U[i, i + 1:i2])
            codes[:, i], Wq[:, i], Err[:, i] = q, wq, err
        if i2 < d:
            Wc[:, i2:] -= Err[:, i1:i2] @ U[i1:i2, i2:]
    return {"codes": codes, "scales": scales, "zeros": zeros, "Wq": Wq, "Err": Err}


def rtn_quantize(W, bits: int, group_size: int = 0):
    """Round-to-nearest on the same grid, no compensation ([FDE] section 01 and "The problem")."""
    W = np.asarray(W, dtype=np.float64)
    m, d = W.shape
    n_groups = 1 if group_size == 0 else d // group_size
    gs = d if group_size == 0 else group_size
    codes = np.zeros((m, d), dtype=np.int64)
    scales = np.zeros((m, n_groups), dtype=np.float32)
    zeros = np.zeros((m, n_groups), dtype=np.int64)
    for g in range(n_groups):
        cols = W[:, g * gs:(g + 1) * gs]
        s, z = grid_params(cols.min(axis=1), cols.max(axis=1), bits)
        scales[:, g], zeros[:, g] = s, z
        codes[:, g * gs:(g + 1) * gs] = quantize_codes(cols, s[:, None], z[:, None], bits)
    Wq = np.zeros((m, d))
    for g in range(n_groups):
        Wq[:, g * gs:(g + 1) * gs] = dequantize(codes[:, g * gs:(g + 1) * gs],
                                                scales[:, g:g + 1], zeros[:, g:g + 1])
    return {"codes": codes, "scales": scales, "zeros": zeros, "Wq": Wq}


# --------------------------------------------------------------------------------------------
# Explicit OBS / OBQ recursion ([NUB] "Builds on Optimal Brain Quantization (OBQ)").  Keeps the
# inverse Hessian of the not-yet-quantized set F and removes column i after quantizing it:
#   W_F -= (w_i - q_i) / Hinv[i,i] * Hinv[i, F];   Hinv <- Hinv - Hinv[:, i] Hinv[i, :] / Hinv[i,i].
# Used only to pin the Cholesky form (small d).
# --------------------------------------------------------------------------------------------
def obs_quantize(W, Hd, bits: int, group_size: int = 0, order=None):
    """``order`` (default: natural) is the sequence in which columns are quantized; the recursion
    needs no permuted matrices: it removes each quantized column from the free set F directly.  A
    group is ``group_size`` consecutive steps of the order; its grid comes from the current values of
    the group's columns at its first step."""
    Wc = np.array(W, dtype=np.float64)
    m, d = Wc.shape
    order = np.arange(d) if order is None else np.asarray(order)
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=np.float64))
    n_groups = 1 if group_size == 0 else d // group_size
    scales = np.zeros((m, n_groups), dtype=np.float32)
    zeros = np.zeros((m, n_groups), dtype=np.int64)
    codes = np.zeros((m, d), dtype=np.int64)
    free = np.ones(d, dtype=bool)
    if group_size == 0:
        s, z = grid_params(Wc.min(axis=1), Wc.max(axis=1), bits)
        scales[:, 0], zeros[:, 0] = s, z
    for k, i in enumerate(order):
        if group_size and k % group_size == 0:
            cols = Wc[:, order[k:k + group_size]]
            s, z = grid_params(cols.min(axis=1), cols.max(axis=1), bits)
            scales[:, k // group_size], zeros[:, k // group_size] = s, z
        g = k // group_size if group_size else 0
        q = quantize_codes(Wc[:, i], scales[:, g], zeros[:, g], bits)
        delta = Wc[:, i] - dequantize(q, scales[:, g], zeros[:, g])
        hii = Hinv[i, i]
        free[i] = False
        Wc[:, free] -= np.outer(delta / hii, Hinv[i, free])
        Hinv = Hinv - np.outer(Hinv[:, i], Hinv[i, :]) / hii
        codes[:, i] = q
    return {"codes": codes, "scales": scales, "zeros": zeros}


def conditional_ls_values(w, Hd, wq_prefix):
    """Minimiser of (w - v)^T Hd (w - v) over v[k:] with v[:k] = wq_prefix fixed (the layer-wise
    objective of [ZLY] 数学基础 / [FDE] section 01 restricted to the free columns)."""
    w = np.asarray(w, dtype=np.float64)
    Hd = np.asarray(Hd, dtype=np.float64)
    k = len(wq_prefix)
    dF = w[:k] - np.asarray(wq_prefix, dtype=np.float64)
    return w[k:] + np.linalg.solve(Hd[k:, k:], Hd[k:, :k] @ dF)


def bruteforce_best_codes(w, Hd, bits: int, scale, zero):
    """Exhaustive minimum of (w - deq(q))^T Hd (w - deq(q)) over all code vectors q (tiny d)."""
    w = np.asarray(w, dtype=np.float64)
    d = w.shape[0]
    levels = 2 ** bits
    grids = np.meshgrid(*[np.arange(levels)] * d, indexing="ij")
    Q = np.stack([g.ravel() for g in grids], axis=1)
    D = w[None, :] - dequantize(Q, scale, zero)
    obj = np.einsum("ni,ij,nj->n", D, np.asarray(Hd, dtype=np.float64), D)
    k = int(np.argmin(obj))
    return Q[k], float(obj[k])


# --------------------------------------------------------------------------------------------
# A8  Reconstruction error of the layer ([ZLY] 数学基础 "minimize ||Wx - Ŵx||^2"; [FDE] section 01
#     "the layer's outputs on a small calibration set X should change as little as possible").
#     With the undamped H = 2 X^T X: ||(W - Ŵ) X^T||_F^2 = 1/2 tr(dW H dW^T).
# --------------------------------------------------------------------------------------------
def reconstruction_error(W, Wq, H) -> float:
    dW = np.asarray(W, dtype=np.float64) - np.asarray(Wq, dtype=np.float64)
    return 0.5 * float(np.einsum("ij,jk,ik->", dW, np.asarray(H, dtype=np.float64), dW))


# --------------------------------------------------------------------------------------------
# A7  Packing into int32 words.  [FDE] figure: 3-bit weights stored (350 GB -> 66 GB) and read by
#     the inference kernel.  Layout reading: per row, code j occupies bits [j*b, (j+1)*b) of a
#     little-endian bit stream; word k holds stream bits [32k, 32k+32); row stride ceil(d*b/32).
# --------------------------------------------------------------------------------------------
def pack_codes(codes, bits: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    m, d = codes.shape
    n_words = (d * bits + 31) // 32
    out = np.zeros((m, n_words), dtype=np.uint64)
    for j in range(d):
        bit = j * bits
        w, sh = divmod(bit, 32)
        v = codes[:, j].astype(np.uint64)
        out[:, w] |= (v << np.uint64(sh)) & np.uint64(0xFFFFFFFF)
        if sh + bits > 32:
            out[:, w + 1] |= v >> np.uint64(32 - sh)
    return out.astype(np.uint32).view(np.int32)


def unpack_codes(packed, bits: int, d: int) -> np.ndarray:
    p = np.asarray(packed).view(np.uint32).astype(np.uint64)
    m = p.shape[0]
    mask = np.uint64(2 ** bits - 1)
    out = np.zeros((m, d), dtype=np.int64)
    for j in range(d):
        w, sh = divmod(j * bits, 32)
        v = p[:, w] >> np.uint64(sh)
        if sh + bits > 32:
            v = v | (p[:, w + 1] << np.uint64(32 - sh))
        out[:, j] = (v & mask).astype(np.int64)
    return out


# --------------------------------------------------------------------------------------------
# Act-order ("desc_act").  [ZLY] 实践指南 lists desc_act (off by default); [CSDN] 关键参数说明 lists
# it among the quantizer's settings.  The pages do not define the order beyond its name ("sort by
# activation"); reading: the columns are quantized in descending order of diag(H) (the channels with
# the largest calibration activations first), ties in column order.  The method itself is unchanged:
# it runs on the permuted problem (H -> P H P^T, W -> W P^T), and the codes are put back in the
# original column order.  Groups are consecutive columns of the quantization order, so group k
# holds the original columns perm[k*g : (k+1)*g].
# --------------------------------------------------------------------------------------------
def act_order_permutation(H) -> np.ndarray:
    """perm[i] = the original column quantized at step i: descending diag(H), ties by column index."""
    diag = np.diag(np.asarray(H, dtype=np.float64))
    return np.argsort(-diag, kind="stable")


def act_order_group_index(perm, group_size: int) -> np.ndarray:
    """Group of each original column: the step at which it is quantized, divided by the group size."""
    perm = np.asarray(perm)
    step = np.empty_like(perm)
    step[perm] = np.arange(perm.shape[0])
    return step // group_size if group_size else np.zeros_like(step)


def gptq_quantize_act_order(W, H, bits: int, group_size: int = 0, block_size: int = 0, damp: float = 0.01,
                            perm=None):
    """The column loop in act-order.  Returns codes and Wq in the original column order, the grids of
    the groups of the quantization order, perm, the group index of every original column, and the
    factor U of the permuted dampened Hessian."""
    H = np.asarray(H, dtype=np.float64)
    if perm is None:
        perm = act_order_permutation(H)
    perm = np.asarray(perm)
    U = inverse_upper_cholesky(dampen(H[np.ix_(perm, perm)], damp))
    r = gptq_quantize(np.asarray(W, dtype=np.float64)[:, perm], U, bits, group_size, block_size)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.shape[0])
    return {"codes": r["codes"][:, inv], "Wq": r["Wq"][:, inv], "scales": r["scales"], "zeros": r["zeros"],
            "perm": perm, "g_idx": act_order_group_index(perm, group_size), "U": U,
            "codes_in_order": r["codes"]}


# --------------------------------------------------------------------------------------------
# Inference with the packed weights.  [FDE] section 01, last paragraph: custom kernels read the 3-bit
# weights and dequantize them on the fly (the 3.25x generation speed-up on A100).  What that kernel
# computes is the layer's product with the dequantized weights: Y = X_in @ What^T with
# What[r, j] = scale[r, g(j)] * (q[r, j] - zero[r, g(j)]), g(j) = j // group_size (0 per-row), the codes
# read from the packed words (A7 layout).  X_in [batch, d] -> Y [batch, m].
# --------------------------------------------------------------------------------------------
def dequant_matmul(packed, scales, zeros, bits: int, group_size: int, d: int, X_in) -> np.ndarray:
    codes = unpack_codes(packed, bits, d)
    m = codes.shape[0]
    gs = d if group_size == 0 else group_size
    s = np.repeat(np.asarray(scales, dtype=np.float64).reshape(m, -1), gs, axis=1)
    z = np.repeat(np.asarray(zeros, dtype=np.float64).reshape(m, -1), gs, axis=1)
    What = dequantize(codes, s, z)
    return np.asarray(X_in, dtype=np.float64) @ What.T


# --------------------------------------------------------------------------------------------
# The whole layer: A1 -> A2 -> A3 -> A5/A6 -> A7.
# --------------------------------------------------------------------------------------------
def gptq_layer(W, X, bits: int, group_size: int = 0, block_size: int = 128, damp: float = 0.01,
               H=None):
    """Everything the solver produces for one layer, in fp64.  ``H`` (2 X^T X) may be passed in
    when the caller accumulated it chunk by chunk."""
    if H is None:
        H = hessian(X)
    Hd = dampen(H, damp)
    U = inverse_upper_cholesky(Hd)
    res = gptq_quantize(W, U, bits, group_size, block_size)
    res.update(H=H, Hd=Hd, U=U, packed=pack_codes(res["codes"], bits),
               E=reconstruction_error(W, res["Wq"], H))
    return res
