"""Helpers shared by the GPU parity tests: run a stage through the C ABI, compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import post_weight_quantization_21_b200 as g

# Tolerances (from the solver's parity targets; readings in the design notes):
H_REL_FRO = 1e-5        # Hessian, relative Frobenius error against fp64 on the same inputs
CODES_MIN_AGREE = 0.995  # share of identical codes; a row's first mismatch is exactly one level
SCALE_REL = 1e-5         # scales relative error (per-row: all rows; per-group: rows whose earlier codes match)
E_REL = 0.02             # layer reconstruction error, relative


# every compare_quantization call appends (label, stats) here; the session summary prints them
PARITY_LOG: list[tuple[str, dict]] = []
# other measured figures a test wants in the session summary (label, text)
NOTES: list[tuple[str, str]] = []


def dev():
    return torch.device("cuda", 0)


def hessian(X: torch.Tensor, accumulate_into: torch.Tensor | None = None, scale: float = 2.0):
    n, d = X.shape
    H = accumulate_into if accumulate_into is not None else torch.empty(d, d, device=X.device)
    ws = torch.empty(max(g.gptq_hessian_workspace_size(n, d, X.dtype), 256), dtype=torch.uint8, device=X.device)
    st = torch.zeros(4, dtype=torch.int32, device=X.device)
    g.gptq_hessian_accumulate(X, H, st, ws, scale, accumulate_into is not None)
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_OK, (code, detail)
    return H


def prepare(H: torch.Tensor, damp: float = 0.01, expect_ok: bool = True):
    d = H.shape[0]
    U = torch.empty_like(H)
    ws = torch.empty(g.gptq_prepare_workspace_size(d), dtype=torch.uint8, device=H.device)
    st = torch.zeros(4, dtype=torch.int32, device=H.device)
    g.gptq_prepare_uinv(H, U, st, ws, damp)
    code, detail = g.gptq_read_status(st)
    if expect_ok:
        assert code == g.GPTQ_OK, (code, detail)
        return U
    return U, code, detail


def quantize(W: torch.Tensor, U: torch.Tensor, bits: int, group_size: int, block_size: int, rows=None,
             flags: int = 0):
    """Codes, scales, zeros of the whole layer (of ``rows`` only when given) as int64/fp32 host arrays."""
    m, d = W.shape
    n_groups = 1 if group_size == 0 else d // group_size
    codes = torch.empty(m, d, dtype=torch.uint8, device=W.device)
    scales = torch.empty(m, n_groups, dtype=torch.float32, device=W.device)
    zeros = torch.empty(m, n_groups, dtype=torch.int32, device=W.device)
    ws = torch.empty(g.gptq_quantize_workspace_size(m, d, bits, group_size, block_size), dtype=torch.uint8,
                     device=W.device)
    st = torch.zeros(4, dtype=torch.int32, device=W.device)
    g.gptq_quantize_layer(W, U, codes, scales, zeros, st, ws, bits, group_size, block_size, flags)
    code, detail = g.gptq_read_status(st)
    assert code == g.GPTQ_OK, (code, detail)
    if rows is not None:
        idx = torch.as_tensor(rows, device=W.device)
        codes, scales, zeros = codes[idx], scales[idx], zeros[idx]
    return codes.cpu().numpy().astype(np.int64), scales.cpu().numpy(), zeros.cpu().numpy().astype(np.int64)


def pack(codes_u8: torch.Tensor, bits: int):
    m, d = codes_u8.shape
    out = torch.empty(m, d * bits // 32, dtype=torch.int32, device=codes_u8.device)
    g.gptq_pack(codes_u8, bits, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def upper_rel_fro(A_gpu: np.ndarray, A_ref: np.ndarray) -> float:
    iu = np.triu_indices(A_ref.shape[0])
    return float(np.linalg.norm(A_gpu[iu] - A_ref[iu]) / np.linalg.norm(A_ref[iu]))


def dequant(codes, scales, zeros, group_size):
    m, d = codes.shape
    gs = d if group_size == 0 else group_size
    s = np.repeat(scales.astype(np.float64), gs, axis=1)
    z = np.repeat(zeros.astype(np.float64), gs, axis=1)
    return s * (codes - z)


def compare_quantization(gpu, ref, group_size, W=None, H=None, E_ref=None, label=""):
    """Checks codes / scales / zeros (and E when W, H given) of the GPU against the oracle; returns stats."""
    codes, scales, zeros = gpu
    rc, rs, rz = ref["codes"], ref["scales"], ref["zeros"]
    diff = codes - rc
    agree = float(np.mean(diff == 0))
    if agree < CODES_MIN_AGREE:
        PARITY_LOG.append((label, {"agree": agree, "mismatches": int(np.sum(diff != 0)), "failed": True}))
    assert agree >= CODES_MIN_AGREE, f"{label}: codes agree {agree:.5f}"
    m, d = codes.shape
    bad_rows = (diff != 0).any(axis=1)
    first_bad = np.where(bad_rows, np.argmax(diff != 0, axis=1), d)
    # at a row's first mismatch both trajectories are still identical: a near-tie, one level apart
    firsts = diff[bad_rows, first_bad[bad_rows]]
    assert np.all(np.abs(firsts) == 1), f"{label}: a first mismatch differs by more than one level"
    if group_size == 0:
        # one fixed grid per row: later mismatches stay one level apart as well
        assert np.all(np.abs(diff) <= 1), f"{label}: a code differs by more than one level"
        rel = np.abs(scales - rs) / np.abs(rs)
        assert rel.max() <= SCALE_REL, f"{label}: scale rel err {rel.max()}"
        assert np.array_equal(zeros, rz), f"{label}: zeros differ"
        checked = m
    else:
        # per-group grids depend on the row's earlier codes.  Groups before the row's first mismatch
        # must match (scales within tolerance, zeros equal); in the group of the first mismatch the
        # scale must match and the zero point may sit one level off (its rounding is a near-tie of
        # the same kind as a code's); later groups follow a different trajectory and are counted.
        ng = d // group_size
        gstart = np.arange(ng)[None, :] * group_size
        before = gstart + group_size <= first_bad[:, None]
        at = (gstart <= first_bad[:, None]) & ~before
        rel = np.abs(scales - rs) / np.abs(rs)
        upto = before | at
        assert rel[upto].max() <= SCALE_REL, f"{label}: group scale rel err {rel[upto].max()}"
        assert np.array_equal(zeros[before], rz[before]), f"{label}: group zeros differ"
        assert np.all(np.abs(zeros[at] - rz[at]) <= 1), f"{label}: zero point off by more than one"
        checked = int(upto.sum())
    stats = {"agree": agree, "mismatches": int(np.sum(diff != 0)), "rows_diverged": int(bad_rows.sum()),
             "max_level_diff": int(np.abs(diff).max()), "grids_checked": checked}
    PARITY_LOG.append((label, stats))
    if W is not None and H is not None:
        import oracle
        E_gpu = oracle.reconstruction_error(W, dequant(codes, scales, zeros, group_size), H)
        E_o = E_ref if E_ref is not None else oracle.reconstruction_error(W, ref["Wq"], H)
        stats["E_rel"] = abs(E_gpu - E_o) / E_o
        assert stats["E_rel"] <= E_REL, f"{label}: E rel {stats['E_rel']}"
    return stats
