"""GPU parity of the inference product with the packed weights (gptq_dequant_matmul) against the
oracle's dequantized product on the same packed codes, grids and inputs."""
import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_21_b200 as g

import gpu_support as S

pytestmark = pytest.mark.gpu


def _case(m, d, bits, gs, seed):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 2 ** bits, size=(m, d))
    ng = 1 if gs == 0 else d // gs
    scales = rng.uniform(0.001, 0.05, size=(m, ng)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, size=(m, ng)).astype(np.int32)
    return codes, oracle.pack_codes(codes, bits), scales, zeros


# several row blocks and column tiles with ragged ends, every width, per-row and group grids
CASES = [
    # m, d, bits, group, batch, x dtype
    (1, 32, 4, 0, 1, torch.float32),
    (33, 96, 3, 32, 1, torch.float16),
    (100, 4096 + 512, 3, 0, 1, torch.float16),
    (257, 8192, 4, 128, 3, torch.bfloat16),
    (64, 12288, 2, 64, 4, torch.float16),
    (40, 4096, 3, 128, 7, torch.float32),
]


@pytest.mark.parametrize("m,d,bits,gs,batch,xdt", CASES)
def test_dequant_matmul_matches_oracle(m, d, bits, gs, batch, xdt):
    codes, packed, scales, zeros = _case(m, d, bits, gs, seed=m + d + bits)
    X = torch.randn(batch, d, generator=torch.Generator().manual_seed(d)).to(xdt)
    ref = oracle.dequant_matmul(packed, scales, zeros, bits, gs, d, X.double().numpy())
    dev = S.dev()
    Y = torch.full((batch, m), float("nan"), device=dev)
    ws = torch.empty(g.gptq_dequant_matmul_workspace_size(m, d, batch), dtype=torch.uint8, device=dev)
    st = torch.zeros(2, dtype=torch.int32, device=dev)
    g.gptq_dequant_matmul(torch.from_numpy(packed).to(dev), torch.from_numpy(scales).to(dev),
                          torch.from_numpy(zeros).to(dev), bits, gs, X.to(dev), Y, st, ws)
    assert g.gptq_read_status(st)[0] == g.GPTQ_OK
    got = Y.cpu().double().numpy()
    _check(got, ref, codes, scales, zeros, bits, gs, X.double().numpy())


def _check(got, ref, codes, scales, zeros, bits, gs, X):
    """fp32 arithmetic: every product q_j x_j is formed exactly and rounded once, the unit sums of 32
    such products and of the inputs are fp32 sums, and each unit adds scale (sum q x - zero sum x); the
    rounding error is a few tens of ulps of scale sum_j |x_j| (|q_j| + |zero|) <= sum_j |x_j| (|What_j|
    + 2^(b+1) scale), so 64 ulps of that bound."""
    d = codes.shape[1]
    rep = d if gs == 0 else gs
    s_rep = np.repeat(scales.astype(np.float64), rep, axis=1)
    Wq = np.abs(oracle.dequantize(codes, s_rep, np.repeat(zeros.astype(np.float64), rep, axis=1)))
    scale_terms = np.abs(X) @ (Wq + (2 ** (bits + 1)) * s_rep).T
    err = np.abs(got - ref)
    assert np.all(err <= 64 * 6e-8 * scale_terms + 1e-30), (err / scale_terms).max()


@pytest.mark.parametrize("batch", [1, 2])
def test_dequant_matmul_large_sampled_rows(batch):
    """6144 x 49152 3-bit per-row words (uniform random codes): the staged form's column tiles run 16
    chunks each, so every warp's ring of stages wraps around several times.  Sampled rows against the
    oracle."""
    m, d, bits = 6144, 49152, 3
    rng = np.random.default_rng(11)
    packed = rng.integers(-2 ** 31, 2 ** 31, size=(m, d * bits // 32), dtype=np.int64).astype(np.int32)
    scales = rng.uniform(0.001, 0.05, size=(m, 1)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, size=(m, 1)).astype(np.int32)
    X = torch.randn(batch, d, generator=torch.Generator().manual_seed(5)).to(torch.float16)
    dev = S.dev()
    Y = torch.full((batch, m), float("nan"), device=dev)
    ws = torch.empty(g.gptq_dequant_matmul_workspace_size(m, d, batch), dtype=torch.uint8, device=dev)
    st = torch.zeros(2, dtype=torch.int32, device=dev)
    g.gptq_dequant_matmul(torch.from_numpy(packed).to(dev), torch.from_numpy(scales).to(dev),
                          torch.from_numpy(zeros).to(dev), bits, 0, X.to(dev), Y, st, ws)
    assert g.gptq_read_status(st)[0] == g.GPTQ_OK
    rows = np.unique(np.concatenate([rng.choice(m, 94, replace=False), [0, m - 1]]))
    Xd = X.double().numpy()
    ref = oracle.dequant_matmul(packed[rows], scales[rows], zeros[rows], bits, 0, d, Xd)
    got = Y.cpu().double().numpy()[:, rows]
    assert np.isfinite(Y.cpu().numpy()).all()
    _check(got, ref, oracle.unpack_codes(packed[rows], bits, d), scales[rows], zeros[rows], bits, 0, Xd)
