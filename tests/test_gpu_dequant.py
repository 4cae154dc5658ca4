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
    g.gptq_dequant_matmul(torch.from_numpy(packed).to(dev), torch.from_numpy(scales).to(dev),
                          torch.from_numpy(zeros).to(dev), bits, gs, X.to(dev), Y, ws)
    got = Y.cpu().double().numpy()
    # fp32 arithmetic: each unit of 32 codes sums (1 + q/2^b) x_j and removes sum x_j, so its rounding
    # error scales with 2^b * scale * sum |x_j| besides the terms |What x|; 64 ulps covers the sums
    rep = d if gs == 0 else gs
    s_rep = np.repeat(scales.astype(np.float64), rep, axis=1)
    Wq = np.abs(oracle.dequantize(codes, s_rep, np.repeat(zeros.astype(np.float64), rep, axis=1)))
    scale_terms = np.abs(X.double().numpy()) @ (Wq + (2 ** bits) * s_rep).T
    err = np.abs(got - ref)
    assert np.all(err <= 64 * 6e-8 * scale_terms + 1e-30), (err / scale_terms).max()
