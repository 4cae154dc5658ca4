"""GPU parity of the sequential block pipeline (synthetic OPT-style block, two blocks in sequence).

Each stage is checked against the oracle on the inputs the pipeline itself produced at that point:
the block forward against the fp64 block, every Hessian against fp64 on the collected bf16 inputs,
every layer's codes against the oracle's column loop on the oracle's U of that Hessian, the
dequantized weights against the codes and grids, and the next block's inputs against the fp64 block
run with the dequantized weights.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import block as OB
from post_weight_quantization_21_b200 import pipeline as P

import gpu_support as S

pytestmark = pytest.mark.gpu

CFG = P.BlockConfig(d_model=128, n_heads=4, d_ffn=512, seq_len=64, bits=4, group_size=0, block_size=128)


def _np(p):
    return {k: v.double().cpu().numpy() for k, v in p.items()}


@pytest.mark.parametrize("cfg", [CFG, P.BlockConfig(d_model=256, n_heads=8, d_ffn=1024, seq_len=128, bits=3,
                                                    group_size=128, block_size=128)],
                         ids=["d128_4bit_row", "d256_3bit_g128"])
def test_two_blocks_in_sequence_match_the_oracle(cfg):
    n_seq = 24
    X = (torch.randn(n_seq * cfg.seq_len, cfg.d_model, generator=torch.Generator().manual_seed(7))).to(torch.bfloat16)
    bq = P.BlockQuantizer(cfg, device=S.dev(), chunk_seqs=8, keep_inputs=True)
    x = X.to(S.dev())
    for b in range(2):
        p = P.make_block(cfg, seed=100 + b, device=S.dev())
        pn = _np(p)
        # the forward pass the pipeline runs, against the fp64 block on the same inputs
        y_gpu = P.block_forward(cfg, p, x).double().cpu().numpy()
        y_ref = OB.block_forward(pn, x.double().cpu().numpy(), cfg.n_heads, cfg.seq_len)
        assert np.abs(y_gpu - y_ref).max() <= 1e-4 * np.abs(y_ref).max()
        q, y_next = bq.quantize_block(p, x)
        for name_in, layers in P.INPUTS.items():
            acts = torch.cat(bq.inputs[name_in]).double().cpu().numpy()  # the bf16 inputs the Hessian saw
            H_ref = oracle.hessian(acts)
            assert S.upper_rel_fro(bq.H[name_in].cpu().numpy(), H_ref) <= S.H_REL_FRO
            U_ref = oracle.inverse_upper_cholesky(oracle.dampen(H_ref, cfg.damp))
            for nm in layers:
                ref = oracle.gptq_quantize(pn[nm], U_ref, cfg.bits, cfg.group_size, cfg.block_size)
                gpu = (q[nm].codes.cpu().numpy().astype(np.int64), q[nm].scales.cpu().numpy(),
                       q[nm].zeros.cpu().numpy().astype(np.int64))
                S.compare_quantization(gpu, ref, cfg.group_size, pn[nm], H_ref, label=f"block {b} {nm}")
                np.testing.assert_array_equal(q[nm].packed.cpu().numpy(), oracle.pack_codes(gpu[0], cfg.bits))
                # the dequantized weights: scale * (q - zero) as one fp32 product, rounded to fp16
                gs = cfg.group_size or cfg.shape(nm)[1]
                s_rep = np.repeat(gpu[1].astype(np.float32), gs, axis=1)
                z_rep = np.repeat(gpu[2], gs, axis=1)
                deq = (s_rep * (gpu[0] - z_rep).astype(np.float32)).astype(np.float16)
                np.testing.assert_array_equal(q[nm].W_hat.cpu().numpy(), deq)
        # the next block's inputs: the block with its dequantized weights, against fp64
        W_hat = {nm: q[nm].W_hat.double().cpu().numpy() for nm in P.LINEARS}
        y_q_ref = OB.block_forward(pn, x.double().cpu().numpy(), cfg.n_heads, cfg.seq_len, weights=W_hat)
        yq = y_next.double().cpu().numpy()
        # y_next is stored in the calibration dtype (bf16): one rounding of relative size 2^-8
        assert np.abs(yq - y_q_ref).max() <= 2 ** -8 * np.abs(y_q_ref).max() * 1.01
        S.NOTES.append((f"pipeline {cfg.d_model} block {b}", ", ".join(f"{k} {v:.3f} ms" for k, v in bq.timing.items())))
        x = y_next
