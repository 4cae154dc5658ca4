"""The partitioned solve of one layer across ranks (token-sharded Hessian + all-reduce, replicated or
broadcast U, row-sharded column loop), run as world-size-2 gloo process groups on CPU.

The partitioning is the product's; the compute steps are injected, and here they are the oracle's
(test infrastructure), so the gathered result must equal the single-process oracle on the whole
layer: H and U to fp64 rounding (the token sum is split differently), codes, grids and packed
words exactly.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from post_weight_quantization_21_b200.sharded import ShardedLayerSolver, ShardOps, shard_range

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("n,world,align", [(1000, 2, 64), (37, 3, 1), (5, 4, 1), (0, 2, 64), (4096, 8, 64)])
def test_shard_range_covers_in_order(n, world, align):
    got = [shard_range(n, world, r, align) for r in range(world)]
    assert got[0][0] == 0 and got[-1][1] == n
    for (a, b), (c, _) in zip(got, got[1:]):
        assert b == c and a <= b
    for a, b in got[:-1]:
        assert b % align == 0 or b == n
    sizes = [b - a for a, b in got]
    assert max(sizes) - min(sizes) <= align


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_ops(bits, gs, B, damp):
    import oracle

    def hessian(X, H):
        H.copy_(torch.from_numpy(oracle.hessian(X.double().numpy())))

    def prepare(H, U):
        U.copy_(torch.from_numpy(oracle.inverse_upper_cholesky(oracle.dampen(H.numpy(), damp))))

    def quantize(W, U, codes, scales, zeros):
        if W.shape[0] == 0:
            return
        r = oracle.gptq_quantize(W.double().numpy(), U.numpy(), bits, gs, B)
        codes.copy_(torch.from_numpy(r["codes"].astype(np.uint8)))
        scales.copy_(torch.from_numpy(r["scales"]))
        zeros.copy_(torch.from_numpy(r["zeros"].astype(np.int32)))

    def pack(codes, packed):
        if codes.shape[0] == 0:
            return
        packed.copy_(torch.from_numpy(oracle.pack_codes(codes.numpy().astype(np.int64), bits)))

    return ShardOps(hessian, prepare, quantize, pack)


def _inputs(m, d, n, seed):
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(n, d, generator=gen, dtype=torch.float64) @ (torch.randn(d, d, generator=gen, dtype=torch.float64)
                                                                / d ** 0.5)
    W = torch.randn(m, d, generator=gen, dtype=torch.float64) * 0.02
    return X.float(), W.float()


def _rank_main(rank, world, port, case, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        m, d, n, bits, gs, B, u_source = case
        X, W = _inputs(m, d, n, seed=m + d + n)
        s = ShardedLayerSolver(m, d, n, bits, gs, B, 0.01, torch.float32, torch.float32, "cpu",
                               ops=_oracle_ops(bits, gs, B, 0.01), u_source=u_source, h_dtype=torch.float64)
        t0, t1 = s.tokens
        r0, r1 = s.rows
        s.X_local.copy_(X[t0:t1])
        s.W_local.copy_(W[r0:r1])
        s.run()
        codes, scales, zeros, packed = s.gather_results()
        torch.save({"H": s.H, "U": s.U, "codes": codes, "scales": scales, "zeros": zeros, "packed": packed,
                    "tokens": s.tokens, "rows": s.rows}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


CASES = [
    # m, d, n, bits, group, block, U from
    (37, 64, 1000, 4, 0, 32, "replicated"),      # ragged rows and tokens
    (40, 64, 640, 3, 32, 32, "broadcast"),
]


@pytest.mark.parametrize("case", CASES)
def test_sharded_layer_matches_single_process_oracle(case, tmp_path):
    import oracle
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), case, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    m, d, n, bits, gs, B, _ = case
    X, W = _inputs(m, d, n, seed=m + d + n)
    ref = oracle.gptq_layer(W.double().numpy(), X.double().numpy(), bits, gs, B, 0.01)
    shards = [torch.load(os.path.join(tmp_path, f"rank{r}.pt")) for r in range(world)]
    assert shards[0]["tokens"][1] == shards[1]["tokens"][0] and shards[1]["tokens"][1] == n
    assert shards[0]["tokens"][1] % 64 == 0
    for sh in shards:
        np.testing.assert_allclose(np.triu(sh["H"].numpy()), np.triu(ref["H"]), rtol=1e-12, atol=1e-9)
        np.testing.assert_allclose(sh["U"].numpy(), ref["U"], rtol=1e-9, atol=1e-12)
        np.testing.assert_array_equal(sh["codes"].numpy(), ref["codes"])
        np.testing.assert_array_equal(sh["scales"].numpy(), ref["scales"])
        np.testing.assert_array_equal(sh["zeros"].numpy(), ref["zeros"])
        np.testing.assert_array_equal(sh["packed"].numpy(), ref["packed"])
    # every rank holds the same U (replicated: computed from the same all-reduced H; broadcast: rank 0's)
    np.testing.assert_array_equal(shards[0]["U"].numpy(), shards[1]["U"].numpy())
