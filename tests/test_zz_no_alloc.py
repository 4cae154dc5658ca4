"""The allocation-free prepare entry point (gptq_prepare_uinv_static).

Callers that cannot allocate device memory (a plugin whose host application owns every buffer, a
path where no allocator may run) use this variant: its scratch is a fixed array inside the library.
The test calls it through the C ABI twice in a row and compares each result with the workspace
entry point's on the same input, on both prepare paths: the one-launch kernel (d <= 1024) and the
blocked path above it, with tensor-core tiles (d = 2048) and fp32 tiles (d = 1030, rows not 16-byte
aligned).  Each result is also held to the oracle's U.  It also checks that an order above the
array's limit is refused before any work is enqueued.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import post_weight_quantization_21_b200 as g

pytestmark = pytest.mark.gpu

U_REL = 1e-5  # the prepare tests' floor on the relative Frobenius error of U


def _spd_hessian(d, seed):
    gen = torch.Generator().manual_seed(seed)
    X = torch.randn(4 * d, d, generator=gen, dtype=torch.float64)
    X = X @ (torch.randn(d, d, generator=gen, dtype=torch.float64) / d ** 0.5)
    return 2.0 * X.T @ X


# 200, 768: one-launch kernel; 2048: blocked path, tensor-core tiles; 1030: blocked path, fp32 tiles
@pytest.mark.parametrize("d", [200, 768, 2048, 1030])
def test_static_prepare_matches_workspace_prepare(d):
    lib = g.lib()
    H64 = _spd_hessian(d, seed=d)
    H = H64.float().cuda()
    Hd = oracle.dampen(H.double().cpu().numpy(), 0.01)
    Uo = oracle.inverse_upper_cholesky(Hd)
    kappa = np.linalg.cond(Hd)
    o_tol = max(1e-5, 10 * kappa * 6e-8)  # the prepare parity tests' bound against the oracle
    stream = torch.cuda.current_stream().cuda_stream
    status = torch.zeros(4, dtype=torch.int32, device="cuda")
    ws = torch.empty(g.gptq_prepare_workspace_size(d), dtype=torch.uint8, device="cuda")
    U_ref = torch.empty_like(H)
    st = lib.gptq_prepare_uinv(H.data_ptr(), d, 0.01, U_ref.data_ptr(), status.data_ptr(), ws.data_ptr(),
                               ws.numel(), stream)
    assert st == g.GPTQ_OK
    assert g.gptq_read_status(status)[0] == g.GPTQ_OK
    ref = U_ref.double().cpu().numpy()
    for _ in range(2):  # two calls in a row share the library's scratch array
        U = torch.full_like(H, float("nan"))
        st = lib.gptq_prepare_uinv_static(H.data_ptr(), d, 0.01, U.data_ptr(), status.data_ptr(), stream)
        assert st == g.GPTQ_OK
        code, detail = g.gptq_read_status(status)
        assert code == g.GPTQ_OK, (code, detail)
        got = U.double().cpu().numpy()
        rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        # above d = 1024 the two entry points group the trailing updates differently (the workspace
        # entry point updates in two levels on CTA pairs), so they agree to fp32 rounding amplified
        # by the condition number: the prepare tests' bound
        assert rel <= (U_REL if d <= 1024 else o_tol), (rel, o_tol)
        assert np.all(np.tril(got, -1) == 0.0)
        rel_o = np.linalg.norm(got - Uo) / np.linalg.norm(Uo)
        assert rel_o <= o_tol, (rel_o, kappa)


def test_static_prepare_refuses_orders_above_its_scratch():
    lib = g.lib()
    fake = ctypes.c_void_p(4096)
    other = ctypes.c_void_p(1 << 20)
    d = g.PREPARE_STATIC_MAX_D + 1
    assert lib.gptq_prepare_uinv_static(fake, d, 0.01, other, fake, None) == g.GPTQ_ERR_WORKSPACE
