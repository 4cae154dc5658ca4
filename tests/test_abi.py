"""The C-ABI library: it loads, exports every entry point include/gptq.h declares, and its host-side
validation rejects bad arguments before any device work (no GPU needed for these calls)."""
import ctypes
import os
import re

import pytest

import post_weight_quantization_21_b200 as g
from post_weight_quantization_21_b200 import build as gbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "gptq.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(g.LIB_PATH):
        gbuild.build()
    return g.lib()


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"GPTQ_API\s+[\w\s\*]+?\b(gptq_\w+)\s*\(", src)


def test_header_declares_the_four_calls():
    names = set(declared_functions())
    for n in ("gptq_hessian_accumulate", "gptq_prepare_uinv", "gptq_quantize_layer", "gptq_pack"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(g.ABI_FUNCTIONS)
    assert lib.gptq_abi_version() == 2


def test_status_strings(lib):
    assert g.gptq_status_string(0) == "ok"
    assert "positive definite" in g.gptq_status_string(3)


def test_workspace_sizes(lib):
    import torch
    assert g.gptq_hessian_workspace_size(262144, 768, torch.bfloat16) > 0
    assert g.gptq_prepare_workspace_size(4096) >= 4096 * 32 * 4
    w = g.gptq_quantize_workspace_size(64, 128, 4, 0, 32)
    assert w >= 64 * 128 * 4 + 64 * 32 * 4
    assert g.gptq_quantize_workspace_size(64, 128, 5, 0, 32) == 0       # bits out of range
    assert g.gptq_quantize_workspace_size(64, 100, 4, 0, 32) == 0       # block does not divide d
    assert lib.gptq_prepare_workspace_size(0) == 0


def other_ptr():
    return ctypes.c_void_p(8192)


def test_validation_rejects_bad_arguments_without_a_device(lib):
    cfg = g.QuantCfg(4, 0, 128, 0)
    fake = ctypes.c_void_p(256)  # never dereferenced: validation fails first
    st = lib.gptq_quantize_layer(fake, 1, 8, 100, fake, ctypes.byref(cfg), fake, fake, fake, fake, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG                               # d % 32 != 0
    bad = g.QuantCfg(5, 0, 128, 0)
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(bad), fake, fake, fake, fake, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG                               # bits = 5
    act = g.QuantCfg(4, 0, 128, g.GPTQ_FLAG_ACT_ORDER)
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(act), fake, fake, fake, fake, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG                               # act-order needs the permutation argument
    assert lib.gptq_quantize_act_order_workspace_size(8, 128, ctypes.byref(act)) > \
        lib.gptq_quantize_workspace_size(8, 128, ctypes.byref(cfg))
    st = lib.gptq_quantize_layer_act_order(fake, 1, 8, 128, fake, None, ctypes.byref(act), fake, fake, fake, fake,
                                           fake, 1 << 24, None)
    assert st == g.GPTQ_ERR_ARG                               # no permutation
    st = lib.gptq_quantize_layer_act_order(fake, 1, 8, 128, fake, fake, ctypes.byref(act), fake, fake, fake, fake,
                                           fake, 16, None)
    assert st == g.GPTQ_ERR_WORKSPACE
    odd = ctypes.c_void_p(257)
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(cfg), odd, fake, fake, fake, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG                               # codes not 4-byte aligned
    assert lib.gptq_act_order(fake, 16, fake, fake, fake, None) == g.GPTQ_ERR_ARG      # H_perm aliases H
    assert lib.gptq_act_order(fake, 0, fake, other_ptr(), fake, None) == g.GPTQ_ERR_ARG
    grp = g.QuantCfg(4, 96, 128, 0)                           # 96 and 128 do not divide one another
    st = lib.gptq_quantize_layer(fake, 1, 8, 384, fake, ctypes.byref(grp), fake, fake, fake, fake, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG
    unknown = g.QuantCfg(4, 0, 128, 4)                        # no such flag bit
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(unknown), fake, fake, fake, fake, fake, 1 << 20,
                                 None)
    assert st == g.GPTQ_ERR_ARG
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(cfg), fake, fake, fake, None, fake, 1 << 20, None)
    assert st == g.GPTQ_ERR_ARG                               # no status word
    fma = g.QuantCfg(4, 0, 128, g.GPTQ_FLAG_FP32_FMA)
    assert lib.gptq_quantize_workspace_size(8, 128, ctypes.byref(fma)) > 0
    st = lib.gptq_quantize_layer(fake, 1, 8, 128, fake, ctypes.byref(cfg), fake, fake, fake, fake, None, 0, None)
    assert st == g.GPTQ_ERR_WORKSPACE
    assert lib.gptq_pack(fake, 4, 48, 3, fake, None) == g.GPTQ_ERR_ARG        # d % 32
    assert lib.gptq_pack(fake, 4, 64, 5, fake, None) == g.GPTQ_ERR_ARG        # bits
    # orders past the documented maximum are refused, not launched
    assert lib.gptq_pack(fake, 4, (1 << 20) + 32, 4, fake, None) == g.GPTQ_ERR_ARG
    assert lib.gptq_hessian_accumulate(fake, 0, 16, 12, fake, 2.0, 0, fake, fake, 1 << 20, None) == g.GPTQ_ERR_ARG
    assert lib.gptq_hessian_accumulate(fake, 7, 16, 16, fake, 2.0, 0, fake, fake, 1 << 20, None) == g.GPTQ_ERR_ARG
    other = ctypes.c_void_p(4096)
    assert lib.gptq_prepare_uinv(fake, 16, 0.01, other, fake, None, 0, None) == g.GPTQ_ERR_WORKSPACE
    assert lib.gptq_prepare_uinv(fake, 16, -1.0, other, fake, fake, 1 << 20, None) == g.GPTQ_ERR_ARG
    assert lib.gptq_prepare_uinv(fake, 16, 0.01, fake, fake, fake, 1 << 20, None) == g.GPTQ_ERR_ARG  # H == U


def test_tensor_core_phase_mask_without_a_device():
    import torch
    assert g.gptq_tensor_core_phases(768, 768, 262144, torch.bfloat16, 4) == g.GPTQ_TC_HESSIAN
    all3 = g.GPTQ_TC_HESSIAN | g.GPTQ_TC_PREPARE | g.GPTQ_TC_LAZY
    assert g.gptq_tensor_core_phases(4096, 4096, 262144, torch.bfloat16, 3, 128) == all3
    assert g.gptq_tensor_core_phases(4096, 4096, 262144, torch.bfloat16, 3, 128,
                                     flags=g.GPTQ_FLAG_FP32_FMA) == g.GPTQ_TC_HESSIAN | g.GPTQ_TC_PREPARE
    assert g.gptq_tensor_core_phases(64, 4224, 256, torch.float32, 4) == g.GPTQ_TC_PREPARE | g.GPTQ_TC_LAZY
    assert g.gptq_tensor_core_phases(64, 100, 256, torch.float32, 4) == -1   # block does not divide d


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """No fallback: without libgptq.so every call raises instead of computing anything elsewhere."""
    monkeypatch.setattr(g, "LIB_PATH", str(tmp_path / "libgptq.so"))
    monkeypatch.setattr(g, "_lib", None)
    with pytest.raises(ImportError):
        g.lib()
    with pytest.raises(ImportError):
        g.gptq_prepare_workspace_size(128)
