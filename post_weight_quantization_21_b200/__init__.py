"""GPTQ layer-wise quantization solver for NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libgptq.so`` (C ABI in ``include/gptq.h``).  The functions keep the C
names and only marshal arguments: torch tensors supply device memory and streams, and every step of
the solver runs in the library's CUDA kernels.  There is no CPU fallback; if the library is missing,
the first call raises.

    H = 2 X^T X                       gptq_hessian_accumulate
    U = chol((H + l*mean(diag H) I)^-1) gptq_prepare_uinv
    codes, scales, zeros              gptq_quantize_layer   (column loop + lazy block updates)
    packed int32 words                gptq_pack
    act-order (desc_act)              gptq_act_order + gptq_quantize_layer_act_order

``LayerSolver`` strings the four calls together over preallocated buffers.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "GPTQError", "lib", "gptq_hessian_accumulate", "gptq_hessian_workspace_size", "gptq_prepare_uinv",
    "gptq_prepare_workspace_size", "gptq_prepare_uinv_static", "gptq_quantize_layer", "gptq_quantize_workspace_size", "gptq_pack",
    "gptq_read_status", "gptq_status_string", "gptq_kernel_launches", "gptq_tensor_core_phases", "LayerSolver", "LIB_PATH", "ABI_FUNCTIONS",
    "gptq_act_order", "gptq_quantize_layer_act_order", "gptq_quantize_act_order_workspace_size", "act_order_group_index",
    "gptq_dequant_matmul", "gptq_dequant_matmul_workspace_size", "gptq_dequantize",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq.so")

GPTQ_OK, GPTQ_ERR_ARG, GPTQ_ERR_UNSUPPORTED, GPTQ_ERR_NOT_PD = 0, 1, 2, 3
GPTQ_ERR_CUDA, GPTQ_ERR_TIMEOUT, GPTQ_ERR_WORKSPACE = 4, 5, 6
GPTQ_BF16, GPTQ_FP16, GPTQ_FP32 = 0, 1, 2
GPTQ_FLAG_ACT_ORDER = 1
GPTQ_FLAG_FP32_FMA = 2
GPTQ_TC_HESSIAN, GPTQ_TC_PREPARE, GPTQ_TC_LAZY = 1, 2, 4

_DTYPES = {torch.bfloat16: GPTQ_BF16, torch.float16: GPTQ_FP16, torch.float32: GPTQ_FP32}


class QuantCfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("flags", ctypes.c_uint32)]


_i32, _i64, _sz, _vp, _f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_float
ABI_FUNCTIONS = {
    "gptq_hessian_accumulate": (_i32, [_vp, _i32, _i64, _i64, _vp, _f32, _i32, _vp, _vp, _sz, _vp]),
    "gptq_hessian_workspace_size": (_sz, [_i64, _i64, _i32]),
    "gptq_prepare_uinv": (_i32, [_vp, _i64, _f32, _vp, _vp, _vp, _sz, _vp]),
    "gptq_prepare_workspace_size": (_sz, [_i64]),
    "gptq_prepare_uinv_static": (_i32, [_vp, _i64, _f32, _vp, _vp, _vp]),
    "gptq_quantize_layer": (_i32, [_vp, _i32, _i64, _i64, _vp, ctypes.POINTER(QuantCfg), _vp, _vp, _vp,
                                   _vp, _vp, _sz, _vp]),
    "gptq_quantize_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(QuantCfg)]),
    "gptq_pack": (_i32, [_vp, _i64, _i64, _i32, _vp, _vp]),
    "gptq_act_order": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp]),
    "gptq_quantize_layer_act_order": (_i32, [_vp, _i32, _i64, _i64, _vp, _vp, ctypes.POINTER(QuantCfg), _vp, _vp,
                                             _vp, _vp, _vp, _sz, _vp]),
    "gptq_quantize_act_order_workspace_size": (_sz, [_i64, _i64, ctypes.POINTER(QuantCfg)]),
    "gptq_test_hessian_timeout": (None, [_i64]),
    "gptq_dequant_matmul": (_i32, [_vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp, _i32, _i64, _vp, _vp, _vp, _sz,
                                   _vp]),
    "gptq_dequant_matmul_workspace_size": (_sz, [_i64, _i64, _i64]),
    "gptq_dequantize": (_i32, [_vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp, _i32, _vp]),
    "gptq_read_status": (_i32, [_vp, _vp, ctypes.POINTER(_i64)]),
    "gptq_status_string": (ctypes.c_char_p, [_i32]),
    "gptq_abi_version": (_i32, []),
    "gptq_kernel_launches": (ctypes.c_uint64, []),
    "gptq_tensor_core_phases": (_i32, [_i64, _i64, _i64, _i32, ctypes.POINTER(QuantCfg)]),
}

_lib = None


def lib():
    """The loaded library (loaded on first use; raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m post_weight_quantization_21_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in ABI_FUNCTIONS.items():
            fn = getattr(handle, name)
            fn.restype, fn.argtypes = res, args
        _lib = handle
    return _lib


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str, detail: int | None = None):
        self.status, self.detail = status, detail
        msg = f"{where}: {gptq_status_string(status)} (status {status})"
        if detail is not None:
            msg += f", detail {detail}"
        super().__init__(msg)


def gptq_status_string(status: int) -> str:
    return lib().gptq_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != GPTQ_OK:
        raise GPTQError(status, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cfg(bits: int, group_size: int, block_size: int, flags: int = 0) -> QuantCfg:
    return QuantCfg(bits, group_size, block_size, flags)


def _contig(t: torch.Tensor, name: str):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")


# ------------------------------------------------------------------------------------------ A1
def gptq_hessian_workspace_size(n_tokens: int, d: int, x_dtype: torch.dtype) -> int:
    return lib().gptq_hessian_workspace_size(n_tokens, d, _DTYPES[x_dtype])


def gptq_hessian_accumulate(X: torch.Tensor, H: torch.Tensor, status: torch.Tensor, workspace: torch.Tensor,
                            scale: float = 2.0, accumulate: bool = False, stream=None):
    """H (upper triangle) = [H +] scale * X^T X for X [tokens, d] on the device."""
    _contig(X, "X"), _contig(H, "H")
    n, d = X.shape
    st = lib().gptq_hessian_accumulate(_ptr(X), _DTYPES[X.dtype], n, d, _ptr(H), scale, int(accumulate),
                                       _ptr(status), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream))
    _check(st, "gptq_hessian_accumulate")


# ------------------------------------------------------------------------------------------ A2 + A3
def gptq_prepare_workspace_size(d: int) -> int:
    return lib().gptq_prepare_workspace_size(d)


def gptq_prepare_uinv(H: torch.Tensor, U: torch.Tensor, status: torch.Tensor, workspace: torch.Tensor,
                      damp: float = 0.01, stream=None):
    """U = upper Cholesky factor of (H + damp*mean(diag H)*I)^-1 (device status in ``status``)."""
    _contig(H, "H"), _contig(U, "U")
    st = lib().gptq_prepare_uinv(_ptr(H), H.shape[0], damp, _ptr(U), _ptr(status), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "gptq_prepare_uinv")


PREPARE_STATIC_MAX_D = 8192


def gptq_prepare_uinv_static(H: torch.Tensor, U: torch.Tensor, status: torch.Tensor, damp: float = 0.01,
                             stream=None):
    """gptq_prepare_uinv without a workspace, for callers that cannot allocate: the library's own
    fixed scratch array (d <= PREPARE_STATIC_MAX_D) is used.  Calls overlapping on the GPU race."""
    _contig(H, "H"), _contig(U, "U")
    st = lib().gptq_prepare_uinv_static(_ptr(H), H.shape[0], damp, _ptr(U), _ptr(status), _stream(stream))
    _check(st, "gptq_prepare_uinv_static")


# ------------------------------------------------------------------------------------------ A4 - A6
def gptq_quantize_workspace_size(m: int, d: int, bits: int, group_size: int, block_size: int) -> int:
    c = _cfg(bits, group_size, block_size)
    return lib().gptq_quantize_workspace_size(m, d, ctypes.byref(c))


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
                        zeros: torch.Tensor, status: torch.Tensor, workspace: torch.Tensor, bits: int,
                        group_size: int = 0, block_size: int = 128, flags: int = 0, stream=None):
    """Column loop with lazy block updates: fills codes [m, d] u8, scales/zeros [m, n_groups]."""
    for t, n in ((W, "W"), (U, "U"), (codes, "codes"), (scales, "scales"), (zeros, "zeros"), (status, "status")):
        _contig(t, n)
    m, d = W.shape
    c = _cfg(bits, group_size, block_size, flags)
    st = lib().gptq_quantize_layer(_ptr(W), _DTYPES[W.dtype], m, d, _ptr(U), ctypes.byref(c), _ptr(codes),
                                   _ptr(scales), _ptr(zeros), _ptr(status), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "gptq_quantize_layer")


# ------------------------------------------------------------------------------------------ act-order
def gptq_act_order(H: torch.Tensor, perm: torch.Tensor, H_perm: torch.Tensor, status: torch.Tensor, stream=None):
    """perm (int32 [d]) = columns by descending diag(H); H_perm (upper) = P H P^T."""
    for t, n in ((H, "H"), (perm, "perm"), (H_perm, "H_perm"), (status, "status")):
        _contig(t, n)
    _check(lib().gptq_act_order(_ptr(H), H.shape[0], _ptr(perm), _ptr(H_perm), _ptr(status), _stream(stream)),
           "gptq_act_order")


def gptq_quantize_act_order_workspace_size(m: int, d: int, bits: int, group_size: int, block_size: int) -> int:
    c = _cfg(bits, group_size, block_size, GPTQ_FLAG_ACT_ORDER)
    return lib().gptq_quantize_act_order_workspace_size(m, d, ctypes.byref(c))


def gptq_quantize_layer_act_order(W: torch.Tensor, U_perm: torch.Tensor, perm: torch.Tensor, codes: torch.Tensor,
                                  scales: torch.Tensor, zeros: torch.Tensor, status: torch.Tensor,
                                  workspace: torch.Tensor, bits: int, group_size: int = 0, block_size: int = 128,
                                  flags: int = 0, stream=None):
    """The column loop in the order ``perm`` (W in its original column order, U of the permuted Hessian);
    codes come back in the original column order, grids per group of the quantization order."""
    for t, n in ((W, "W"), (U_perm, "U_perm"), (perm, "perm"), (codes, "codes"), (scales, "scales"),
                 (zeros, "zeros"), (status, "status")):
        _contig(t, n)
    m, d = W.shape
    c = _cfg(bits, group_size, block_size, flags | GPTQ_FLAG_ACT_ORDER)
    st = lib().gptq_quantize_layer_act_order(_ptr(W), _DTYPES[W.dtype], m, d, _ptr(U_perm), _ptr(perm),
                                             ctypes.byref(c), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(status),
                                             _ptr(workspace), workspace.numel() * workspace.element_size(),
                                             _stream(stream))
    _check(st, "gptq_quantize_layer_act_order")


def act_order_group_index(perm: torch.Tensor, group_size: int) -> torch.Tensor:
    """Group of every original column under act-order: its step in ``perm`` // group_size (index
    bookkeeping for dequantization; no arithmetic of the method)."""
    step = torch.empty_like(perm)
    step[perm.long()] = torch.arange(perm.numel(), dtype=perm.dtype, device=perm.device)
    return step // group_size if group_size else torch.zeros_like(step)


# ------------------------------------------------------------------------------------------ A7
def gptq_pack(codes: torch.Tensor, bits: int, packed: torch.Tensor, stream=None):
    _contig(codes, "codes"), _contig(packed, "packed")
    m, d = codes.shape
    _check(lib().gptq_pack(_ptr(codes), m, d, bits, _ptr(packed), _stream(stream)), "gptq_pack")


# ------------------------------------------------------------------------------------------ inference
def gptq_dequant_matmul_workspace_size(m: int, d: int, batch: int) -> int:
    return lib().gptq_dequant_matmul_workspace_size(m, d, batch)


def gptq_dequant_matmul(packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bits: int, group_size: int,
                        X: torch.Tensor, Y: torch.Tensor, status: torch.Tensor, workspace: torch.Tensor, stream=None):
    """Y [batch, m] (fp32) = X [batch, d] @ What^T, What dequantized on the fly from the packed codes."""
    for t, n in ((packed, "packed"), (scales, "scales"), (zeros, "zeros"), (X, "X"), (Y, "Y"), (status, "status")):
        _contig(t, n)
    m = packed.shape[0]
    batch, d = X.shape
    st = lib().gptq_dequant_matmul(_ptr(packed), _ptr(scales), _ptr(zeros), m, d, bits, group_size, _ptr(X),
                                   _DTYPES[X.dtype], batch, _ptr(Y), _ptr(status), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "gptq_dequant_matmul")


def gptq_dequantize(packed: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, bits: int, group_size: int,
                    W_hat: torch.Tensor, stream=None):
    """W_hat [m, d] (fp16 / bf16 / fp32) = the dequantized weights of the packed codes."""
    for t, n in ((packed, "packed"), (scales, "scales"), (zeros, "zeros"), (W_hat, "W_hat")):
        _contig(t, n)
    m, d = W_hat.shape
    _check(lib().gptq_dequantize(_ptr(packed), _ptr(scales), _ptr(zeros), m, d, bits, group_size, _ptr(W_hat),
                                 _DTYPES[W_hat.dtype], _stream(stream)), "gptq_dequantize")


def gptq_tensor_core_phases(m: int, d: int, n_tokens: int, x_dtype, bits: int, group_size: int = 0,
                            block_size: int = 128, flags: int = 0) -> int:
    """Bit mask of the phases whose block products run on the tensor cores (GPTQ_TC_*)."""
    c = _cfg(bits, group_size, block_size, flags)
    return int(lib().gptq_tensor_core_phases(m, d, n_tokens, _DTYPES[x_dtype], ctypes.byref(c)))


def gptq_kernel_launches() -> int:
    """Kernels launched by the library so far in this process (host-side counter)."""
    return int(lib().gptq_kernel_launches())


def gptq_read_status(status: torch.Tensor, stream=None) -> tuple[int, int]:
    detail = ctypes.c_int64(0)
    code = lib().gptq_read_status(_ptr(status), _stream(stream), ctypes.byref(detail))
    return int(code), int(detail.value)


# ------------------------------------------------------------------------------------------ solver
class LayerSolver:
    """Device buffers for one layer shape, and the four calls in order.

    ``run()`` works on the device-resident ``X``/``W`` buffers; ``run_host()`` copies pinned host
    inputs in, runs, and copies the packed codes, scales and zeros back out.
    """

    HOST_CHUNK_TOKENS = 16384  # tokens of X per host -> device copy in run_host (a multiple of 64)


    def __init__(self, m: int, d: int, n_tokens: int, bits: int, group_size: int = 0, block_size: int = 128,
                 damp: float = 0.01, x_dtype=torch.bfloat16, w_dtype=torch.float16, device="cuda", flags: int = 0,
                 act_order: bool = False):
        self.m, self.d, self.n_tokens, self.flags = m, d, n_tokens, flags
        self.act_order = act_order
        self.bits, self.group_size, self.block_size, self.damp = bits, group_size, block_size, damp
        n_groups = 1 if group_size == 0 else d // group_size
        dev = torch.device(device)
        u8 = torch.uint8
        self.X = torch.empty(n_tokens, d, dtype=x_dtype, device=dev)
        self.W = torch.empty(m, d, dtype=w_dtype, device=dev)
        self.H = torch.empty(d, d, dtype=torch.float32, device=dev)
        self.U = torch.empty(d, d, dtype=torch.float32, device=dev)
        self.codes = torch.empty(m, d, dtype=u8, device=dev)
        self.scales = torch.empty(m, n_groups, dtype=torch.float32, device=dev)
        self.zeros = torch.empty(m, n_groups, dtype=torch.int32, device=dev)
        self.packed = torch.empty(m, d * bits // 32, dtype=torch.int32, device=dev)
        # one device status word per call (prepare and quantize clear theirs when they start)
        # rows: hessian, prepare, quantize, act-order permutation
        self.status = torch.zeros(4, 2, dtype=torch.int32, device=dev)
        self.host_chunk = min(n_tokens, self.HOST_CHUNK_TOKENS)
        q_ws = (gptq_quantize_act_order_workspace_size(m, d, bits, group_size, block_size) if act_order
                else gptq_quantize_workspace_size(m, d, bits, group_size, block_size))
        if act_order:
            self.perm = torch.empty(d, dtype=torch.int32, device=dev)
            self.H_perm = torch.empty(d, d, dtype=torch.float32, device=dev)
        ws = max(gptq_hessian_workspace_size(n_tokens, d, x_dtype),
                 gptq_hessian_workspace_size(self.host_chunk, d, x_dtype) if self.host_chunk else 0,
                 gptq_prepare_workspace_size(d), q_ws, 256)
        self.workspace = torch.empty(ws, dtype=u8, device=dev)
        self._copy_stream = None

    def hessian(self, stream=None):
        gptq_hessian_accumulate(self.X, self.H, self.status[0], self.workspace, 2.0, False, stream)

    def prepare(self, stream=None):
        """U of the dampened Hessian; with act-order, the permutation first and U of P H P^T."""
        if self.act_order:
            gptq_act_order(self.H, self.perm, self.H_perm, self.status[3], stream)
            gptq_prepare_uinv(self.H_perm, self.U, self.status[1], self.workspace, self.damp, stream)
        else:
            gptq_prepare_uinv(self.H, self.U, self.status[1], self.workspace, self.damp, stream)

    def quantize(self, stream=None):
        if self.act_order:
            gptq_quantize_layer_act_order(self.W, self.U, self.perm, self.codes, self.scales, self.zeros,
                                          self.status[2], self.workspace, self.bits, self.group_size,
                                          self.block_size, self.flags, stream)
        else:
            gptq_quantize_layer(self.W, self.U, self.codes, self.scales, self.zeros, self.status[2], self.workspace,
                                self.bits, self.group_size, self.block_size, self.flags, stream)

    def pack(self, stream=None):
        gptq_pack(self.codes, self.bits, self.packed, stream)

    def run(self, stream=None):
        self.hessian(stream)
        self.prepare(stream)
        self.quantize(stream)
        self.pack(stream)

    def check_status(self, stream=None):
        """Raises GPTQError with the first failure any of the calls recorded on the device."""
        for word in self.status:
            code, detail = gptq_read_status(word, stream)
            if code != GPTQ_OK:
                raise GPTQError(code, "device status", detail)

    def run_host(self, W_host: torch.Tensor, X_host: torch.Tensor, out_packed: torch.Tensor,
                 out_scales: torch.Tensor, out_zeros: torch.Tensor, stream=None):
        """Host -> device copies of W and X, the four calls, device -> host copies of the results.

        X crosses in chunks of HOST_CHUNK_TOKENS tokens on a copy stream, and the Hessian of each chunk
        accumulates (gptq_hessian_accumulate with accumulate = 1) as soon as the chunk has landed, so
        the copy of chunk c + 1 overlaps the product of chunk c.  W crosses first.  Inputs should be
        pinned for the copies to be asynchronous.
        """
        s = stream if stream is not None else torch.cuda.current_stream(self.X.device)
        if self._copy_stream is None:
            self._copy_stream = torch.cuda.Stream(device=self.X.device)
        copy = self._copy_stream
        copy.wait_stream(s)  # the device buffers are free once the caller's earlier work is done
        step = max(self.host_chunk, 1)
        landed = []
        with torch.cuda.stream(copy):
            self.W.copy_(W_host, non_blocking=True)
            for t0 in range(0, self.n_tokens, step):
                self.X[t0:t0 + step].copy_(X_host[t0:t0 + step], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy)
                landed.append(ev)
        if not landed:  # no tokens: H = 0
            s.wait_stream(copy)
            gptq_hessian_accumulate(self.X, self.H, self.status[0], self.workspace, 2.0, False, s)
        for c, t0 in enumerate(range(0, self.n_tokens, step)):
            s.wait_event(landed[c])
            gptq_hessian_accumulate(self.X[t0:t0 + step], self.H, self.status[0], self.workspace, 2.0, c > 0, s)
        self.prepare(s)
        self.quantize(s)
        self.pack(s)
        with torch.cuda.stream(s):
            out_packed.copy_(self.packed, non_blocking=True)
            out_scales.copy_(self.scales, non_blocking=True)
            out_zeros.copy_(self.zeros, non_blocking=True)
