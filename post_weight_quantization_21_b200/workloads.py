"""Seeded synthetic layers for the GPTQ solver: weights W[out, in] and calibration inputs X[tokens, in].

This module holds no arithmetic of the GPTQ method itself. It only draws random numbers with the
shapes, dtypes and value distributions of the layers the solver is measured on, so that the CUDA
path and the fp64 oracle can be fed identical inputs.

The layer shapes follow the GPTQ paper's setting (IST Austria / ETH Zurich, ICLR 2023, as summarised
on the fdeinterviews.com breakdown, section 01 and the figure "THE IDEA, VISUALLY"): one linear
layer at a time, a calibration set of 128 sequences of 2,048 tokens (262,144 tokens). The C4
calibration text and the trained OPT / LLaMA weights are not available, so synthetic inputs of the
same shapes stand in for them:

* tiny_64x128           W fp32 [64,128] ~ N(0, 0.02^2); X fp32 [256,128] = Z A (correlated)
* opt125m_768x768       W fp16 ~ N(0, 0.02^2), 0.1% entries x10; X bf16, AR(1) rho=0.5, 1% channels x20
* llama7b_q_4096x4096   W fp16 ~ N(0, 0.015^2); X bf16 Student-t(5), 1% channels x20; 3-bit g128
* llama7b_up_11008x4096 W fp16 ~ N(0, 0.015^2); X bf16 N(0,1); 4-bit g128
* llama7b_down_4096x11008 W fp16 ~ N(0, 0.015^2); X bf16 ReLU(N(0,1)); 4-bit g128
* opt175b_fc2_12288x49152 W fp16 ~ N(0, 0.01^2), 0.1% x10; X bf16 ReLU(N(0,1)), 1% channels x20; 3-bit

X is drawn in chunks of 2,048 tokens; chunk c uses the seed ``seed * 1000003 + c`` so any token range
can be regenerated on its own.  Draws happen on the requested device ("cpu" or "cuda"); the two
devices give different (each deterministic) streams, so one test always uses one device for both
sides.
"""
from __future__ import annotations

import dataclasses
import math

import torch

CHUNK_TOKENS = 2048
CAL_TOKENS = 128 * 2048  # 128 sequences of 2,048 tokens


@dataclasses.dataclass(frozen=True)
class Layer:
    name: str
    m: int                 # out features (rows of W)
    d: int                 # in features (columns of W, channels of X)
    n_tokens: int          # calibration tokens (rows of X)
    bits: int
    group_size: int        # 0 = one grid per row
    block_size: int
    seed: int
    w_dtype: torch.dtype
    x_dtype: torch.dtype
    w_std: float
    w_outlier_frac: float  # fraction of W entries multiplied by 10
    x_kind: str            # "za" | "ar1" | "student5" | "normal" | "relu"
    x_outlier_frac: float  # fraction of X channels multiplied by 20
    damp: float = 0.01

    @property
    def n_groups(self) -> int:
        return 1 if self.group_size == 0 else self.d // self.group_size

    def with_tokens(self, n_tokens: int) -> "Layer":
        return dataclasses.replace(self, n_tokens=n_tokens)


LAYERS = {
    "tiny_64x128": Layer("tiny_64x128", 64, 128, 256, 4, 0, 32, 0, torch.float32, torch.float32,
                         0.02, 0.0, "za", 0.0),
    "opt125m_768x768": Layer("opt125m_768x768", 768, 768, CAL_TOKENS, 4, 0, 128, 1,
                             torch.float16, torch.bfloat16, 0.02, 0.001, "ar1", 0.01),
    "llama7b_q_4096x4096": Layer("llama7b_q_4096x4096", 4096, 4096, CAL_TOKENS, 3, 128, 128, 2,
                                 torch.float16, torch.bfloat16, 0.015, 0.0, "student5", 0.01),
    "llama7b_up_11008x4096": Layer("llama7b_up_11008x4096", 11008, 4096, CAL_TOKENS, 4, 128, 128, 3,
                                   torch.float16, torch.bfloat16, 0.015, 0.0, "normal", 0.0),
    "llama7b_down_4096x11008": Layer("llama7b_down_4096x11008", 4096, 11008, CAL_TOKENS, 4, 128, 128,
                                     4, torch.float16, torch.bfloat16, 0.015, 0.0, "relu", 0.0),
    "opt175b_fc2_12288x49152": Layer("opt175b_fc2_12288x49152", 12288, 49152, CAL_TOKENS, 3, 0, 128,
                                     5, torch.float16, torch.bfloat16, 0.01, 0.001, "relu", 0.01),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _prefix_perm(n: int, k: int, seed: int) -> torch.Tensor:
    """First k entries of a seeded permutation of range(n) (drawn on the CPU)."""
    return torch.randperm(n, generator=_gen(seed, "cpu"))[:k]


def make_w(layer: Layer, device="cpu") -> torch.Tensor:
    """W [m, d] in the layer's weight dtype."""
    g = _gen(layer.seed, device)
    w = torch.randn(layer.m, layer.d, generator=g, device=device, dtype=torch.float32) * layer.w_std
    k = round(layer.w_outlier_frac * layer.m * layer.d)
    if k:
        idx = _prefix_perm(layer.m * layer.d, k, layer.seed * 7 + 1).to(device)
        w.view(-1)[idx] *= 10.0
    return w.to(layer.w_dtype)


def _za_mixing(layer: Layer) -> torch.Tensor:
    g = _gen(layer.seed * 7 + 2, "cpu")
    return torch.randn(layer.d, layer.d, generator=g, dtype=torch.float64) / math.sqrt(layer.d)


def outlier_channels(layer: Layer) -> torch.Tensor:
    k = round(layer.x_outlier_frac * layer.d)
    return _prefix_perm(layer.d, k, layer.seed * 7 + 3)


def make_x_chunk(layer: Layer, c: int, device="cpu") -> torch.Tensor:
    """Tokens [c*2048, (c+1)*2048) of X (fewer for a final partial chunk), in the layer's X dtype."""
    t0 = c * CHUNK_TOKENS
    n = min(CHUNK_TOKENS, layer.n_tokens - t0)
    if n <= 0:
        raise ValueError("chunk out of range")
    g = _gen(layer.seed * 1000003 + c, device)
    d = layer.d
    if layer.x_kind == "za":
        z = torch.randn(n, d, generator=g, device=device, dtype=torch.float64)
        x = z @ _za_mixing(layer).to(device)
    elif layer.x_kind == "ar1":
        e = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
        x = torch.empty_like(e)
        x[:, 0] = e[:, 0]
        s = math.sqrt(0.75)
        for ch in range(1, d):
            x[:, ch] = 0.5 * x[:, ch - 1] + s * e[:, ch]
    elif layer.x_kind == "student5":
        z = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
        chi = torch.zeros_like(z)
        for _ in range(5):
            chi += torch.randn(n, d, generator=g, device=device, dtype=torch.float32).square()
        x = z / torch.sqrt(chi / 5.0)
    elif layer.x_kind == "normal":
        x = torch.randn(n, d, generator=g, device=device, dtype=torch.float32)
    elif layer.x_kind == "relu":
        x = torch.randn(n, d, generator=g, device=device, dtype=torch.float32).clamp_min_(0.0)
    else:
        raise ValueError(layer.x_kind)
    oc = outlier_channels(layer)
    if oc.numel():
        x[:, oc.to(device)] *= 20.0
    return x.to(layer.x_dtype)


def make_upper(d: int, seed: int, device="cpu", rows_per_chunk: int = 1024) -> torch.Tensor:
    """A seeded upper-triangular fp32 matrix [d, d] with a positive diagonal, used as a stand-in U input.

    Diagonal ~ U(0.5, 1.5); entry (i, j > i) = U_ii * 0.5 * N(0, 1) / (1 + j - i), so each row's
    off-diagonal weights decay away from the diagonal the way a correlated layer's do.  Rows are drawn
    in chunks of ``rows_per_chunk``, chunk c from seed * 1000003 + c, on ``device``.
    """
    U = torch.empty(d, d, dtype=torch.float32, device=device)
    col = torch.arange(d, device=device, dtype=torch.float32)
    for c, r0 in enumerate(range(0, d, rows_per_chunk)):
        r1 = min(d, r0 + rows_per_chunk)
        g = _gen(seed * 1000003 + c, device)
        diag = torch.rand(r1 - r0, generator=g, device=device, dtype=torch.float32) + 0.5
        off = torch.randn(r1 - r0, d, generator=g, device=device, dtype=torch.float32)
        rows = torch.arange(r0, r1, device=device, dtype=torch.float32)[:, None]
        dist = col[None, :] - rows
        blk = diag[:, None] * 0.5 * off / (1.0 + dist.clamp_min(0.0))
        blk = torch.where(dist > 0, blk, torch.zeros((), device=device))
        blk[torch.arange(r1 - r0, device=device), torch.arange(r0, r1, device=device)] = diag
        U[r0:r1] = blk
    return U


def make_x(layer: Layer, device="cpu", out: torch.Tensor | None = None) -> torch.Tensor:
    """The whole X [n_tokens, d]; written into ``out`` when given (e.g. a preallocated device buffer)."""
    if out is None:
        out = torch.empty(layer.n_tokens, layer.d, dtype=layer.x_dtype, device=device)
    n_chunks = (layer.n_tokens + CHUNK_TOKENS - 1) // CHUNK_TOKENS
    for c in range(n_chunks):
        t0 = c * CHUNK_TOKENS
        chunk = make_x_chunk(layer, c, device)
        out[t0:t0 + chunk.shape[0]].copy_(chunk)
    return out
