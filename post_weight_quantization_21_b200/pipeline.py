"""Sequential quantization of a Transformer block: the step before the layer solve.

GPTQ quantizes a model one Transformer block at a time on the calibration set (FDE Interviews
breakdown of GPTQ, figure "THE IDEA, VISUALLY": 128 sequences of 2,048 tokens, one block at a time;
section 01: each layer is solved on its own inputs).  For one block:

  1. run the block with its original weights on the block's calibration inputs and, as the activations
     stream past, accumulate the Hessian of every linear layer's input with gptq_hessian_accumulate
     (q, k and v share their input, so they share one Hessian);
  2. solve every linear layer with gptq_prepare_uinv / gptq_quantize_layer / gptq_pack;
  3. run the block again with the dequantized weights (gptq_dequantize): its outputs are the next
     block's calibration inputs.

The block is an OPT-style pre-LayerNorm decoder block (the pages' models are OPT, BLOOM and LLaMA; the
pages do not fix a block, so the plainest one is used): h = x + Wo attn(LN1(x)), y = h + W2 relu(W1
LN2(h)), causal multi-head attention over each sequence, biases on every linear layer.  The weights are
synthetic (seeded); no trained weights are involved.  The block's forward pass is plumbing in torch
(fp32); every step of the GPTQ solve runs in the library's kernels.
"""
from __future__ import annotations

import dataclasses
import math

import torch

import post_weight_quantization_21_b200 as g

LINEARS = ("q", "k", "v", "out", "fc1", "fc2")
# the linear layers that read each collected input (q, k and v read the same one)
INPUTS = {"attn_in": ("q", "k", "v"), "out_in": ("out",), "fc1_in": ("fc1",), "fc2_in": ("fc2",)}


@dataclasses.dataclass(frozen=True)
class BlockConfig:
    d_model: int
    n_heads: int
    d_ffn: int
    seq_len: int
    bits: int = 4
    group_size: int = 0
    block_size: int = 128
    damp: float = 0.01

    def shape(self, name: str) -> tuple[int, int]:
        """[out_features, in_features] of a linear layer."""
        d, f = self.d_model, self.d_ffn
        return {"q": (d, d), "k": (d, d), "v": (d, d), "out": (d, d), "fc1": (f, d), "fc2": (d, f)}[name]


def make_block(cfg: BlockConfig, seed: int, device="cpu") -> dict[str, torch.Tensor]:
    """Seeded synthetic weights: fp16 W ~ N(0, 1/in_features), fp32 biases ~ N(0, 0.02^2), LayerNorm
    gains 1 + N(0, 0.05^2) and shifts N(0, 0.02^2)."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    p = {}
    for name in LINEARS:
        o, i = cfg.shape(name)
        p[name] = (torch.randn(o, i, generator=gen) / math.sqrt(i)).half().to(device)
        p[name + "_b"] = (torch.randn(o, generator=gen) * 0.02).to(device)
    for ln in ("ln1", "ln2"):
        p[ln + "_g"] = (1.0 + 0.05 * torch.randn(cfg.d_model, generator=gen)).to(device)
        p[ln + "_b"] = (0.02 * torch.randn(cfg.d_model, generator=gen)).to(device)
    return p


def block_forward(cfg: BlockConfig, p: dict[str, torch.Tensor], x: torch.Tensor, collect=None,
                  weights: dict[str, torch.Tensor] | None = None) -> torch.Tensor:
    """y = block(x) for x [n_seq * seq_len, d] (fp32 math).  ``collect(name, act)`` is called with the
    input of every linear group (INPUTS) as it is produced; ``weights`` overrides the linear weights
    (the dequantized ones)."""
    W = {n: (weights[n] if weights is not None else p[n]).float() for n in LINEARS}
    d, H = cfg.d_model, cfg.n_heads
    x = x.float()
    a_in = torch.nn.functional.layer_norm(x, (d,), p["ln1_g"], p["ln1_b"])
    if collect:
        collect("attn_in", a_in)
    q = a_in @ W["q"].t() + p["q_b"]
    k = a_in @ W["k"].t() + p["k_b"]
    v = a_in @ W["v"].t() + p["v_b"]
    S = cfg.seq_len
    n_seq = x.shape[0] // S

    def heads(t):
        return t.view(n_seq, S, H, d // H).transpose(1, 2)

    att = torch.nn.functional.scaled_dot_product_attention(heads(q), heads(k), heads(v), is_causal=True)
    o_in = att.transpose(1, 2).reshape(n_seq * S, d)
    if collect:
        collect("out_in", o_in)
    h = x + o_in @ W["out"].t() + p["out_b"]
    f_in = torch.nn.functional.layer_norm(h, (d,), p["ln2_g"], p["ln2_b"])
    if collect:
        collect("fc1_in", f_in)
    a = torch.relu(f_in @ W["fc1"].t() + p["fc1_b"])
    if collect:
        collect("fc2_in", a)
    return h + a @ W["fc2"].t() + p["fc2_b"]


@dataclasses.dataclass
class QuantizedLinear:
    codes: torch.Tensor     # [m, d] uint8
    scales: torch.Tensor    # [m, n_groups] fp32
    zeros: torch.Tensor     # [m, n_groups] int32
    packed: torch.Tensor    # [m, d*b/32] int32
    W_hat: torch.Tensor     # [m, d] fp16, the dequantized weights


class BlockQuantizer:
    """Quantizes blocks one after another on the GPU; see the module notes for the three steps.

    The calibration inputs stream through the block in chunks of ``chunk_seqs`` sequences; each
    chunk's activations are cast to bf16 (the calibration dtype) and added to the Hessians at once, so
    only one chunk of activations is alive at a time.  ``keep_inputs`` also keeps every collected
    input (tests use it to check the Hessians)."""

    def __init__(self, cfg: BlockConfig, device="cuda", chunk_seqs: int = 16, keep_inputs: bool = False):
        self.cfg, self.dev, self.chunk_seqs, self.keep_inputs = cfg, torch.device(device), chunk_seqs, keep_inputs
        self.inputs: dict[str, list[torch.Tensor]] = {}
        dims = {"attn_in": cfg.d_model, "out_in": cfg.d_model, "fc1_in": cfg.d_model, "fc2_in": cfg.d_ffn}
        self.H = {k: torch.empty(n, n, device=self.dev) for k, n in dims.items()}
        # one status word per call whose failure must survive the later calls: 4 Hessians, 4 prepare
        # steps, 6 layer solves
        self.status = torch.zeros(14, 2, dtype=torch.int32, device=self.dev)
        self._row = {**{k: i for i, k in enumerate(INPUTS)}, **{"U_" + k: 4 + i for i, k in enumerate(INPUTS)},
                     **{"Q_" + k: 8 + i for i, k in enumerate(LINEARS)}}
        chunk_tokens = chunk_seqs * cfg.seq_len
        ws = [256, max(g.gptq_prepare_workspace_size(n) for n in dims.values())]
        ws += [g.gptq_hessian_workspace_size(chunk_tokens, n, torch.bfloat16) for n in dims.values()]
        ws += [g.gptq_quantize_workspace_size(*cfg.shape(nm), cfg.bits, cfg.group_size, cfg.block_size)
               for nm in LINEARS]
        self.workspace = torch.empty(max(ws), dtype=torch.uint8, device=self.dev)
        self.timing: dict[str, float] = {}

    def _hessians(self, p, X):
        started = set()

        def collect(name, act):
            a16 = act.to(torch.bfloat16).contiguous()
            g.gptq_hessian_accumulate(a16, self.H[name], self.status[self._row[name]], self.workspace, 2.0,
                                      name in started)
            started.add(name)
            if self.keep_inputs:
                self.inputs.setdefault(name, []).append(a16)

        S = self.cfg.seq_len
        step = self.chunk_seqs * S
        for t0 in range(0, X.shape[0], step):
            block_forward(self.cfg, p, X[t0:t0 + step], collect)

    def quantize_block(self, p: dict[str, torch.Tensor], X: torch.Tensor):
        """(quantized layers by name, next block's inputs) for calibration inputs X [n_seq*seq_len, d]."""
        cfg = self.cfg
        self.inputs = {}
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record()
        self._hessians(p, X)
        ev[1].record()
        U = {}
        for name, Hm in self.H.items():
            n = Hm.shape[0]
            U[name] = torch.empty(n, n, device=self.dev)
            g.gptq_prepare_uinv(Hm, U[name], self.status[self._row["U_" + name]], self.workspace, cfg.damp)
        out = {}
        for name_in, layers in INPUTS.items():
            for nm in layers:
                m, d = cfg.shape(nm)
                ng = 1 if cfg.group_size == 0 else d // cfg.group_size
                q = QuantizedLinear(torch.empty(m, d, dtype=torch.uint8, device=self.dev),
                                    torch.empty(m, ng, device=self.dev),
                                    torch.empty(m, ng, dtype=torch.int32, device=self.dev),
                                    torch.empty(m, d * cfg.bits // 32, dtype=torch.int32, device=self.dev),
                                    torch.empty(m, d, dtype=torch.float16, device=self.dev))
                g.gptq_quantize_layer(p[nm], U[name_in], q.codes, q.scales, q.zeros, self.status[self._row["Q_" + nm]],
                                      self.workspace, cfg.bits, cfg.group_size, cfg.block_size)
                g.gptq_pack(q.codes, cfg.bits, q.packed)
                g.gptq_dequantize(q.packed, q.scales, q.zeros, cfg.bits, cfg.group_size, q.W_hat)
                out[nm] = q
        ev[2].record()
        S = cfg.seq_len
        step = self.chunk_seqs * S
        W_hat = {nm: out[nm].W_hat for nm in LINEARS}
        Y = torch.empty(X.shape[0], cfg.d_model, dtype=X.dtype, device=self.dev)
        for t0 in range(0, X.shape[0], step):
            Y[t0:t0 + step] = block_forward(cfg, p, X[t0:t0 + step], weights=W_hat).to(X.dtype)
        ev[3].record()
        torch.cuda.synchronize(self.dev)
        for word in self.status:
            code, detail = g.gptq_read_status(word)
            if code != g.GPTQ_OK:
                raise g.GPTQError(code, "block pipeline", detail)
        self.timing = {"forward_and_hessians_ms": ev[0].elapsed_time(ev[1]),
                       "solve_ms": ev[1].elapsed_time(ev[2]), "quantized_forward_ms": ev[2].elapsed_time(ev[3])}
        self.U = U
        return out, Y
