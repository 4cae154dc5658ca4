"""The synthetic Transformer block of the sequential pipeline, in fp64: the oracle of its forward pass.

TEST INFRASTRUCTURE ONLY (like the rest of ``oracle/``).  GPTQ quantizes one Transformer block at a
time, each block's calibration inputs being the previous (quantized) block's outputs (FDE Interviews
breakdown of GPTQ, figure "THE IDEA, VISUALLY"; section 01).  The pages do not print a block; the
reading used is an OPT-style pre-LayerNorm decoder block (OPT is the pages' model family):
    a = LN1(x);  h = x + (attn(a Wq^T + bq, a Wk^T + bk, a Wv^T + bv)) Wo^T + bo
    f = LN2(h);  y = h + relu(f W1^T + b1) W2^T + b2
with causal softmax attention over each sequence of ``seq_len`` tokens, ``n_heads`` heads, scale
1/sqrt(head_dim), LayerNorm eps 1e-5.  Written out with plain NumPy (fp64) operations.
"""
from __future__ import annotations

import numpy as np


def layer_norm(x, gain, shift, eps: float = 1e-5):
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gain + shift


def causal_attention(q, k, v, n_heads: int, seq_len: int):
    """Per sequence and head: softmax(q k^T / sqrt(dh) + causal mask) v."""
    n, d = q.shape
    dh = d // n_heads
    out = np.zeros((n, d))
    mask = np.triu(np.full((seq_len, seq_len), -np.inf), k=1)
    for s0 in range(0, n, seq_len):
        for h in range(n_heads):
            cols = slice(h * dh, (h + 1) * dh)
            Q, K, V = q[s0:s0 + seq_len, cols], k[s0:s0 + seq_len, cols], v[s0:s0 + seq_len, cols]
            logits = Q @ K.T / np.sqrt(dh) + mask
            logits -= logits.max(axis=1, keepdims=True)
            w = np.exp(logits)
            w /= w.sum(axis=1, keepdims=True)
            out[s0:s0 + seq_len, cols] = w @ V
    return out


def block_forward(p: dict, x, n_heads: int, seq_len: int, weights: dict | None = None, collect: dict | None = None):
    """y = block(x) in fp64.  ``p`` holds the weights (q, k, v, out, fc1, fc2: [out, in]) and the biases
    and LayerNorm parameters; ``weights`` overrides the linear weights; ``collect`` receives the input of
    every linear group (attn_in, out_in, fc1_in, fc2_in)."""
    f64 = {k: np.asarray(v, dtype=np.float64) for k, v in p.items()}
    W = {n: np.asarray((weights or {}).get(n, f64[n]), dtype=np.float64) for n in ("q", "k", "v", "out", "fc1", "fc2")}
    x = np.asarray(x, dtype=np.float64)
    a = layer_norm(x, f64["ln1_g"], f64["ln1_b"])
    q = a @ W["q"].T + f64["q_b"]
    k = a @ W["k"].T + f64["k_b"]
    v = a @ W["v"].T + f64["v_b"]
    o_in = causal_attention(q, k, v, n_heads, seq_len)
    h = x + o_in @ W["out"].T + f64["out_b"]
    f = layer_norm(h, f64["ln2_g"], f64["ln2_b"])
    r = np.maximum(f @ W["fc1"].T + f64["fc1_b"], 0.0)
    if collect is not None:
        collect.update(attn_in=a, out_in=o_in, fc1_in=f, fc2_in=r)
    return h + r @ W["fc2"].T + f64["fc2_b"]
