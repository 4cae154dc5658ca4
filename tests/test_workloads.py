"""The seeded synthetic layers: shapes, dtypes, determinism and the stated value distributions."""
import numpy as np
import torch

from post_weight_quantization_21_b200 import workloads as wl


def test_tiny_layer_shapes_and_determinism():
    L = wl.LAYERS["tiny_64x128"]
    W1, W2 = wl.make_w(L), wl.make_w(L)
    X1, X2 = wl.make_x(L), wl.make_x(L)
    assert W1.shape == (64, 128) and W1.dtype == torch.float32
    assert X1.shape == (256, 128) and X1.dtype == torch.float32
    assert torch.equal(W1, W2) and torch.equal(X1, X2)
    assert abs(W1.std().item() - 0.02) < 0.002


def test_chunks_regenerate_independently():
    L = wl.LAYERS["opt125m_768x768"].with_tokens(3 * wl.CHUNK_TOKENS)
    X = wl.make_x(L)
    c1 = wl.make_x_chunk(L, 1)
    assert torch.equal(X[wl.CHUNK_TOKENS:2 * wl.CHUNK_TOKENS], c1)


def test_opt125m_like_distribution():
    L = wl.LAYERS["opt125m_768x768"].with_tokens(2 * wl.CHUNK_TOKENS)
    X = wl.make_x(L).double().numpy()
    oc = wl.outlier_channels(L).numpy()
    assert len(oc) == 8
    std = X.std(axis=0)
    assert np.all(std[oc] > 10.0)
    normal = np.setdiff1d(np.arange(768), oc)
    normal = normal[(normal > 0) & ~np.isin(normal - 1, oc)]
    # AR(1) with rho = 0.5 and unit variance on the ordinary channels
    c = np.mean([np.corrcoef(X[:, j - 1], X[:, j])[0, 1] for j in normal[:50]])
    assert abs(c - 0.5) < 0.05
    W = wl.make_w(L)
    assert W.dtype == torch.float16
    assert (W.abs() > 0.1).float().mean().item() > 0.0005  # the x10 outlier entries


def test_relu_and_student_inputs():
    L = wl.LAYERS["llama7b_down_4096x11008"].with_tokens(256)
    x = wl.make_x_chunk(L, 0).float()
    assert x.shape == (256, 11008) and (x >= 0).all()
    assert abs((x == 0).float().mean().item() - 0.5) < 0.02
    L = wl.LAYERS["llama7b_q_4096x4096"].with_tokens(512)
    x = wl.make_x_chunk(L, 0).float()
    assert len(wl.outlier_channels(L)) == 41
