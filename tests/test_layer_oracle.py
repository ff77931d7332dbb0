"""Pins of the layer oracle (oracle/layer_oracle.py), which the multi-layer GPU tests
compare the projection kernels and the whole attention block against:

* a two-token, hidden = 2, d = 1 block worked out by hand
  (tests/golden/layer_hand_example.json);
* with one host the block's attention is dense causal attention: the block equals the
  same block written with a textbook masked softmax (a second formulation);
* W_o = 0 leaves x unchanged exactly; scaling x by c > 0 leaves q, k, v unchanged
  (RMSNorm with eps = 0); the stack applies blocks in order;
* a planted mistake (a norm over the wrong axis, a transposed W_qkv, a dropped
  residual) fails one of these pins.
"""

import json
import math
import os

import numpy as np
import pytest

from oracle import layer_oracle as lo

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "layer_hand_example.json")


def _hand():
    ex = json.load(open(GOLDEN))
    x = np.array(ex["x"], dtype=np.float64)
    w_qkv = np.array(ex["w_qkv"], dtype=np.float64)
    w_o = np.array(ex["w_o"], dtype=np.float64)
    return ex, x, w_qkv, w_o


def _hand_expected():
    r2 = math.sqrt(2.0)
    v0 = 7 * r2 / 5
    a, b = math.exp(4 * r2 / 5), math.exp(-1.0)
    o1 = a * v0 / (a + b)
    x1 = np.array([[3 + v0, 4 + 2 * v0], [1 + o1, -1 + 2 * o1]])
    lse = np.array([[24 / 25, math.log(a + b)]])
    return x1, lse


def test_hand_example():
    ex, x, w_qkv, w_o = _hand()
    r = lo.attention_block(x, w_qkv, w_o, 1, 1, 1, [2], 0, 0, 1, eps=ex["eps"], scale=1.0)
    want_x, want_lse = _hand_expected()
    np.testing.assert_allclose(r["x"], want_x, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], want_lse, rtol=0, atol=1e-12)


def test_hand_example_catches_planted_mistakes():
    ex, x, w_qkv, w_o = _hand()
    want_x, _ = _hand_expected()
    # norm over the wrong axis
    h = x / np.sqrt(np.mean(x * x, axis=0, keepdims=True))
    assert not np.allclose(h @ w_qkv.T, lo.rms_norm(x, 0.0) @ w_qkv.T)
    # transposed weights (w_qkv used as [in, out]) cannot even be applied to hidden = 2 ... 3
    with pytest.raises(ValueError):
        lo.attention_block(x, w_qkv.T, w_o, 1, 1, 1, [2], 0, 0, 1, eps=0.0, scale=1.0)
    # dropped residual
    r = lo.attention_block(x, w_qkv, w_o, 1, 1, 1, [2], 0, 0, 1, eps=0.0, scale=1.0)
    assert not np.allclose(r["x"] - x, want_x)


def _random_block(rng, T=40, hidden=16, hq=4, hkv=2, d=4):
    x = rng.standard_normal((T, hidden))
    w_qkv = rng.standard_normal(((hq + 2 * hkv) * d, hidden)) / math.sqrt(hidden)
    w_o = rng.standard_normal((hidden, hq * d)) / math.sqrt(hq * d)
    return x, w_qkv, w_o


def _dense_causal_textbook(q, k, v, scale):
    """softmax(q k^T * scale + causal mask) v, one head at a time."""
    T, hq, d = q.shape
    G = hq // k.shape[1]
    O = np.empty_like(q)
    for c in range(hq):
        s = q[:, c, :] @ k[:, c // G, :].T * scale
        s = np.where(np.tril(np.ones((T, T), dtype=bool)), s, -np.inf)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        O[:, c, :] = (p / p.sum(axis=1, keepdims=True)) @ v[:, c // G, :]
    return O


def test_one_host_block_is_dense_causal():
    rng = np.random.default_rng(11)
    hq, hkv, d = 4, 2, 4
    x, w_qkv, w_o = _random_block(rng, hq=hq, hkv=hkv, d=d)
    T = x.shape[0]
    r = lo.attention_block(x, w_qkv, w_o, hq, hkv, d, [T], 0, 0, 4, eps=1e-6)
    h = x / np.sqrt((x ** 2).mean(axis=1, keepdims=True) + 1e-6)
    q = (h @ w_qkv[:hq * d].T).reshape(T, hq, d)
    k = (h @ w_qkv[hq * d:(hq + hkv) * d].T).reshape(T, hkv, d)
    v = (h @ w_qkv[(hq + hkv) * d:].T).reshape(T, hkv, d)
    O = _dense_causal_textbook(q, k, v, 1 / math.sqrt(d))
    np.testing.assert_allclose(r["x"], x + O.reshape(T, -1) @ w_o.T, rtol=1e-12, atol=1e-12)


def test_zero_output_projection_and_scale_invariance():
    rng = np.random.default_rng(12)
    x, w_qkv, w_o = _random_block(rng)
    sizes = [16, 24]
    r0 = lo.attention_block(x, w_qkv, np.zeros_like(w_o), 4, 2, 4, sizes, 4, 4, 4, eps=0.0)
    np.testing.assert_array_equal(r0["x"], x)
    r1 = lo.attention_block(x, w_qkv, w_o, 4, 2, 4, sizes, 4, 4, 4, eps=0.0)
    r2 = lo.attention_block(3.5 * x, w_qkv, w_o, 4, 2, 4, sizes, 4, 4, 4, eps=0.0)
    for name in ("q", "k", "v", "O"):
        np.testing.assert_allclose(r2[name], r1[name], rtol=1e-12, atol=1e-12)


def test_stack_applies_blocks_in_order():
    rng = np.random.default_rng(13)
    x, w_qkv, w_o = _random_block(rng)
    _, w_qkv2, w_o2 = _random_block(rng)
    sizes = [16, 24]
    layers = [{"w_qkv": w_qkv, "w_o": w_o}, {"w_qkv": w_qkv2, "w_o": w_o2}]
    out = lo.attention_stack(x, layers, 4, 2, 4, sizes, 4, 4, 4)
    a = lo.attention_block(x, w_qkv, w_o, 4, 2, 4, sizes, 4, 4, 4)
    b = lo.attention_block(a["x"], w_qkv2, w_o2, 4, 2, 4, sizes, 4, 4, 4)
    np.testing.assert_array_equal(out[1]["x"], b["x"])
    # with the selection given back, the same result
    again = lo.attention_stack(x, layers, 4, 2, 4, sizes, 4, 4, 4, sels=[o["sel"] for o in out])
    np.testing.assert_array_equal(again[1]["x"], out[1]["x"])
