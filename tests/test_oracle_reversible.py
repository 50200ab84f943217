"""Pins for the oracle's chunked feed-forward and reversible block (CPU only).

Sources: "Reformer: The Efficient Transformer" (research.elamur.ai summary
page), Key points, "Reversible layers" bullet (reversible residual layers
after Gomez et al. 2017; feed-forward layers processed in chunks with
unchanged results), and the reversible residual form y1 = x1 + F(x2),
y2 = x2 + G(y1) of the cited paper.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import lsh_oracle as orc
from oracle import rev_ff_oracle as rev

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    with open(os.path.join(GOLDEN, "ff_worked_example.json")) as f:
        return json.load(f)


def _arr(g, k):
    return np.asarray(g[k], dtype=np.float64)


def test_ff_worked_example_forward():
    g = _golden()
    y = rev.ff_forward(_arr(g, "x"), _arr(g, "W1"), _arr(g, "b1"), _arr(g, "W2"), _arr(g, "b2"))
    assert np.array_equal(y, _arr(g, "y"))


def test_ff_worked_example_backward():
    g = _golden()
    dx, dW1, db1, dW2, db2 = rev.ff_backward(_arr(g, "x"), _arr(g, "W1"), _arr(g, "b1"),
                                              _arr(g, "W2"), _arr(g, "b2"), _arr(g, "dy"))
    for got, k in ((dx, "dx"), (dW1, "dW1"), (db1, "db1"), (dW2, "dW2"), (db2, "db2")):
        assert np.array_equal(got, _arr(g, k)), k


def test_ff_relu_kink_has_zero_slope():
    """A pre-activation of exactly 0 passes no gradient (relu'(0) = 0)."""
    x = np.array([[1.0, 1.0]])
    W1 = np.array([[1.0], [-1.0]])          # pre = 0
    W2 = np.array([[3.0, -2.0]])
    dx, dW1, db1, dW2, db2 = rev.ff_backward(x, W1, np.zeros(1), W2, np.zeros(2), np.ones((1, 2)))
    assert np.all(dx == 0.0) and np.all(dW1 == 0.0) and np.all(db1 == 0.0)
    assert np.all(dW2 == 0.0) and np.array_equal(db2, np.ones(2))


def _ff_params(rng, d, dff, n):
    while True:
        x = rng.standard_normal((n, d))
        W1 = rng.standard_normal((d, dff)) / math.sqrt(d)
        b1 = 0.1 * rng.standard_normal(dff)
        W2 = rng.standard_normal((dff, d)) / math.sqrt(dff)
        b2 = 0.1 * rng.standard_normal(d)
        if np.abs(x @ W1 + b1).min() > 1e-2:   # keep away from the kink for differences
            return x, W1, b1, W2, b2


def test_ff_backward_central_differences():
    rng = np.random.default_rng(11)
    x, W1, b1, W2, b2 = _ff_params(rng, 4, 6, 5)
    dy = rng.standard_normal((5, 4))
    dx, dW1, db1, dW2, db2 = rev.ff_backward(x, W1, b1, W2, b2, dy)
    loss = lambda x_, W1_, b1_, W2_, b2_: float((rev.ff_forward(x_, W1_, b1_, W2_, b2_) * dy).sum())
    eps = 1e-6
    args = [x, W1, b1, W2, b2]
    grads = [dx, dW1, db1, dW2, db2]
    for k in range(5):
        for idx in [tuple(rng.integers(0, s) for s in args[k].shape) for _ in range(4)]:
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[k][idx] += eps
            minus[k][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert abs(fd - grads[k][idx]) < 1e-6 * (1 + abs(fd)), (k, idx)


@pytest.mark.parametrize("chunk", [1, 2, 3, 7, 64])
def test_ff_chunked_matches_whole(chunk):
    """Chunking the positions does not change the feed-forward's results."""
    rng = np.random.default_rng(chunk)
    x, W1, b1, W2, b2 = _ff_params(rng, 8, 16, 21)
    whole = rev.ff_forward(x, W1, b1, W2, b2)
    part = rev.ff_forward_chunked(x, W1, b1, W2, b2, chunk)
    assert np.allclose(part, whole, rtol=0, atol=1e-13)


def test_ff_rows_are_independent():
    """Changing one position changes that position's output only."""
    rng = np.random.default_rng(3)
    x, W1, b1, W2, b2 = _ff_params(rng, 8, 16, 9)
    y = rev.ff_forward(x, W1, b1, W2, b2)
    x2 = x.copy()
    x2[4] += rng.standard_normal(8)
    y2 = rev.ff_forward(x2, W1, b1, W2, b2)
    changed = np.any(y2 != y, axis=1)
    assert changed[4] and not changed[np.arange(9) != 4].any()


def test_head_token_layout():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((2, 3, 5, 4))
    t = rev.heads_to_tokens(a)
    assert t.shape == (10, 12)
    for b, h, l, e in [(0, 0, 0, 0), (1, 2, 4, 3), (0, 1, 3, 2), (1, 0, 2, 1)]:
        assert t[b * 5 + l, h * 4 + e] == a[b, h, l, e]
    assert np.array_equal(rev.tokens_to_heads(t, 2, 3, 5), a)


def _block(seed, B=1, H=2, L=16, d=8, m=4, n_r=2, dff=24, causal=True):
    rng = np.random.default_rng(seed)
    x1 = rng.standard_normal((B, H, L, d))
    x2 = rng.standard_normal((B, H, L, d))
    R = rng.standard_normal((n_r, d, 2))
    bucket, _ = orc.hash_buckets(x2, R)
    perm = orc.sort_positions(bucket)
    W1 = rng.standard_normal((H * d, dff)) / math.sqrt(H * d)
    b1 = 0.1 * rng.standard_normal(dff)
    W2 = rng.standard_normal((dff, H * d)) / math.sqrt(dff)
    b2 = 0.1 * rng.standard_normal(H * d)
    return dict(x1=x1, x2=x2, perm=perm, m=m, causal=causal, scale=1.0 / math.sqrt(d),
                W1=W1, b1=b1, W2=W2, b2=b2)


def _fwd(k, **over):
    a = dict(k)
    a.update(over)
    return rev.rev_forward(a["x1"], a["x2"], a["perm"], a["m"], a["causal"], a["scale"],
                           a["W1"], a["b1"], a["W2"], a["b2"])


@pytest.mark.parametrize("causal", [True, False])
def test_reversible_inverse_recovers_inputs(causal):
    k = _block(1, causal=causal)
    y1, y2 = _fwd(k)
    x1, x2 = rev.rev_backward(y1, y2, np.zeros_like(y1), np.zeros_like(y2), k["perm"], k["m"],
                              k["causal"], k["scale"], k["W1"], k["b1"], k["W2"], k["b2"])[:2]
    assert np.abs(x1 - k["x1"]).max() < 1e-12
    assert np.abs(x2 - k["x2"]).max() < 1e-12


def test_reversible_with_zero_G_is_attention_residual():
    """With W2 = 0 and b2 = 0, G vanishes: y2 = x2 exactly and y1 - x1 = F(x2)."""
    k = _block(2)
    y1, y2 = _fwd(k, W2=np.zeros_like(k["W2"]), b2=np.zeros_like(k["b2"]))
    assert np.array_equal(y2, k["x2"])
    O, _ = orc.forward(k["x2"], k["x2"], k["perm"], k["m"], k["causal"], k["scale"])
    assert np.abs((y1 - k["x1"]) - O).max() < 1e-14


def test_reversible_backward_central_differences():
    """Gradients of sum(c1 * y1 + c2 * y2) against central differences, for
    both inputs and all four feed-forward parameters (permutation fixed)."""
    k = _block(4)
    rng = np.random.default_rng(40)
    y1, y2 = _fwd(k)
    pre = rev.heads_to_tokens(y1) @ k["W1"] + k["b1"]
    assert np.abs(pre).min() > 1e-3       # no kink within the differences
    c1 = rng.standard_normal(y1.shape)
    c2 = rng.standard_normal(y2.shape)
    out = rev.rev_backward(y1, y2, c1, c2, k["perm"], k["m"], k["causal"], k["scale"],
                           k["W1"], k["b1"], k["W2"], k["b2"])
    grads = dict(x1=out[2], x2=out[3], W1=out[4], b1=out[5], W2=out[6], b2=out[7])

    def loss(**over):
        a1, a2 = _fwd(k, **over)
        return float((c1 * a1).sum() + (c2 * a2).sum())

    eps = 1e-6
    for name, g in grads.items():
        for _ in range(4):
            idx = tuple(int(rng.integers(0, s)) for s in k[name].shape)
            p = k[name].copy()
            q = k[name].copy()
            p[idx] += eps
            q[idx] -= eps
            fd = (loss(**{name: p}) - loss(**{name: q})) / (2 * eps)
            assert abs(fd - g[idx]) < 2e-6 * (1 + abs(fd)), (name, idx, fd, g[idx])
