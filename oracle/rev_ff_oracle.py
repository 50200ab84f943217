"""CPU oracle for the reversible residual block and the chunked feed-forward
that surround LSH attention in a Reformer layer (float64, numpy).

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module. The product path
never calls it, and it never imports the product.

What it computes, in the order of the source pages:

* "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
  Key points, the "Reversible layers" bullet: reversible residual layers
  (its reference 8, Gomez et al. 2017, "The reversible residual network")
  take the number of layers out of the activation memory, because a layer's
  inputs are recomputed from its outputs in the backward pass; running the
  feed-forward layers chunk by chunk takes the d_ff factor out and leaves the
  results numerically unchanged.
* "The Reformer - Pushing the limits of language modeling" (Hugging Face blog
  page), Summary: a Reformer layer combines LSH self-attention with chunked
  feed-forward layers and reversible residual layers.
* The reversible residual form is that of the cited paper: the activations
  are split in two halves, y1 = x1 + F(x2) and y2 = x2 + G(y1), which invert
  as x2 = y2 - G(y1) and x1 = y1 - F(x2). In the Reformer F is the attention
  and G the feed-forward.

Readings where the pages are silent:
  G is the position-wise feed-forward max(0, x W1 + b1) W2 + b2 (the pages
  name no activation; ReLU is the plain Transformer one) with relu'(0) = 0;
  F is LSH attention of x2 with the shared query/key and the values both
  equal to x2 (the projection weights are outside this path); the block's
  activations are [B, H, L, 64] arrays and a token's d_model = 64 H features
  are its H head rows side by side; the backward keeps the forward's sort
  permutation (a bucket id is a discrete function of x2, and the
  reconstructed x2 equals the original only up to rounding).

Every function is pinned by ``tests/test_oracle_reversible.py``: a hand-worked
feed-forward example, central differences for both backward passes, the
inverse identity of the reversible block and its G = 0 special case.
Parity status: pinned.
"""
from __future__ import annotations

import numpy as np

from oracle import lsh_oracle as lsh


# --------------------------------------------------------------------------
# Layout: [B, H, L, 64] head rows <-> [B * L, 64 H] token rows
# --------------------------------------------------------------------------

def heads_to_tokens(a: np.ndarray) -> np.ndarray:
    """[B, H, L, d] -> [B * L, H * d]: token (b, l) gets its H head rows side by side."""
    B, H, L, d = a.shape
    return np.ascontiguousarray(np.transpose(a, (0, 2, 1, 3))).reshape(B * L, H * d)


def tokens_to_heads(t: np.ndarray, B: int, H: int, L: int) -> np.ndarray:
    """Inverse of ``heads_to_tokens``."""
    d = t.shape[1] // H
    return np.ascontiguousarray(np.transpose(t.reshape(B, L, H, d), (0, 2, 1, 3)))


# --------------------------------------------------------------------------
# Position-wise feed-forward G(x) = max(0, x W1 + b1) W2 + b2
# --------------------------------------------------------------------------

def ff_forward(x, W1, b1, W2, b2):
    """G of every row of x [n, d_model]; W1 [d_model, d_ff], W2 [d_ff, d_model]."""
    x = np.asarray(x, dtype=np.float64)
    pre = x @ W1 + b1
    h = np.maximum(pre, 0.0)
    return h @ W2 + b2


def ff_forward_chunked(x, W1, b1, W2, b2, chunk: int):
    """The same feed-forward, applied to ``chunk`` rows at a time; only a
    [chunk, d_ff] hidden block exists at once."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty((x.shape[0], np.asarray(W2).shape[1]))
    for r0 in range(0, x.shape[0], chunk):
        out[r0:r0 + chunk] = ff_forward(x[r0:r0 + chunk], W1, b1, W2, b2)
    return out


def ff_backward(x, W1, b1, W2, b2, dy):
    """Gradients of sum(G(x) * dy): (dx, dW1, db1, dW2, db2)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    pre = x @ W1 + b1
    h = np.maximum(pre, 0.0)
    dh = (dy @ np.asarray(W2, dtype=np.float64).T) * (pre > 0.0)
    dW2 = h.T @ dy
    db2 = dy.sum(axis=0)
    dW1 = x.T @ dh
    db1 = dh.sum(axis=0)
    dx = dh @ np.asarray(W1, dtype=np.float64).T
    return dx, dW1, db1, dW2, db2


# --------------------------------------------------------------------------
# Reversible block: y1 = x1 + F(x2), y2 = x2 + G(y1)
# --------------------------------------------------------------------------

def attention_F(x2, perm, m, causal, scale):
    """F(x2): LSH attention with qk = v = x2 under the given permutation.
    Returns (O, LSE), both needed again by the backward."""
    return lsh.forward(x2, x2, perm, m, causal, scale)


def rev_forward(x1, x2, perm, m, causal, scale, W1, b1, W2, b2):
    """(y1, y2) of the block for inputs x1, x2 [B, H, L, 64]."""
    x1 = np.asarray(x1, dtype=np.float64)
    x2 = np.asarray(x2, dtype=np.float64)
    B, H, L, _ = x1.shape
    O, _ = attention_F(x2, perm, m, causal, scale)
    y1 = x1 + O
    g = ff_forward(heads_to_tokens(y1), W1, b1, W2, b2)
    y2 = x2 + tokens_to_heads(g, B, H, L)
    return y1, y2


def rev_backward(y1, y2, dy1, dy2, perm, m, causal, scale, W1, b1, W2, b2):
    """Backward of the block from its outputs alone.

    G half: x2 = y2 - G(y1); dz1 = dy1 + (dG/dy1)^T dy2, with G's weight
    gradients. F half: x1 = y1 - F(x2); dx2 = dy2 + (dF/dx2)^T dz1, where F's
    input feeds both the shared query/key and the values; dx1 = dz1.
    Returns (x1, x2, dx1, dx2, dW1, db1, dW2, db2).
    """
    y1 = np.asarray(y1, dtype=np.float64)
    y2 = np.asarray(y2, dtype=np.float64)
    B, H, L, _ = y1.shape
    t1 = heads_to_tokens(y1)
    g = ff_forward(t1, W1, b1, W2, b2)
    x2 = y2 - tokens_to_heads(g, B, H, L)
    dt1, dW1, db1, dW2, db2 = ff_backward(t1, W1, b1, W2, b2, heads_to_tokens(dy2))
    dz1 = np.asarray(dy1, dtype=np.float64) + tokens_to_heads(dt1, B, H, L)
    O, LSE = attention_F(x2, perm, m, causal, scale)
    x1 = y1 - O
    dqk, dv = lsh.backward(x2, x2, perm, m, causal, scale, O, LSE, dz1)
    dx2 = np.asarray(dy2, dtype=np.float64) + dqk + dv
    return x1, x2, dz1, dx2, dW1, db1, dW2, db2
