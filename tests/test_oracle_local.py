"""Pins for the oracle's local chunked attention (CPU only).

Source: "The Reformer - Pushing the limits of language modeling" (yomu.fyi
summary of the Hugging Face blog post), Approach and Takeaways: the input is
cut into chunks of length l_c, and each chunk also sees overlap from
preceding and following chunks. Queries and keys are the shared qk vectors
with the self-mask of "Reformer: The Efficient Transformer" (Key points,
"Shared-QK Transformer").
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lsh_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(seed, B, H, L, d):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, L, d)), rng.standard_normal((B, H, L, d)),
            rng.standard_normal((B, H, L, d)))


def _loops(x, v, m, n_back, n_fwd, causal, scale):
    """Local attention of one (b, h) written with explicit loops over keys."""
    L = x.shape[0]
    O = np.zeros_like(v)
    LSE = np.full(L, -np.inf)
    for i in range(L):
        c = i // m
        lo, hi = max(0, (c - n_back) * m), min(L, (c + 1 + n_fwd) * m)
        keys = [j for j in range(lo, hi) if j != i and (not causal or j < i)]
        if not keys:
            O[i] = v[i]
            continue
        logits = [scale * float(np.dot(x[i], x[j])) for j in keys]
        mx = max(logits)
        w = [math.exp(t - mx) for t in logits]
        z = sum(w)
        LSE[i] = mx + math.log(z)
        for wj, j in zip(w, keys):
            O[i] += (wj / z) * v[j]
    return O, LSE


def test_local_hand_worked_example():
    with open(os.path.join(GOLDEN, "local_attention_worked_example.json")) as f:
        g = json.load(f)
    qk = np.array(g["qk"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    for key, causal in (("non_causal", False), ("causal", True)):
        O, LSE = orc.local_forward(qk, v, g["chunk"], g["n_back"], g["n_fwd"], causal, 1.0)
        np.testing.assert_allclose(O[0, 0], np.array(g[key]["O"]), rtol=0, atol=1e-15)
        exp = np.array([-np.inf if t is None else t for t in g[key]["LSE"]])
        np.testing.assert_allclose(LSE[0, 0], exp, rtol=0, atol=1e-15)


def test_planted_mistake_dropping_look_ahead_breaks_the_worked_example(monkeypatch):
    with open(os.path.join(GOLDEN, "local_attention_worked_example.json")) as f:
        g = json.load(f)
    qk = np.array(g["qk"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    monkeypatch.setattr(orc, "local_window",
                        lambda c, m, L, nb, nf: range(max(0, (c - nb) * m), (c + 1) * m))
    O, _ = orc.local_forward(qk, v, g["chunk"], g["n_back"], g["n_fwd"], False, 1.0)
    assert not np.allclose(O[0, 0], np.array(g["non_causal"]["O"]))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_back,n_fwd", [(0, 0), (1, 0), (0, 1), (2, 1), (1, 3)])
def test_local_matches_explicit_loops(causal, n_back, n_fwd):
    qk, v, _ = _rand(3, 1, 2, 24, 5)
    O, LSE = orc.local_forward(qk, v, 4, n_back, n_fwd, causal, 0.4)
    for h in range(2):
        Oe, Le = _loops(qk[0, h], v[0, h], 4, n_back, n_fwd, causal, 0.4)
        np.testing.assert_allclose(O[0, h], Oe, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(np.isfinite(LSE[0, h]), np.isfinite(Le))
        f = np.isfinite(Le)
        np.testing.assert_allclose(LSE[0, h][f], Le[f], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_window_covering_the_sequence_is_full_attention(causal):
    # enough look-back and look-ahead that every chunk sees every position:
    # dense softmax attention with the self-mask
    qk, v, _ = _rand(5, 1, 1, 20, 6)
    x = qk[0, 0]
    O, LSE = orc.local_forward(qk, v, 4, 5, 5, causal, 0.3)
    S = 0.3 * x @ x.T
    mask = ~np.eye(20, dtype=bool)
    if causal:
        mask &= np.tri(20, k=-1, dtype=bool)
    Sm = np.where(mask, S, -np.inf)
    mx = Sm.max(axis=1, keepdims=True)
    has = np.isfinite(mx[:, 0])
    P = np.where(mask, np.exp(Sm - np.where(has[:, None], mx, 0.0)), 0.0)
    Z = P.sum(axis=1, keepdims=True)
    Od = np.where(has[:, None], (P / np.where(Z > 0, Z, 1.0)) @ v[0, 0], v[0, 0])
    np.testing.assert_allclose(O[0, 0], Od, rtol=1e-12, atol=1e-12)
    f = np.isfinite(LSE[0, 0])
    np.testing.assert_array_equal(f, has)
    np.testing.assert_allclose(LSE[0, 0][f], (mx[:, 0] + np.log(Z[:, 0]))[f], rtol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_look_back_one_is_the_identity_order_lsh_window(causal):
    # one chunk of look-back and none ahead is the LSH layer's window (a chunk
    # and the one before it) with every position in its own order, one round
    qk, v, dO = _rand(7, 2, 1, 32, 4)
    perm = np.broadcast_to(np.arange(32), (2, 1, 1, 32)).copy()
    O, LSE = orc.local_forward(qk, v, 8, 1, 0, causal, 0.5)
    O2, LSE2 = orc.forward(qk, v, perm, 8, causal, 0.5)
    np.testing.assert_allclose(O, O2, rtol=1e-12, atol=1e-12)
    np.testing.assert_array_equal(LSE, LSE2)
    g = orc.local_backward(qk, v, 8, 1, 0, causal, 0.5, O, LSE, dO)
    g2 = orc.backward(qk, v, perm, 8, causal, 0.5, O2, LSE2, dO)
    np.testing.assert_allclose(g[0], g2[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[1], g2[1], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_local_backward_central_differences(causal):
    qk, v, dO = _rand(9, 1, 1, 12, 3)
    m, nb, nf, sc = 3, 1, 1, 0.7
    O, LSE = orc.local_forward(qk, v, m, nb, nf, causal, sc)
    dqk, dv = orc.local_backward(qk, v, m, nb, nf, causal, sc, O, LSE, dO)

    def loss(q, w):
        return float((orc.local_forward(q, w, m, nb, nf, causal, sc)[0] * dO).sum())

    eps = 1e-6
    for arr, grad, which in ((qk, dqk, 0), (v, dv, 1)):
        for idx in [(0, 0, 0, 0), (0, 0, 4, 1), (0, 0, 7, 2), (0, 0, 11, 0), (0, 0, 2, 1)]:
            a, b = arr.copy(), arr.copy()
            a[idx] += eps
            b[idx] -= eps
            if which == 0:
                num = (loss(a, v) - loss(b, v)) / (2 * eps)
            else:
                num = (loss(qk, a) - loss(qk, b)) / (2 * eps)
            assert abs(num - grad[idx]) < 1e-6 * max(1.0, abs(num))


def test_local_backward_matches_autograd_of_dense_masked_form():
    qk, v, dO = _rand(11, 1, 1, 16, 4)
    m, nb, nf, sc = 4, 1, 2, 0.5
    O, LSE = orc.local_forward(qk, v, m, nb, nf, True, sc)
    dqk, dv = orc.local_backward(qk, v, m, nb, nf, True, sc, O, LSE, dO)
    L = 16
    mask = np.zeros((L, L), dtype=bool)
    for i in range(L):
        c = i // m
        for j in range(max(0, (c - nb) * m), min(L, (c + 1 + nf) * m)):
            mask[i, j] = j < i
    x = torch.tensor(qk[0, 0], requires_grad=True)
    w = torch.tensor(v[0, 0], requires_grad=True)
    M = torch.tensor(mask)
    S = sc * x @ x.T
    S = torch.where(M, S, torch.tensor(-torch.inf, dtype=torch.float64))
    has = M.any(dim=1)
    P = torch.softmax(torch.where(has[:, None], S, torch.zeros_like(S)), dim=1)
    P = torch.where(M, P, torch.zeros_like(P))
    out = torch.where(has[:, None], P @ w, w)
    (out * torch.tensor(dO[0, 0])).sum().backward()
    np.testing.assert_allclose(dqk[0, 0], x.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv[0, 0], w.grad.numpy(), rtol=1e-10, atol=1e-12)
