"""Pins for the oracle's chunk attention, round combine and backward (CPU only).

Sources: "Reformer: The Efficient Transformer" (research.elamur.ai summary
page), Key points "LSH attention" (a chunk attends to itself and the chunk
before it), "Shared-QK Transformer" (no attending to oneself unless there is
no other valid target) and "Number of hash rounds" (several rounds).
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
    return rng.standard_normal((B, H, L, d)), rng.standard_normal((B, H, L, d))


def _identity_perm(B, H, n_r, L):
    return np.broadcast_to(np.arange(L), (B, H, n_r, L)).copy()


def _random_perm(seed, B, H, n_r, L):
    rng = np.random.default_rng(seed)
    p = np.empty((B, H, n_r, L), dtype=np.int64)
    for idx in np.ndindex(B, H, n_r):
        p[idx] = rng.permutation(L)
    return p


# ---------------------------------------------------------------- worked example

def test_attention_hand_worked_example():
    with open(os.path.join(GOLDEN, "attention_worked_example.json")) as f:
        g = json.load(f)
    qk = np.array(g["qk"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    perm = _identity_perm(1, 1, 1, 4)
    for key, causal in (("non_causal", False), ("causal", True)):
        O, LSE = orc.forward(qk, v, perm, g["chunk"], causal, 1.0)
        np.testing.assert_allclose(O[0, 0], np.array(g[key]["O"]), rtol=0, atol=1e-15)
        exp = np.array([-np.inf if t is None else t for t in g[key]["LSE"]])
        np.testing.assert_allclose(LSE[0, 0], exp, rtol=0, atol=1e-15)


# ----------------------------------------------------------- dense brute force

def _dense_full_attention(x, v, scale, causal):
    """Full softmax attention with the self-mask, written from scratch with loops."""
    L, d = x.shape
    O = np.zeros_like(v)
    LSE = np.full(L, -np.inf)
    for i in range(L):
        keys = [j for j in range(L) if j != i and (not causal or j < i)]
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


@pytest.mark.parametrize("causal", [False, True])
def test_one_chunk_spanning_sequence_is_full_attention(causal):
    # m = L, one round: the only chunk holds every position, so LSH attention
    # must equal full attention under the same masks, whatever the sort order.
    qk, v = _rand(10, 1, 2, 48, 16)
    perm = _random_perm(11, 1, 2, 1, 48)
    O, LSE = orc.forward(qk, v, perm, 48, causal, 0.25)
    for h in range(2):
        Od, Ld = _dense_full_attention(qk[0, h], v[0, h], 0.25, causal)
        np.testing.assert_allclose(O[0, h], Od, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(LSE[0, h], Ld, rtol=1e-12, atol=1e-12)


def test_causal_first_position_attends_to_itself():
    qk, v = _rand(12, 2, 2, 64, 8)
    R = np.random.default_rng(13).standard_normal((3, 8, 4))
    res = orc.lsh_attention(qk, v, R, 16, True, 1 / math.sqrt(8))
    np.testing.assert_array_equal(res["O"][:, :, 0], v[:, :, 0])
    assert np.all(np.isneginf(res["LSE"][:, :, 0]))


def test_rows_sum_to_one_constant_value_column():
    qk, v = _rand(14, 1, 2, 96, 8)
    v[..., 3] = 2.5
    R = np.random.default_rng(15).standard_normal((2, 8, 6))
    for causal in (False, True):
        res = orc.lsh_attention(qk, v, R, 16, causal, 0.3)
        np.testing.assert_allclose(res["O"][..., 3], 2.5, rtol=0, atol=1e-13)


# ------------------------------------------- multi-round: dense count matrix

def _count_matrix(perm_bh, m, causal):
    """C[i, j] = number of rounds in which key j is in query i's window and valid."""
    n_r, L = perm_bh.shape
    C = np.zeros((L, L))
    for r in range(n_r):
        p = perm_bh[r]
        for t in range(L):
            i = p[t]
            c = t // m
            for u in range(max(0, (c - 1) * m), (c + 1) * m):
                j = p[u]
                if j != i and (not causal or j < i):
                    C[i, j] += 1
    return C


def _dense_union_softmax(x, v, C, scale):
    """O_i = sum_j C_ij e^{s_ij} v_j / sum_j C_ij e^{s_ij}; v_i when row i of C is 0."""
    s = scale * (x @ x.T)
    O = np.array(v, copy=True)
    LSE = np.full(x.shape[0], -np.inf)
    for i in range(x.shape[0]):
        if C[i].sum() == 0:
            continue
        mx = s[i][C[i] > 0].max()
        w = C[i] * np.exp(s[i] - mx)
        O[i] = w @ v / w.sum()
        LSE[i] = mx + np.log(w.sum())
    return O, LSE


@pytest.mark.parametrize("causal", [False, True])
def test_round_combine_equals_union_softmax(causal):
    qk, v = _rand(16, 1, 2, 40, 8)
    R = np.random.default_rng(17).standard_normal((3, 8, 3))
    res = orc.lsh_attention(qk, v, R, 8, causal, 0.35)
    for h in range(2):
        C = _count_matrix(res["perm"][0, h], 8, causal)
        Od, Ld = _dense_union_softmax(qk[0, h], v[0, h], C, 0.35)
        np.testing.assert_allclose(res["O"][0, h], Od, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(res["LSE"][0, h], Ld, rtol=1e-12, atol=1e-12)


def test_identical_rounds_equal_one_round():
    qk, v = _rand(18, 1, 1, 64, 8)
    R1 = np.random.default_rng(19).standard_normal((1, 8, 4))
    R4 = np.repeat(R1, 4, axis=0)
    a = orc.lsh_attention(qk, v, R1, 16, True, 0.3)
    b = orc.lsh_attention(qk, v, R4, 16, True, 0.3)
    np.testing.assert_allclose(b["O"], a["O"], rtol=1e-12, atol=1e-13)
    fin = np.isfinite(a["LSE"])
    np.testing.assert_allclose(b["LSE"][fin], a["LSE"][fin] + math.log(4), rtol=1e-13)
    assert np.array_equal(np.isfinite(b["LSE"]), fin)


@pytest.mark.parametrize("causal", [False, True])
def test_forward_rows_matches_forward(causal):
    qk, v = _rand(20, 2, 2, 96, 8)
    perm = _random_perm(21, 2, 2, 3, 96)
    O, LSE = orc.forward(qk, v, perm, 16, causal, 0.3)
    rows = [0, 1, 15, 16, 17, 50, 95]
    for b in range(2):
        for h in range(2):
            Or, Lr = orc.forward_rows(qk, v, perm, 16, causal, 0.3, b, h, rows)
            np.testing.assert_allclose(Or, O[b, h, rows], rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(Lr, LSE[b, h, rows], rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- backward

def _loss(qk, v, perm, m, causal, scale, dO):
    O, _ = orc.forward(qk, v, perm, m, causal, scale)
    return float((O * dO).sum())


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_central_differences(causal):
    B, H, L, d, m, n_r = 1, 1, 16, 4, 4, 2
    qk, v = _rand(22, B, H, L, d)
    dO = np.random.default_rng(23).standard_normal((B, H, L, d))
    perm = _random_perm(24, B, H, n_r, L)
    scale = 0.5
    O, LSE = orc.forward(qk, v, perm, m, causal, scale)
    dqk, dv = orc.backward(qk, v, perm, m, causal, scale, O, LSE, dO)
    eps = 1e-6
    num_qk = np.zeros_like(qk)
    num_v = np.zeros_like(v)
    for idx in np.ndindex(*qk.shape):
        for arr, out in ((qk, num_qk), (v, num_v)):
            old = arr[idx]
            arr[idx] = old + eps
            fp = _loss(qk, v, perm, m, causal, scale, dO)
            arr[idx] = old - eps
            fm = _loss(qk, v, perm, m, causal, scale, dO)
            arr[idx] = old
            out[idx] = (fp - fm) / (2 * eps)
    np.testing.assert_allclose(dqk, num_qk, rtol=1e-6, atol=1e-7)
    np.testing.assert_allclose(dv, num_v, rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_autograd_of_dense_union_softmax(causal):
    # torch.autograd in float64 through the dense count-matrix formulation,
    # which shares no code with the oracle's chunked backward.
    B, H, L, d, m, n_r = 1, 2, 32, 8, 8, 3
    qk, v = _rand(25, B, H, L, d)
    dO = np.random.default_rng(26).standard_normal((B, H, L, d))
    R = np.random.default_rng(27).standard_normal((n_r, d, 4))
    scale = 0.3
    res = orc.lsh_attention(qk, v, R, m, causal, scale)
    dqk, dv = orc.backward(qk, v, res["perm"], m, causal, scale, res["O"], res["LSE"], dO)
    for h in range(H):
        C = torch.tensor(_count_matrix(res["perm"][0, h], m, causal))
        x = torch.tensor(qk[0, h], requires_grad=True)
        vv = torch.tensor(v[0, h], requires_grad=True)
        s = scale * (x @ x.T)
        has = C.sum(1) > 0
        w = C * torch.exp(s - s.detach().max(1, keepdim=True).values)
        att = w / torch.where(has, w.sum(1), torch.ones(L, dtype=w.dtype))[:, None]
        O = torch.where(has[:, None], att @ vv, vv)
        (O * torch.tensor(dO[0, h])).sum().backward()
        np.testing.assert_allclose(dqk[0, h], x.grad.numpy(), rtol=1e-10, atol=1e-11)
        np.testing.assert_allclose(dv[0, h], vv.grad.numpy(), rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_rows_matches_backward(causal):
    B, H, L, d, m, n_r = 1, 2, 64, 8, 8, 3
    qk, v = _rand(28, B, H, L, d)
    dO = np.random.default_rng(29).standard_normal((B, H, L, d))
    perm = _random_perm(30, B, H, n_r, L)
    O, LSE = orc.forward(qk, v, perm, m, causal, 0.3)
    dqk, dv = orc.backward(qk, v, perm, m, causal, 0.3, O, LSE, dO)
    rows = [0, 1, 7, 8, 33, 63]
    for h in range(H):
        a, b = orc.backward_rows(qk, v, perm, m, causal, 0.3, dO, 0, h, rows)
        np.testing.assert_allclose(a, dqk[0, h, rows], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(b, dv[0, h, rows], rtol=1e-11, atol=1e-12)


def test_backward_identical_rounds_equal_one_round():
    qk, v = _rand(31, 1, 1, 48, 8)
    dO = np.random.default_rng(32).standard_normal((1, 1, 48, 8))
    R1 = np.random.default_rng(33).standard_normal((1, 8, 4))
    out = []
    for R in (R1, np.repeat(R1, 3, axis=0)):
        res = orc.lsh_attention(qk, v, R, 8, True, 0.3)
        out.append(orc.backward(qk, v, res["perm"], 8, True, 0.3, res["O"], res["LSE"], dO))
    np.testing.assert_allclose(out[1][0], out[0][0], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out[1][1], out[0][1], rtol=1e-11, atol=1e-12)


# ------------------------------------------------ planted mistakes are caught

def test_planted_mistakes_fail_the_pins(monkeypatch):
    """Each plausible mistake, planted in the oracle, breaks at least one pin."""
    qk, v = _rand(40, 1, 1, 32, 8)
    perm = _random_perm(41, 1, 1, 1, 32)

    def pins_hold():
        try:
            test_one_chunk_spanning_sequence_is_full_attention(False)
            test_one_chunk_spanning_sequence_is_full_attention(True)
            test_round_combine_equals_union_softmax(True)
            test_attention_hand_worked_example()
            return True
        except AssertionError:
            return False

    assert pins_hold()
    real_valid = orc._valid
    # 1) self-mask dropped
    monkeypatch.setattr(orc, "_valid", lambda q, k, c: (k[None, :] <= q[:, None]) if c
                        else np.ones((len(q), len(k)), bool))
    assert not pins_hold()
    monkeypatch.setattr(orc, "_valid", real_valid)
    # 2) causal mask with the wrong direction
    monkeypatch.setattr(orc, "_valid", lambda q, k, c: (k[None, :] != q[:, None]) &
                        ((k[None, :] > q[:, None]) if c else True))
    assert not pins_hold()
    monkeypatch.setattr(orc, "_valid", real_valid)
    # 3) rounds averaged instead of weighted by their log-sum-exps
    real_combine = orc.combine_rounds

    def mean_combine(o_r, lse_r, v):
        O, LSE = real_combine(o_r, lse_r, v)
        fin = np.isfinite(lse_r)
        cnt = np.maximum(fin.sum(0), 1)
        return np.where(fin.any(0)[..., None], o_r.sum(0) / cnt[..., None], O), LSE
    monkeypatch.setattr(orc, "combine_rounds", mean_combine)
    assert not pins_hold()
    monkeypatch.setattr(orc, "combine_rounds", real_combine)
    assert pins_hold()
