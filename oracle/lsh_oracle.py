"""CPU oracle for Reformer LSH self-attention (float64, numpy).

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module. The product path
(the CUDA library and its Python binding) never calls it, and the oracle never
imports the product: both take their inputs from the seeded generator module,
which holds no attention arithmetic.

What it computes, step by step, in the order of the source pages:

* "Reformer: The Efficient Transformer" (research.elamur.ai summary page),
  Summary paragraph: queries and keys come from one shared projection, are
  hashed with random rotations, sorted by bucket, and attention runs inside
  small fixed-size chunks; several hashing rounds are used.
* Same page, Key points, "LSH attention": h(x) = argmax([xR; -xR]) with a
  random matrix R; after sorting, each chunk of m positions attends to itself
  and the chunk before it.
* Same page, Key points, "Shared-QK Transformer": keys equal queries; a token
  may not attend to itself unless it has no other valid target.
* Same page, Key points, "Number of hash rounds": several rounds, each an
  independent hash.

Readings where the pages are silent:
  scale = 1/sqrt(d) on the logits; argmax ties go to the lowest index; the
  sort is stable by position; the window is the chunk and the previous chunk
  of the same round, with no wrap-around; causal masking is by original
  position; the self-mask fallback is decided over the union of all rounds;
  rounds are combined by a softmax over their per-round log-sum-exps (a key
  seen in k rounds counts k times); the backward pass recomputes the
  attention weights from the final log-sum-exp.

Every function is pinned by tests in ``tests/test_oracle_*.py`` against
closed forms, exact rational brute force, dense full attention, a dense
count-matrix formulation of the round combine and finite differences.
Parity status: pinned (no function here is "parity unpinned").
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# --------------------------------------------------------------------------
# Hashing: h(x) = argmax([xR; -xR])  (Key points, "LSH attention")
# --------------------------------------------------------------------------

def hash_round(x: np.ndarray, R_r: np.ndarray):
    """Bucket ids of the rows of ``x`` under one random rotation ``R_r``.

    x: [n, d]; R_r: [d, n_b/2]. Returns (bucket [n] int64, gap [n] float64).
    u = [xR, -xR] has n_b entries; bucket = first index of max(u).
    gap = (u_max - u_second) / u_max; 0 when u_max == 0 (a tie by definition).
    """
    x = np.asarray(x, dtype=np.float64)
    R_r = np.asarray(R_r, dtype=np.float64)
    s = x @ R_r
    u = np.concatenate([s, -s], axis=1)
    bucket = np.argmax(u, axis=1)           # numpy: first occurrence on ties
    rows = np.arange(u.shape[0])
    top = u[rows, bucket]
    u[rows, bucket] = NEG_INF
    second = u.max(axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        gap = np.where(top > 0, (top - second) / np.where(top > 0, top, 1.0), 0.0)
    return bucket.astype(np.int64), gap


def hash_buckets(qk: np.ndarray, R: np.ndarray, row_block: int = 8192):
    """Bucket ids for every (batch, head, round, position).

    qk: [B, H, L, d]; R: [n_rounds, d, n_b/2].
    Returns (bucket [B, H, n_rounds, L] int64, gap [B, H, n_rounds, L]).
    """
    B, H, L, _ = qk.shape
    n_r = R.shape[0]
    bucket = np.empty((B, H, n_r, L), dtype=np.int64)
    gap = np.empty((B, H, n_r, L), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r in range(n_r):
                for i0 in range(0, L, row_block):
                    i1 = min(L, i0 + row_block)
                    bk, gp = hash_round(qk[b, h, i0:i1], R[r])
                    bucket[b, h, r, i0:i1] = bk
                    gap[b, h, r, i0:i1] = gp
    return bucket, gap


# --------------------------------------------------------------------------
# Sorting by bucket  (Summary; Key points, "LSH attention")
# --------------------------------------------------------------------------

def sort_positions(bucket: np.ndarray) -> np.ndarray:
    """Stable sort of positions by bucket, separately for each (b, h, round).

    perm[..., t] = original position held by sorted slot t. Stability makes
    this the sort by the packed key (round, bucket, position).
    """
    return np.argsort(bucket, axis=-1, kind="stable").astype(np.int64)


def slots_of_positions(perm_r: np.ndarray) -> np.ndarray:
    """Inverse permutation: slot[i] = sorted slot that holds position i."""
    inv = np.empty_like(perm_r)
    inv[perm_r] = np.arange(perm_r.shape[0], dtype=perm_r.dtype)
    return inv


def window_slots(t: int, m: int) -> range:
    """Key slots seen by the query in sorted slot ``t``: its chunk and the one before."""
    c = t // m
    return range(max(0, (c - 1) * m), (c + 1) * m)


def _valid(q_pos: np.ndarray, k_pos: np.ndarray, causal: bool) -> np.ndarray:
    """Mask [len(q), len(k)]: not itself, and (causal) keys at earlier positions."""
    v = k_pos[None, :] != q_pos[:, None]
    if causal:
        v &= k_pos[None, :] < q_pos[:, None]
    return v


def _masked_lse(s: np.ndarray, valid: np.ndarray):
    """Row log-sum-exp over valid entries; -inf for rows with none."""
    sm = np.where(valid, s, NEG_INF)
    mx = sm.max(axis=1)
    has = np.isfinite(mx)
    safe = np.where(has, mx, 0.0)
    with np.errstate(under="ignore"):
        tot = np.where(valid, np.exp(sm - safe[:, None]), 0.0).sum(axis=1)
    with np.errstate(divide="ignore"):
        lse = np.where(has, safe + np.log(np.where(has, tot, 1.0)), NEG_INF)
    return lse


# --------------------------------------------------------------------------
# Forward: chunked attention per round, then the round combine
# --------------------------------------------------------------------------

def forward_rounds(qk, v, perm, m, causal, scale):
    """Per-round outputs o_r and log-sum-exps lse_r, in original order.

    qk, v: [B, H, L, d]; perm: [B, H, n_r, L].
    Returns o_r [n_r, B, H, L, d] and lse_r [n_r, B, H, L]; rows with no
    valid key in a round get o = 0 and lse = -inf.
    """
    qk = np.asarray(qk, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, L, d = qk.shape
    n_r = perm.shape[2]
    if L % m:
        raise ValueError("L must be a multiple of the chunk size")
    o_r = np.zeros((n_r, B, H, L, d))
    lse_r = np.full((n_r, B, H, L), NEG_INF)
    for b in range(B):
        for h in range(H):
            X, V = qk[b, h], v[b, h]
            for r in range(n_r):
                p = perm[b, h, r]
                for c in range(L // m):
                    qi = p[c * m:(c + 1) * m]
                    kj = p[max(0, (c - 1) * m):(c + 1) * m]
                    s = scale * (X[qi] @ X[kj].T)
                    valid = _valid(qi, kj, causal)
                    lse = _masked_lse(s, valid)
                    fin = np.isfinite(lse)
                    with np.errstate(under="ignore"):
                        w = np.where(valid & fin[:, None],
                                     np.exp(s - np.where(fin, lse, 0.0)[:, None]), 0.0)
                    o_r[r, b, h, qi] = w @ V[kj]
                    lse_r[r, b, h, qi] = lse
    return o_r, lse_r


def combine_rounds(o_r, lse_r, v):
    """Softmax over the per-round log-sum-exps.

    LSE = log sum_r exp(lse_r); O = sum_r exp(lse_r - LSE) o_r. A row with no
    valid key in any round attends only to itself: O = v, LSE = -inf.
    """
    v = np.asarray(v, dtype=np.float64)
    mx = lse_r.max(axis=0)
    has = np.isfinite(mx)
    safe = np.where(has, mx, 0.0)
    with np.errstate(under="ignore"):
        wsum = np.exp(lse_r - safe).sum(axis=0)
    with np.errstate(divide="ignore"):
        LSE = np.where(has, safe + np.log(np.where(has, wsum, 1.0)), NEG_INF)
    with np.errstate(under="ignore", invalid="ignore"):
        w = np.where(np.isfinite(lse_r), np.exp(lse_r - np.where(has, LSE, 0.0)), 0.0)
    O = (w[..., None] * o_r).sum(axis=0)
    O = np.where(has[..., None], O, v)
    return O, LSE


def forward(qk, v, perm, m, causal, scale):
    """Full LSH-attention forward: (O [B,H,L,d], LSE [B,H,L])."""
    o_r, lse_r = forward_rounds(qk, v, perm, m, causal, scale)
    return combine_rounds(o_r, lse_r, v)


def forward_rows(qk, v, perm, m, causal, scale, b, h, rows):
    """Forward for selected positions of one (b, h), one query at a time.

    Returns (O [len(rows), d], LSE [len(rows)]). Used at sizes where the full
    forward would take too long; agrees with ``forward`` (tested).
    """
    X = np.asarray(qk[b, h], dtype=np.float64)
    V = np.asarray(v[b, h], dtype=np.float64)
    n_r = perm.shape[2]
    inv = [slots_of_positions(perm[b, h, r]) for r in range(n_r)]
    rows = np.asarray(rows, dtype=np.int64)
    O = np.zeros((len(rows), X.shape[1]))
    LSE = np.full(len(rows), NEG_INF)
    for n, i in enumerate(rows):
        lses, outs = [], []
        for r in range(n_r):
            kj = perm[b, h, r][list(window_slots(int(inv[r][i]), m))]
            s = scale * (X[kj] @ X[i])
            valid = _valid(np.array([i]), kj, causal)[0]
            if not valid.any():
                continue
            sv = s[valid]
            mx = sv.max()
            lse = mx + np.log(np.exp(sv - mx).sum())
            lses.append(lse)
            outs.append(np.exp(sv - lse) @ V[kj[valid]])
        if not lses:
            O[n] = V[i]
            continue
        lses = np.array(lses)
        mx = lses.max()
        tot = mx + np.log(np.exp(lses - mx).sum())
        LSE[n] = tot
        O[n] = sum(np.exp(l - tot) * o for l, o in zip(lses, outs))
    return O, LSE


# --------------------------------------------------------------------------
# Backward by recomputation (attention weights rebuilt from the final LSE)
# --------------------------------------------------------------------------

def backward(qk, v, perm, m, causal, scale, O, LSE, dO):
    """Gradients of sum(O * dO) with respect to the shared qk and v.

    The combined output is one softmax over the union of all rounds' windows,
    so P_ij = exp(s_ij - LSE_i) for every (round, window) occurrence of j, and
    dS = P * (dO_i . v_j - D_i) with D_i = dO_i . O_i. Because queries and keys
    are the same vectors, both the query-side and the key-side terms land in
    dqk. Rows that fell back to themselves (LSE = -inf) pass dO straight to dv.
    """
    qk = np.asarray(qk, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    O = np.asarray(O, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, H, L, d = qk.shape
    n_r = perm.shape[2]
    dqk = np.zeros_like(qk)
    dv = np.zeros_like(v)
    D = (dO * O).sum(axis=-1)
    for b in range(B):
        for h in range(H):
            X, V, G = qk[b, h], v[b, h], dO[b, h]
            lse_all = LSE[b, h]
            for r in range(n_r):
                p = perm[b, h, r]
                for c in range(L // m):
                    qi = p[c * m:(c + 1) * m]
                    kj = p[max(0, (c - 1) * m):(c + 1) * m]
                    s = scale * (X[qi] @ X[kj].T)
                    lq = lse_all[qi]
                    fin = np.isfinite(lq)
                    valid = _valid(qi, kj, causal) & fin[:, None]
                    with np.errstate(under="ignore"):
                        P = np.where(valid, np.exp(s - np.where(fin, lq, 0.0)[:, None]), 0.0)
                    dP = G[qi] @ V[kj].T
                    dS = P * (dP - D[b, h, qi][:, None])
                    dqk[b, h, qi] += scale * (dS @ X[kj])
                    dqk[b, h, kj] += scale * (dS.T @ X[qi])
                    dv[b, h, kj] += P.T @ G[qi]
            fb = ~np.isfinite(lse_all)
            dv[b, h, fb] += G[fb]
    return dqk, dv


def backward_rows(qk, v, perm, m, causal, scale, dO, b, h, rows):
    """Gradients at selected positions of one (b, h), built from per-row terms.

    For each target j: its own query-side term, the key-side terms from every
    query whose window holds j in some round, and the fall-back pass-through.
    The needed queries' O and LSE come from ``forward_rows``.
    Returns (dqk [len(rows), d], dv [len(rows), d]).
    """
    X = np.asarray(qk[b, h], dtype=np.float64)
    V = np.asarray(v[b, h], dtype=np.float64)
    G = np.asarray(dO[b, h], dtype=np.float64)
    L = X.shape[0]
    n_r = perm.shape[2]
    inv = [slots_of_positions(perm[b, h, r]) for r in range(n_r)]
    rows = [int(j) for j in rows]
    target = {j: n for n, j in enumerate(rows)}
    need = set(rows)
    for j in rows:
        for r in range(n_r):
            c = int(inv[r][j]) // m
            lo, hi = c * m, min(L, (c + 2) * m)
            need.update(int(q) for q in perm[b, h, r][lo:hi])
    need = np.array(sorted(need), dtype=np.int64)
    On, Ln = forward_rows(qk, v, perm, m, causal, scale, b, h, need)
    Dn = (G[need] * On).sum(axis=1)
    lse_of = dict(zip(need.tolist(), Ln.tolist()))
    d_of = dict(zip(need.tolist(), Dn.tolist()))
    dqk = np.zeros((len(rows), X.shape[1]))
    dv = np.zeros((len(rows), X.shape[1]))
    for i in need.tolist():
        lse_i = lse_of[i]
        if not np.isfinite(lse_i):
            continue
        for r in range(n_r):
            kj = perm[b, h, r][list(window_slots(int(inv[r][i]), m))]
            valid = _valid(np.array([i]), kj, causal)[0]
            kv = kj[valid]
            s = scale * (X[kv] @ X[i])
            P = np.exp(s - lse_i)
            dS = P * (V[kv] @ G[i] - d_of[i])
            if i in target:
                dqk[target[i]] += scale * (dS @ X[kv])
            for n, j in enumerate(kv.tolist()):
                if j in target:
                    dqk[target[j]] += scale * dS[n] * X[i]
                    dv[target[j]] += P[n] * G[i]
    for j in rows:
        if not np.isfinite(lse_of[j]):
            dv[target[j]] += G[j]
    return dqk, dv


def lsh_attention(qk, v, R, m, causal, scale):
    """Whole forward path: hash, sort, chunk attention, combine."""
    bucket, gap = hash_buckets(qk, R)
    perm = sort_positions(bucket)
    O, LSE = forward(qk, v, perm, m, causal, scale)
    return {"bucket": bucket, "gap": gap, "perm": perm, "O": O, "LSE": LSE}


# --------------------------------------------------------------------------
# Local chunked self-attention ("The Reformer – Pushing the limits of
# language modeling", Approach and Takeaways: the input is cut into chunks of
# length l_c, and each chunk also sees a configurable overlap of preceding
# and following chunks). Readings where the page is silent: the overlap is a
# whole number of chunks (n_back before, n_fwd after, clipped at the sequence
# ends); queries and keys are the shared qk vectors with the same self-mask
# and fall-back as the LSH layer, and causal masking is by position.
# --------------------------------------------------------------------------

def local_window(c: int, m: int, L: int, n_back: int, n_fwd: int) -> range:
    """Key positions seen by the queries of chunk ``c``."""
    return range(max(0, (c - n_back) * m), min(L, (c + 1 + n_fwd) * m))


def local_forward(qk, v, m, n_back, n_fwd, causal, scale):
    """Local attention forward: (O [B,H,L,d], LSE [B,H,L]).

    Chunk c's queries (positions [cm, (c+1)m)) attend to the keys of
    ``local_window``; a query with no valid key attends to itself (O = v,
    LSE = -inf).
    """
    qk = np.asarray(qk, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, L, d = qk.shape
    if L % m:
        raise ValueError("L must be a multiple of the chunk size")
    O = np.zeros_like(v)
    LSE = np.full((B, H, L), NEG_INF)
    for b in range(B):
        for h in range(H):
            X, V = qk[b, h], v[b, h]
            for c in range(L // m):
                qi = np.arange(c * m, (c + 1) * m)
                kj = np.array(local_window(c, m, L, n_back, n_fwd))
                s = scale * (X[qi] @ X[kj].T)
                valid = _valid(qi, kj, causal)
                lse = _masked_lse(s, valid)
                fin = np.isfinite(lse)
                with np.errstate(under="ignore"):
                    w = np.where(valid & fin[:, None],
                                 np.exp(s - np.where(fin, lse, 0.0)[:, None]), 0.0)
                O[b, h, qi] = np.where(fin[:, None], w @ V[kj], V[qi])
                LSE[b, h, qi] = lse
    return O, LSE


def local_backward(qk, v, m, n_back, n_fwd, causal, scale, O, LSE, dO):
    """Gradients of sum(O * dO) for local attention, by recomputation.

    Same algebra as ``backward`` with the local windows: P = exp(s - LSE),
    dS = P (dO_i . v_j - D_i), both query- and key-side terms into dqk, and
    rows that fell back to themselves pass dO to dv.
    """
    qk = np.asarray(qk, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, H, L, d = qk.shape
    dqk = np.zeros_like(qk)
    dv = np.zeros_like(v)
    D = (dO * np.asarray(O, dtype=np.float64)).sum(axis=-1)
    for b in range(B):
        for h in range(H):
            X, V, G = qk[b, h], v[b, h], dO[b, h]
            for c in range(L // m):
                qi = np.arange(c * m, (c + 1) * m)
                kj = np.array(local_window(c, m, L, n_back, n_fwd))
                s = scale * (X[qi] @ X[kj].T)
                lq = LSE[b, h, qi]
                fin = np.isfinite(lq)
                valid = _valid(qi, kj, causal) & fin[:, None]
                with np.errstate(under="ignore"):
                    P = np.where(valid, np.exp(s - np.where(fin, lq, 0.0)[:, None]), 0.0)
                dS = P * (G[qi] @ V[kj].T - D[b, h, qi][:, None])
                dqk[b, h, qi] += scale * (dS @ X[kj])
                dqk[b, h, kj] += scale * (dS.T @ X[qi])
                dv[b, h, kj] += P.T @ G[qi]
            fb = ~np.isfinite(LSE[b, h])
            dv[b, h, fb] += G[fb]
    return dqk, dv
