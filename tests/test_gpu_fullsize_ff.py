"""The chunked feed-forward at the full size the benchmark times (the 64K
workload's 8 heads as d_model 512, d_ff 2048, 8192 positions per chunk),
through the same C-ABI calls, against the float64 oracle on sampled outputs:
token rows of y, dx and the reconstruction, hidden units of dW1, db1 and dW2
(each needs only its own column of the hidden layer), and all of db2.

Source: "Reformer: The Efficient Transformer" (research.elamur.ai summary
page), Key points, "Reversible layers" bullet: the feed-forward runs chunk by
chunk. Tolerances as in test_gpu_reversible: bf16 roundings of h, dh and of
each output (2^-8 with margin) plus float32 accumulation.
"""
import numpy as np
import pytest

from efficient_transformer_lsh_b200.workloads import BLOCK_FF, WORKLOADS, generate_block
from oracle import rev_ff_oracle as rev

pytestmark = pytest.mark.gpu

U = 2.0 ** -8


def test_feed_forward_full_size_sampled():
    import torch
    from efficient_transformer_lsh_b200 import _lib

    w = WORKLOADS["enwik8-64k-bf16"]
    cfg = BLOCK_FF[w.name]
    d_ff, chunk = cfg["d_ff"], cfg["ff_chunk"]
    inp = generate_block(w, d_ff)
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(a).to(dev).to(torch.float32 if k in ("b1", "b2") else torch.bfloat16)
         for k, a in inp.items()}
    f = _lib.make_ff_problem(w.B, w.H, w.L, d_ff, chunk)
    n = _lib.lsh_ff_workspace_size(f)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    W = (t["W1"], t["b1"], t["W2"], t["b2"])
    D = w.H * w.d
    # y = x2 + G(x1), then the backward with dy = dy2, dres = dy1, y_in = y
    y = torch.empty_like(t["x1"])
    _lib.lsh_ff_fwd(f, t["x1"], *W, t["x2"], y, ws, n)
    rec, dx = torch.empty_like(y), torch.empty_like(y)
    g = [torch.full(s, float("nan"), dtype=torch.float32, device=dev)
         for s in ((D, d_ff), (d_ff,), (d_ff, D), (D,))]
    _lib.lsh_ff_bwd(f, t["x1"], *W, t["dy2"], t["dy1"], y, rec, dx, *g, ws, n)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0

    def tok(a):
        return rev.heads_to_tokens(np.asarray(a, dtype=np.float64))

    def gpu_tok(x):
        return tok(x.to(torch.float64).cpu().numpy())

    X, RES, DY, DRES = tok(inp["x1"]), tok(inp["x2"]), tok(inp["dy2"]), tok(inp["dy1"])
    W1, W2 = inp["W1"].astype(np.float64), inp["W2"].astype(np.float64)
    b1, b2 = inp["b1"].astype(np.float64), inp["b2"].astype(np.float64)
    Y, REC, DX = gpu_tok(y), gpu_tok(rec), gpu_tok(dx)
    T = X.shape[0]
    rng = np.random.default_rng(5)
    # token rows: both ends of every chunk plus random ones
    rows = np.unique(np.concatenate([np.arange(0, T, chunk), np.arange(chunk - 1, T, chunk),
                                     rng.choice(T, 240, replace=False)]))
    x = X[rows]
    pre = x @ W1 + b1
    h = np.maximum(pre, 0.0)
    bound = U * (h @ np.abs(W2))
    ref_y = RES[rows] + h @ W2 + b2
    assert (np.abs(Y[rows] - ref_y) <= U * np.abs(ref_y) + bound + 1e-3).all()
    ref_rec = Y[rows] - (h @ W2 + b2)
    assert (np.abs(REC[rows] - ref_rec) <= U * np.abs(ref_rec) + bound + 1e-3).all()
    dh = (DY[rows] @ W2.T) * (pre > 0)
    ref_dx = DRES[rows] + dh @ W1.T
    assert (np.abs(DX[rows] - ref_dx) <= U * np.abs(ref_dx) + U * (np.abs(dh) @ np.abs(W1.T))
            + 1e-3).all()

    # hidden units J: their column of h and dh over all 65536 positions
    J = np.unique(np.concatenate([[0, d_ff - 1], rng.choice(d_ff, 30, replace=False)]))
    preJ = X @ W1[:, J] + b1[J]
    hJ = np.maximum(preJ, 0.0)
    dhJ = (DY @ W2[J].T) * (preJ > 0)
    dW1, db1, dW2, db2 = (x_.double().cpu().numpy() for x_ in g)
    assert (np.abs(dW2[J] - hJ.T @ DY) <= U * (hJ.T @ np.abs(DY)) + 1e-3).all()
    assert (np.abs(dW1[:, J] - X.T @ dhJ) <= U * (np.abs(X).T @ np.abs(dhJ)) + 1e-3).all()
    assert (np.abs(db1[J] - dhJ.sum(0)) <= U * np.abs(dhJ).sum(0) + 1e-3).all()
    # db2 = sum of the bf16 dy over all positions, added in float32
    assert (np.abs(db2 - DY.sum(0)) <= 2.0 ** -14 * np.abs(DY).sum(0) + 1e-3).all()
