"""GPU parity of the chunked feed-forward and the reversible block against the
float64 oracle, through the C ABI.

Sources: "Reformer: The Efficient Transformer" (research.elamur.ai summary
page), Key points, "Reversible layers" bullet: reversible residual layers
recompute a layer's inputs in the backward pass; the feed-forward runs in
chunks with unchanged results. The chunking claim is checked bit for bit.

Tolerances come from the arithmetic: the tensor-core products take bf16
operands exactly and accumulate in float32; the path rounds the hidden
activations h (and their gradient dh) to bf16 per chunk and every output to
bf16, each a relative error of at most 2^-9. So an output y = sum_j h_j W2_jk
+ ... may differ from the float64 value by 2^-8 |y| (its own rounding, with
margin) plus 2^-8 sum_j |h_j W2_jk| (the rounding of h), plus float32 noise.
"""
import math

import numpy as np
import pytest

from oracle import lsh_oracle as orc
from oracle import rev_ff_oracle as rev

pytestmark = pytest.mark.gpu

U = 2.0 ** -8          # a bf16 rounding (2^-9) with a factor 2 of margin


def _dev():
    import torch
    return torch.device("cuda")


def _bf(a):
    """Round to bf16 on the host (what the GPU receives), as float64."""
    import torch
    return torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16).to(
        torch.float64).numpy()


def _to(a, dtype):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(_dev()).to(dtype)


def _np(t):
    import torch
    return t.to(torch.float64).cpu().numpy()


def _weights(rng, D, dff):
    W1 = _bf(rng.standard_normal((D, dff)) / math.sqrt(D))
    b1 = (0.1 * rng.standard_normal(dff)).astype(np.float32).astype(np.float64)
    W2 = _bf(rng.standard_normal((dff, D)) / math.sqrt(dff))
    b2 = (0.1 * rng.standard_normal(D)).astype(np.float32).astype(np.float64)
    return W1, b1, W2, b2


def _ff_bound(x_tok, W1, b1, W2):
    """2^-8 sum_j |h_j W2_jk|: the effect of rounding the hidden layer."""
    h = np.maximum(x_tok @ W1 + b1, 0.0)
    return U * (np.abs(h) @ np.abs(W2))


def _ff_run(f, x, W, res=None):
    import torch
    from efficient_transformer_lsh_b200 import _lib
    W1, b1, W2, b2 = W
    n = _lib.lsh_ff_workspace_size(f)
    ws = torch.empty(n, dtype=torch.uint8, device=_dev())
    y = torch.empty_like(x)
    _lib.lsh_ff_fwd(f, x, _to(W1, torch.bfloat16), _to(b1, torch.float32), _to(W2, torch.bfloat16),
                    _to(b2, torch.float32), res, y, ws, n)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    return y


def _ff_bwd_run(f, x, W, dy, dres=None, y_in=None):
    import torch
    from efficient_transformer_lsh_b200 import _lib
    W1, b1, W2, b2 = W
    D, dff = W1.shape
    n = _lib.lsh_ff_workspace_size(f)
    ws = torch.empty(n, dtype=torch.uint8, device=_dev())
    dx = torch.empty_like(x)
    rec = torch.empty_like(x) if y_in is not None else None
    g = [torch.full(s, float("nan"), dtype=torch.float32, device=_dev())
         for s in ((D, dff), (dff,), (dff, D), (D,))]
    _lib.lsh_ff_bwd(f, x, _to(W1, torch.bfloat16), _to(b1, torch.float32), _to(W2, torch.bfloat16),
                    _to(b2, torch.float32), dy, dres, y_in, rec, dx, g[0], g[1], g[2], g[3], ws, n)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    return dx, rec, g


@pytest.mark.parametrize("B,H,L,dff,chunk", [
    (1, 2, 256, 256, 128),     # two chunks
    (2, 3, 384, 384, 256),     # odd H (64-wide N tiles), chunks across the batch edge, ragged tail
    (1, 1, 128, 128, 128),     # d_model 64: one K block, one 64-wide tile
    (2, 4, 256, 512, 384),     # d_model 256, ragged last chunk
])
def test_feed_forward_forward_matches_oracle(B, H, L, dff, chunk):
    import torch
    from efficient_transformer_lsh_b200 import _lib
    rng = np.random.default_rng(B * 1000 + H * 100 + L + dff)
    D = 64 * H
    x = _bf(rng.standard_normal((B, H, L, 64)))
    res = _bf(rng.standard_normal((B, H, L, 64)))
    W = _weights(rng, D, dff)
    f = _lib.make_ff_problem(B, H, L, dff, chunk)
    y = _np(_ff_run(f, _to(x, torch.bfloat16), W, _to(res, torch.bfloat16)))
    xt = rev.heads_to_tokens(x)
    ref = rev.heads_to_tokens(res) + rev.ff_forward(xt, *W)
    tol = U * np.abs(ref) + _ff_bound(xt, W[0], W[1], W[2]) + 1e-3
    err = np.abs(rev.heads_to_tokens(y) - ref)
    assert (err <= tol).all(), float((err - tol).max())


def test_feed_forward_chunking_is_bit_identical():
    """The pages' claim: chunking the feed-forward leaves the results unchanged.
    y, dx and the reconstruction are compared bit for bit across chunk sizes."""
    import torch
    from efficient_transformer_lsh_b200 import _lib
    rng = np.random.default_rng(7)
    B, H, L, dff = 2, 2, 512, 256
    x = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    res = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    dy = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    W = _weights(rng, 64 * H, dff)
    outs = []
    for chunk in (128, 384, B * L):
        f = _lib.make_ff_problem(B, H, L, dff, chunk)
        y = _ff_run(f, x, W, res)
        dx, rec, g = _ff_bwd_run(f, x, W, dy, dres=res, y_in=y)
        outs.append((y, dx, rec, g))
    y0, dx0, rec0, g0 = outs[0]
    for y, dx, rec, g in outs[1:]:
        assert torch.equal(y, y0) and torch.equal(dx, dx0) and torch.equal(rec, rec0)
        # weight gradients sum over chunks in chunk order: equal up to float32 rounding
        for a, b in zip(g, g0):
            assert torch.allclose(a, b, rtol=1e-4, atol=1e-3)


@pytest.mark.parametrize("B,H,L,dff,chunk", [
    (1, 2, 256, 256, 128),
    (2, 3, 384, 384, 256),
    (2, 2, 512, 256, 1024),    # 16 K blocks per weight-gradient product: split along K
])
def test_feed_forward_backward_matches_oracle(B, H, L, dff, chunk):
    import torch
    from efficient_transformer_lsh_b200 import _lib
    rng = np.random.default_rng(100 + H)
    D = 64 * H
    x = _bf(rng.standard_normal((B, H, L, 64)))
    dy = _bf(rng.standard_normal((B, H, L, 64)))
    dres = _bf(rng.standard_normal((B, H, L, 64)))
    y_in = _bf(rng.standard_normal((B, H, L, 64)))
    W = _weights(rng, D, dff)
    f = _lib.make_ff_problem(B, H, L, dff, chunk)
    dx, rec, g = _ff_bwd_run(f, _to(x, torch.bfloat16), W, _to(dy, torch.bfloat16),
                             dres=_to(dres, torch.bfloat16), y_in=_to(y_in, torch.bfloat16))
    xt, dyt = rev.heads_to_tokens(x), rev.heads_to_tokens(dy)
    rdx, rdW1, rdb1, rdW2, rdb2 = rev.ff_backward(xt, *W, dyt)
    W1, b1, W2, b2 = W
    pre = xt @ W1 + b1
    h = np.maximum(pre, 0.0)
    dh = (dyt @ W2.T) * (pre > 0)
    # reconstruction y_in - G(x)
    rrec = rev.heads_to_tokens(y_in) - rev.ff_forward(xt, *W)
    tol = U * np.abs(rrec) + _ff_bound(xt, W1, b1, W2) + 1e-3
    assert (np.abs(rev.heads_to_tokens(_np(rec)) - rrec) <= tol).all()
    # dx = dres + dh W1^T with dh rounded to bf16
    ref = rev.heads_to_tokens(dres) + rdx
    tol = U * np.abs(ref) + U * (np.abs(dh) @ np.abs(W1.T)) + 1e-3
    assert (np.abs(rev.heads_to_tokens(_np(dx)) - ref) <= tol).all()
    # weight and bias gradients: sums over tokens of bf16-rounded h / dh terms
    tW2 = U * (np.abs(h).T @ np.abs(dyt)) + 1e-3
    assert (np.abs(_np(g[2]) - rdW2) <= tW2).all()
    tW1 = U * (np.abs(xt).T @ np.abs(dh)) + 1e-3
    assert (np.abs(_np(g[0]) - rdW1) <= tW1).all()
    assert (np.abs(_np(g[1]) - rdb1) <= U * np.abs(dh).sum(0) + 1e-3).all()
    assert np.abs(_np(g[3]) - rdb2).max() <= 1e-3


def _block_inputs(seed, B, H, L, n_r, nb):
    rng = np.random.default_rng(seed)
    x1 = _bf(rng.standard_normal((B, H, L, 64)))
    x2 = _bf(rng.standard_normal((B, H, L, 64)))
    R = _bf(rng.standard_normal((n_r, 64, nb // 2)))
    dy1 = _bf(rng.standard_normal((B, H, L, 64)))
    dy2 = _bf(rng.standard_normal((B, H, L, 64)))
    return rng, x1, x2, R, dy1, dy2


@pytest.mark.parametrize("causal", [True, False])
def test_reversible_block_matches_oracle(causal):
    """Forward y1, y2 and backward (reconstructed x1, x2; dx1, dx2; weight
    gradients) of the block against the oracle, which is given the GPU's
    permutation (the hash and sort have their own bit-exact tests)."""
    import torch
    from efficient_transformer_lsh_b200 import _lib
    B, H, L, n_r, nb, m, dff = 1, 2, 512, 2, 16, 64, 256
    rng, x1, x2, R, dy1, dy2 = _block_inputs(3 + causal, B, H, L, n_r, nb)
    W = _weights(rng, 64 * H, dff)
    W1, b1, W2, b2 = W
    scale = 1.0 / 8.0
    p = _lib.make_problem(B, H, L, 64, nb, n_r, m, causal, scale, "bf16")
    f = _lib.make_ff_problem(B, H, L, dff, 256)
    bf, f32 = torch.bfloat16, torch.float32
    t = {k: _to(a, bf) for k, a in dict(x1=x1, x2=x2, R=R, dy1=dy1, dy2=dy2, W1=W1, W2=W2).items()}
    tb1, tb2 = _to(b1, f32), _to(b2, f32)
    y1 = torch.empty_like(t["x1"])
    y2 = torch.empty_like(t["x1"])
    perm = torch.empty((B, H, n_r, L), dtype=torch.int32, device=_dev())
    n = _lib.lsh_rev_fwd_workspace_size(p, f)
    ws = torch.empty(n, dtype=torch.uint8, device=_dev())
    _lib.lsh_rev_fwd(p, f, t["x1"], t["x2"], t["R"], t["W1"], tb1, t["W2"], tb2, y1, y2, perm,
                     ws, n)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    P = perm.cpu().numpy().astype(np.int64)
    for b in range(B):
        for h in range(H):
            for r in range(n_r):
                assert np.array_equal(np.sort(P[b, h, r]), np.arange(L))
    gy1, gy2 = _np(y1), _np(y2)
    # y1 = x1 + F(x2): the attention's own tolerance plus the rounding of y1
    O, _ = orc.forward(x2, x2, P, m, causal, scale)
    assert (np.abs(gy1 - (x1 + O)) <= 2e-2 + U * np.abs(x1 + O)).all()
    # y2 = x2 + G(y1), G applied to the GPU's y1
    yt = rev.heads_to_tokens(gy1)
    ry2 = rev.heads_to_tokens(x2) + rev.ff_forward(yt, *W)
    tol = U * np.abs(ry2) + _ff_bound(yt, W1, b1, W2) + 1e-3
    assert (np.abs(rev.heads_to_tokens(gy2) - ry2) <= tol).all()

    # backward from the GPU's outputs, against the oracle's backward from the same
    outs = {k: torch.empty_like(t["x1"]) for k in ("x1", "x2", "dx1", "dx2")}
    D = 64 * H
    g = [torch.full(s, float("nan"), dtype=f32, device=_dev())
         for s in ((D, dff), (dff,), (dff, D), (D,))]
    nb_ = _lib.lsh_rev_bwd_workspace_size(p, f)
    wsb = torch.empty(nb_, dtype=torch.uint8, device=_dev())
    _lib.lsh_rev_bwd(p, f, y1, y2, t["dy1"], t["dy2"], perm, t["W1"], tb1, t["W2"], tb2,
                     outs["x1"], outs["x2"], outs["dx1"], outs["dx2"], g[0], g[1], g[2], g[3],
                     wsb, nb_)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    rx1, rx2, rdx1, rdx2, rdW1, rdb1, rdW2, rdb2 = rev.rev_backward(
        gy1, gy2, dy1, dy2, P, m, causal, scale, W1, b1, W2, b2)
    tt = rev.heads_to_tokens
    # G half: reconstruction x2 = y2 - G(y1), dx1 = dy1 + (dG/dy1)^T dy2, weight gradients
    tol = U * np.abs(tt(rx2)) + _ff_bound(yt, W1, b1, W2) + 1e-3
    assert (np.abs(tt(_np(outs["x2"])) - tt(rx2)) <= tol).all()
    dyt = tt(dy2)
    pre = yt @ W1 + b1
    dh = (dyt @ W2.T) * (pre > 0)
    tol = U * np.abs(tt(rdx1)) + U * (np.abs(dh) @ np.abs(W1.T)) + 1e-3
    assert (np.abs(tt(_np(outs["dx1"])) - tt(rdx1)) <= tol).all()
    assert (np.abs(_np(g[2]) - rdW2) <= U * (np.maximum(pre, 0).T @ np.abs(dyt)) + 1e-3).all()
    assert (np.abs(_np(g[0]) - rdW1) <= U * (np.abs(yt).T @ np.abs(dh)) + 1e-3).all()
    assert (np.abs(_np(g[1]) - rdb1) <= U * np.abs(dh).sum(0) + 1e-3).all()
    assert np.abs(_np(g[3]) - rdb2).max() <= 1e-3
    # F half: x1 = y1 - F(x2), dx2 = dy2 + dqk + dv (the attention's tolerance, twice)
    assert (np.abs(_np(outs["x1"]) - rx1) <= 2e-2 + U * np.abs(rx1)).all()
    assert (np.abs(_np(outs["dx2"]) - rdx2) <= 4e-2 + U * np.abs(rdx2)).all()
    # and the inverse recovers the original inputs up to the roundings of y
    assert np.abs(_np(outs["x2"]) - x2).max() < 4 * U * max(1.0, np.abs(gy2).max())
    assert np.abs(_np(outs["x1"]) - x1).max() < 4 * U * max(1.0, np.abs(gy1).max()) + 2e-2


def test_feed_forward_outputs_only_16_byte_aligned_are_bit_identical():
    """Outputs 16-byte aligned but not 32 (the ABI's rule is 16): the GEMM
    epilogue then stores each 16-column piece with two 128-bit stores instead
    of one 256-bit store; y, dx, the reconstruction and the weight gradients
    must not change by a bit."""
    import torch
    from efficient_transformer_lsh_b200 import _lib
    rng = np.random.default_rng(11)
    B, H, L, dff, chunk = 2, 2, 512, 256, 1024     # the weight gradients split along K
    x = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    res = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    dy = _to(rng.standard_normal((B, H, L, 64)), torch.bfloat16)
    W = _weights(rng, 64 * H, dff)
    f = _lib.make_ff_problem(B, H, L, dff, chunk)
    y = _ff_run(f, x, W, res)
    dx, rec, g = _ff_bwd_run(f, x, W, dy, dres=res, y_in=y)

    def off16(shape, dtype):
        n = int(np.prod(shape))
        pad = 16 // torch.tensor([], dtype=dtype).element_size()
        t = torch.full((n + pad,), float("nan"), dtype=dtype, device=_dev())[pad:]
        assert t.data_ptr() % 32 == 16
        return t.view(shape)

    W1, b1, W2, b2 = W
    Wd = (_to(W1, torch.bfloat16), _to(b1, torch.float32), _to(W2, torch.bfloat16),
          _to(b2, torch.float32))
    n = _lib.lsh_ff_workspace_size(f)
    ws = torch.empty(n, dtype=torch.uint8, device=_dev())
    y2 = off16(x.shape, torch.bfloat16)
    _lib.lsh_ff_fwd(f, x, *Wd, res, y2, ws, n)
    dx2, rec2 = off16(x.shape, torch.bfloat16), off16(x.shape, torch.bfloat16)
    g2 = [off16(t.shape, torch.float32) for t in g]
    _lib.lsh_ff_bwd(f, x, *Wd, dy, res, y, rec2, dx2, g2[0], g2[1], g2[2], g2[3], ws, n)
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    assert torch.equal(y2, y) and torch.equal(dx2, dx) and torch.equal(rec2, rec)
    for a, b in zip(g2, g):
        assert torch.equal(a, b)
