"""Torch-facing driver of the C ABI: owns output and workspace buffers.

PyTorch only allocates device memory and provides streams here; every step
(hash, sort, chunk attention, round combine, backward) runs in liblsh.so.
"""
from __future__ import annotations

import math
from typing import Optional

import torch

from . import _lib

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


class LSHAttention:
    """Reformer LSH self-attention for one fixed problem shape.

    Buffers: bucket/perm [B,H,n_rounds,L] int32, out and out_lo [B,H,L,d]
    (input dtype; out_lo only for bf16), lse [B,H,L] float32, dqk/dv [B,H,L,d] float32, and the three workspaces.
    """

    def __init__(self, B, H, L, n_buckets, n_rounds, chunk, causal, dtype="bf16", d=64,
                 scale: Optional[float] = None, device="cuda"):
        self.dtype = dtype
        self.tdtype = _TORCH_DTYPE[dtype]
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        self.p = _lib.make_problem(B, H, L, d, n_buckets, n_rounds, chunk, causal, scale, dtype)
        self.shape = (B, H, L, d)
        dev = torch.device(device)
        i32 = dict(dtype=torch.int32, device=dev)
        self.bucket = torch.empty((B, H, n_rounds, L), **i32)
        self.perm = torch.empty((B, H, n_rounds, L), **i32)
        self.out = torch.empty(self.shape, dtype=self.tdtype, device=dev)
        # rounding residual of out (bf16 problems): keeps D = dout . O accurate
        self.out_lo = torch.empty(self.shape, dtype=self.tdtype, device=dev) if dtype == "bf16" \
            else None
        self.lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        self.dqk = torch.empty(self.shape, dtype=torch.float32, device=dev)
        self.dv = torch.empty(self.shape, dtype=torch.float32, device=dev)
        self.ws_sort_bytes = _lib.lsh_sort_workspace_size(self.p)
        self.ws_fwd_bytes = _lib.lsh_fwd_workspace_size(self.p)
        self.ws_bwd_bytes = _lib.lsh_bwd_workspace_size(self.p)
        if min(self.ws_sort_bytes, self.ws_fwd_bytes, self.ws_bwd_bytes) == 0 and B * H * L > 0:
            raise _lib.LshError(1, "workspace size query (problem rejected)")
        u8 = dict(dtype=torch.uint8, device=dev)
        self.ws_sort = torch.empty(max(1, self.ws_sort_bytes), **u8)
        self.ws_fwd = torch.empty(max(1, self.ws_fwd_bytes), **u8)
        self.ws_bwd = torch.empty(max(1, self.ws_bwd_bytes), **u8)

    def hash(self, qk, R, stream=None):
        _lib.lsh_hash(self.p, qk, R, self.bucket, stream)
        return self.bucket

    def sort(self, bucket=None, stream=None):
        _lib.lsh_sort(self.p, self.bucket if bucket is None else bucket, self.perm, self.ws_sort,
                      self.ws_sort_bytes, stream)
        return self.perm

    def attend(self, qk, v, perm=None, stream=None):
        _lib.lsh_attn_fwd(self.p, qk, v, self.perm if perm is None else perm, self.out,
                          self.out_lo, self.lse, self.ws_fwd, self.ws_fwd_bytes, stream)
        return self.out, self.lse

    def forward(self, qk, v, R, stream=None):
        """hash -> sort -> chunk attention + round combine. Returns (out, lse)."""
        self.hash(qk, R, stream)
        self.sort(None, stream)
        return self.attend(qk, v, None, stream)

    def backward(self, qk, v, dout, perm=None, stream=None):
        """Gradients of sum(out * dout) w.r.t. qk and v (float32)."""
        _lib.lsh_attn_bwd(self.p, qk, v, self.perm if perm is None else perm, self.out,
                          self.out_lo, self.lse, dout, self.dqk, self.dv, self.ws_bwd,
                          self.ws_bwd_bytes, stream)
        return self.dqk, self.dv


class LocalAttention:
    """Local chunked self-attention for one fixed shape: the queries of chunk c
    attend to chunks c - n_back .. c + n_fwd (identity order, shared qk with
    the self-mask). Buffers: out/out_lo [B,H,L,d], lse [B,H,L], dqk/dv
    [B,H,L,d] float32, and the two workspaces."""

    def __init__(self, B, H, L, chunk, n_back, n_fwd, causal, dtype="bf16", d=64,
                 scale: Optional[float] = None, device="cuda"):
        self.dtype = dtype
        self.tdtype = _TORCH_DTYPE[dtype]
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        self.n_back, self.n_fwd = int(n_back), int(n_fwd)
        self.p = _lib.make_problem(B, H, L, d, 2, 1, chunk, causal, scale, dtype)
        self.shape = (B, H, L, d)
        dev = torch.device(device)
        self.out = torch.empty(self.shape, dtype=self.tdtype, device=dev)
        self.out_lo = torch.empty(self.shape, dtype=self.tdtype, device=dev) if dtype == "bf16" \
            else None
        self.lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
        self.dqk = torch.empty(self.shape, dtype=torch.float32, device=dev)
        self.dv = torch.empty(self.shape, dtype=torch.float32, device=dev)
        self.ws_fwd_bytes = _lib.lsh_local_fwd_workspace_size(self.p, self.n_back, self.n_fwd)
        self.ws_bwd_bytes = _lib.lsh_local_bwd_workspace_size(self.p, self.n_back, self.n_fwd)
        if min(self.ws_fwd_bytes, self.ws_bwd_bytes) == 0 and B * H * L > 0:
            raise _lib.LshError(1, "workspace size query (problem rejected)")
        u8 = dict(dtype=torch.uint8, device=dev)
        self.ws_fwd = torch.empty(max(1, self.ws_fwd_bytes), **u8)
        self.ws_bwd = torch.empty(max(1, self.ws_bwd_bytes), **u8)

    def forward(self, qk, v, stream=None):
        _lib.lsh_local_attn_fwd(self.p, self.n_back, self.n_fwd, qk, v, self.out, self.out_lo,
                                self.lse, self.ws_fwd, self.ws_fwd_bytes, stream)
        return self.out, self.lse

    def backward(self, qk, v, dout, stream=None):
        _lib.lsh_local_attn_bwd(self.p, self.n_back, self.n_fwd, qk, v, self.out, self.out_lo,
                                self.lse, dout, self.dqk, self.dv, self.ws_bwd, self.ws_bwd_bytes,
                                stream)
        return self.dqk, self.dv


class ReversibleLSHBlock:
    """Reversible residual block y1 = x1 + F(x2), y2 = x2 + G(y1) with F the
    LSH attention of x2 (qk = v = x2) and G the chunked feed-forward
    max(0, x W1 + b1) W2 + b2, for one fixed shape. The backward rebuilds
    x1, x2 from y1, y2 (nothing of the forward is kept but the sort
    permutation). Activations and their gradients [B, H, L, 64] bf16
    (d_model = 64 H); W1 [64 H, d_ff], W2 [d_ff, 64 H] bf16; b1, b2 and the
    weight gradients float32."""

    def __init__(self, B, H, L, n_buckets, n_rounds, chunk, causal, d_ff, ff_chunk,
                 scale: Optional[float] = None, device="cuda"):
        if scale is None:
            scale = 1.0 / 8.0
        self.p = _lib.make_problem(B, H, L, 64, n_buckets, n_rounds, chunk, causal, scale, "bf16")
        self.f = _lib.make_ff_problem(B, H, L, d_ff, ff_chunk)
        self.shape = (B, H, L, 64)
        dev = torch.device(device)
        D = 64 * H
        self.perm = torch.empty((B, H, n_rounds, L), dtype=torch.int32, device=dev)
        self.y1 = torch.empty(self.shape, dtype=torch.bfloat16, device=dev)
        self.y2 = torch.empty_like(self.y1)
        self.x1 = torch.empty_like(self.y1)
        self.x2 = torch.empty_like(self.y1)
        self.dx1 = torch.empty_like(self.y1)
        self.dx2 = torch.empty_like(self.y1)
        f32 = dict(dtype=torch.float32, device=dev)
        self.dW1 = torch.empty((D, d_ff), **f32)
        self.db1 = torch.empty((d_ff,), **f32)
        self.dW2 = torch.empty((d_ff, D), **f32)
        self.db2 = torch.empty((D,), **f32)
        self.ws_fwd_bytes = _lib.lsh_rev_fwd_workspace_size(self.p, self.f)
        self.ws_bwd_bytes = _lib.lsh_rev_bwd_workspace_size(self.p, self.f)
        if min(self.ws_fwd_bytes, self.ws_bwd_bytes) == 0 and B * H * L > 0:
            raise _lib.LshError(1, "workspace size query (problem rejected)")
        u8 = dict(dtype=torch.uint8, device=dev)
        self.ws_fwd = torch.empty(max(1, self.ws_fwd_bytes), **u8)
        self.ws_bwd = torch.empty(max(1, self.ws_bwd_bytes), **u8)

    def forward(self, x1, x2, R, W1, b1, W2, b2, stream=None):
        _lib.lsh_rev_fwd(self.p, self.f, x1, x2, R, W1, b1, W2, b2, self.y1, self.y2, self.perm,
                         self.ws_fwd, self.ws_fwd_bytes, stream)
        return self.y1, self.y2

    def backward(self, y1, y2, dy1, dy2, W1, b1, W2, b2, stream=None):
        """Returns (x1, x2, dx1, dx2, dW1, db1, dW2, db2)."""
        _lib.lsh_rev_bwd(self.p, self.f, y1, y2, dy1, dy2, self.perm, W1, b1, W2, b2, self.x1,
                         self.x2, self.dx1, self.dx2, self.dW1, self.db1, self.dW2, self.db2,
                         self.ws_bwd, self.ws_bwd_bytes, stream)
        return self.x1, self.x2, self.dx1, self.dx2, self.dW1, self.db1, self.dW2, self.db2


class _LSHAttentionFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, qk, v, R, runner: LSHAttention):
        qk = qk.contiguous()
        v = v.contiguous()
        out, lse = runner.forward(qk, v, R.contiguous())
        ctx.runner = runner
        ctx.save_for_backward(qk, v)
        return out.clone(), lse.clone()

    @staticmethod
    def backward(ctx, dout, dlse):
        qk, v = ctx.saved_tensors
        dqk, dv = ctx.runner.backward(qk, v, dout.contiguous().to(qk.dtype))
        return dqk.to(qk.dtype), dv.to(v.dtype), None, None


def lsh_attention(qk: torch.Tensor, v: torch.Tensor, R: torch.Tensor, n_buckets: int, chunk: int,
                  causal: bool = True, scale: Optional[float] = None):
    """Autograd-aware LSH self-attention. qk, v: [B,H,L,d]; R: [n_rounds,d,n_buckets/2].

    Returns (out [B,H,L,d], lse [B,H,L]); gradients flow to qk and v (the
    gradient of lse is not propagated).
    """
    B, H, L, d = qk.shape
    dtype = {torch.float32: "f32", torch.bfloat16: "bf16"}[qk.dtype]
    runner = LSHAttention(B, H, L, n_buckets, R.shape[0], chunk, causal, dtype, d, scale,
                          qk.device)
    return _LSHAttentionFn.apply(qk, v, R, runner)
