"""Approximation error of LSH attention against full attention as the number
of hash rounds grows.

"Reformer: The Efficient Transformer" (research.elamur.ai summary page), Key
points, "Number of hash rounds": more rounds bring LSH attention closer to
full attention. For one input and rotations drawn for n_rounds rounds, this
runs the LSH forward (hash, sort, chunk attention, round combine) and full
attention with the same shared-QK self-mask (local attention whose window
covers the sequence) through the C ABI, and reports
||O_lsh - O_full|| / ||O_full|| (Frobenius, over all tokens).

Plumbing only: every attention step runs in liblsh.so; torch forms the norms.
"""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import torch

from .attention import LocalAttention, LSHAttention
from .workloads import Workload, generate


def full_attention(qk, v, chunk: int, causal: bool, scale: float, dtype: str):
    """Self-masked softmax attention over the whole sequence: local attention
    whose look-back covers every chunk."""
    B, H, L, d = qk.shape
    run = LocalAttention(B, H, L, chunk, L // chunk, L // chunk, causal, dtype, d, scale, qk.device)
    out, lse = run.forward(qk, v)
    return out.float().clone(), lse.clone()


def rounds_sweep(w: Workload, rounds: Iterable[int] = (1, 2, 4, 8), device="cuda",
                 seed: Optional[int] = None) -> Dict[int, float]:
    """Relative error of the LSH output against full attention for each
    number of hash rounds. Round r's rotation is the same in every run (the
    first r rotations of the largest run), so runs differ only by the
    rounds added."""
    rounds = sorted(set(int(r) for r in rounds))
    big = w.with_sizes(n_rounds=max(rounds))
    inp = generate(big, seed=seed, with_grad=False)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = torch.device(device)
    qk = torch.from_numpy(inp["qk"]).to(dev).to(td).contiguous()
    v = torch.from_numpy(inp["v"]).to(dev).to(td).contiguous()
    R_all = torch.from_numpy(inp["R"]).to(dev).to(td).contiguous()
    ref, _ = full_attention(qk, v, w.chunk, w.causal, w.scale, w.dtype)
    ref_norm = torch.linalg.vector_norm(ref.double())
    errs = {}
    for n_r in rounds:
        run = LSHAttention(w.B, w.H, w.L, w.n_buckets, n_r, w.chunk, w.causal, w.dtype, w.d,
                           w.scale, dev)
        out, _ = run.forward(qk, v, R_all[:n_r].contiguous())
        diff = torch.linalg.vector_norm((out.double() - ref.double()))
        errs[n_r] = float(diff / ref_norm)
    return errs
