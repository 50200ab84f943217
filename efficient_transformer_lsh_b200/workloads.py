"""Seeded synthetic workloads for LSH self-attention.

This module only draws random numbers and rounds them to the input dtype.
It holds none of the attention arithmetic, so the CUDA path and the CPU
oracle can both take their inputs from it without sharing any of the method.

Recipe (one per named workload):
  * generator: numpy PCG64; every array of every (batch, head) slice has its
    own stream, seeded by SeedSequence([seed, array id, slice index]) with
    ``seed = 20200 + index``, so any contiguous range of slices (one rank's
    shard of a problem) can be drawn on its own and equals the same slices
    of the whole problem; R and the mixture's cluster centres have streams
    of their own;
  * values are drawn in float64 and rounded once to the input dtype
    (round-to-nearest-even); bf16 values are returned as float32 arrays whose
    values are exactly representable in bf16, so widening them is exact;
  * qk, v, dO have shape [B, H, L, d]; R has shape [n_rounds, d, n_buckets/2]
    (one random rotation per hash round, shared by every batch and head);
  * ``qk="mixture"`` draws 256 cluster centres ~ N(0, I) (shared by all
    slices) and gives every token a uniformly chosen centre plus
    N(0, 0.1^2) noise, which makes bucket occupancy uneven the way real text
    does; every other array is N(0, 1).

The sizes mirror the experiments named on the Reformer pages (64K-token
enwik8, 12K-token imagenet-64, half-million-token sequences); the datasets
themselves are not used: these synthetic arrays stand in for them.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    dtype: str          # "f32" or "bf16"
    B: int
    H: int
    L: int
    d: int
    n_buckets: int
    chunk: int
    n_rounds: int
    causal: bool
    backward: bool
    qk: str = "normal"  # "normal" or "mixture"
    n_clusters: int = 256
    cluster_sigma: float = 0.1

    @property
    def tokens(self) -> int:
        """Tokens per call, B*L (the unit of the tokens/s metric)."""
        return self.B * self.L

    @property
    def rows(self) -> int:
        """Token-heads, B*H*L."""
        return self.B * self.H * self.L

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))

    def with_sizes(self, **kw) -> "Workload":
        """Same recipe at other sizes (parity cases the oracle finishes in seconds)."""
        return dataclasses.replace(self, **kw)

    def describe(self) -> Dict[str, object]:
        return {
            "workload": self.name, "dtype": self.dtype, "B": self.B, "H": self.H,
            "L": self.L, "d_head": self.d, "n_buckets": self.n_buckets,
            "chunk": self.chunk, "n_rounds": self.n_rounds, "causal": self.causal,
            "pass": "fwd+bwd" if self.backward else "fwd", "qk": self.qk,
        }


WORKLOADS: Dict[str, Workload] = {
    w.name: w for w in [
        Workload("toy-f32-L1024", 1, "f32", 1, 1, 1024, 64, 32, 64, 1, False, False),
        Workload("toy-f32-L1024-fullchunk", 1, "f32", 1, 1, 1024, 64, 32, 1024, 1, False, False),
        Workload("batch-bf16-8x8x4096", 2, "bf16", 8, 8, 4096, 64, 64, 64, 2, True, False),
        Workload("enwik8-64k-bf16", 3, "bf16", 1, 8, 65536, 64, 1024, 64, 4, True, True,
                 qk="mixture"),
        Workload("imagenet64-12k-bf16", 4, "bf16", 4, 8, 12288, 64, 192, 64, 8, True, True),
        Workload("halfmillion-bf16", 5, "bf16", 1, 2, 524288, 64, 8192, 64, 1, True, False),
    ]
}

# The throughput workload: 64K tokens, 8 heads, 4 hash rounds, forward + backward.
HEADLINE = "enwik8-64k-bf16"


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float64/float32 values to the nearest bf16 (ties to even).

    Returns float32 holding exactly representable bf16 values.
    """
    f = np.ascontiguousarray(a, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    bits = (bits + 0x7FFF + ((bits >> 16) & 1)) & 0xFFFF0000
    return bits.astype(np.uint32).view(np.float32)


def _to_dtype(a: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return a.astype(np.float32)
    if dtype == "bf16":
        return round_to_bf16(a)
    raise ValueError(dtype)


_QK, _V, _DO, _R, _CENTRES = 0, 1, 2, 3, 4
_W1, _B1, _W2, _B2, _DY1 = 5, 6, 7, 8, 9


def _stream(seed: int, array: int, k: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, array, k])))


def generate_slices(w: Workload, lo: int, hi: int, seed: Optional[int] = None,
                    with_grad: Optional[bool] = None):
    """Draw the (batch, head) slices [lo, hi) of workload ``w`` (flattened
    index b * H + h). Returns qk, v (and dO) of shape [hi - lo, L, d] and R."""
    if seed is None:
        seed = 20200 + w.index
    if with_grad is None:
        with_grad = w.backward
    n = hi - lo
    shape = (n, w.L, w.d)
    out = {}
    if w.qk == "mixture":
        centres = _stream(seed, _CENTRES).standard_normal((w.n_clusters, w.d))
    qk = np.empty(shape)
    for i, k in enumerate(range(lo, hi)):
        g = _stream(seed, _QK, k)
        if w.qk == "mixture":
            assign = g.integers(0, w.n_clusters, size=w.L)
            qk[i] = centres[assign] + w.cluster_sigma * g.standard_normal((w.L, w.d))
        elif w.qk == "normal":
            qk[i] = g.standard_normal((w.L, w.d))
        else:
            raise ValueError(w.qk)
    out["qk"] = _to_dtype(qk, w.dtype)
    del qk
    out["v"] = _to_dtype(np.stack([_stream(seed, _V, k).standard_normal((w.L, w.d))
                                   for k in range(lo, hi)]) if n else np.empty(shape), w.dtype)
    out["R"] = _to_dtype(_stream(seed, _R).standard_normal((w.n_rounds, w.d, w.n_buckets // 2)),
                         w.dtype)
    if with_grad:
        out["dO"] = _to_dtype(np.stack([_stream(seed, _DO, k).standard_normal((w.L, w.d))
                                        for k in range(lo, hi)]) if n else np.empty(shape),
                              w.dtype)
    return out


def generate(w: Workload, seed: Optional[int] = None, with_grad: Optional[bool] = None):
    """Draw the inputs of workload ``w``.

    Returns a dict of float32 numpy arrays: qk, v, R and (when a backward pass
    is wanted) dO. Values are exactly representable in ``w.dtype``.
    """
    out = generate_slices(w, 0, w.B * w.H, seed, with_grad)
    for k in ("qk", "v", "dO"):
        if k in out:
            out[k] = out[k].reshape(w.B, w.H, w.L, w.d)
    return out


# The reversible block around the attention (one Reformer layer) on a workload:
# d_model = 64 H, a feed-forward of width 4 d_model run ff_chunk positions at a
# time.
BLOCK_FF = {"enwik8-64k-bf16": dict(d_ff=2048, ff_chunk=8192)}


def generate_block(w: Workload, d_ff: int, seed: Optional[int] = None):
    """Inputs of the reversible block on workload ``w`` (bf16): x2 = the
    workload's qk (so the hash sees its bucket structure), x1 = its v,
    dy2 = its dO, dy1 ~ N(0, 1), all [B, H, L, d]; R as drawn; W1 [64 H, d_ff]
    ~ N(0, 1/(64 H)), W2 [d_ff, 64 H] ~ N(0, 1/d_ff) (bf16) and b1, b2 ~
    N(0, 0.1^2) (float32)."""
    if seed is None:
        seed = 20200 + w.index
    base = generate(w, seed, with_grad=True)
    D = w.H * w.d
    out = {"x1": base["v"], "x2": base["qk"], "R": base["R"], "dy2": base["dO"]}
    out["dy1"] = round_to_bf16(np.stack([_stream(seed, _DY1, k).standard_normal((w.L, w.d))
                                         for k in range(w.B * w.H)])).reshape(w.B, w.H, w.L, w.d)
    out["W1"] = round_to_bf16(_stream(seed, _W1).standard_normal((D, d_ff)) / np.sqrt(D))
    out["W2"] = round_to_bf16(_stream(seed, _W2).standard_normal((d_ff, D)) / np.sqrt(d_ff))
    out["b1"] = (0.1 * _stream(seed, _B1).standard_normal(d_ff)).astype(np.float32)
    out["b2"] = (0.1 * _stream(seed, _B2).standard_normal(D)).astype(np.float32)
    return out
