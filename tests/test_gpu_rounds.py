"""Hash-round sweep ("Reformer: The Efficient Transformer", Key points,
"Number of hash rounds": more rounds come closer to full attention).

The GPU sweep's relative errors against full attention equal the oracle's
(the oracle's LSH forward at each round count against its dense,
self-masked attention, on the same bucket ids); and on clustered inputs the
error falls as rounds are added."""
import numpy as np
import pytest

from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
from oracle import lsh_oracle as orc


@pytest.mark.gpu
def test_rounds_sweep_matches_oracle_and_falls():
    import torch
    from efficient_transformer_lsh_b200.rounds import rounds_sweep
    w = WORKLOADS["enwik8-64k-bf16"].with_sizes(H=2, L=2048, n_buckets=32, n_clusters=16)
    rounds = (1, 2, 4, 8)
    errs = rounds_sweep(w, rounds)
    big = w.with_sizes(n_rounds=8)
    inp = generate(big, with_grad=False)
    f = {k: a.astype(np.float64) for k, a in inp.items()}
    full, _ = orc.local_forward(f["qk"], f["v"], w.chunk, w.L // w.chunk, w.L // w.chunk,
                                w.causal, w.scale)
    for n_r in rounds:
        res = orc.lsh_attention(f["qk"], f["v"], f["R"][:n_r], w.chunk, w.causal, w.scale)
        e_or = np.linalg.norm(res["O"] - full) / np.linalg.norm(full)
        # bf16 outputs and near-tie bucket ids: the two sweeps agree to a
        # small fraction of the error itself
        assert abs(errs[n_r] - e_or) <= 0.02 * e_or + 2e-3, (n_r, errs[n_r], e_or)
    assert errs[8] < errs[4] < errs[2] < errs[1], errs
