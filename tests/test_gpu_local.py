"""GPU parity of local chunked attention (lsh_local_attn_fwd / _bwd) against
the oracle's local_forward / local_backward, element by element.

Source: "The Reformer - Pushing the limits of language modeling" (yomu.fyi
summary of the Hugging Face blog post), Approach and Takeaways: chunks of
length l_c with overlap from preceding and following chunks. Look-back 1 /
look-ahead 0 on bf16 chunk-64 problems runs on the tensor-core kernels;
every other window on the CUDA-core kernels."""
import numpy as np
import pytest

from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
from oracle import lsh_oracle as orc

TOL = {"f32": 1e-4, "bf16": 2e-2}
BASE = WORKLOADS["batch-bf16-8x8x4096"]

CASES = {
    # name: (dtype, B, H, L, chunk, n_back, n_fwd, causal)
    "tc-causal-b1f0": ("bf16", 1, 2, 1472, 64, 1, 0, True),
    "tc-noncausal-b1f0": ("bf16", 2, 1, 1728, 64, 1, 0, False),
    "simt-bf16-b2f1": ("bf16", 1, 2, 1216, 64, 2, 1, True),
    "simt-bf16-m128-b1f1": ("bf16", 1, 1, 1664, 128, 1, 1, False),
    "simt-f32-b0f1": ("f32", 1, 2, 960, 64, 0, 1, False),
    "simt-f32-b0f0-causal": ("f32", 1, 1, 640, 64, 0, 0, True),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_local_parity(name):
    import torch
    from efficient_transformer_lsh_b200 import _lib
    from efficient_transformer_lsh_b200.attention import LocalAttention
    dtype, B, H, L, m, nb, nf, causal = CASES[name]
    w = BASE.with_sizes(dtype=dtype, B=B, H=H, L=L, chunk=m, n_rounds=1, causal=causal,
                        backward=True)
    inp = generate(w)
    f = {k: a.astype(np.float64) for k, a in inp.items()}
    O, LSE = orc.local_forward(f["qk"], f["v"], m, nb, nf, causal, w.scale)
    dqk, dv = orc.local_backward(f["qk"], f["v"], m, nb, nf, causal, w.scale, O, LSE, f["dO"])
    dev = torch.device("cuda")
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = {k: torch.from_numpy(a).to(dev).to(td).contiguous() for k, a in inp.items()}
    run = LocalAttention(B, H, L, m, nb, nf, causal, dtype, 64, w.scale, dev)
    out, lse = run.forward(t["qk"], t["v"])
    g_dqk, g_dv = run.backward(t["qk"], t["v"], t["dO"])
    torch.cuda.synchronize()
    assert _lib.lsh_device_status() == 0
    tol = TOL[dtype]
    lse_g = lse.cpu().numpy()
    fin = np.isfinite(LSE)
    assert np.array_equal(np.isfinite(lse_g), fin)
    err = {"O": np.abs(out.float().cpu().numpy() - O).max(),
           "lse": np.abs(lse_g[fin] - LSE[fin]).max() if fin.any() else 0.0,
           "dqk": np.abs(g_dqk.cpu().numpy() - dqk).max(),
           "dv": np.abs(g_dv.cpu().numpy() - dv).max()}
    print(name, err)
    for k, e in err.items():
        assert e <= tol, f"{name}: {k} err {e}"
