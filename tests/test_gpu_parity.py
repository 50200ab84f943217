"""GPU parity against the oracle at sizes the oracle finishes in seconds.

Each case keeps a workload's recipe (dtype, bucket count, rounds, causal,
value distribution) at smaller B, H, L, chosen to span several tiles of every
kernel and to leave ragged tails: odd chunk counts, partial sort tiles,
token counts that are not multiples of the hashing tile.
"""
import numpy as np
import pytest

from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
from parity_common import compare, gpu_run, oracle_run

W = WORKLOADS

CASES = {
    # float32 (CUDA-core path), several rounds, causal, backward
    "f32-causal-3rounds": W["toy-f32-L1024"].with_sizes(B=1, H=2, L=1472, n_buckets=24,
                                                         n_rounds=3, causal=True, backward=True),
    "f32-toy-full": W["toy-f32-L1024"].with_sizes(backward=True),
    "f32-toy-fullchunk": W["toy-f32-L1024-fullchunk"].with_sizes(backward=True),
    # bf16 recipes
    "batch-small": W["batch-bf16-8x8x4096"].with_sizes(B=2, H=2, L=1472, backward=True),
    "enwik8-small": W["enwik8-64k-bf16"].with_sizes(H=2, L=4160),
    "imagenet-small": W["imagenet64-12k-bf16"].with_sizes(B=2, H=2, L=1536),
    "halfmillion-small": W["halfmillion-bf16"].with_sizes(H=1, L=8256, backward=True),
    # non-causal, chunk 128, odd chunk count
    "bf16-noncausal-m128": W["batch-bf16-8x8x4096"].with_sizes(B=1, H=3, L=1664, chunk=128,
                                                                causal=False, backward=True),
    # single chunk per sequence (m = L): full attention with the self-mask
    "bf16-one-chunk": W["batch-bf16-8x8x4096"].with_sizes(B=1, H=2, L=256, chunk=256,
                                                           n_rounds=1, backward=True),
    # smallest bucket count, one chunk of 64
    "bf16-two-buckets": W["batch-bf16-8x8x4096"].with_sizes(B=1, H=1, L=64, n_buckets=2,
                                                             backward=True),
}


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(CASES))
def test_parity_small(name):
    w = CASES[name]
    inp = generate(w)
    ref = oracle_run(w, inp, w.backward)
    got = gpu_run(w, inp, ref["bucket"], w.backward)
    compare(w, ref, got, w.backward, label=name)


@pytest.mark.gpu
def test_identical_tokens_all_in_one_bucket():
    # every token identical: one bucket, identity permutation, uniform weights
    w = W["batch-bf16-8x8x4096"].with_sizes(B=1, H=1, L=320, n_rounds=2, backward=True)
    inp = generate(w)
    inp["qk"][:] = inp["qk"][:, :, :1, :]
    ref = oracle_run(w, inp, True)
    for r in range(w.n_rounds):     # one bucket per round
        assert np.all(ref["bucket"][:, :, r] == ref["bucket"][0, 0, r, 0])
    got = gpu_run(w, inp, ref["bucket"], True)
    compare(w, ref, got, True, label="identical")


@pytest.mark.gpu
def test_out_of_range_bucket_is_reported_not_faulted():
    import torch
    from efficient_transformer_lsh_b200 import _lib
    from efficient_transformer_lsh_b200.attention import LSHAttention

    run = LSHAttention(1, 1, 128, 16, 1, 64, True, "bf16")
    bad = torch.zeros((1, 1, 1, 128), dtype=torch.int32, device="cuda")
    bad[0, 0, 0, 5] = 999
    run.sort(bad)
    assert _lib.lsh_device_status() == 6      # LSH_ERR_DEVICE_CHECK
    assert _lib.lsh_device_status() == 0      # cleared by the read
    run.sort(torch.zeros_like(bad))
    assert _lib.lsh_device_status() == 0


@pytest.mark.gpu
def test_launch_counter_moves():
    import torch
    from efficient_transformer_lsh_b200 import _lib
    w = CASES["bf16-two-buckets"]
    inp = generate(w)
    n0 = _lib.lsh_launch_count()
    ref = oracle_run(w, inp, True)
    gpu_run(w, inp, ref["bucket"], True)
    assert _lib.lsh_launch_count() > n0


@pytest.mark.gpu
def test_autograd_wrapper_matches_oracle():
    import torch
    from efficient_transformer_lsh_b200.attention import lsh_attention
    # one chunk spanning the sequence: the result does not depend on bucket ids
    w = CASES["bf16-one-chunk"]
    inp = generate(w)
    ref = oracle_run(w, inp, True)
    dev = torch.device("cuda")
    qk = torch.from_numpy(inp["qk"]).to(dev).to(torch.bfloat16).requires_grad_(True)
    v = torch.from_numpy(inp["v"]).to(dev).to(torch.bfloat16).requires_grad_(True)
    R = torch.from_numpy(inp["R"]).to(dev).to(torch.bfloat16)
    out, lse = lsh_attention(qk, v, R, w.n_buckets, w.chunk, w.causal, w.scale)
    (out.float() * torch.from_numpy(inp["dO"]).to(dev)).sum().backward()
    assert np.abs(out.detach().float().cpu().numpy() - ref["O"]).max() <= 2e-2
    # bf16 gradients: the tolerance includes one bf16 rounding of the result
    assert np.abs(qk.grad.float().cpu().numpy() - ref["dqk"]).max() <= 4e-2
    assert np.abs(v.grad.float().cpu().numpy() - ref["dv"]).max() <= 4e-2
