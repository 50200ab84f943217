"""Failure paths of the CUDA library, made on the host and GPU-safe: no test
here faults, traps or hangs a GPU.

* values outside the fp16 range on the tensor-core path are reported as
  LSH_ERR_RANGE (the kernels check every result they write);
* an out-of-range position in `perm` is clamped by the attention kernels and
  reported as LSH_ERR_DEVICE_CHECK;
* a bounded wait that runs out records LSH_ERR_TIMEOUT (through the health
  check that waits on a barrier nothing completes);
and after each, the next call runs cleanly."""
import numpy as np
import pytest

from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate

OK, TIMEOUT, DEVICE_CHECK, RANGE = 0, 5, 6, 7
W = WORKLOADS["batch-bf16-8x8x4096"].with_sizes(B=1, H=2, L=640, n_rounds=2, backward=True)


def _setup(w=W, dtype="bf16"):
    import torch
    from efficient_transformer_lsh_b200.attention import LSHAttention
    inp = generate(w)
    dev = torch.device("cuda")
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = {k: torch.from_numpy(a).to(dev).to(td).contiguous() for k, a in inp.items()}
    run = LSHAttention(w.B, w.H, w.L, w.n_buckets, w.n_rounds, w.chunk, w.causal, dtype)
    return run, t


def _status():
    from efficient_transformer_lsh_b200 import _lib
    return _lib.lsh_device_status()


def _clean_call(run, t):
    run.forward(t["qk"], t["v"], t["R"])
    run.backward(t["qk"], t["v"], t["dO"])
    assert _status() == OK


@pytest.mark.gpu
def test_v_outside_fp16_range_is_reported_by_forward():
    run, t = _setup()
    assert _status() == OK
    t["v"][0, 1, 100, :3] = 1e5           # a bf16 value the fp16 path cannot hold
    run.forward(t["qk"], t["v"], t["R"])
    assert _status() == RANGE
    t["v"][0, 1, 100, :3] = 0.5
    _clean_call(run, t)


@pytest.mark.gpu
def test_qk_outside_fp16_range_forward_exact_backward_reported():
    import torch
    run, t = _setup()
    _clean_call(run, t)
    out_ref = run.out.float().clone()
    # the forward's Q K^T runs on bf16 operands: a large qk entry is fine there
    t["qk"][0, 0, 200, 5] = 7.0e4
    run.forward(t["qk"], t["v"], t["R"])
    assert _status() == OK
    assert torch.isfinite(run.out.float()).all()
    # the backward's gradient products pass qk through fp16: reported
    run.backward(t["qk"], t["v"], t["dO"])
    assert _status() == RANGE
    t["qk"][0, 0, 200, 5] = 0.25
    _clean_call(run, t)
    assert out_ref.shape == run.out.shape


@pytest.mark.gpu
def test_dout_outside_fp16_range_is_reported_by_backward():
    run, t = _setup()
    run.forward(t["qk"], t["v"], t["R"])
    assert _status() == OK
    t["dO"][0, 0, 7, 63] = -1e5
    run.backward(t["qk"], t["v"], t["dO"])
    assert _status() == RANGE
    t["dO"][0, 0, 7, 63] = 1.0
    _clean_call(run, t)


@pytest.mark.gpu
def test_float32_inputs_take_the_cuda_core_path_without_range_limit():
    import torch
    run, t = _setup(dtype="f32")
    t["v"][0, 1, 100, :3] = 1e5
    run.forward(t["qk"], t["v"], t["R"])
    run.backward(t["qk"], t["v"], t["dO"])
    assert _status() == OK
    assert torch.isfinite(run.out).all() and torch.isfinite(run.dv).all()


@pytest.mark.gpu
@pytest.mark.parametrize("bad", [-1, 640, 1 << 30])
def test_out_of_range_perm_is_clamped_and_reported(bad):
    import torch
    run, t = _setup()
    run.hash(t["qk"], t["R"])
    run.sort()
    perm = run.perm.clone()
    perm[0, 1, 1, 77] = bad
    run.attend(t["qk"], t["v"], perm)
    assert _status() == DEVICE_CHECK
    assert _status() == OK                 # cleared by the read
    run.backward(t["qk"], t["v"], t["dO"], perm)
    assert _status() == DEVICE_CHECK
    _clean_call(run, t)


@pytest.mark.gpu
def test_bounded_wait_times_out_and_context_stays_usable():
    from efficient_transformer_lsh_b200 import _lib
    run, t = _setup()
    _lib.lsh_check_wait_timeout(20_000)    # 20 us on a barrier nothing completes
    assert _status() == TIMEOUT
    assert _status() == OK
    _clean_call(run, t)
    # the first recorded error is the one reported
    _lib.lsh_check_wait_timeout(5_000)
    perm = run.perm.clone()
    perm[0, 0, 0, 3] = -5
    run.attend(t["qk"], t["v"], perm)
    assert _status() == TIMEOUT
    _clean_call(run, t)
