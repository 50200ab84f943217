"""Shared helpers for the GPU-vs-oracle parity tests.

The oracle and the CUDA path get the same seeded host arrays. Bucket ids must
match exactly except where the oracle's top two rotated scores differ by less
than 1e-5 relative (near-ties, counted and reported); the oracle's bucket ids
then feed the GPU sort, so every later comparison sees the same permutation.
Tolerances (max-abs): 1e-4 for float32 problems, 2e-2 for bf16 inputs with
float32 accumulation.
"""
from __future__ import annotations

import numpy as np

from oracle import lsh_oracle as orc

TOL = {"f32": 1e-4, "bf16": 2e-2}
NEAR_TIE = 1e-5


def oracle_run(w, inp, backward):
    qk = inp["qk"].astype(np.float64)
    v = inp["v"].astype(np.float64)
    R = inp["R"].astype(np.float64)
    bucket, gap = orc.hash_buckets(qk, R)
    perm = orc.sort_positions(bucket)
    O, LSE = orc.forward(qk, v, perm, w.chunk, w.causal, w.scale)
    res = {"bucket": bucket, "gap": gap, "perm": perm, "O": O, "LSE": LSE}
    if backward:
        dO = inp["dO"].astype(np.float64)
        res["dqk"], res["dv"] = orc.backward(qk, v, perm, w.chunk, w.causal, w.scale, O, LSE, dO)
    return res


def gpu_run(w, inp, bucket_for_sort, backward):
    """Runs the CUDA path through the C ABI. Returns numpy arrays."""
    import torch
    from efficient_transformer_lsh_b200 import _lib
    from efficient_transformer_lsh_b200.attention import LSHAttention

    dev = torch.device("cuda")
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def put(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(td).contiguous()

    qk, v, R = put(inp["qk"]), put(inp["v"]), put(inp["R"])
    run = LSHAttention(w.B, w.H, w.L, w.n_buckets, w.n_rounds, w.chunk, w.causal, w.dtype, w.d,
                       w.scale, dev)
    gpu_bucket = run.hash(qk, R).clone()
    ob = torch.from_numpy(bucket_for_sort.astype(np.int32)).to(dev)
    perm = run.sort(ob).clone()
    out, lse = run.attend(qk, v, perm)
    res = {"bucket": gpu_bucket, "perm": perm, "O": out.float().clone(), "LSE": lse.clone()}
    # the GPU's own buckets through the GPU sort (checked by properties)
    run.sort(gpu_bucket)
    res["perm_own"] = run.perm.clone()
    if backward:
        dO = put(inp["dO"])
        run.attend(qk, v, perm)
        dqk, dv = run.backward(qk, v, dO, perm)
        res["dqk"], res["dv"] = dqk.clone(), dv.clone()
    torch.cuda.synchronize()
    status = _lib.lsh_device_status()
    assert status == 0, f"device status {status}"
    return {k: t.cpu().numpy() for k, t in res.items()}


def check_sorted_by(perm, bucket):
    """perm is, per segment, the stable sort of positions by bucket."""
    L = perm.shape[-1]
    P = perm.reshape(-1, L)
    Bk = bucket.reshape(-1, L)
    for s in range(P.shape[0]):
        p = P[s]
        assert np.array_equal(np.sort(p), np.arange(L))
        kb = Bk[s][p]
        assert np.all(np.diff(kb) >= 0)
        same = np.diff(kb) == 0
        assert np.all(np.diff(p)[same] > 0)


def compare(w, ref, got, backward, label=""):
    tol = TOL[w.dtype]
    report = {}
    # bucket ids: exact outside near-ties
    near = ref["gap"] < NEAR_TIE
    mism = ref["bucket"] != got["bucket"]
    bad = mism & ~near
    report["near_ties"] = int(near.sum())
    report["near_tie_mismatches"] = int((mism & near).sum())
    assert not bad.any(), f"{label}: {int(bad.sum())} bucket ids differ outside near-ties"
    # sort: bit-exact on the oracle's bucket ids; valid on the GPU's own ids
    assert np.array_equal(got["perm"], ref["perm"]), f"{label}: perm differs"
    check_sorted_by(got["perm_own"], got["bucket"])
    # forward
    fin = np.isfinite(ref["LSE"])
    assert np.array_equal(np.isfinite(got["LSE"]), fin), f"{label}: -inf pattern of lse differs"
    report["lse_err"] = float(np.abs(got["LSE"][fin] - ref["LSE"][fin]).max()) if fin.any() else 0.0
    report["O_err"] = float(np.abs(got["O"] - ref["O"]).max())
    assert report["lse_err"] <= tol, f"{label}: lse err {report['lse_err']}"
    assert report["O_err"] <= tol, f"{label}: O err {report['O_err']}"
    if backward:
        report["dqk_err"] = float(np.abs(got["dqk"] - ref["dqk"]).max())
        report["dv_err"] = float(np.abs(got["dv"] - ref["dv"]).max())
        assert report["dqk_err"] <= tol, f"{label}: dqk err {report['dqk_err']}"
        assert report["dv_err"] <= tol, f"{label}: dv err {report['dv_err']}"
    print(label, report)
    return report
