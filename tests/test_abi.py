"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from efficient_transformer_lsh_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "lsh.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(lsh_[a-z_0-9]+)\s*\(", src)))


def _ensure_built():
    if not os.path.exists(_lib.LIB_PATH):
        from efficient_transformer_lsh_b200 import build
        build.build()


def test_library_exports_every_declared_symbol():
    _ensure_built()
    L = _lib.lib()
    declared = _declared_symbols()
    assert set(declared) == set(_lib.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name


def test_status_strings():
    _ensure_built()
    for code in range(8):
        assert _lib.status_string(code)
    assert "fp16" in _lib.status_string(7)
    assert _lib.status_string(0) == "ok"


def _p(**kw):
    base = dict(B=1, H=2, L=256, d=64, n_buckets=16, n_rounds=2, chunk=64, causal=1,
                scale=0.125, dtype=1)
    base.update(kw)
    # raw struct: no normalisation of the fields, so bad values reach the library
    return _lib.lsh_problem(*[base[k] for k, _ in _lib.lsh_problem._fields_])


FAKE = 1 << 20  # non-null, 256-aligned fake address: never dereferenced on the host


@pytest.mark.parametrize("kw,code", [
    (dict(d=32), 2), (dict(d=0), 1), (dict(n_buckets=15), 1), (dict(n_buckets=0), 1),
    (dict(n_buckets=65538), 1), (dict(n_rounds=0), 1), (dict(n_rounds=65), 1),
    (dict(chunk=0), 1), (dict(L=250), 1), (dict(chunk=32, L=256), 2), (dict(causal=2), 1),
    (dict(scale=float("inf")), 1), (dict(dtype=7), 1), (dict(B=-1), 1),
])
def test_bad_problem_rejected_before_launch(kw, code):
    _ensure_built()
    L = _lib.lib()
    p = _p(**kw)
    r = L.lsh_hash(ctypes.byref(p), FAKE, FAKE, FAKE, None)
    assert r == code
    assert L.lsh_sort_workspace_size(ctypes.byref(p)) == 0
    assert L.lsh_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 1 << 30,
                          None) == code


def test_null_pointers_and_workspace_rejected():
    _ensure_built()
    L = _lib.lib()
    p = _p()
    assert L.lsh_hash(None, FAKE, FAKE, FAKE, None) == 1
    assert L.lsh_hash(ctypes.byref(p), None, FAKE, FAKE, None) == 1
    assert L.lsh_hash(ctypes.byref(p), FAKE + 8, FAKE, FAKE, None) == 1   # misaligned qk
    need = L.lsh_sort_workspace_size(ctypes.byref(p))
    assert need > 0
    assert L.lsh_sort(ctypes.byref(p), FAKE, FAKE, FAKE, need - 1, None) == 3
    assert L.lsh_sort(ctypes.byref(p), FAKE, FAKE, None, need, None) == 3
    assert L.lsh_sort(ctypes.byref(p), FAKE, FAKE, FAKE + 16, need, None) == 3
    assert L.lsh_sort(ctypes.byref(p), None, FAKE, FAKE, need, None) == 1
    nf = L.lsh_fwd_workspace_size(ctypes.byref(p))
    assert L.lsh_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, nf - 1,
                          None) == 3
    assert L.lsh_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE + 8, FAKE, FAKE, nf,
                          None) == 1   # misaligned out_lo
    nb = L.lsh_bwd_workspace_size(ctypes.byref(p))
    assert L.lsh_attn_bwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE,
                          FAKE, nb - 1, None) == 3
    assert L.lsh_attn_bwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, None, FAKE, None, FAKE, FAKE,
                          FAKE, nb, None) == 1


def test_empty_problem_is_a_noop():
    _ensure_built()
    L = _lib.lib()
    for kw in (dict(B=0), dict(H=0), dict(L=0)):
        p = _p(**kw)
        assert L.lsh_hash(ctypes.byref(p), None, None, None, None) == 0
        assert L.lsh_sort(ctypes.byref(p), None, None, None, 0, None) == 0
        assert L.lsh_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None, 0,
                              None) == 0
        assert L.lsh_attn_bwd(ctypes.byref(p), None, None, None, None, None, None, None, None,
                              None, None, 0, None) == 0


def test_workspace_sizes_grow_with_problem():
    _ensure_built()
    L = _lib.lib()
    a = _p()
    b = _p(L=262144)   # spans several sort blocks per segment
    for f in (L.lsh_sort_workspace_size, L.lsh_fwd_workspace_size, L.lsh_bwd_workspace_size):
        assert 0 < f(ctypes.byref(a)) < f(ctypes.byref(b))
        assert f(ctypes.byref(a)) % 256 == 0


def test_missing_library_fails_loudly(monkeypatch):
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/liblsh.so")
    with pytest.raises(_lib.LshLibraryMissing):
        _lib.lib()


def test_wait_timeout_check_rejects_bad_limits_before_launch():
    _ensure_built()
    L = _lib.lib()
    assert L.lsh_check_wait_timeout(0, None) == 1               # LSH_ERR_INVALID_ARG
    assert L.lsh_check_wait_timeout(2_000_000_000, None) == 1


def test_local_attention_rejects_bad_arguments_before_launch():
    _ensure_built()
    L = _lib.lib()
    p = _p(n_rounds=1)
    assert L.lsh_local_fwd_workspace_size(ctypes.byref(p), 1, 0) > 0
    assert L.lsh_local_fwd_workspace_size(ctypes.byref(p), -1, 0) == 0
    assert L.lsh_local_bwd_workspace_size(ctypes.byref(_p(n_rounds=2)), 1, 0) == 0
    args = [FAKE] * 5 + [FAKE, 1 << 30, None]
    assert L.lsh_local_attn_fwd(ctypes.byref(_p(n_rounds=2)), 1, 0, *args) == 1
    assert L.lsh_local_attn_fwd(ctypes.byref(p), 0, -3, *args) == 1
    assert L.lsh_local_attn_fwd(ctypes.byref(p), 1, 0, FAKE, FAKE, FAKE, None, FAKE, FAKE, 16,
                                None) == 3                       # workspace too small
    empty = _p(n_rounds=1, B=0)
    assert L.lsh_local_attn_fwd(ctypes.byref(empty), 1, 1, None, None, None, None, None, None, 0,
                                None) == 0


def _f(**kw):
    base = dict(B=1, H=2, L=256, d_ff=256, ff_chunk=128)
    base.update(kw)
    return _lib.lsh_ff_problem(*[base[k] for k, _ in _lib.lsh_ff_problem._fields_])


@pytest.mark.parametrize("kw,code", [
    (dict(L=192), 1), (dict(d_ff=192), 1), (dict(d_ff=0), 1), (dict(ff_chunk=64), 1),
    (dict(ff_chunk=200), 1), (dict(H=0), 1), (dict(B=-1), 1), (dict(d_ff=65536 + 128), 2),
    (dict(H=1025), 2),
])
def test_feed_forward_rejects_bad_problem_before_launch(kw, code):
    _ensure_built()
    L = _lib.lib()
    f = _f(**kw)
    assert L.lsh_ff_workspace_size(ctypes.byref(f)) == 0
    args = [FAKE] * 5 + [None, FAKE * 2, FAKE, 1 << 30, None]
    assert L.lsh_ff_fwd(ctypes.byref(f), *args) == code


def test_feed_forward_and_block_check_pointers_and_workspace():
    _ensure_built()
    L = _lib.lib()
    f = _f()
    n = L.lsh_ff_workspace_size(ctypes.byref(f))
    assert n > 0 and n % 256 == 0
    ok = [FAKE] * 5 + [None, FAKE * 2]
    assert L.lsh_ff_fwd(ctypes.byref(f), *ok, FAKE, n - 1, None) == 3
    assert L.lsh_ff_fwd(ctypes.byref(f), *ok, None, n, None) == 3
    assert L.lsh_ff_fwd(ctypes.byref(f), None, *ok[1:], FAKE, n, None) == 1
    assert L.lsh_ff_fwd(ctypes.byref(f), FAKE, *ok[1:6], FAKE, FAKE, n, None) == 1   # y aliases x
    assert L.lsh_ff_fwd(ctypes.byref(f), FAKE + 8, *ok[1:], FAKE, n, None) == 1      # misaligned x
    bwd = [FAKE] * 6 + [None, None, None] + [FAKE] * 5
    assert L.lsh_ff_bwd(ctypes.byref(f), *bwd, FAKE, n - 1, None) == 3
    bad = list(bwd)
    bad[7] = FAKE                      # y_in without rec
    assert L.lsh_ff_bwd(ctypes.byref(f), *bad, FAKE, n, None) == 1
    p = _p(n_rounds=2)
    assert L.lsh_rev_fwd_workspace_size(ctypes.byref(p), ctypes.byref(f)) > 0
    assert L.lsh_rev_bwd_workspace_size(ctypes.byref(p), ctypes.byref(f)) > 0
    # the attention must match the block's B, H, L and be bf16
    for pk in (dict(H=3), dict(L=512), dict(dtype=0)):
        q = _p(**pk)
        assert L.lsh_rev_fwd_workspace_size(ctypes.byref(q), ctypes.byref(f)) == 0
        assert L.lsh_rev_fwd(ctypes.byref(q), ctypes.byref(f), *([FAKE] * 10), FAKE, 1 << 30,
                             None) in (1, 2)
    nr = L.lsh_rev_bwd_workspace_size(ctypes.byref(p), ctypes.byref(f))
    assert L.lsh_rev_bwd(ctypes.byref(p), ctypes.byref(f), *([FAKE] * 17), FAKE, nr - 1,
                         None) == 3


def test_feed_forward_and_block_empty_problem_is_a_noop():
    _ensure_built()
    L = _lib.lib()
    f = _f(B=0)
    assert L.lsh_ff_fwd(ctypes.byref(f), *([None] * 8), 0, None) == 0
    assert L.lsh_ff_bwd(ctypes.byref(f), *([None] * 15), 0, None) == 0
    p = _p(B=0)
    assert L.lsh_rev_fwd(ctypes.byref(p), ctypes.byref(f), *([None] * 11), 0, None) == 0
    assert L.lsh_rev_bwd(ctypes.byref(p), ctypes.byref(f), *([None] * 18), 0, None) == 0
