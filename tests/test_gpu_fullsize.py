"""GPU parity against the oracle at the full sizes of every named workload,
element by element, through the same C-ABI calls the benchmark times.

The oracle runs the whole problem in float64 (about a minute per large
workload on a few host cores)."""
import pytest

from efficient_transformer_lsh_b200.workloads import WORKLOADS, generate
from parity_common import compare, gpu_run, oracle_run


@pytest.mark.gpu
@pytest.mark.parametrize("name", list(WORKLOADS))
def test_parity_full_size(name):
    w = WORKLOADS[name]
    inp = generate(w)
    ref = oracle_run(w, inp, w.backward)
    got = gpu_run(w, inp, ref["bucket"], w.backward)
    compare(w, ref, got, w.backward, label=name)
