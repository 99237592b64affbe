"""NSA prefill backward on the GPU against the fp64 oracle (oracle/backward.py).

Both sides take the selection the oracle's forward makes (the backward treats
it as a constant) and the compressed cache as the forward stored it (the
CUDA compression is checked bit-exact against the oracle's first).

Tolerance: the kernels compute in fp32 (inputs exact in fp32 or bf16). A
gradient entry is a sum of at most a few thousand terms (keys, or rows that
attend to a key) with one cancellation per key, p (dO . v - D); fp32 rounding
(6e-8) grown by ~sqrt(2000) = 45 over such sums and by up to ~10 in the
cancellation gives ~3e-5 of the gradient's largest magnitude, so the bound is
5e-5 of it (observed: below 1e-6). A dropped term, wrong sign or misplaced
scatter changes a gradient by a sizeable fraction of its magnitude.
"""
import pytest

from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu

TOL = 5e-5


@pytest.mark.parametrize("name,over", [
    ("nsa_prefill_f32_t1024", dict(T=300)),                                  # ragged blocks
    ("nsa_prefill_bf16_t8192", dict(T=260, Hq=16, Hkv=1)),                   # the bf16 shape
    ("nsa_prefill_f32_t1024", dict(B=2, T=130, Hq=8, Hkv=2, d=64, cmp_block=8, cmp_stride=4,
                                   sel_block=16, top_n=3, window=20)),       # many blocks, GQA 4
    ("nsa_prefill_f32_t1024", dict(T=200, gate_mode=1, fixed_gates=(0.3, 0.5, 0.2))),
    ("nsa_prefill_f32_t1024", dict(T=200, top_p=0.6, top_n=4)),              # unused slots
    ("nsa_prefill_f32_t1024", dict(T=20)),                                   # no compressed block
])
def test_prefill_backward_matches_the_oracle(name, over):
    gc.run_backward(inputs.workload(name, **over), seed=31, tol=TOL)


def test_prefill_backward_runs_its_kernels(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    nsa.trace_enable(True, 64)
    try:
        gc.run_backward(inputs.workload("nsa_prefill_f32_t1024", T=100), seed=32, tol=TOL)
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    assert {"bwd_rows", "bwd_compress", "bwd_dw", "bwd_dwg"} <= names, names
