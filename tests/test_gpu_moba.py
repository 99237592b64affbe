"""GPU parity of MoBA prefill against the fp64 oracle."""
import pytest
import torch

from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    torch.cuda.synchronize()
    yield


def test_moba_f32_small_all_rows():
    w = inputs.workload("moba_prefill_bf16_t131072", B=1, T=1500, Hq=2, Hkv=2, d=64, block=128,
                        top_k=3, dtype="f32")
    st = gc.run_moba(w)
    assert st["max_err"] <= 1e-4


def test_moba_bf16_gqa_ragged():
    w = inputs.workload("moba_prefill_bf16_t131072", B=2, T=3000, Hq=4, Hkv=2)
    gc.run_moba(w, rows=gc.sample_rows(3000, 300, B=2))


def test_moba_bf16_top1_and_all_blocks():
    for k in (1, 8):
        w = inputs.workload("moba_prefill_bf16_t131072", T=2560, Hq=2, Hkv=2, top_k=k)
        gc.run_moba(w, rows=gc.sample_rows(2560, 200))


def test_moba_bf16_full_size_sampled():
    w = inputs.workload("moba_prefill_bf16_t131072")
    gc.run_moba(w, rows=gc.sample_rows(w["T"], 24), heads=[0, 13, 31])


# Tensor-core MoBA path (bf16, d = 128, block a multiple of 128): bucket tiles,
# ragged query tiles, a sequence shorter than one block, GQA, up to 7 picks.
@pytest.mark.parametrize("over", [
    dict(T=1000, Hq=2, Hkv=2, block=128, top_k=4),
    dict(T=300, Hq=2, Hkv=2),
    dict(B=2, T=1536, Hq=4, Hkv=1, block=256, top_k=2),
    dict(T=4096, Hq=2, Hkv=2, block=512, top_k=8),
])
def test_moba_bf16_tensor_core_edges(over):
    w = inputs.workload("moba_prefill_bf16_t131072", **over)
    gc.run_moba(w, seed=9)


def test_moba_bf16_more_than_two_gate_chunks():
    # 320 blocks of 128: the gate scores up to 319 past blocks in three
    # 128-block chunks, reusing its two score buffers; ragged last tile
    w = inputs.workload("moba_prefill_bf16_t131072", T=41000, Hq=2, Hkv=1, block=128, top_k=4)
    rows = gc.sample_rows(41000, 160) + [(0, 40999), (0, 32768), (0, 32767), (0, 16384)]
    gc.run_moba(w, rows=rows, seed=5)


def test_moba_bf16_runs_the_tensor_core_kernels():
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("moba_prefill_bf16_t131072", T=2048, Hq=2, Hkv=2, block=256, top_k=3)
    nsa.trace_enable(True, 64)
    try:
        gc.run_moba(w, rows=gc.sample_rows(2048, 100))
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    assert {"moba_gate", "moba_blk", "moba_own"} <= names, names
