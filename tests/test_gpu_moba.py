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
