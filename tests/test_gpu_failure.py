"""Failure detection on the GPU without a GPU fault.

A bounded device wait on a flag nothing sets must end with the error word set,
nsa_check must report NSA_ERR_DEVICE_TIMEOUT, and the context must stay usable.
A decode sequence length out of range is reported the same way.
"""
import ctypes

import pytest
import torch

from dynamic_block_sparse_nsa_b200 import nsa

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_ok):
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = nsa.LIB.nsa_debug_bounded_wait(ctypes.c_void_p(flag.data_ptr()), 2000,
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    assert nsa.status_of_check() == 5  # NSA_ERR_DEVICE_TIMEOUT
    assert nsa.status_of_check() == 0  # the word was cleared
    # the context still runs work
    x = torch.randn(1024, device="cuda")
    assert torch.isfinite(x.sum()).item()


def test_flag_already_set_returns_ok(cuda_ok):
    flag = torch.ones(1, dtype=torch.int32, device="cuda")
    nsa.LIB.nsa_debug_bounded_wait(ctypes.c_void_p(flag.data_ptr()), 10,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert nsa.status_of_check() == 0


def test_decode_bad_seq_len_reported(cuda_ok):
    B, T, Hq, Hkv, d = 2, 256, 4, 1, 64
    p = nsa.params(B, T, Hq, Hkv, d, top_n=2, window=32, dtype=torch.float32)
    q = torch.randn(B, Hq, d, device="cuda")
    k = torch.randn(B, T, Hkv, d, device="cuda")
    v = torch.randn(B, T, Hkv, d, device="cuda")
    w = torch.randn(32, device="cuda")
    kc, vc = nsa.nsa_compress_kv(p, k, v, w)
    lens = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    wg = torch.randn(d, 3, device="cuda")
    out, sel = nsa.nsa_decode(p, q, k, v, lens, kc, vc, wg)
    assert nsa.status_of_check() == 1
    assert torch.all(out[0] == 0).item() and torch.all(sel[0] == -1).item()
    assert torch.isfinite(out[1]).all().item()
