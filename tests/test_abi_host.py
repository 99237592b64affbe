"""Host-only checks of the C ABI (no GPU needed, no kernel launched).

* the library loads and exports every function include/nsa.h declares;
* argument validation happens on the host before any CUDA call.
"""
import ctypes

import torch
import os
import re

import pytest

from tests.conftest import ROOT

nsa = pytest.importorskip("dynamic_block_sparse_nsa_b200.nsa")


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nsa.h")).read()
    return sorted(set(re.findall(r"NSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(nsa.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(nsa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    for code, name in nsa.STATUS.items():
        assert nsa.LIB.nsa_status_string(code).decode() == name


def test_num_cmp_blocks():
    assert nsa.num_cmp_blocks(65536, 32, 16) == 4095
    assert nsa.num_cmp_blocks(8192, 32, 16) == 511
    assert nsa.num_cmp_blocks(31, 32, 16) == 0


def _status(fn, *args):
    return fn(*args)


def test_workspace_size_validation():
    n = ctypes.c_size_t(7)
    assert nsa.LIB.nsa_workspace_size(None, 0, ctypes.byref(n)) == 1
    p = nsa.params(1, 1024, 4, 1, 64)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(p), 99, ctypes.byref(n)) == 1
    bad = nsa.params(1, 1024, 4, 1, 96)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 2
    assert b"head dim" in nsa.LIB.nsa_last_error_detail()
    bad = nsa.params(1, 1024, 6, 4, 64)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 1
    bad = nsa.params(1, 1024, 4, 1, 64, top_p=1.5)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 1
    assert b"top_p" in nsa.LIB.nsa_last_error_detail()
    bad = nsa.params(1, 1024, 4, 1, 64, cmp_block=8, cmp_stride=16)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 1
    # MoBA: block means [B, T/m, Hkv, d] fp32; the tensor-core path (bf16,
    # d = 128) adds the selection, bucket counts / offsets / tile offsets /
    # cursors, bucket rows, partial outputs and their log-sum-exp
    def a256(x):
        return (x + 255) // 256 * 256
    B, T, H, m, k = 2, 131072, 32, 512, 3
    kbar = a256(B * (T // m) * H * 128 * 4)
    rows, nb = B * T * H, B * H * (T // m)
    moba = nsa.params(B, T, H, H, 128, sel_block=m, top_n=k)
    rows_g = max(32, -(-(T // m) // 32) * 32)  # block rows per part, padded to 32-row boxes
    parts = a256(B * H * 3 * rows_g * 128 * 2 + 4)  # the means split into three bf16 parts
    assert nsa.workspace_size(moba, nsa.OP_MOBA_PREFILL) == (
        kbar + a256(rows * k * 4) + 4 * a256((nb + 1) * 4) + a256(rows * (k - 1) * 4 + 4) +
        a256(rows * (k - 1) * 128 * 2 + 4) + a256(rows * (k - 1) * 4 + 4) + parts +
        a256((nb + rows * (k - 1) // 128 + 2) * 16))  # a descriptor per 128-row bucket tile
    moba32 = nsa.params(B, T, H, H, 128, sel_block=m, top_n=k, dtype=torch.float32)
    assert nsa.workspace_size(moba32, nsa.OP_MOBA_PREFILL) == kbar  # CUDA-core path


def test_calls_reject_null_pointers_before_launching():
    p = nsa.params(1, 1024, 4, 1, 64)
    L = nsa.LIB
    assert L.nsa_compress_kv(ctypes.byref(p), None, None, None, None, None, None) == 1
    assert L.nsa_prefill(ctypes.byref(p), None, None, None, None, None, None, None, None, None,
                         0, None) == 1
    assert L.nsa_decode(ctypes.byref(p), None, None, None, None, None, None, None, None, None,
                        None, 0, None) == 1
    assert L.moba_prefill(ctypes.byref(p), None, None, None, None, None, None, 0, None) == 1
    assert L.nsa_debug_bounded_wait(None, 10, None) == 1
    assert L.nsa_block_bounds(ctypes.byref(p), None, None, None, None) == 1
    assert L.nsa_append_bounds(ctypes.byref(p), None, None, None, None) == 1
    # the Quest decode needs sel_mode 1, then its pointers (k_bounds included)
    assert L.nsa_decode_quest(ctypes.byref(p), *([None] * 11), 0, None) == 1
    assert b"sel_mode" in L.nsa_last_error_detail()
    pq = nsa.params(2, 4096, 32, 2, 128, sel_mode=1)
    args = [ctypes.c_void_p(256)] * 11
    args[6] = None  # k_bounds
    assert L.nsa_decode_quest(ctypes.byref(pq), *args, 0, None) == 1
    assert b"k_bounds" in L.nsa_last_error_detail()
    # gate weights are required for learned gates only
    fake = ctypes.c_void_p(256)
    assert L.nsa_prefill(ctypes.byref(p), fake, fake, fake, fake, fake, None, fake, None, None,
                         0, None) == 1
    assert b"w_gate" in L.nsa_last_error_detail()


def test_moba_rejects_small_workspace_before_launching():
    p = nsa.params(1, 4096, 4, 4, 128, sel_block=512, top_n=3)
    fake = ctypes.c_void_p(256)
    need = nsa.workspace_size(p, nsa.OP_MOBA_PREFILL)
    st = nsa.LIB.moba_prefill(ctypes.byref(p), fake, fake, fake, fake, None, fake, need - 1, None)
    assert st == 3
    st = nsa.LIB.moba_prefill(ctypes.byref(p), fake, fake, fake, fake, None, ctypes.c_void_p(264),
                              need, None)
    assert st == 1  # misaligned workspace


def test_backward_workspace_and_argument_checks():
    """Backward scratch: dK~ and dV~ fp32 [B, Nc, Hkv, d] and the gate
    gradients dz fp32 [B, T, Hq, 3], each 256-byte aligned; the calls reject
    NULL pointers and top_n > 64 before touching the device."""
    def a256(x):
        return (x + 255) // 256 * 256
    B, T, Hq, Hkv, d = 2, 8192, 64, 4, 128
    p = nsa.params(B, T, Hq, Hkv, d)
    Nc = nsa.LIB.nsa_num_cmp_blocks(T, 32, 16)
    assert nsa.workspace_size(p, nsa.OP_PREFILL_BACKWARD) == (
        2 * a256(B * Nc * Hkv * d * 4) + a256(B * T * Hq * 3 * 4))
    L = nsa.LIB
    assert L.nsa_prefill_backward(ctypes.byref(p), *([None] * 15), 0, None) == 1
    fake = ctypes.c_void_p(256)
    big = nsa.params(1, 1024, 4, 1, 64, top_n=65)
    assert L.nsa_prefill_backward(ctypes.byref(big), *([fake] * 15), 1 << 30, None) == 2
    assert b"top_n" in L.nsa_last_error_detail()


def test_selection_mode_checks():
    """sel_mode: 0 or 1; the Quest bound (1) ranks raw bounds, not a probability
    mass, so it takes no top-p threshold."""
    n = ctypes.c_size_t()
    ok = nsa.params(1, 1024, 4, 1, 64, sel_mode=1)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(ok), nsa.OP_PREFILL, ctypes.byref(n)) == 0
    bad = nsa.params(1, 1024, 4, 1, 64, sel_mode=2)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 1
    bad = nsa.params(1, 1024, 4, 1, 64, sel_mode=1, top_p=0.5)
    assert nsa.LIB.nsa_workspace_size(ctypes.byref(bad), nsa.OP_PREFILL, ctypes.byref(n)) == 1
    assert b"top_p" in nsa.LIB.nsa_last_error_detail()
    # the tensor-core prefill takes the Quest bound with a block-bounds table and
    # a score matrix in its workspace
    fast = nsa.params(1, 8192, 64, 4, 128)
    base = nsa.workspace_size(fast, nsa.OP_PREFILL)
    assert base > 0
    nblk = 8192 // 64
    quest = nsa.workspace_size(nsa.params(1, 8192, 64, 4, 128, sel_mode=1), nsa.OP_PREFILL)
    assert quest >= nblk * 4 * 2 * 128 * 2 + 8192 * 4 * nblk * 4
