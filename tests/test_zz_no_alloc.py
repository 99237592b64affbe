"""The no-allocation decode entry point against the workspace one.

nsa_decode_noalloc serves callers that cannot allocate device memory (work
enqueued during a CUDA-graph stream capture, real-time threads, hosts whose
device memory belongs to another runtime's pool): it runs the same decode with
the library's static scratch in place of a caller workspace. This file is
collected last so a failure here never hides the other tests; it passes alone
in a fresh process too (the first call there does the per-device set-up).
"""
import ctypes

import pytest
import torch

from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc
from tests import parity

pytestmark = pytest.mark.gpu


def _c_abi_noalloc(nsa, p, dev, kc, vc, out, sel):
    """One call straight through the C ABI (no Python wrapper)."""
    P = ctypes.c_void_p
    return nsa.LIB.nsa_decode_noalloc(
        ctypes.byref(p), P(dev["q"].data_ptr()), P(dev["k"].data_ptr()), P(dev["v"].data_ptr()),
        P(dev["seq_lens"].data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()),
        P(dev["w_gate"].data_ptr()), P(out.data_ptr()), P(sel.data_ptr()),
        P(torch.cuda.current_stream().cuda_stream))


def _decode_case(nsa, B, T, seed, lens):
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=B, T=T)
    inp = inputs.make_decode(w, seed=seed, seq_lens=lens)
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    return p, dev, kc, vc


def test_noalloc_decode_matches_workspace_decode_twice(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    # A first call of another shape leaves its own contents in the static
    # scratch: other batch size, lengths shorter than one compressed block (no
    # compressed key at all) and a different selection count.
    p0, dev0, kc0, vc0 = _decode_case(nsa, 3, 5000, 4, [5000, 20, 1])
    assert nsa.workspace_size(p0, nsa.OP_DECODE) > 0
    out0 = torch.empty(3, p0.Hq, p0.d, dtype=torch.bfloat16, device="cuda")
    sel0 = torch.empty(3, p0.Hkv, p0.top_n, dtype=torch.int32, device="cuda")
    assert _c_abi_noalloc(nsa, p0, dev0, kc0, vc0, out0, sel0) == 0
    nsa.nsa_check()

    p, dev, kc, vc = _decode_case(nsa, 6, 12000, 11, [12000, 9000, 4097, 777, 64, 11999])
    # the fast decode path is the one that uses the scratch
    assert nsa.workspace_size(p, nsa.OP_DECODE) > 0
    ref_out, ref_sel = nsa.nsa_decode(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                      dev["w_gate"])
    nsa.nsa_check()
    for _ in range(2):  # the static scratch keeps the previous call's contents
        out = torch.full_like(ref_out, float("nan"))
        sel = torch.full_like(ref_sel, -7)
        assert _c_abi_noalloc(nsa, p, dev, kc, vc, out, sel) == 0
        nsa.nsa_check()
        parity.check_output(out.float().cpu().numpy(), ref_out.float().cpu().numpy(), "bf16")
        assert torch.equal(sel, ref_sel)

    # the first shape again, after the second one wrote over the scratch
    ref0, rsel0 = nsa.nsa_decode(p0, dev0["q"], dev0["k"], dev0["v"], dev0["seq_lens"], kc0, vc0,
                                 dev0["w_gate"])
    assert _c_abi_noalloc(nsa, p0, dev0, kc0, vc0, out0, sel0) == 0
    nsa.nsa_check()
    parity.check_output(out0.float().cpu().numpy(), ref0.float().cpu().numpy(), "bf16")
    assert torch.equal(sel0, rsel0)


def test_noalloc_python_wrapper(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    p, dev, kc, vc = _decode_case(nsa, 2, 3000, 12, [3000, 1500])
    ref_out, ref_sel = nsa.nsa_decode(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                      dev["w_gate"])
    out, sel = nsa.nsa_decode_noalloc(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                      dev["w_gate"])
    nsa.nsa_check()
    parity.check_output(out.float().cpu().numpy(), ref_out.float().cpu().numpy(), "bf16")
    assert torch.equal(sel, ref_sel)


def test_noalloc_rejects_shapes_beyond_the_static_scratch(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    p = nsa.params(128, 65536, 64, 4, 128)  # needs about 91 MiB of decode scratch
    null = ctypes.c_void_p(0)
    st = nsa.LIB.nsa_decode_noalloc(ctypes.byref(p), *([null] * 10))
    assert st == 2  # NSA_ERR_UNSUPPORTED, before anything is launched
    assert b"static scratch" in nsa.LIB.nsa_last_error_detail()
