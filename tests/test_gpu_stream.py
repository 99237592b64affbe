"""Streaming decode: nsa_append_kv grows the caches token by token.

A compressed block written by an append must equal the oracle's compression of
the same tokens bit for bit (both are the correctly rounded exact sum), and a
decode over the grown caches must match the oracle at every step.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


def _start(w, src, L0):
    """Caches holding the first L0[b] tokens of the stream (the rest zero), and
    their compression (entries of blocks not yet complete are filled by appends)."""
    from dynamic_block_sparse_nsa_b200 import nsa
    p = gc.nsa_params_for(w)
    k = torch.zeros_like(src["k"])
    v = torch.zeros_like(src["v"])
    for b, L in enumerate(L0):
        k[b, :L] = src["k"][b, :L]
        v[b, :L] = src["v"][b, :L]
    k, v = k.cuda(), v.cuda()
    kc, vc = nsa.nsa_compress_kv(p, k, v, src["w_cmp"].cuda())
    return p, k, v, kc, vc


def _append(p, src, k, v, kc, vc, lens):
    from dynamic_block_sparse_nsa_b200 import nsa
    B = len(lens)
    kn = torch.stack([src["k"][b, lens[b]] for b in range(B)]).cuda()
    vn = torch.stack([src["v"][b, lens[b]] for b in range(B)]).cuda()
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nsa.nsa_append_kv(p, kn, vn, pos, k, v, src["w_cmp"].cuda(), kc, vc)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_appends_reproduce_the_full_compression(cuda_ok, dtype):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=3, T=400, Hq=16, Hkv=2, dtype=dtype)
    src = inputs.make_decode(w, seed=21)
    L0 = [0, 17, 100]
    p, k, v, kc, vc = _start(w, src, L0)
    lens = list(L0)
    for _ in range(230):
        _append(p, src, k, v, kc, vc, lens)
        lens = [x + 1 for x in lens]
    nsa.nsa_check()
    op = gc.oracle_params_for(dict(w, B=1))
    l, s = w["cmp_block"], w["cmp_stride"]
    for b, L in enumerate(lens):
        assert torch.equal(k[b, :L].cpu(), src["k"][b, :L])
        assert torch.equal(v[b, :L].cpu(), src["v"][b, :L])
        kc64, vc64 = oracle.compress(dict(op, T=L), gc.f64(src["k"][b:b + 1, :L]),
                                     gc.f64(src["v"][b:b + 1, :L]), gc.f64(src["w_cmp"]))
        n = (L - l) // s + 1 if L >= l else 0  # blocks complete within L tokens
        np.testing.assert_array_equal(gc.f64(kc[b:b + 1, :n]), kc64[:, :n])
        np.testing.assert_array_equal(gc.f64(vc[b:b + 1, :n]), vc64[:, :n])


def test_generation_steps_match_the_oracle(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=2, T=2200, Hq=16, Hkv=1)
    src = inputs.make_decode(w, seed=22)
    L0 = [900, 1503]  # one append closes a compressed block for the second sequence
    p, k, v, kc, vc = _start(w, src, L0)
    lens = list(L0)
    op = gc.oracle_params_for(dict(w, B=1))
    gen = torch.Generator().manual_seed(23)
    for step in range(4):
        _append(p, src, k, v, kc, vc, lens)
        lens = [x + 1 for x in lens]
        q = (torch.randn(2, 16, 128, generator=gen) / np.sqrt(128)).to(torch.bfloat16)
        seq = torch.tensor(lens, dtype=torch.int32, device="cuda")
        out, sel = nsa.nsa_decode(p, q.cuda(), k, v, seq, kc, vc, src["w_gate"].cuda())
        nsa.nsa_check()
        for b, L in enumerate(lens):
            k64 = gc.f64(src["k"][b:b + 1, :L])
            v64 = gc.f64(src["v"][b:b + 1, :L])
            opl = dict(op, T=L)
            kc64, vc64 = oracle.compress(opl, k64, v64, gc.f64(src["w_cmp"]))
            gc.compare_nsa_rows(w, opl, [0], [L - 1], gc.f64(q[b:b + 1]), k64, v64, kc64, vc64,
                                gc.f64(src["w_gate"]), gc.f64(out[b:b + 1]),
                                sel[b:b + 1].cpu().numpy())


def test_append_rejects_positions_outside_the_cache(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=2, T=64, Hq=16, Hkv=1)
    src = inputs.make_decode(w, seed=24)
    p, k, v, kc, vc = _start(w, src, [10, 64])
    k0, kc0 = k.clone(), kc.clone()
    kn = torch.ones(2, 1, 128, dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor([64, -1], dtype=torch.int32, device="cuda")
    nsa.nsa_append_kv(p, kn, kn, pos, k, v, src["w_cmp"].cuda(), kc, vc)
    with pytest.raises(nsa.NsaError) as e:
        nsa.nsa_check()
    assert e.value.status == 1  # NSA_ERR_INVALID_ARGUMENT
    assert torch.equal(k, k0) and torch.equal(kc, kc0)
