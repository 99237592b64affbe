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
import numpy as np
import pytest
import torch

import oracle
from oracle import backward as obwd
from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu

TOL = 5e-5


def run_backward(w, seed):
    from dynamic_block_sparse_nsa_b200 import nsa
    inp = inputs.make_prefill(w, seed)
    p = gc.nsa_params_for(w)
    op = gc.oracle_params_for(w)
    B, T, Hq, d = inp["q"].shape
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    q64, k64, v64 = gc.f64(inp["q"]), gc.f64(inp["k"]), gc.f64(inp["v"])
    wc64, wg64 = gc.f64(inp["w_cmp"]), gc.f64(inp["w_gate"])
    kc64, vc64 = oracle.compress(op, k64, v64, wc64)
    np.testing.assert_array_equal(gc.f64(kc), kc64)
    fwd = oracle.nsa_prefill(op, q64, k64, v64, wc64, wg64)
    sel = fwd["sel"].reshape(B, T, p.Hkv, p.top_n)
    gen = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, T, Hq, d, generator=gen).to(inp["q"].dtype)
    got = nsa.nsa_prefill_backward(p, dev["q"], dev["k"], dev["v"], kc, vc, dev["w_cmp"],
                                   dev["w_gate"], torch.from_numpy(sel).cuda(), dout.cuda())
    nsa.nsa_check()
    ref = obwd.nsa_prefill_backward(op, q64, k64, v64, wc64, wg64, gc.f64(dout), sel,
                                    kc=kc64, vc=vc64)
    stats = {}
    for name, g in zip(("dq", "dk", "dv", "dw_cmp", "dwg"), got):
        r = ref[name]
        err = float(np.abs(gc.f64(g) - r).max()) if r.size else 0.0
        scale = max(float(np.abs(r).max()) if r.size else 0.0, 1e-6)
        stats[name] = (err, scale)
    print(w["dtype"], w["T"], {k_: f"{e / s:.2e}" for k_, (e, s) in stats.items()})
    for name, (err, scale) in stats.items():
        assert err <= TOL * scale, (name, err, scale)
    return stats


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
    run_backward(inputs.workload(name, **over), seed=31)


def test_prefill_backward_runs_its_kernels(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    nsa.trace_enable(True, 64)
    try:
        run_backward(inputs.workload("nsa_prefill_f32_t1024", T=100), seed=32)
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    assert {"bwd_rows", "bwd_compress", "bwd_dw", "bwd_dwg"} <= names, names
