"""Quest-style selection for decode (EP94 notes §八, the selection ablation's
Quest bound): the block-bounds table beside the cache (nsa_block_bounds, kept
current by nsa_append_bounds) and nsa_decode_quest, against plain tensor
reductions and the fp64 oracle's score_mode 2 (which computes the bounds from
the keys themselves)."""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_nsa_b200 import inputs
from tests import gpu_cases as gc

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_cuda(cuda_ok):
    torch.cuda.synchronize()
    yield


def _ref_bounds(k, lens, bs):
    """[B, nblk, Hkv, 2, d] from max / min over each block's tokens < len."""
    B, T, Hkv, d = k.shape
    nblk = -(-T // bs)
    ref = {}
    for b in range(B):
        for j in range(nblk):
            u0, u1 = j * bs, min(j * bs + bs, int(lens[b]))
            if u0 >= u1:
                continue
            blk = k[b, u0:u1].float()
            ref[(b, j)] = torch.stack([blk.amax(0), blk.amin(0)], 1)  # [Hkv, 2, d]
    return ref


@pytest.mark.parametrize("dtype,bs", [("bf16", 64), ("f32", 16)])
def test_block_bounds_are_the_block_extremes(dtype, bs):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=3, T=1000, Hq=8, Hkv=2, d=64,
                        dtype=dtype, sel_block=bs)
    lens = [1000, 130, 1]
    inp = inputs.make_decode(w, seed=3, seq_lens=lens)
    p = gc.nsa_params_for(w)
    k = inp["k"].cuda()
    kb = nsa.nsa_block_bounds(p, k, inp["seq_lens"].cuda())
    nsa.nsa_check()
    kb = kb.cpu().float()
    for (b, j), r in _ref_bounds(inp["k"], lens, bs).items():
        assert torch.equal(kb[b, j], r), (b, j)


def test_append_bounds_track_a_growing_cache():
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=2, T=300)
    inp = inputs.make_decode(w, seed=4)
    p = gc.nsa_params_for(w)
    k = inp["k"].cuda()
    lens0 = torch.tensor([60, 127], dtype=torch.int32)
    kb = nsa.nsa_block_bounds(p, k, lens0.cuda())
    pos = lens0.clone()
    for _ in range(70):  # crosses the block boundaries at 64, 128 and 192
        knew = torch.stack([inp["k"][b, int(pos[b])] for b in range(2)]).cuda()
        nsa.nsa_append_bounds(p, knew, pos.cuda(), kb)
        pos += 1
    nsa.nsa_check()
    kb = kb.cpu().float()
    for (b, j), r in _ref_bounds(inp["k"], pos.tolist(), 64).items():
        assert torch.equal(kb[b, j], r), (b, j)


@pytest.mark.parametrize("over,lens", [
    (dict(B=4, T=5000), [5000, 3001, 700, 64]),
    (dict(B=3, T=9000, top_n=7, window=300), [9000, 4097, 129]),
    (dict(B=2, T=200, top_n=16), [200, 40]),                  # fewer candidates than n
    (dict(B=2, T=3000, gate_mode=1, fixed_gates=(0.0, 1.0, 0.0)), [3000, 2049]),
])
def test_decode_quest_fast_path(over, lens):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", sel_mode=1, **over)
    nsa.trace_enable(True, 64)
    try:
        gc.run_nsa_decode(w, lens, seed=19, quest_table=True)
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    assert "dec_quest_select" in names and "dec_select" not in names, names
    assert "nsa_rows_simt" not in names, names


def test_decode_quest_other_shapes_use_the_cuda_core_path():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=2, T=2000, dtype="f32", Hq=8, Hkv=2,
                        d=64, top_n=5, window=100, sel_mode=1)
    gc.run_nsa_decode(w, [2000, 777], seed=20, quest_table=True)


def test_decode_quest_with_appended_bounds_matches_a_rebuilt_table():
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=2, T=1200, sel_mode=1)
    inp = inputs.make_decode(w, seed=21, seq_lens=[1100, 900])
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    lens = torch.tensor([1030, 840], dtype=torch.int32)
    kb = nsa.nsa_block_bounds(p, dev["k"], lens.cuda())
    pos = lens.clone()
    while int(pos[0]) < 1100:
        knew = torch.stack([inp["k"][b, int(pos[b])] for b in range(2)]).cuda()
        nsa.nsa_append_bounds(p, knew, pos.cuda(), kb)
        pos += 1
    ref = nsa.nsa_block_bounds(p, dev["k"], dev["seq_lens"])
    out1, sel1 = nsa.nsa_decode_quest(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                      kb, dev["w_gate"])
    out2, sel2 = nsa.nsa_decode_quest(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                      ref, dev["w_gate"])
    nsa.nsa_check()
    assert torch.equal(sel1, sel2) and torch.equal(out1, out2)
    assert int(pos[1]) == 910
