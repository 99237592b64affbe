"""GPU parity of NSA compression, prefill and decode against the fp64 oracle.

Each test calls the C ABI (through the ctypes binding) on seeded inputs and
compares with the oracle on the same inputs: compressed blocks bit-exact,
block selection exact outside 1e-5-relative near-ties, outputs within
1e-4 (fp32) or 2e-2 max / 2e-3 mean (bf16).
"""
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


def test_prefill_f32_t1024_all_rows():
    w = inputs.workload("nsa_prefill_f32_t1024")
    st = gc.run_nsa_prefill(w)
    assert st["max_err"] <= 1e-4


def test_prefill_bf16_t8192_sampled_rows():
    w = inputs.workload("nsa_prefill_bf16_t8192")
    gc.run_nsa_prefill(w, rows=gc.sample_rows(w["T"], 160))


@pytest.mark.parametrize("over", [
    dict(T=20),                                           # no compressed block visible
    dict(T=1000),                                         # ragged last selection block
    dict(T=1000, top_n=32, window=2000),                  # keep every block, window > T
    dict(T=777, Hq=4, Hkv=4),                             # G = 1
    dict(B=2, T=600, window=64),
    dict(T=900, gate_mode=1, fixed_gates=(0.2, 0.5, 0.3)),
    dict(T=700, d=128, Hq=8, Hkv=2, top_n=3, window=100),
])
def test_prefill_f32_edge_cases(over):
    w = inputs.workload("nsa_prefill_f32_t1024", **over)
    gc.run_nsa_prefill(w, seed=3)


@pytest.mark.parametrize("over", [
    dict(T=4000, Hq=16, Hkv=1, d=64),
    dict(T=3000, Hq=32, Hkv=2, d=128, top_n=8, window=256),
])
def test_prefill_bf16_small_all_rows(over):
    w = inputs.workload("nsa_prefill_bf16_t8192", **over)
    gc.run_nsa_prefill(w, rows=gc.sample_rows(w["T"], 400))


# Tensor-core prefill path (bf16, d = 128, 16 query heads per KV head): edges of
# its 8-token row tiles, 128-key tiles and the selection.
@pytest.mark.parametrize("over", [
    dict(T=1003),                                  # ragged last row tile and key tiles
    dict(B=2, T=517, window=100),                  # two sequences
    dict(T=20),                                    # no compressed block visible
    dict(T=300, window=1, top_n=2),                # window of one token
    dict(T=700, window=3000, top_n=16),            # window longer than the sequence
    dict(T=640, top_n=16),                         # every block selected up to t = 639
    dict(T=1500, gate_mode=1, fixed_gates=(0.2, 0.5, 0.3), top_n=5),
    dict(T=1200, Hq=32, Hkv=2, top_n=7, window=200),
])
def test_prefill_bf16_tensor_core_edges(over):
    w = inputs.workload("nsa_prefill_bf16_t8192", **dict(dict(Hq=16, Hkv=1), **over))
    gc.run_nsa_prefill(w, seed=7)


# Each branch alone on the tensor-core path, with unit-variance q, k, v so the
# outputs are O(1) and the absolute bf16 bounds are tight: a late-row error in
# one branch cannot hide behind the others or behind a small output scale.
@pytest.mark.parametrize("gates", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0)])
def test_prefill_bf16_tensor_core_branch_alone(gates):
    w = inputs.workload("nsa_prefill_bf16_t8192", T=1403, Hq=16, Hkv=1, qkv_scale=1.0,
                        gate_mode=1, fixed_gates=gates, top_n=6, window=300)
    rows = [(0, t) for t in list(range(0, 1403, 7)) + list(range(1350, 1403))]
    gc.run_nsa_prefill(w, rows=rows, seed=17)


@pytest.mark.parametrize("gates", [(1.0, 0.0, 0.0), (0.0, 1.0, 0.0), (0.0, 0.0, 1.0)])
def test_decode_bf16_fast_path_branch_alone(gates):
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=4, T=6000, gate_mode=1,
                        fixed_gates=gates)
    gc.run_nsa_decode(w, [6000, 4033, 999, 70], seed=18)


@pytest.mark.parametrize("top_n", [16, 5])
def test_prefill_bf16_tensor_core_exact_ties(top_n):
    # q = 0: every compressed score is 0, so all visible compressed blocks get
    # the same probability and every selection block fully covered by visible
    # ones gets bit-identical scores here and in the oracle. Only the rule
    # "ties go to the lower index" decides, so the selections must be equal.
    w = inputs.workload("nsa_prefill_bf16_t8192", T=3000, Hq=16, Hkv=1, top_n=top_n)
    inp = inputs.make_prefill(w, seed=23)
    inp["q"].zero_()
    rows = [(0, t) for t in [0, 63, 64, 600, 1023, 1024, 1500, 2047, 2048, 2999]]
    gc.run_nsa_prefill(w, rows=rows, inp=inp, exact_sel=True)


def test_prefill_bf16_runs_the_tensor_core_kernels():
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_prefill_bf16_t8192", T=600, Hq=16, Hkv=1)
    nsa.trace_enable(True, 64)
    try:
        gc.run_nsa_prefill(w, rows=gc.sample_rows(w["T"], 50))
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    assert {"pf_cmp_win", "pf_slc_attn"} <= names, names


def test_prefill_bf16_t65536_sampled_rows():
    w = inputs.workload("nsa_prefill_bf16_t65536")
    gc.run_nsa_prefill(w, rows=gc.sample_rows(w["T"], 40))


def test_decode_bf16_ragged():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=6, T=5000)
    lens = [1, 31, 32, 700, 4999, 5000]
    for st in gc.run_nsa_decode(w, lens):
        assert st["max_err"] <= 2e-2


def test_decode_f32_ragged():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=4, T=3000, dtype="f32", Hq=8, Hkv=2,
                        d=64, top_n=6, window=100)
    gc.run_nsa_decode(w, [17, 1025, 2999, 3000])


def test_decode_bf16_full_size_sampled_sequences():
    w = inputs.workload("nsa_decode_bf16_b32_l65536")
    gc.run_nsa_decode(w, None, check_b=[0, 13, 31])


def test_decode_bf16_many_units_ragged():
    # many (sequence, KV head) units per CTA and units split across CTAs
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=16, T=20000)
    lens = inputs.ragged_lens(16, 20000, seed=5, lo=1)
    gc.run_nsa_decode(w, lens, check_b=[0, 3, 7, 11, 15])


# Fast decode path (bf16, d = 128, 16 heads per KV head): small caches and the
# degenerate selections and gates; the trace shows the four fast kernels ran.
@pytest.mark.parametrize("over,lens", [
    (dict(B=4, T=64), [64, 40, 20, 1]),                         # a cache of one selection block
    (dict(B=3, T=33, window=1, top_n=1), [33, 32, 31]),         # one compressed block at most
    (dict(B=2, T=200, gate_mode=1, fixed_gates=(0.0, 1.0, 0.0)), [200, 129]),
    (dict(B=2, T=130, top_n=64, window=3000), [130, 65]),       # n above the candidates
])
def test_decode_bf16_fast_path_edges(over, lens):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", **over)
    nsa.trace_enable(True, 64)
    try:
        gc.run_nsa_decode(w, lens)
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    want = {"dec_select", "dec_sel_win", "dec_combine"}
    if max(lens) >= w["cmp_block"]:
        want.add("dec_cmp_partial")
    assert want <= names, names


# Quest-style block-bound selection (sel_mode 1, the pages' selection ablation)
# against the oracle's score_mode 2: bf16 with d = 128 and 16 heads per KV head
# runs the block-bounds table, its scores and top-n ahead of the tensor-core
# kernels; other shapes and fp32 run the CUDA-core row kernel.
@pytest.mark.parametrize("name,over,tc", [
    ("nsa_prefill_bf16_t8192", dict(T=300, Hq=16, Hkv=1, sel_mode=1), True),
    ("nsa_prefill_bf16_t8192", dict(B=2, T=1403, Hq=32, Hkv=2, top_n=7, window=200,
                                    sel_mode=1), True),
    ("nsa_prefill_bf16_t8192", dict(T=2100, Hq=16, Hkv=1, qkv_scale=1.0, top_n=9,
                                    sel_mode=1), True),
    ("nsa_prefill_bf16_t8192", dict(T=700, Hq=16, Hkv=1, top_n=16, sel_mode=1), True),
    ("nsa_prefill_bf16_t8192", dict(T=500, Hq=8, Hkv=1, sel_mode=1), False),
    ("nsa_prefill_f32_t1024", dict(T=400, sel_mode=1), False),
    ("nsa_prefill_f32_t1024", dict(B=2, T=130, Hq=8, Hkv=2, cmp_block=8, cmp_stride=4,
                                   sel_block=16, top_n=3, window=20, sel_mode=1), False),
])
def test_prefill_quest_selection(name, over, tc):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload(name, **over)
    nsa.trace_enable(True, 64)
    try:
        gc.run_nsa_prefill(w, rows=None if w["T"] <= 1500 else gc.sample_rows(w["T"], 300))
        recs, _ = nsa.trace_records()
        names = {nm for nm, _ in recs}
    finally:
        nsa.trace_enable(False)
    if tc:
        assert {"quest_scores", "quest_select", "pf_cmp_win", "pf_slc_attn"} <= names, names
        assert "nsa_rows_simt" not in names, names
    else:
        assert "nsa_rows_simt" in names and "pf_cmp_win" not in names, names


def test_prefill_quest_t8192_sampled_rows():
    w = inputs.workload("nsa_prefill_bf16_t8192", sel_mode=1)
    gc.run_nsa_prefill(w, rows=gc.sample_rows(w["T"], 96))


def test_decode_quest_selection():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=3, T=3000, sel_mode=1)
    gc.run_nsa_decode(w, [3000, 1777, 65])


def test_decode_bf16_group_of_8_generic_path():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=3, T=4000, Hq=32, Hkv=4)
    gc.run_nsa_decode(w, [4000, 1234, 64])


def test_decode_repeat_is_deterministic(cuda_ok):
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=4, T=9000)
    inp = inputs.make_decode(w, seq_lens=[9000, 5000, 777, 8999])
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    outs = [nsa.nsa_decode(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                           dev["w_gate"]) for _ in range(3)]
    nsa.nsa_check()
    for o, s in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(s, outs[0][1])


def test_decode_independent_of_stale_workspace(cuda_ok):
    # Workspace contents left by an earlier call (another shape) must not leak
    # into a later one: fill the workspace with garbage and compare.
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=6, T=12000)
    inp = inputs.make_decode(w, seed=11, seq_lens=[12000, 9000, 4097, 777, 64, 11999])
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    outs = []
    for fill in (0, 0x7f, 0x3c):
        ws = nsa.workspace(p, nsa.OP_DECODE)
        ws.fill_(fill)
        outs.append(nsa.nsa_decode(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                   dev["w_gate"], ws=ws))
    nsa.nsa_check()
    for o, s in outs[1:]:
        assert torch.equal(o, outs[0][0]) and torch.equal(s, outs[0][1])
    gc.run_nsa_decode(w, [12000, 9000, 4097, 777, 64, 11999], seed=11)


@pytest.mark.parametrize("want_sel", [False, True])
def test_prefill_bf16_dense_closed_form(want_sel):
    # Gates fixed to (0, 0, 1) and a window covering the sequence reduce NSA to
    # dense causal attention; the tensor-core path then skips the zero-gated
    # branches (and the selection, unless sel_idx is requested).
    from dynamic_block_sparse_nsa_b200 import nsa
    from tests import dense_ref, parity
    T = 700
    w = inputs.workload("nsa_prefill_bf16_t8192", T=T, Hq=16, Hkv=1, window=4096, gate_mode=1,
                        fixed_gates=(0.0, 0.0, 1.0))
    inp = inputs.make_prefill(w, 5)
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    out, sel = nsa.nsa_prefill(p, dev["q"], dev["k"], dev["v"], kc, vc, None, want_sel=want_sel)
    nsa.nsa_check()
    q, k, v = gc.f64(inp["q"])[0], gc.f64(inp["k"])[0], gc.f64(inp["v"])[0]
    ref = np.stack([dense_ref.masked_attention(q[:, h], k[:, 0], v[:, 0], dense_ref.causal_mask(T),
                                               1.0 / np.sqrt(128))[0] for h in range(16)], axis=1)
    parity.check_output(gc.f64(out)[0], ref, "bf16")
    if want_sel:
        s = sel.cpu().numpy()[0, :, 0]
        assert (s[:, 0] == 0).all()
        for t in range(T):
            row = s[t][s[t] >= 0]
            assert len(row) == min(w["top_n"], t // 64 + 1) and (np.diff(row) > 0).all()


# Adaptive (top-p) selection on every selection implementation. Unit-variance
# queries and keys make the block scores uneven enough that the cumulative
# rule stops before n blocks for many rows.
@pytest.mark.parametrize("top_p", [0.2, 0.5, 0.95])
def test_prefill_bf16_top_p_tensor_core(top_p):
    w = inputs.workload("nsa_prefill_bf16_t8192", T=1500, Hq=16, Hkv=1, qkv_scale=1.0, top_p=top_p)
    gc.run_nsa_prefill(w, seed=31)


def test_prefill_f32_top_p_generic():
    w = inputs.workload("nsa_prefill_f32_t1024", top_n=8, top_p=0.4)
    gc.run_nsa_prefill(w, seed=32)


@pytest.mark.parametrize("top_p", [0.3, 0.7])
def test_decode_bf16_top_p_fast(top_p):
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=4, T=5000, top_p=top_p)
    gc.run_nsa_decode(w, [5000, 3001, 700, 64])


def test_decode_f32_top_p_generic():
    w = inputs.workload("nsa_decode_bf16_b32_l65536", B=3, T=3000, dtype="f32", Hq=8, Hkv=2,
                        d=64, top_n=6, window=100, top_p=0.5)
    gc.run_nsa_decode(w, [2999, 1500, 200])


def test_prefill_top_p_stops_before_n():
    from dynamic_block_sparse_nsa_b200 import nsa
    w = inputs.workload("nsa_prefill_bf16_t8192", T=1500, Hq=16, Hkv=1, qkv_scale=1.0, top_p=0.2)
    inp = inputs.make_prefill(w, 31)
    p = gc.nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    _, sel = nsa.nsa_prefill(p, dev["q"], dev["k"], dev["v"], kc, vc, dev["w_gate"])
    nsa.nsa_check()
    counts = (sel[0, 1100:, 0] >= 0).sum(-1)
    assert int(counts.min()) < w["top_n"] and int(counts.max()) >= 2
