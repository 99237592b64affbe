"""Runners shared by the GPU parity tests: one GPU call through the C ABI, the
oracle on the same seeded inputs, and the parity rules of tests/parity.py."""
import numpy as np
import torch

import oracle
from dynamic_block_sparse_nsa_b200 import inputs
from dynamic_block_sparse_nsa_b200 import nsa
from tests import parity


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def nsa_params_for(w, **kw):
    return nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], cmp_block=w["cmp_block"],
                      cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                      window=w["window"], gate_mode=w.get("gate_mode", 0),
                      fixed_gates=w.get("fixed_gates", (0.0, 0.0, 0.0)),
                      dtype=inputs.DTYPES[w["dtype"]], top_p=w.get("top_p", 0.0),
                      sel_mode=w.get("sel_mode", 0), **kw)


def oracle_params_for(w):
    return dict(B=w["B"], T=w["T"], Hq=w["Hq"], Hkv=w["Hkv"], d=w["d"],
                cmp_block=w["cmp_block"], cmp_stride=w["cmp_stride"], sel_block=w["sel_block"],
                top_n=w["top_n"], window=w["window"], scale=0.0,
                gate_mode=w.get("gate_mode", 0), fixed_gates=w.get("fixed_gates", (0.0, 0.0, 0.0)),
                store=w["dtype"], score_mode=2 if w.get("sel_mode", 0) == 1 else 0,
                top_p=w.get("top_p", 0.0))


def compare_nsa_rows(w, op, rows_b, rows_t, q_rows, k64, v64, kc64, vc64, wg64, gpu_out, gpu_sel,
                     exact_sel=False):
    """Oracle on the listed rows, selection rule, forced re-run, output check.
    exact_sel: the selections must be equal element by element (inputs whose
    block scores tie exactly on both sides, where only the tie rule decides)."""
    res = oracle.nsa_rows(op, rows_b, rows_t, q_rows, k64, v64, kc64, vc64, wg64)
    if exact_sel:
        np.testing.assert_array_equal(gpu_sel, res["sel"])
    n, bs = w["top_n"], w["sel_block"]
    differ = np.zeros(len(rows_b), dtype=bool)
    for r, t in enumerate(rows_t):
        for g in range(w["Hkv"]):
            if w.get("top_p", 0.0) > 0.0:
                same = parity.check_selection_topp(gpu_sel[r, g], res["sel"][r, g],
                                                   res["scores"][r, g], t // bs + 1, n, w["top_p"])
            else:
                # Quest bounds can sit near zero: their near-tie scale is the
                # row's largest score magnitude
                sc = res["scores"][r, g]
                abs_scale = (float(np.abs(sc[:t // bs + 1]).max())
                             if w.get("sel_mode", 0) == 1 else 0.0)
                same = parity.check_selection(gpu_sel[r, g], res["sel"][r, g], sc, t // bs + 1, n,
                                              abs_scale=abs_scale)
            differ[r] |= not same
    if differ.any():
        idx = np.nonzero(differ)[0]
        forced = oracle.nsa_rows(op, np.asarray(rows_b)[idx], np.asarray(rows_t)[idx],
                                 q_rows[idx], k64, v64, kc64, vc64, wg64,
                                 forced_sel=gpu_sel[idx])
        res["out"][idx] = forced["out"]
    stats = parity.check_output(gpu_out, res["out"], w["dtype"])
    return dict(max_err=stats[0], mean_err=stats[1], sel_near_ties=int(differ.sum()))


def run_nsa_prefill(w, rows=None, seed=None, inp=None, exact_sel=False):
    """GPU compress + prefill on workload w; oracle on `rows` (list of (b, t))."""
    if inp is None:
        inp = inputs.make_prefill(w, seed)
    p = nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    wg = dev["w_gate"] if w.get("gate_mode", 0) == 0 else None
    out, sel = nsa.nsa_prefill(p, dev["q"], dev["k"], dev["v"], kc, vc, wg)
    nsa.nsa_check()
    op = oracle_params_for(w)
    k64, v64 = f64(inp["k"]), f64(inp["v"])
    kc64, vc64 = oracle.compress(op, k64, v64, f64(inp["w_cmp"]))
    # the compressed blocks are the correctly rounded exact sums on both sides
    np.testing.assert_array_equal(f64(kc), kc64)
    np.testing.assert_array_equal(f64(vc), vc64)
    if rows is None:
        rows = [(b, t) for b in range(w["B"]) for t in range(w["T"])]
    rb = np.array([r[0] for r in rows])
    rt = np.array([r[1] for r in rows])
    q64 = f64(inp["q"])
    out_h = f64(out)[rb, rt]
    sel_h = sel.cpu().numpy()[rb, rt]
    return compare_nsa_rows(w, op, rb, rt, q64[rb, rt], k64, v64, kc64, vc64,
                            f64(inp["w_gate"]), out_h, sel_h, exact_sel=exact_sel)


def run_nsa_decode(w, seq_lens, check_b=None, seed=None, inp=None, quest_table=False):
    """GPU decode against the oracle. quest_table: the Quest-style selection
    through nsa_decode_quest with a block-bounds table from nsa_block_bounds."""
    if inp is None:
        inp = inputs.make_decode(w, seed, seq_lens)
    p = nsa_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    if quest_table:
        kb = nsa.nsa_block_bounds(p, dev["k"], dev["seq_lens"])
        out, sel = nsa.nsa_decode_quest(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                        kb, dev["w_gate"])
    else:
        out, sel = nsa.nsa_decode(p, dev["q"], dev["k"], dev["v"], dev["seq_lens"], kc, vc,
                                  dev["w_gate"])
    nsa.nsa_check()
    if check_b is None:
        check_b = list(range(w["B"]))
    op = oracle_params_for(dict(w, B=1))
    wc64, wg64 = f64(inp["w_cmp"]), f64(inp["w_gate"])
    out_h, sel_h = f64(out), sel.cpu().numpy()
    stats = []
    for b in check_b:
        L = int(inp["seq_lens"][b])
        k64 = f64(inp["k"][b:b + 1])
        v64 = f64(inp["v"][b:b + 1])
        kc64, vc64 = oracle.compress(op, k64, v64, wc64)
        np.testing.assert_array_equal(f64(kc[b:b + 1]), kc64)
        stats.append(compare_nsa_rows(w, op, [0], [L - 1], f64(inp["q"][b:b + 1]), k64, v64,
                                      kc64, vc64, wg64, out_h[b:b + 1], sel_h[b:b + 1]))
    return stats


def moba_params_for(w):
    return nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], sel_block=w["block"],
                      top_n=w["top_k"], dtype=inputs.DTYPES[w["dtype"]])


def run_moba(w, rows=None, heads=None, seed=None):
    """GPU MoBA prefill; oracle on rows x heads (heads: a subset, MHA only)."""
    inp = inputs.make_prefill(w, seed)
    p = moba_params_for(w)
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    out, sel = nsa.moba_prefill(p, dev["q"], dev["k"], dev["v"])
    nsa.nsa_check()
    if rows is None:
        rows = [(b, t) for b in range(w["B"]) for t in range(w["T"])]
    rb = np.array([r[0] for r in rows])
    rt = np.array([r[1] for r in rows])
    q, k, v = inp["q"], inp["k"], inp["v"]
    Hq, Hkv = w["Hq"], w["Hkv"]
    if heads is not None:
        assert Hq == Hkv, "head subsets need independent heads (MHA)"
        q, k, v = q[:, :, heads], k[:, :, heads], v[:, :, heads]
        Hq = Hkv = len(heads)
    op = dict(B=w["B"], T=w["T"], Hq=Hq, Hkv=Hkv, d=w["d"], block=w["block"], top_k=w["top_k"],
              scale=0.0)
    q64 = f64(q)
    res = oracle.moba_rows(op, rb, rt, q64[rb, rt], f64(k), f64(v))
    out_h = f64(out)[rb, rt]
    sel_h = sel.cpu().numpy()[rb, rt]
    if heads is not None:
        out_h, sel_h = out_h[:, heads], sel_h[:, heads]
    m, K = w["block"], w["top_k"]
    differ = np.zeros(len(rb), dtype=bool)
    for r, t in enumerate(rt):
        own = t // m
        for h in range(Hq):
            if own <= K - 1:
                assert sorted(sel_h[r, h][sel_h[r, h] >= 0]) == list(range(own + 1))
                continue
            same = parity.check_selection(sel_h[r, h], res["sel"][r, h], res["scores"][r, h],
                                          own, K, forced_first=False, forced_block=own)
            differ[r] |= not same
    if differ.any():
        idx = np.nonzero(differ)[0]
        forced = oracle.moba_rows(op, rb[idx], rt[idx], q64[rb[idx], rt[idx]], f64(k), f64(v),
                                  forced_sel=sel_h[idx])
        res["out"][idx] = forced["out"]
    st = parity.check_output(out_h, res["out"], w["dtype"])
    return dict(max_err=st[0], mean_err=st[1], sel_near_ties=int(differ.sum()))


def sample_rows(T, n, seed=0, B=1):
    """Rows spanning the first compressed blocks, block edges, random middle, last."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 30, 31, 32, 63, 64, 65, 127, 128, 511, 512, 513, T - 2, T - 1]
    fixed = [t for t in fixed if 0 <= t < T]
    extra = list(rng.integers(0, T, max(0, n - len(fixed))))
    ts = sorted(set(fixed + [int(x) for x in extra]))
    return [(b, t) for b in range(B) for t in ts]


def run_backward(w, seed, tol):
    """GPU prefill backward against the fp64 backward oracle (selection and
    compressed cache from the oracle's forward); asserts every gradient within
    tol of its largest magnitude and returns the relative errors."""
    from oracle import backward as obwd
    inp = inputs.make_prefill(w, seed)
    p = nsa_params_for(w)
    op = oracle_params_for(w)
    B, T, Hq, d = inp["q"].shape
    dev = {k_: v_.cuda() for k_, v_ in inp.items()}
    kc, vc = nsa.nsa_compress_kv(p, dev["k"], dev["v"], dev["w_cmp"])
    q64, k64, v64 = f64(inp["q"]), f64(inp["k"]), f64(inp["v"])
    wc64, wg64 = f64(inp["w_cmp"]), f64(inp["w_gate"])
    kc64, vc64 = oracle.compress(op, k64, v64, wc64)
    np.testing.assert_array_equal(f64(kc), kc64)
    fwd = oracle.nsa_prefill(op, q64, k64, v64, wc64, wg64)
    sel = fwd["sel"].reshape(B, T, p.Hkv, p.top_n)
    gen = torch.Generator().manual_seed(seed + 1)
    dout = torch.randn(B, T, Hq, d, generator=gen).to(inp["q"].dtype)
    got = nsa.nsa_prefill_backward(p, dev["q"], dev["k"], dev["v"], kc, vc, dev["w_cmp"],
                                   dev["w_gate"], torch.from_numpy(sel).cuda(), dout.cuda())
    nsa.nsa_check()
    ref = obwd.nsa_prefill_backward(op, q64, k64, v64, wc64, wg64, f64(dout), sel,
                                    kc=kc64, vc=vc64)
    stats = {}
    for name, g in zip(("dq", "dk", "dv", "dw_cmp", "dwg"), got):
        r = ref[name]
        err = float(np.abs(f64(g) - r).max()) if r.size else 0.0
        scale = max(float(np.abs(r).max()) if r.size else 0.0, 1e-6)
        stats[name] = (err, scale)
    for name, (err, scale) in stats.items():
        assert err <= tol * scale, (name, err, scale)
    return {k_: e / s for k_, (e, s) in stats.items()}
