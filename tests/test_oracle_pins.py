"""Pins for the fp64 oracle: it is checked against things other than itself.

* an independent dense-mask formulation (tests/dense_ref.py) on small inputs;
* closed forms: full selection + full window = dense causal attention;
  l = s = 1 compression = dense causal attention; w = 1 window = v_t;
  n = 1 = attention over block 0; MoBA with k >= #blocks = dense causal,
  k = 1 = block-local causal;
* the tie rule (q = 0 gives equal scores: the lowest indices win);
* invariants: softmax mass 1, no weight on future keys, block 0 always kept,
  score totals, gates in (0, 1);
* storage rounding against torch/numpy casts and brute-force nearest search.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from tests import dense_ref

RNG = np.random.default_rng(1234)


def base_params(**kw):
    p = dict(B=1, T=192, Hq=4, Hkv=2, d=16, cmp_block=8, cmp_stride=4, sel_block=16,
             top_n=3, window=24, scale=0.0, gate_mode=0, fixed_gates=(0.0, 0.0, 0.0),
             store="none", score_mode=0)
    p.update(kw)
    return p


def rand_inputs(p, rng=RNG, qscale=1.0):
    T, Hq, Hkv, d = p["T"], p["Hq"], p["Hkv"], p["d"]
    q = rng.standard_normal((1, T, Hq, d)) * qscale
    k = rng.standard_normal((1, T, Hkv, d))
    v = rng.standard_normal((1, T, Hkv, d))
    w = rng.standard_normal(p["cmp_block"]) / math.sqrt(p["cmp_block"])
    wg = rng.standard_normal((d, 3)) / math.sqrt(d)
    return q, k, v, w, wg


def dense_causal(q, k, v, scale):
    """Textbook causal softmax attention, per head, full matrices. q [T,Hq,d]."""
    T, Hq, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros_like(q)
    for h in range(Hq):
        out[:, h], _, _ = dense_ref.masked_attention(
            q[:, h], k[:, h // G], v[:, h // G], dense_ref.causal_mask(T), scale)
    return out


# --------------------------------------------------------------------------
# storage rounding
# --------------------------------------------------------------------------

def test_round_bf16_matches_torch_cast_on_fp32_values():
    x = (RNG.standard_normal(20000) * np.exp(RNG.uniform(-30, 30, 20000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.round_store(x.astype(np.float64), "bf16")
    np.testing.assert_array_equal(got, want)


def test_round_f32_matches_numpy_cast():
    x = RNG.standard_normal(20000) * np.exp(RNG.uniform(-60, 60, 20000))
    got = oracle.round_store(x, "f32")
    np.testing.assert_array_equal(got, x.astype(np.float32).astype(np.float64))


def test_round_bf16_is_nearest_even_on_fp64_values():
    # brute force: the result is a bf16 value and no bf16 neighbour is nearer;
    # at an exact midpoint the even significand wins.
    x = RNG.standard_normal(4000) * np.exp(RNG.uniform(-20, 20, 4000))
    got = oracle.round_store(x, "bf16")
    for xi, r in zip(x, got):
        bits = np.float32(r).view(np.uint32)
        assert bits & 0xFFFF == 0 and float(np.float32(r)) == r
        e = math.frexp(r)[1]
        ulp = 2.0 ** (e - 8)
        for nb in (r - ulp, r + ulp, r - ulp / 2, r + ulp / 2):
            nb32 = np.float32(nb)
            if float(nb32) == nb and np.uint32(nb32.view(np.uint32)) & 0xFFFF == 0:
                assert abs(xi - r) <= abs(xi - nb)


def test_round_bf16_ties_and_limits():
    r = lambda x: oracle.round_store(np.array([x]), "bf16")[0]
    assert r(1.0 + 2.0 ** -8) == 1.0                     # tie -> even (down)
    assert r(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6     # tie -> even (up)
    assert r(1.0 + 2.0 ** -8 + 2.0 ** -30) == 1.0 + 2.0 ** -7
    assert r(2.0 ** 128 * (1 - 2.0 ** -9)) == math.inf   # rounds past the largest finite
    assert r(2.0 ** -134) == 0.0                          # half the smallest subnormal -> even 0
    assert r(3 * 2.0 ** -134) == 2.0 ** -132


# --------------------------------------------------------------------------
# compression
# --------------------------------------------------------------------------

def test_num_cmp_sizes():
    assert oracle.num_cmp(1024, 32, 16) == 63
    assert oracle.num_cmp(8192, 32, 16) == 511
    assert oracle.num_cmp(65536, 32, 16) == 4095
    assert oracle.num_cmp(31, 32, 16) == 0
    assert oracle.num_cmp(32, 32, 16) == 1


@pytest.mark.parametrize("j0", [0, 3, 7])
def test_compress_one_hot_picks_token(j0):
    p = base_params()
    _, k, v, _, _ = rand_inputs(p)
    w = np.zeros(p["cmp_block"])
    w[j0] = 1.0
    kc, vc = oracle.compress(p, k, v, w)
    Nc = kc.shape[1]
    np.testing.assert_array_equal(kc[0], k[0, j0:j0 + Nc * p["cmp_stride"]:p["cmp_stride"]])
    np.testing.assert_array_equal(vc[0], v[0, j0:j0 + Nc * p["cmp_stride"]:p["cmp_stride"]])


def test_compress_mean_weights_give_block_means():
    p = base_params(cmp_block=8, cmp_stride=8)
    _, k, v, _, _ = rand_inputs(p)
    kc, _ = oracle.compress(p, k, v, np.full(8, 1 / 8))
    want = k[0].reshape(p["T"] // 8, 8, p["Hkv"], p["d"]).mean(axis=1)
    np.testing.assert_allclose(kc[0], want, rtol=0, atol=1e-14)


def test_compress_bf16_store_is_rounded_exact_sum():
    p = base_params(store="bf16")
    _, k, v, w, _ = rand_inputs(p)
    kc, _ = oracle.compress(p, k, v, w)
    C = dense_ref.compression_matrix(p["T"], p["cmp_block"], p["cmp_stride"], w)
    exact = np.einsum("it,tgd->igd", C, k[0])
    np.testing.assert_allclose(kc[0], oracle.round_store(exact, "bf16"), rtol=0, atol=0)
    assert np.max(np.abs(kc[0] - exact) / np.maximum(np.abs(exact), 1e-300)) <= 2.0 ** -8


# --------------------------------------------------------------------------
# whole NSA against the independent dense-mask formulation
# --------------------------------------------------------------------------

@pytest.mark.parametrize("kw", [
    dict(),
    dict(T=257, Hq=6, Hkv=3, window=1),
    dict(T=130, Hq=2, Hkv=2, top_n=1, window=200),
    dict(T=256, Hq=8, Hkv=1, d=8, top_n=5, score_mode=1),
    dict(T=96, cmp_block=32, cmp_stride=16, sel_block=64, top_n=2, window=40),
])
def test_nsa_matches_dense_mask_formulation(kw):
    p = base_params(**kw)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    want = dense_ref.nsa_dense(p, q[0], k[0], v[0], w, wg)
    for key in ("o_cmp", "o_slc", "o_win", "gates", "out"):
        np.testing.assert_allclose(got[key], want[key], rtol=0, atol=1e-12, err_msg=key)
    fin = np.isfinite(want["scores"])
    np.testing.assert_array_equal(np.isfinite(got["scores"]), fin)
    np.testing.assert_allclose(got["scores"][fin], want["scores"][fin], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(got["sel"], want["sel"])
    lf = np.isfinite(want["lse_cmp"])
    np.testing.assert_array_equal(np.isfinite(got["lse_cmp"]), lf)
    np.testing.assert_allclose(got["lse_cmp"][lf], want["lse_cmp"][lf], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("gates", [(0.0, 1.0, 0.0), (0.0, 0.0, 1.0)])
def test_full_selection_and_window_is_dense_causal(gates):
    p = base_params(T=200, top_n=13, window=200, gate_mode=1, fixed_gates=gates)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    want = dense_causal(q[0], k[0], v[0], 1 / math.sqrt(p["d"]))
    np.testing.assert_allclose(got["out"], want, rtol=0, atol=1e-12)


def test_unit_compression_is_dense_causal_and_scores_are_block_mass():
    p = base_params(T=160, cmp_block=1, cmp_stride=1, sel_block=16)
    q, k, v, _, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, np.ones(1), wg)
    scale = 1 / math.sqrt(p["d"])
    want = dense_causal(q[0], k[0], v[0], scale)
    np.testing.assert_allclose(got["o_cmp"], want, rtol=0, atol=1e-12)
    # block score = sum over the group's heads of the causal attention mass on the block
    T, G = p["T"], p["Hq"] // p["Hkv"]
    for g in range(p["Hkv"]):
        mass = np.zeros((T, T))
        for hh in range(G):
            h = g * G + hh
            z = scale * q[0, :, h] @ k[0, :, g].T
            z[~dense_ref.causal_mask(T)] = -np.inf
            e = np.exp(z - z.max(axis=1, keepdims=True))
            mass += e / e.sum(axis=1, keepdims=True)
        for t in range(T):
            nb = t // 16 + 1
            blk = [mass[t, 16 * j:16 * j + 16].sum() for j in range(nb)]
            np.testing.assert_allclose(got["scores"][t, g, :nb], blk, rtol=0, atol=1e-12)


def test_window_of_one_returns_current_value():
    p = base_params(window=1)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    G = p["Hq"] // p["Hkv"]
    for h in range(p["Hq"]):
        np.testing.assert_array_equal(got["o_win"][:, h], v[0, :, h // G])


def test_top_one_attends_block_zero_only():
    p = base_params(top_n=1)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    assert np.all(got["sel"][:, :, 0] == 0)
    bs, T, G = p["sel_block"], p["T"], p["Hq"] // p["Hkv"]
    mask = dense_ref.causal_mask(T) & (np.arange(T)[None, :] < bs)
    for h in range(p["Hq"]):
        o, _, _ = dense_ref.masked_attention(q[0, :, h], k[0, :, h // G], v[0, :, h // G], mask,
                                             1 / math.sqrt(p["d"]))
        np.testing.assert_allclose(got["o_slc"][:, h], o, rtol=0, atol=1e-12)


def test_equal_scores_pick_lowest_indices():
    # q = 0: every visible compressed key gets the same probability, so all
    # full selection blocks tie; the tie rule keeps the lowest block indices.
    p = base_params(T=256, top_n=4)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, np.zeros_like(q), k, v, w, wg)
    for t in range(128, 256):
        for g in range(p["Hkv"]):
            assert list(got["sel"][t, g]) == [0, 1, 2, 3], (t, got["sel"][t, g])


def test_selection_maximises_score_sum_brute_force():
    p = base_params(T=128, sel_block=8, top_n=4, cmp_block=4, cmp_stride=2)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    n = p["top_n"]
    for t in range(0, 128, 7):
        for g in range(p["Hkv"]):
            nc = t // 8 + 1
            sc = got["scores"][t, g, :nc]
            S = list(got["sel"][t, g][got["sel"][t, g] >= 0])
            if nc <= n:
                assert S == list(range(nc))
                continue
            assert S[0] == 0
            best = max(sum(sc[list(c)]) for c in itertools.combinations(range(1, nc), n - 1))
            assert abs(sum(sc[S[1:]]) - best) <= 1e-12


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_softmax_mass_is_one():
    p = base_params(store="none")
    q, k, v, w, wg = rand_inputs(p)
    ones = np.ones_like(v)
    got = oracle.nsa_prefill(p, q, k, ones, w, wg)
    np.testing.assert_allclose(got["o_slc"], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got["o_win"], 1.0, rtol=0, atol=1e-12)
    vis = np.arange(p["T"]) >= p["cmp_block"] - 1
    np.testing.assert_allclose(got["o_cmp"][vis], w.sum(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(got["o_cmp"][~vis], 0.0)


def test_future_tokens_carry_no_weight():
    p = base_params()
    q, k, v, w, wg = rand_inputs(p)
    a = oracle.nsa_prefill(p, q, k, v, w, wg)
    t0 = 100
    k2, v2 = k.copy(), v.copy()
    k2[0, t0 + 1:] = RNG.standard_normal(k2[0, t0 + 1:].shape) * 5
    v2[0, t0 + 1:] = RNG.standard_normal(v2[0, t0 + 1:].shape) * 5
    b = oracle.nsa_prefill(p, q, k2, v2, w, wg)
    for key in ("out", "o_cmp", "o_slc", "o_win"):
        np.testing.assert_array_equal(a[key][: t0 + 1], b[key][: t0 + 1])
    np.testing.assert_array_equal(a["sel"][: t0 + 1], b["sel"][: t0 + 1])


@pytest.mark.parametrize("score_mode", [0, 1])
def test_score_totals_block_zero_and_gates(score_mode):
    p = base_params(score_mode=score_mode)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    G = p["Hq"] // p["Hkv"]
    T = p["T"]
    assert np.all(got["sel"][:, :, 0] == 0)
    assert np.all((got["gates"] > 0) & (got["gates"] < 1))
    tot = np.where(np.isfinite(got["scores"]), got["scores"], 0).sum(axis=2)
    vis = np.arange(T) >= p["cmp_block"] - 1
    np.testing.assert_array_equal(tot[~vis], 0.0)
    if score_mode == 1:
        np.testing.assert_allclose(tot[vis], G, rtol=0, atol=1e-12)
    else:
        assert np.all(tot[vis] >= G - 1e-12) and np.all(tot[vis] <= 2 * G + 1e-12)


def test_single_head_groups_select_per_head():
    # G = 1: each head's selection is the top set of its own compressed mass
    p = base_params(Hq=3, Hkv=3)
    q, k, v, w, wg = rand_inputs(p)
    got = oracle.nsa_prefill(p, q, k, v, w, wg)
    want = dense_ref.nsa_dense(p, q[0], k[0], v[0], w, wg)
    np.testing.assert_array_equal(got["sel"], want["sel"])


def test_decode_equals_prefill_row_of_prefix():
    p = base_params(B=3, T=150)
    rng = np.random.default_rng(7)
    _, k, v, w, wg = rand_inputs(dict(p, T=150), rng)
    k = rng.standard_normal((3, 150, p["Hkv"], p["d"]))
    v = rng.standard_normal((3, 150, p["Hkv"], p["d"]))
    qd = rng.standard_normal((3, p["Hq"], p["d"]))
    lens = [150, 61, 9]
    kc, vc = oracle.compress(p, k, v, w)
    dec = oracle.nsa_decode(p, qd, k, v, lens, kc, vc, wg)
    for b, L in enumerate(lens):
        pp = dict(p, B=1, T=L)
        qp = np.zeros((1, L, p["Hq"], p["d"]))
        qp[0, L - 1] = qd[b]
        pre = oracle.nsa_prefill(pp, qp, k[b:b + 1, :L], v[b:b + 1, :L], w, wg, rows=[(0, L - 1)])
        np.testing.assert_array_equal(dec["out"][b], pre["out"][0])
        np.testing.assert_array_equal(dec["sel"][b], pre["sel"][0])


# --------------------------------------------------------------------------
# MoBA
# --------------------------------------------------------------------------

def moba_params(**kw):
    p = dict(B=1, T=200, Hq=4, Hkv=2, d=16, block=16, top_k=3, scale=0.0)
    p.update(kw)
    return p


@pytest.mark.parametrize("kw", [dict(), dict(T=256, Hq=3, Hkv=3, top_k=2), dict(top_k=1)])
def test_moba_matches_dense_mask_formulation(kw):
    p = moba_params(**kw)
    q, k, v, _, _ = rand_inputs(dict(p, cmp_block=1))
    got = oracle.moba_prefill(p, q, k, v)
    want = dense_ref.moba_dense(p, q[0], k[0], v[0])
    np.testing.assert_allclose(got["out"], want["out"], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(got["sel"], want["sel"])


def test_moba_all_blocks_is_dense_causal():
    p = moba_params(top_k=13)
    q, k, v, _, _ = rand_inputs(dict(p, cmp_block=1))
    got = oracle.moba_prefill(p, q, k, v)
    np.testing.assert_allclose(got["out"], dense_causal(q[0], k[0], v[0], 1 / math.sqrt(16)),
                               rtol=0, atol=1e-12)


def test_moba_top_one_is_block_local_causal():
    p = moba_params(top_k=1)
    q, k, v, _, _ = rand_inputs(dict(p, cmp_block=1))
    got = oracle.moba_prefill(p, q, k, v)
    T, m = p["T"], p["block"]
    tp = np.arange(T)
    mask = dense_ref.causal_mask(T) & ((tp[:, None] // m) == (tp[None, :] // m))
    G = p["Hq"] // p["Hkv"]
    for h in range(p["Hq"]):
        o, _, _ = dense_ref.masked_attention(q[0, :, h], k[0, :, h // G], v[0, :, h // G], mask,
                                             1 / math.sqrt(16))
        np.testing.assert_allclose(got["out"][:, h], o, rtol=0, atol=1e-12)


def test_moba_block_means():
    p = moba_params()
    _, k, _, _, _ = rand_inputs(dict(p, cmp_block=1))
    kbar = oracle.moba_block_means(p, k)
    want = k[0, :192].reshape(12, 16, p["Hkv"], p["d"]).mean(axis=1)
    np.testing.assert_allclose(kbar[0], want, rtol=0, atol=1e-14)


# --------------------------------------------------------------------------
# adaptive (top-p) selection: lchairun NSA article, adaptive sparsification
# (choose from the most important block on until the chosen scores reach p
# times the total). Properties that fix the rule given the block scores:
# --------------------------------------------------------------------------

def _topp_rows(p):
    q, k, v, w, wg = rand_inputs(p, rng=np.random.default_rng(77), qscale=3.0)
    return oracle.nsa_prefill(p, q, k, v, w, wg)


@pytest.mark.parametrize("top_p", [0.3, 0.6, 0.9])
def test_topp_selection_is_the_shortest_best_prefix(top_p):
    n = 12
    p = base_params(T=256, sel_block=8, top_n=n, cmp_block=4, cmp_stride=2, top_p=top_p)
    got = _topp_rows(p)
    for t in range(0, 256, 5):
        for g in range(p["Hkv"]):
            nc = t // 8 + 1
            sc = got["scores"][t, g, :nc]
            S = [int(j) for j in got["sel"][t, g] if j >= 0]
            assert S[0] == 0 and len(S) <= min(n, nc)          # block 0 kept, at most n
            others = sorted(range(1, nc), key=lambda j: (-sc[j], j))
            m = len(S) - 1
            assert sorted(S[1:]) == sorted(others[:m])          # the m best of the others
            total = sc.sum()
            chosen = sc[0] + sum(sc[j] for j in others[:m])
            if len(S) < min(n, nc):
                assert chosen >= top_p * total - 1e-12         # reaches p of the total
            if m > 0:                                           # and is the shortest such prefix
                assert chosen - sc[others[m - 1]] < top_p * total + 1e-12


def test_topp_grows_with_p_and_tiny_p_keeps_block_zero():
    base = dict(T=256, sel_block=8, top_n=16, cmp_block=4, cmp_stride=2)
    sels = [_topp_rows(base_params(**base, top_p=tp))["sel"] for tp in (1e-12, 0.4, 0.8, 1.0)]
    for t in range(0, 256, 3):
        for g in range(2):
            a = [set(int(j) for j in s[t, g] if j >= 0) for s in sels]
            assert a[0] == {0}
            assert a[0] <= a[1] <= a[2] <= a[3]


# --------------------------------------------------------------------------
# backward oracle (oracle/backward.py)
# --------------------------------------------------------------------------

def _bwd_case(seed, **kw):
    p = base_params(B=2, T=70, Hq=4, Hkv=2, d=8, window=12, **kw)
    rng = np.random.default_rng(seed)
    B, T, Hq, Hkv, d = p["B"], p["T"], p["Hq"], p["Hkv"], p["d"]
    q = rng.standard_normal((B, T, Hq, d))
    k = rng.standard_normal((B, T, Hkv, d))
    v = rng.standard_normal((B, T, Hkv, d))
    w = rng.standard_normal(p["cmp_block"]) / math.sqrt(p["cmp_block"])
    wg = rng.standard_normal((d, 3)) / math.sqrt(d)
    dout = rng.standard_normal((B, T, Hq, d))
    fwd = oracle.nsa_prefill(p, q, k, v, w, wg)
    sel = fwd["sel"].reshape(B, T, Hkv, p["top_n"])
    return p, q, k, v, w, wg, dout, fwd, sel


def test_backward_matches_finite_differences_of_the_forward():
    """Central differences of the C forward oracle (selection held at the
    forward's choice) against the analytic gradient of every input."""
    from oracle import backward
    p, q, k, v, w, wg, dout, fwd, sel = _bwd_case(5)
    B, T, Hq, d = q.shape
    grads = backward.nsa_prefill_backward(p, q, k, v, w, wg, dout, sel)
    np.testing.assert_allclose(grads["out"], fwd["out"].reshape(B, T, Hq, d), atol=1e-12)
    forced = sel.reshape(B * T, p["Hkv"], p["top_n"])

    def loss(q, k, v, w, wg):
        r = oracle.nsa_prefill(p, q, k, v, w, wg, forced_sel=forced)
        return float(np.sum(dout.reshape(-1, Hq, d) * r["out"]))

    args = {"q": q, "k": k, "v": v, "w": w, "wg": wg}
    names = {"q": "dq", "k": "dk", "v": "dv", "w": "dw_cmp", "wg": "dwg"}
    rng = np.random.default_rng(6)
    eps = 1e-6
    for name, arr in args.items():
        for _ in range(10):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus = {a: b.copy() for a, b in args.items()}
            minus = {a: b.copy() for a, b in args.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd = (loss(**plus) - loss(**minus)) / (2 * eps)
            an = grads[names[name]][idx]
            assert abs(fd - an) <= 1e-6 * (1.0 + abs(an)), (name, idx, fd, an)


def test_backward_window_only_equals_autograd_of_softmax_attention():
    """Gates (0, 0, 1): the output is sliding-window attention, whose gradient
    torch autograd gives for a plain masked-softmax formulation in fp64."""
    from oracle import backward
    p, q, k, v, w, wg, dout, _, sel = _bwd_case(7, gate_mode=1, fixed_gates=(0.0, 0.0, 1.0))
    B, T, Hq, d = q.shape
    G = Hq // p["Hkv"]
    grads = backward.nsa_prefill_backward(p, q, k, v, w, wg, dout, sel)
    qt, kt, vt = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    kh = kt.repeat_interleave(G, dim=2)  # [B, T, Hq, d]: head h reads KV head h // G
    vh = vt.repeat_interleave(G, dim=2)
    s = torch.einsum("bthe,buhe->bhtu", qt, kh) / math.sqrt(d)
    t_idx = torch.arange(T)
    allowed = (t_idx[None, :] <= t_idx[:, None]) & (t_idx[None, :] > t_idx[:, None] - p["window"])
    s = s.masked_fill(~allowed, float("-inf"))
    o = torch.einsum("bhtu,buhe->bthe", torch.softmax(s, dim=-1), vh)
    (o * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(grads["dq"], qt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(grads["dk"], kt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(grads["dv"], vt.grad.numpy(), atol=1e-12)
    assert np.all(grads["dw_cmp"] == 0.0) and np.all(grads["dwg"] == 0.0)


def test_backward_value_gradient_sums_to_the_gated_upstream():
    """Softmax weights sum to one, so the value gradients of a branch sum to
    its gated upstream gradient: sum_u dv[u] = sum over rows and the group's
    heads of (g_slc + g_win + g_cmp sum_j w_j [a compressed block is visible]) dout."""
    from oracle import backward
    p, q, k, v, w, wg, dout, fwd, sel = _bwd_case(9)
    B, T, Hq, d = q.shape
    G = Hq // p["Hkv"]
    grads = backward.nsa_prefill_backward(p, q, k, v, w, wg, dout, sel)
    gates = fwd["gates"].reshape(B, T, Hq, 3)
    vis = (np.arange(T) + 1 >= p["cmp_block"]).astype(np.float64)
    coef = gates[..., 1] + gates[..., 2] + gates[..., 0] * w.sum() * vis[None, :, None]
    want = (coef[..., None] * dout).reshape(B, T, p["Hkv"], G, d).sum(axis=(1, 3))
    np.testing.assert_allclose(grads["dv"].sum(axis=1), want, atol=1e-10)


# --------------------------------------------------------------------------
# Quest-style block bound (score_mode 2)
# --------------------------------------------------------------------------

def test_quest_bound_is_the_box_maximum_and_bounds_every_key():
    """The largest q . x over the axis-aligned box of a block's keys is attained
    at a corner; brute force over all 2^d corners (d = 4) must give the score,
    summed over the group's heads, and it bounds q . k of every key."""
    p = base_params(T=90, Hq=4, Hkv=2, d=4, sel_block=8, score_mode=2)
    q, k, v, w, wg = rand_inputs(p, rng=np.random.default_rng(41))
    res = oracle.nsa_prefill(p, q, k, v, w, wg)
    G, bs, d = 2, p["sel_block"], p["d"]
    corners = np.array(list(itertools.product([0, 1], repeat=d)))
    for t in (0, 3, 7, 8, 40, 89):
        for g in range(p["Hkv"]):
            for j in range(t // bs + 1):
                keys = k[0, j * bs:min(j * bs + bs, t + 1), g]
                box = np.where(corners == 0, keys.min(axis=0), keys.max(axis=0))
                want = best = 0.0
                for hh in range(G):
                    qh = q[0, t, g * G + hh]
                    want += (box @ qh).max()
                    best += (keys @ qh).max()
                got = res["scores"][t, g, j]
                assert abs(got - want) <= 1e-12 * (1 + abs(want)), (t, g, j)
                assert got >= best - 1e-12


def test_quest_with_one_token_blocks_selects_by_summed_logits():
    """Blocks of one token: the bound is q . k itself, so the score of token j is
    the group's summed logits and the selection is token 0 plus the n-1 best."""
    p = base_params(T=60, Hq=4, Hkv=2, d=16, sel_block=1, top_n=5, score_mode=2)
    q, k, v, w, wg = rand_inputs(p, rng=np.random.default_rng(42))
    res = oracle.nsa_prefill(p, q, k, v, w, wg)
    G = 2
    for t in (4, 5, 30, 59):
        for g in range(p["Hkv"]):
            logit = sum(k[0, :t + 1, g] @ q[0, t, g * G + hh] for hh in range(G))
            np.testing.assert_allclose(res["scores"][t, g, :t + 1], logit, rtol=0, atol=1e-12)
            order = [j for j in np.argsort(-logit[1:], kind="stable") + 1][:p["top_n"] - 1]
            assert sorted(int(x) for x in res["sel"][t, g]) == sorted([0] + order)


def test_quest_ignores_future_tokens_of_the_current_block():
    p = base_params(T=70, sel_block=16, score_mode=2)
    q, k, v, w, wg = rand_inputs(p, rng=np.random.default_rng(43))
    base = oracle.nsa_prefill(p, q, k, v, w, wg, rows=[(0, 37)])
    k2 = k.copy()
    k2[0, 38:48] += 5.0  # later tokens of block 2, which holds t = 37
    moved = oracle.nsa_prefill(p, q, k2, v, w, wg, rows=[(0, 37)])
    np.testing.assert_array_equal(base["scores"], moved["scores"])


# --------------------------------------------------------------------------
# exact token top-k (oracle/variants.py; oracle-level variant only)
# --------------------------------------------------------------------------

def _topk_case(seed, **kw):
    p = base_params(T=80, Hq=4, Hkv=2, d=8, sel_block=4, top_n=3, window=10, **kw)
    q, k, v, w, wg = rand_inputs(p, rng=np.random.default_rng(seed))
    return p, q, k, v, w, wg


def test_exact_topk_with_every_token_is_dense_causal_attention():
    from oracle import variants
    p, q, k, v, w, wg = _topk_case(51)
    rows = [(0, t) for t in (0, 5, 11, 40, 79)]
    res = variants.exact_topk_rows(p, q, k, v, w, wg, rows, ktok=p["T"])
    G = 2
    for r, (_, t) in enumerate(rows):
        for h in range(p["Hq"]):
            z = k[0, :t + 1, h // G] @ q[0, t, h] / math.sqrt(p["d"])
            pr = np.exp(z - z.max())
            pr /= pr.sum()
            np.testing.assert_allclose(res["o_slc"][r, h], pr @ v[0, :t + 1, h // G], atol=1e-12)


def test_exact_topk_of_one_is_the_value_of_the_heaviest_token():
    from oracle import variants
    p, q, k, v, w, wg = _topk_case(52, gate_mode=1, fixed_gates=(0.0, 1.0, 0.0))
    rows = [(0, t) for t in (3, 20, 79)]
    res = variants.exact_topk_rows(p, q, k, v, w, wg, rows, ktok=1)
    G = 2
    for r, (_, t) in enumerate(rows):
        for g in range(p["Hkv"]):
            mass = np.zeros(t + 1)
            for hh in range(G):
                z = k[0, :t + 1, g] @ q[0, t, g * G + hh] / math.sqrt(p["d"])
                e = np.exp(z - z.max())
                mass += e / e.sum()
            u = int(np.argmax(mass))  # first maximum: the lower index on a tie
            assert res["sel"][r, g, 0] == u
            for hh in range(G):
                np.testing.assert_allclose(res["out"][r, g * G + hh], v[0, u, g], atol=1e-12)


def test_exact_topk_set_is_the_heaviest_tokens():
    from oracle import variants
    p, q, k, v, w, wg = _topk_case(53)
    rows = [(0, t) for t in (12, 50, 79)]
    res = variants.exact_topk_rows(p, q, k, v, w, wg, rows)
    ktok = p["top_n"] * p["sel_block"]
    G = 2
    for r, (_, t) in enumerate(rows):
        for g in range(p["Hkv"]):
            mass = np.zeros(t + 1)
            for hh in range(G):
                z = k[0, :t + 1, g] @ q[0, t, g * G + hh] / math.sqrt(p["d"])
                e = np.exp(z - z.max())
                mass += e / e.sum()
            want = sorted(np.lexsort((np.arange(t + 1), -mass))[:ktok].tolist())
            got = [int(x) for x in res["sel"][r, g] if x >= 0]
            assert got == want
