"""Parity rules shared by the GPU tests.

Selection: the GPU's block set must equal the oracle's wherever the oracle's
last kept and first dropped non-forced candidates differ by more than 1e-5
relative. Elsewhere the GPU set must still be a valid top set of the oracle's
scores within that tolerance; those rows are then re-run through the oracle
with the GPU's selection forced, and outputs are compared on every row.

Outputs: fp32 max |err| <= 1e-4; bf16 max |err| <= 2e-2 and mean |err| <= 2e-3;
and the same bounds times the reference's largest magnitude when it is below 1.
"""
import numpy as np

SEL_REL = 1e-5
TOL = {"f32": dict(max=1e-4, mean=1e-4), "bf16": dict(max=2e-2, mean=2e-3)}


def _ranked(scores, lo, hi):
    """Candidate indices lo..hi-1 sorted by (score desc, index asc)."""
    idx = np.arange(lo, hi)
    return idx[np.lexsort((idx, -scores[lo:hi]))]


def check_selection(gpu_sel, ora_sel, ora_scores, ncand, n_keep, forced_first=True,
                    forced_block=None, abs_scale=0.0):
    """Compare one row's selection. Returns True if the sets are equal, False if
    they differ but the difference is allowed (a near tie); raises otherwise.

    ncand: candidate blocks are 0..ncand-1 (NSA) -- for MoBA pass the number of
    earlier blocks and forced_block = own block. abs_scale: a floor for the
    scale the relative near-tie gap is taken of (scores that can be near zero).
    """
    g = sorted(int(x) for x in gpu_sel if x >= 0)
    o = sorted(int(x) for x in ora_sel if x >= 0)
    if g == o:
        return True
    lo = 1 if forced_first else 0
    want = n_keep - 1  # non-forced picks
    if forced_first and ncand <= n_keep:
        raise AssertionError(f"selection differs with no choice to make: gpu {g} oracle {o}")
    ranked = _ranked(ora_scores, lo, ncand)
    if len(ranked) <= want:
        raise AssertionError(f"selection differs with no choice to make: gpu {g} oracle {o}")
    s_last = ora_scores[ranked[want - 1]]
    s_next = ora_scores[ranked[want]]
    gap = abs(s_last - s_next)
    if gap > SEL_REL * max(abs(s_last), abs_scale):
        raise AssertionError(
            f"selection differs beyond the tie tolerance: gpu {g} oracle {o} "
            f"(gap {gap:.3e}, last kept {s_last:.9e})")
    forced = 0 if forced_first else forced_block
    free = [j for j in g if j != forced]
    if forced is not None:
        assert forced in g, f"forced block {forced} missing from gpu selection {g}"
    assert len(free) == want, f"gpu kept {len(free)} blocks, expected {want}"
    tol = SEL_REL * max(abs(s_last), abs_scale)
    for j in free:
        assert ora_scores[j] >= s_last - tol, f"gpu kept block {j} well below the cut"
    dropped = [j for j in ranked if j not in free]
    for j in dropped:
        assert ora_scores[j] <= s_last + tol, f"gpu dropped block {j} well above the cut"
    return False


def check_selection_topp(gpu_sel, ora_sel, ora_scores, ncand, n_keep, top_p):
    """Compare one row of adaptive (top-p) selection. True if the sets are
    equal; False if they differ only within the tolerances (near-equal scores
    at the cut, or a cumulative sum within SEL_REL of top_p times the total);
    raises otherwise. The GPU set must be block 0 plus a best-first prefix of
    the others that reaches top_p of the total (unless n blocks are taken) and
    is the shortest such prefix."""
    g = sorted(int(x) for x in gpu_sel if x >= 0)
    o = sorted(int(x) for x in ora_sel if x >= 0)
    if g == o:
        return True
    sc = np.asarray(ora_scores[:ncand], dtype=np.float64)
    assert 0 in g, f"block 0 missing from gpu selection {g}"
    assert len(g) <= min(n_keep, ncand), f"gpu kept {len(g)} blocks (n {n_keep}, {ncand} candidates)"
    total = float(sc.sum())
    goal = top_p * total
    tol = SEL_REL * max(abs(total), 1e-30)
    free = [j for j in g if j != 0]
    chosen = float(sc[0] + sc[free].sum()) if free else float(sc[0])
    if free:
        s_min = float(sc[free].min())
        for j in range(1, ncand):
            if j not in free:
                assert sc[j] <= s_min + SEL_REL * abs(s_min), (
                    f"gpu dropped block {j} ({sc[j]:.9e}) above kept {s_min:.9e}: gpu {g} oracle {o}")
        assert chosen - s_min < goal + tol, f"gpu selection {g} is longer than needed (oracle {o})"
    if len(g) < min(n_keep, ncand):
        assert chosen >= goal - tol, f"gpu selection {g} stops short of top_p (oracle {o})"
    return False


def check_output(gpu, ref, dtype, what="out"):
    """The stated bounds on |gpu - ref|, plus the same bounds scaled by the
    reference's largest magnitude when that is below 1 (floored at 1e-2), so
    that outputs of small magnitude (queries and keys scaled by 1/sqrt(d))
    are held to the same relative accuracy as unit-scale ones. Returns
    (max |err|, mean |err|)."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU values"
    err = np.abs(gpu - ref)
    mx, mean = float(err.max(initial=0.0)), float(err.mean()) if err.size else 0.0
    tol = TOL[dtype]
    assert mx <= tol["max"], f"{what}: max |err| {mx:.3e} > {tol['max']}"
    assert mean <= tol["mean"], f"{what}: mean |err| {mean:.3e} > {tol['mean']}"
    mag = min(1.0, max(float(np.abs(ref).max(initial=0.0)), 1e-2))
    assert mx <= tol["max"] * mag, (
        f"{what}: max |err| {mx:.3e} > {tol['max']} x max|ref| {mag:.3e}")
    assert mean <= tol["mean"] * mag, (
        f"{what}: mean |err| {mean:.3e} > {tol['mean']} x max|ref| {mag:.3e}")
    return mx, mean
