"""fp64 CPU oracle for a selection variant without a CUDA path -- TEST INFRASTRUCTURE.

Only ``tests/`` may import this module; the CUDA library never does, and this
module imports nothing from it.

Exact top-k over token scores (EP94 notes section 八: the block-selection
ablation names exact top-k -- the full attention score matrix computed, the
top-k taken -- as the upper bound of top-k methods, above Quest-style block
selection). The pages give no formula; the reading taken here keeps NSA's
GQA-shared rule and token budget:

* token score of key u <= t for the query at t and KV group g: the exact
  attention probability of u summed over the group's heads,
  sum_h softmax_u(scale q_h . k_u);
* the selected branch attends to the k highest-scoring tokens (ties to the
  lower index; all of them when t + 1 <= k), with k = top_n * sel_block so the
  budget equals NSA's;
* the compressed and window branches and the gates are NSA's (taken from the
  C oracle), and out = g_cmp o_cmp + g_slc o_slc + g_win o_win.

Parity status: oracle-level only (no CUDA implementation); pinned by the
all-tokens closed form (dense causal attention), k = 1 (the value of the token
with the largest summed probability), and the set against a brute-force sort
(tests/test_oracle_pins.py).
"""
import math

import numpy as np

from . import compress, nsa_rows


def exact_topk_rows(p, q, k, v, w_cmp, wg, rows, ktok=None):
    """NSA forward with the selected branch replaced by exact token top-k.

    ``rows``: list of (b, t). Returns a dict with ``out``, ``o_slc`` ``[nrows,
    Hq, d]`` and ``sel`` ``[nrows, Hkv, ktok]`` (selected tokens ascending, -1
    padded).
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    scale = p.get("scale", 0.0) or 1.0 / math.sqrt(d)
    if ktok is None:
        ktok = p["top_n"] * p["sel_block"]
    rb = [r[0] for r in rows]
    rt = [r[1] for r in rows]
    kc, vc = compress(p, k, v, w_cmp)
    base = nsa_rows(p, rb, rt, q[rb, rt], k, v, kc, vc, wg)
    nrows = len(rows)
    o_slc = np.zeros((nrows, Hq, d))
    sel = -np.ones((nrows, Hkv, ktok), dtype=np.int64)
    for r, (b, t) in enumerate(rows):
        for g in range(Hkv):
            keys = k[b, :t + 1, g]
            vals = v[b, :t + 1, g]
            # exact probabilities of every causal key, summed over the group
            mass = np.zeros(t + 1)
            for hh in range(G):
                z = scale * (keys @ q[b, t, g * G + hh])
                e = np.exp(z - z.max())
                mass += e / e.sum()
            order = sorted(range(t + 1), key=lambda u: (-mass[u], u))[:ktok]
            chosen = sorted(order)
            sel[r, g, :len(chosen)] = chosen
            for hh in range(G):
                h = g * G + hh
                z = scale * (keys[chosen] @ q[b, t, h])
                e = np.exp(z - z.max())
                o_slc[r, h] = (e / e.sum()) @ vals[chosen]
    gates = base["gates"]
    out = (gates[..., 0:1] * base["o_cmp"] + gates[..., 1:2] * o_slc +
           gates[..., 2:3] * base["o_win"])
    return {"out": out, "o_slc": o_slc, "sel": sel}
