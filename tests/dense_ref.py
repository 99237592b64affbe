"""Independent dense-matrix formulation of each NSA / MoBA branch (test helper).

Where the oracle walks explicit key lists per query, this module builds full
T x T (or T x Nc) boolean masks and evaluates masked softmax attention with
numpy matrix products. The two share no code; the tests compare them.
"""
import numpy as np


def masked_attention(q, k, v, mask, scale):
    """q [T, d], k/v [S, d], mask [T, S] bool -> (out [T, d], p [T, S], lse [T]).

    Rows with no visible key give a zero output and lse = -inf.
    """
    z = scale * (q @ k.T)
    z = np.where(mask, z, -np.inf)
    m = np.max(z, axis=1, keepdims=True)
    empty = ~np.isfinite(m[:, 0])
    m[empty] = 0.0
    e = np.where(mask, np.exp(z - m), 0.0)
    s = e.sum(axis=1, keepdims=True)
    s[empty] = 1.0
    p = e / s
    lse = np.where(empty, -np.inf, m[:, 0] + np.log(s[:, 0]))
    return p @ v, p, lse


def causal_mask(T):
    return np.tril(np.ones((T, T), dtype=bool))


def compression_matrix(T, l, s, w):
    """C [Nc, T] with C[i, i*s + j] = w[j], so K~ = C @ K."""
    Nc = 0 if T < l else (T - l) // s + 1
    C = np.zeros((Nc, T))
    for i in range(Nc):
        C[i, i * s:i * s + l] = w
    return C


def overlap_matrix(T, l, s, bs, Nc, weighted=False):
    """O [Nc, nblk]: 1 (or overlap/l) where compressed block i and selection block j intersect."""
    nblk = -(-T // bs)
    starts_c = np.arange(Nc) * s
    ends_c = starts_c + l - 1
    starts_b = np.arange(nblk) * bs
    ends_b = starts_b + bs - 1
    lo = np.maximum(starts_c[:, None], starts_b[None, :])
    hi = np.minimum(ends_c[:, None], ends_b[None, :])
    ov = np.clip(hi - lo + 1, 0, None).astype(np.float64)
    return ov / l if weighted else (ov > 0).astype(np.float64)


def select_blocks(scores, ncand, n):
    """Top selection of one row: block 0 forced, the rest by score desc, index asc."""
    if ncand <= n:
        return list(range(ncand))
    idx = np.arange(1, ncand)
    order = np.lexsort((idx, -scores[1:ncand]))  # last key primary: -score, then index
    return sorted([0] + list(idx[order[: n - 1]]))


def nsa_dense(p, q, k, v, w_cmp, wg):
    """Full NSA forward for B=1 by dense masks. q [T,Hq,d], k/v [T,Hkv,d]."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    l, s, bs, n, w = p["cmp_block"], p["cmp_stride"], p["sel_block"], p["top_n"], p["window"]
    scale = p.get("scale") or 1.0 / np.sqrt(d)
    C = compression_matrix(T, l, s, np.asarray(w_cmp, dtype=np.float64))
    Nc = C.shape[0]
    O = overlap_matrix(T, l, s, bs, Nc, weighted=p.get("score_mode", 0) == 1)
    nblk = -(-T // bs)
    tpos = np.arange(T)
    cmp_vis = (np.arange(Nc)[None, :] * s + l - 1) <= tpos[:, None]
    ncand = tpos // bs + 1
    win = (tpos[None, :] <= tpos[:, None]) & (tpos[None, :] > tpos[:, None] - w)
    res = {k_: np.zeros((T, Hq, d)) for k_ in ("o_cmp", "o_slc", "o_win", "out")}
    res["scores"] = np.full((T, Hkv, nblk), -np.inf)
    res["sel"] = np.full((T, Hkv, n), -1, dtype=np.int64)
    res["lse_cmp"] = np.zeros((T, Hq))
    res["gates"] = np.zeros((T, Hq, 3))
    for g in range(Hkv):
        kc = C @ k[:, g, :]
        vc = C @ v[:, g, :]
        sc = np.zeros((T, nblk))
        ps = []
        for hh in range(G):
            h = g * G + hh
            o, pc, lse = masked_attention(q[:, h, :], kc, vc, cmp_vis, scale)
            res["o_cmp"][:, h] = o
            res["lse_cmp"][:, h] = lse
            sc += pc @ O
            ps.append(pc)
        for t in range(T):
            res["scores"][t, g, : ncand[t]] = sc[t, : ncand[t]]
        slc_mask = np.zeros((T, T), dtype=bool)
        for t in range(T):
            S = select_blocks(sc[t], ncand[t], n)
            res["sel"][t, g, : len(S)] = S
            blk_ok = np.zeros(nblk, dtype=bool)
            blk_ok[S] = True
            slc_mask[t] = blk_ok[tpos // bs] & (tpos <= t)
        for hh in range(G):
            h = g * G + hh
            res["o_slc"][:, h], _, _ = masked_attention(q[:, h, :], k[:, g], v[:, g], slc_mask, scale)
            res["o_win"][:, h], _, _ = masked_attention(q[:, h, :], k[:, g], v[:, g], win, scale)
    if p.get("gate_mode", 0) == 1:
        gt = np.broadcast_to(np.asarray(p["fixed_gates"], dtype=np.float64), (T, Hq, 3))
    else:
        gt = 1.0 / (1.0 + np.exp(-np.einsum("thd,dc->thc", q, wg)))
    res["gates"] = np.array(gt)
    res["out"] = (gt[..., 0:1] * res["o_cmp"] + gt[..., 1:2] * res["o_slc"]
                  + gt[..., 2:3] * res["o_win"])
    return res


def moba_dense(p, q, k, v):
    """MoBA forward for B=1 by dense masks. q [T,H,d], k/v [T,Hkv,d]."""
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    m, K = p["block"], p["top_k"]
    scale = p.get("scale") or 1.0 / np.sqrt(d)
    nfull = T // m
    tpos = np.arange(T)
    own = tpos // m
    out = np.zeros((T, Hq, d))
    sel = np.full((T, Hq, K), -1, dtype=np.int64)
    for h in range(Hq):
        g = h // G
        kbar = k[: nfull * m, g, :].reshape(nfull, m, d).mean(axis=1)
        sc = q[:, h, :] @ kbar.T                    # [T, nfull]
        mask = np.zeros((T, T), dtype=bool)
        for t in range(T):
            c = own[t]
            past = np.arange(c)
            if c <= K - 1:
                S = list(past) + [c]
            else:
                order = np.lexsort((past, -sc[t, :c]))
                S = sorted(list(past[order[: K - 1]]) + [c])
            sel[t, h, : len(S)] = S
            ok = np.zeros(-(-T // m), dtype=bool)
            ok[S] = True
            mask[t] = ok[tpos // m] & (tpos <= t)
        out[:, h], _, _ = masked_attention(q[:, h, :], k[:, g], v[:, g], mask, scale)
    return dict(out=out, sel=sel)
