"""fp64 CPU oracle for the NSA prefill backward pass -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module. The CUDA library never does, and this
module imports nothing from it.

What is differentiated. The forward is the one ``oracle.c`` computes (EP94
notes section 五; lchairun.cn NSA article, the three squads and the gate):

    K~[i] = sum_j w[j] K[i s + j],  V~ likewise                    (compression)
    o_c   = softmax(sigma q . keys_c) values_c   for c in cmp, slc, win
    g_c   = sigmoid(q . Wg[:, c])  (or fixed gates)
    out   = g_cmp o_cmp + g_slc o_slc + g_win o_win

with the scalar loss L = sum(dout * out). The selected blocks are the ones the
forward chose and enter as constants: the top-n choice is a discrete step, and
the pages say the gradient that trains the selection flows through the
compressed branch (EP94 section 五, branch one; lchairun.cn, the paragraph on
trainability). Gradients are the plain chain rule through each step, in the
order of the forward: gates, the three attentions, then the compression.

Arrays use the library's layouts: q, dout ``[B, T, Hq, d]``, k, v
``[B, T, Hkv, d]``, w_cmp ``[l]``, Wg ``[d, 3]``, sel ``[B, T, Hkv, n]``
(-1 marks an unused slot). Query head h uses KV head h // (Hq / Hkv).

Parity status: pinned by central finite differences of ``oracle.c``'s forward
with the selection held fixed, by the window-only case against autograd of
plain softmax attention, and by the value-gradient sum identity (tests/
test_oracle_pins.py).
"""
import math

import numpy as np


def _attention_backward(q, keys, vals, scale, d_o):
    """One query against an explicit key list: returns (o, dq, dkeys, dvals).

    o = sum_a p_a v_a with p = softmax(scale q . k_a). With dO the upstream
    gradient of o: dp_a = dO . v_a, D = sum_a p_a dp_a, dS_a = p_a (dp_a - D),
    dq = scale sum_a dS_a k_a, dk_a = scale dS_a q, dv_a = p_a dO.
    An empty key list gives o = 0 and no gradient.
    """
    d = q.shape[0]
    if keys.shape[0] == 0:
        return np.zeros(d), np.zeros(d), np.zeros((0, d)), np.zeros((0, d))
    z = scale * (keys @ q)
    p = np.exp(z - z.max())
    p /= p.sum()
    o = p @ vals
    dp = vals @ d_o
    D = float(p @ dp)
    ds = p * (dp - D)
    dq = scale * (ds @ keys)
    dk = scale * np.outer(ds, q)
    dv = np.outer(p, d_o)
    return o, dq, dk, dv


def nsa_prefill_backward(p, q, k, v, w_cmp, wg, dout, sel, kc=None, vc=None):
    """Gradients of L = sum(dout * out) of the causal NSA prefill.

    ``kc``, ``vc``: the compressed keys and values the forward attended to,
    when it stored them rounded (bf16); the rounding is taken as the identity
    in the gradient of the compression. Default: the exact compression.

    Returns a dict with ``dq`` ``[B, T, Hq, d]``, ``dk``, ``dv`` ``[B, T, Hkv,
    d]`` (through the selected and window branches and, via the compression,
    the compressed branch), ``dw_cmp`` ``[l]`` and ``dwg`` ``[d, 3]`` (zero
    with fixed gates); also ``out`` for cross-checks.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    w_cmp = np.asarray(w_cmp, dtype=np.float64)
    wg = np.zeros((q.shape[3], 3)) if wg is None else np.asarray(wg, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    sel = np.asarray(sel)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    l, s, bs, w = p["cmp_block"], p["cmp_stride"], p["sel_block"], p["window"]
    scale = p.get("scale", 0.0) or 1.0 / math.sqrt(d)
    fixed = int(p.get("gate_mode", 0)) == 1
    fg = np.asarray(p.get("fixed_gates", (0.0, 0.0, 0.0)), dtype=np.float64)
    Nc = (T - l) // s + 1 if T >= l else 0

    # compression (its output is what the compressed branch attends to)
    if kc is None:
        kc = np.zeros((B, Nc, Hkv, d))
        vc = np.zeros((B, Nc, Hkv, d))
        for i in range(Nc):
            for j in range(l):
                kc[:, i] += w_cmp[j] * k[:, i * s + j]
                vc[:, i] += w_cmp[j] * v[:, i * s + j]
    else:
        kc = np.asarray(kc, dtype=np.float64)
        vc = np.asarray(vc, dtype=np.float64)

    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dkc = np.zeros_like(kc)
    dvc = np.zeros_like(vc)
    dwg = np.zeros((d, 3))
    out = np.zeros_like(q)

    for b in range(B):
        for t in range(T):
            # compressed block i is visible once it ends: i s + l - 1 <= t
            nvis = (t + 1 - l) // s + 1 if t + 1 >= l else 0
            nvis = min(nvis, Nc)
            w0 = max(0, t - w + 1)
            for g in range(Hkv):
                blocks = [int(j) for j in sel[b, t, g] if j >= 0]
                slc_rows = [u for j in blocks for u in range(j * bs, j * bs + bs) if u <= t]
                win_rows = list(range(w0, t + 1))
                for hh in range(G):
                    h = g * G + hh
                    qh = q[b, t, h]
                    dO = dout[b, t, h]
                    # gates from the raw query
                    if fixed:
                        gt = fg.copy()
                    else:
                        gt = 1.0 / (1.0 + np.exp(-(qh @ wg)))
                    # forward of the three branches
                    o_c, _, _, _ = _attention_backward(qh, kc[b, :nvis, g], vc[b, :nvis, g],
                                                       scale, np.zeros(d))
                    o_s, _, _, _ = _attention_backward(qh, k[b, slc_rows, g], v[b, slc_rows, g],
                                                       scale, np.zeros(d))
                    o_w, _, _, _ = _attention_backward(qh, k[b, win_rows, g], v[b, win_rows, g],
                                                       scale, np.zeros(d))
                    out[b, t, h] = gt[0] * o_c + gt[1] * o_s + gt[2] * o_w
                    # gates: dL/dg_c = dO . o_c, through the sigmoid
                    if not fixed:
                        dg = np.array([dO @ o_c, dO @ o_s, dO @ o_w])
                        dz = dg * gt * (1.0 - gt)
                        dq[b, t, h] += wg @ dz
                        dwg += np.outer(qh, dz)
                    # the three attentions, each with upstream gradient g_c dO
                    _, dq_c, dk_c, dv_c = _attention_backward(qh, kc[b, :nvis, g],
                                                              vc[b, :nvis, g], scale, gt[0] * dO)
                    dq[b, t, h] += dq_c
                    dkc[b, :nvis, g] += dk_c
                    dvc[b, :nvis, g] += dv_c
                    _, dq_s, dk_s, dv_s = _attention_backward(qh, k[b, slc_rows, g],
                                                              v[b, slc_rows, g], scale, gt[1] * dO)
                    dq[b, t, h] += dq_s
                    np.add.at(dk[b, :, g], slc_rows, dk_s)
                    np.add.at(dv[b, :, g], slc_rows, dv_s)
                    _, dq_w, dk_w, dv_w = _attention_backward(qh, k[b, win_rows, g],
                                                              v[b, win_rows, g], scale, gt[2] * dO)
                    dq[b, t, h] += dq_w
                    dk[b, win_rows, g] += dk_w
                    dv[b, win_rows, g] += dv_w

    # compression backward: K~[i] = sum_j w[j] K[i s + j]
    dw_cmp = np.zeros(l)
    for i in range(Nc):
        for j in range(l):
            dk[:, i * s + j] += w_cmp[j] * dkc[:, i]
            dv[:, i * s + j] += w_cmp[j] * dvc[:, i]
            dw_cmp[j] += np.sum(dkc[:, i] * k[:, i * s + j]) + np.sum(dvc[:, i] * v[:, i * s + j])
    return {"dq": dq, "dk": dk, "dv": dv, "dw_cmp": dw_cmp, "dwg": dwg, "out": out}
