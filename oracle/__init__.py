"""fp64 CPU oracle for the NSA and MoBA forward pass -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The CUDA library never does, and this
package imports nothing from it.

The arithmetic lives in ``oracle.c`` (plain loops, fp64, OpenMP over rows);
this module only marshals numpy float64 arrays through ctypes.

Arrays use the layouts of the library: q ``[B, T, Hq, d]``, k/v
``[B, T, Hkv, d]``, compressed k/v ``[B, Nc, Hkv, d]``, gate weights
``[d, 3]``. Values are the exact input values as float64.
"""
import ctypes
import math

import numpy as np

from . import build as _build

STORE = {"none": 0, "f32": 1, "bf16": 2}


class _NsaCfg(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
        ("cmp_block", ctypes.c_int), ("cmp_stride", ctypes.c_int),
        ("sel_block", ctypes.c_int), ("top_n", ctypes.c_int), ("window", ctypes.c_int),
        ("scale", ctypes.c_double), ("gate_mode", ctypes.c_int),
        ("fixed_gates", ctypes.c_double * 3), ("store", ctypes.c_int),
        ("score_mode", ctypes.c_int), ("top_p", ctypes.c_double),
    ]


class _MobaCfg(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int),
        ("Hkv", ctypes.c_int), ("d", ctypes.c_int), ("block", ctypes.c_int),
        ("top_k", ctypes.c_int), ("scale", ctypes.c_double),
    ]


_LIB = None
_D = ctypes.POINTER(ctypes.c_double)
_I = ctypes.POINTER(ctypes.c_int)


def _lib():
    global _LIB
    if _LIB is None:
        lib = ctypes.CDLL(_build.build())
        lib.oracle_round_store.restype = ctypes.c_double
        lib.oracle_round_store.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.oracle_round_store_array.argtypes = [ctypes.c_int, _D, _D, ctypes.c_long]
        lib.oracle_num_cmp.restype = ctypes.c_int
        lib.oracle_num_cmp.argtypes = [ctypes.c_int] * 3
        lib.oracle_compress.argtypes = [ctypes.POINTER(_NsaCfg), _D, _D, _D, _D, _D]
        lib.oracle_nsa_rows.argtypes = [
            ctypes.POINTER(_NsaCfg), ctypes.c_int, _I, _I, _D, _D, _D, _D, _D, _D, _I,
            _D, _D, _D, _D, _D, _D, _D, _I,
        ]
        lib.oracle_moba_block_means.argtypes = [ctypes.POINTER(_MobaCfg), _D, _D]
        lib.oracle_moba_rows.argtypes = [
            ctypes.POINTER(_MobaCfg), ctypes.c_int, _I, _I, _D, _D, _D, _D, _I, _D, _I, _D, _D,
        ]
        _LIB = lib
    return _LIB


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _dp(a):
    return None if a is None else a.ctypes.data_as(_D)


def _ip(a):
    return None if a is None else a.ctypes.data_as(_I)


def _nsa_cfg(p):
    c = _NsaCfg()
    for name in ("B", "T", "Hq", "Hkv", "d", "cmp_block", "cmp_stride", "sel_block",
                 "top_n", "window"):
        setattr(c, name, int(p[name]))
    scale = p.get("scale", 0.0) or 0.0
    c.scale = float(scale) if scale else 1.0 / math.sqrt(p["d"])
    c.gate_mode = int(p.get("gate_mode", 0))
    fg = p.get("fixed_gates", (0.0, 0.0, 0.0))
    for i in range(3):
        c.fixed_gates[i] = float(fg[i])
    c.store = STORE[p.get("store", "none")] if isinstance(p.get("store", "none"), str) else int(p["store"])
    c.score_mode = int(p.get("score_mode", 0))
    c.top_p = float(p.get("top_p", 0.0))
    return c


def _moba_cfg(p):
    c = _MobaCfg()
    for name in ("B", "T", "Hq", "Hkv", "d", "block", "top_k"):
        setattr(c, name, int(p[name]))
    scale = p.get("scale", 0.0) or 0.0
    c.scale = float(scale) if scale else 1.0 / math.sqrt(p["d"])
    return c


def round_store(x, store):
    """Round fp64 values once, to nearest-even, into ``store`` ('none', 'f32', 'bf16')."""
    x = _f64(x)
    y = np.empty_like(x)
    _lib().oracle_round_store_array(STORE[store], _dp(x), _dp(y), x.size)
    return y


def num_cmp(T, l, s):
    return _lib().oracle_num_cmp(int(T), int(l), int(s))


def compress(p, k, v, w):
    """Compressed keys and values ``[B, Nc, Hkv, d]`` (rounded to ``p['store']``)."""
    k, v, w = _f64(k), _f64(v), _f64(w)
    B, T, Hkv, d = k.shape
    q = dict(p, B=B, T=T, Hkv=Hkv, d=d)
    Nc = num_cmp(T, q["cmp_block"], q["cmp_stride"])
    kc = np.zeros((B, Nc, Hkv, d))
    vc = np.zeros((B, Nc, Hkv, d))
    cfg = _nsa_cfg(q)
    _lib().oracle_compress(ctypes.byref(cfg), _dp(k), _dp(v), _dp(w), _dp(kc), _dp(vc))
    return kc, vc


def nsa_rows(p, rows_b, rows_t, q_rows, k, v, kc, vc, wg, forced_sel=None):
    """All intermediates of the NSA forward for the listed query rows.

    ``q_rows`` is ``[nrows, Hq, d]``; row r is the query at position
    ``rows_t[r]`` of sequence ``rows_b[r]``. Returns a dict with ``out``,
    ``o_cmp``, ``o_slc``, ``o_win`` ``[nrows, Hq, d]``, ``gates``
    ``[nrows, Hq, 3]``, ``lse_cmp`` ``[nrows, Hq]``, ``scores``
    ``[nrows, Hkv, ceil(T/sel_block)]`` and ``sel`` ``[nrows, Hkv, n]``.
    """
    k, v, kc, vc = _f64(k), _f64(v), _f64(kc), _f64(vc)
    q_rows = _f64(q_rows)
    wg = _f64(wg if wg is not None else np.zeros((p["d"], 3)))
    rb = np.ascontiguousarray(np.asarray(rows_b, dtype=np.int32))
    rt = np.ascontiguousarray(np.asarray(rows_t, dtype=np.int32))
    nrows = rb.size
    Hq, Hkv, d, n = p["Hq"], p["Hkv"], p["d"], p["top_n"]
    nblk = -(-p["T"] // p["sel_block"])
    assert kc.shape[1] == num_cmp(p["T"], p["cmp_block"], p["cmp_stride"])
    res = {
        "out": np.zeros((nrows, Hq, d)), "o_cmp": np.zeros((nrows, Hq, d)),
        "o_slc": np.zeros((nrows, Hq, d)), "o_win": np.zeros((nrows, Hq, d)),
        "gates": np.zeros((nrows, Hq, 3)), "lse_cmp": np.zeros((nrows, Hq)),
        "scores": np.zeros((nrows, Hkv, nblk)), "sel": np.zeros((nrows, Hkv, n), np.int32),
    }
    fs = None
    if forced_sel is not None:
        fs = np.ascontiguousarray(np.asarray(forced_sel, dtype=np.int32).reshape(nrows, Hkv, n))
    cfg = _nsa_cfg(p)
    _lib().oracle_nsa_rows(
        ctypes.byref(cfg), nrows, _ip(rb), _ip(rt), _dp(q_rows), _dp(k), _dp(v), _dp(kc),
        _dp(vc), _dp(wg), _ip(fs), _dp(res["out"]), _dp(res["o_cmp"]), _dp(res["o_slc"]),
        _dp(res["o_win"]), _dp(res["gates"]), _dp(res["lse_cmp"]), _dp(res["scores"]),
        _ip(res["sel"]),
    )
    return res


def nsa_prefill(p, q, k, v, w_cmp, wg, rows=None, forced_sel=None):
    """NSA causal prefill. ``rows``: list of (b, t) to evaluate (default: all)."""
    q = _f64(q)
    B, T = q.shape[:2]
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(T)]
    rb = [r[0] for r in rows]
    rt = [r[1] for r in rows]
    kc, vc = compress(p, k, v, w_cmp)
    res = nsa_rows(p, rb, rt, q[rb, rt], k, v, kc, vc, wg, forced_sel)
    res["k_cmp"], res["v_cmp"] = kc, vc
    return res


def nsa_decode(p, q, k_cache, v_cache, seq_lens, kc, vc, wg, forced_sel=None):
    """NSA single-token decode: query ``[B, Hq, d]`` at position seq_len - 1."""
    q = _f64(q)
    B = q.shape[0]
    lens = [int(x) for x in seq_lens]
    return nsa_rows(p, list(range(B)), [x - 1 for x in lens], q, k_cache, v_cache, kc, vc, wg,
                    forced_sel)


def moba_block_means(p, k):
    k = _f64(k)
    B, T, Hkv, d = k.shape
    q = dict(p, B=B, T=T, Hkv=Hkv, d=d)
    kbar = np.zeros((B, T // q["block"], Hkv, d))
    cfg = _moba_cfg(q)
    _lib().oracle_moba_block_means(ctypes.byref(cfg), _dp(k), _dp(kbar))
    return kbar


def moba_rows(p, rows_b, rows_t, q_rows, k, v, kbar=None, forced_sel=None):
    k, v, q_rows = _f64(k), _f64(v), _f64(q_rows)
    if kbar is None:
        kbar = moba_block_means(p, k)
    kbar = _f64(kbar)
    rb = np.ascontiguousarray(np.asarray(rows_b, dtype=np.int32))
    rt = np.ascontiguousarray(np.asarray(rows_t, dtype=np.int32))
    nrows = rb.size
    Hq, d, K = p["Hq"], p["d"], p["top_k"]
    nblk = -(-p["T"] // p["block"])
    res = {
        "out": np.zeros((nrows, Hq, d)), "sel": np.zeros((nrows, Hq, K), np.int32),
        "scores": np.zeros((nrows, Hq, nblk)), "lse": np.zeros((nrows, Hq)),
    }
    fs = None
    if forced_sel is not None:
        fs = np.ascontiguousarray(np.asarray(forced_sel, dtype=np.int32).reshape(nrows, Hq, K))
    cfg = _moba_cfg(p)
    _lib().oracle_moba_rows(
        ctypes.byref(cfg), nrows, _ip(rb), _ip(rt), _dp(q_rows), _dp(k), _dp(v), _dp(kbar),
        _ip(fs), _dp(res["out"]), _ip(res["sel"]), _dp(res["scores"]), _dp(res["lse"]),
    )
    return res


def moba_prefill(p, q, k, v, rows=None, forced_sel=None):
    q = _f64(q)
    B, T = q.shape[:2]
    if rows is None:
        rows = [(b, t) for b in range(B) for t in range(T)]
    rb = [r[0] for r in rows]
    rt = [r[1] for r in rows]
    return moba_rows(p, rb, rt, q[rb, rt], k, v, forced_sel=forced_sel)
