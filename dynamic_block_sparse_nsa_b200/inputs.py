"""Seeded synthetic inputs and the named workloads.

This module holds shapes, value distributions and random draws only -- none
of the method's arithmetic. Both the CUDA path (tests, benchmark) and the fp64
oracle receive the arrays it returns.

Recipe: one CPU ``torch.Generator`` per call, seeded with the workload's
seed, draws in this fixed order: q, k, v, w_cmp, w_gate. q/k/v are standard
normal times ``qkv_scale`` and are then cast to the run dtype (the cast values
are the inputs both sides see). w_cmp ~ N(0, 1/l) and w_gate ~ N(0, 1/d) stay
fp32. For decode, k and v are drawn one sequence at a time (k for every
sequence, then v for every sequence) to bound host memory.
"""
import math

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}

# Workloads, named by what they are. Shapes and distributions follow the
# problem statement of each run (NSA block 64 / top-16 and MoBA block 512 /
# top-3 are the pages' parameter table; l = 32, s = 16, w = 512 fixed here).
WORKLOADS = {
    # fp32 parity case small enough for the oracle in full.
    "nsa_prefill_f32_t1024": dict(
        kind="prefill", B=1, T=1024, Hq=4, Hkv=1, d=64, cmp_block=32, cmp_stride=16,
        sel_block=64, top_n=4, window=128, dtype="f32", qkv_scale=1.0, seed=0),
    "nsa_prefill_bf16_t8192": dict(
        kind="prefill", B=1, T=8192, Hq=64, Hkv=4, d=128, cmp_block=32, cmp_stride=16,
        sel_block=64, top_n=16, window=512, dtype="bf16", qkv_scale=1.0 / math.sqrt(128),
        seed=0),
    "nsa_decode_bf16_b32_l65536": dict(
        kind="decode", B=32, T=65536, Hq=64, Hkv=4, d=128, cmp_block=32, cmp_stride=16,
        sel_block=64, top_n=16, window=512, dtype="bf16", qkv_scale=1.0, seed=0),
    "nsa_prefill_bf16_t65536": dict(
        kind="prefill", B=1, T=65536, Hq=64, Hkv=4, d=128, cmp_block=32, cmp_stride=16,
        sel_block=64, top_n=16, window=512, dtype="bf16", qkv_scale=1.0 / math.sqrt(128),
        seed=0),
    "moba_prefill_bf16_t131072": dict(
        kind="moba", B=1, T=131072, Hq=32, Hkv=32, d=128, block=512, top_k=3, dtype="bf16",
        qkv_scale=1.0, seed=0),
}


def workload(name, **overrides):
    w = dict(WORKLOADS[name])
    w.update(overrides)
    return w


def _randn(gen, shape, scale, dtype):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=gen.device)
    if scale != 1.0:
        x.mul_(scale)
    return x.to(dtype)


def _gen(seed, device):
    return torch.Generator(device=device or "cpu").manual_seed(seed)


def make_prefill(w, seed=None, device=None):
    """q [B,T,Hq,d], k/v [B,T,Hkv,d] in the run dtype; w_cmp [l], w_gate [d,3] fp32.

    device=None draws on the CPU generator (the recipe the tests use); a CUDA
    device draws the same distributions from a CUDA generator (other numbers,
    used by the benchmark to skip the host draw of multi-GB inputs)."""
    gen = _gen(w["seed"] if seed is None else seed, device)
    dt = DTYPES[w["dtype"]]
    B, T, Hq, Hkv, d = w["B"], w["T"], w["Hq"], w["Hkv"], w["d"]
    sc = w.get("qkv_scale", 1.0)
    q = _randn(gen, (B, T, Hq, d), sc, dt)
    k = _randn(gen, (B, T, Hkv, d), sc, dt)
    v = _randn(gen, (B, T, Hkv, d), sc, dt)
    out = dict(q=q, k=k, v=v)
    if "cmp_block" in w:
        l = w["cmp_block"]
        out["w_cmp"] = torch.randn(l, generator=gen, device=gen.device) * math.sqrt(1.0 / l)
        out["w_gate"] = torch.randn(d, 3, generator=gen, device=gen.device) * math.sqrt(1.0 / d)
    return out


def make_decode(w, seed=None, seq_lens=None, device=None):
    """q [B,Hq,d], k/v caches [B,T,Hkv,d], seq_lens [B] int32 (default: all T)."""
    gen = _gen(w["seed"] if seed is None else seed, device)
    dt = DTYPES[w["dtype"]]
    B, T, Hq, Hkv, d = w["B"], w["T"], w["Hq"], w["Hkv"], w["d"]
    sc = w.get("qkv_scale", 1.0)
    q = _randn(gen, (B, Hq, d), sc, dt)
    k = torch.empty(B, T, Hkv, d, dtype=dt, device=gen.device)
    v = torch.empty(B, T, Hkv, d, dtype=dt, device=gen.device)
    for b in range(B):
        k[b] = _randn(gen, (T, Hkv, d), sc, dt)
    for b in range(B):
        v[b] = _randn(gen, (T, Hkv, d), sc, dt)
    l = w["cmp_block"]
    w_cmp = torch.randn(l, generator=gen, device=gen.device) * math.sqrt(1.0 / l)
    w_gate = torch.randn(d, 3, generator=gen, device=gen.device) * math.sqrt(1.0 / d)
    if seq_lens is None:
        seq_lens = [T] * B
    lens = torch.tensor(seq_lens, dtype=torch.int32, device=gen.device)
    return dict(q=q, k=k, v=v, w_cmp=w_cmp, w_gate=w_gate, seq_lens=lens)


def ragged_lens(B, T, seed, lo=1):
    """Seeded ragged sequence lengths in [lo, T] (the last one is T)."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, T + 1, (B,), generator=gen).tolist()
    lens[-1] = T
    return lens
