#!/usr/bin/env python
"""NSA / MoBA forward benchmark on B200 (one JSON line on rank 0).

Default workload: NSA single-token decode, 32 sequences x 65536-token KV
cache, 64 query heads / 4 KV heads, d = 128, bf16, top-16 blocks of 64,
window 512 (metric: algorithmic KV GB/s). ``--workload`` selects the NSA
prefill (TFLOP/s) or MoBA prefill (TFLOP/s) workloads instead.

A step is one call of the hot path over one batch of inputs already resident
in HBM. Timing: W warm-up steps, then exactly K steps between CUDA events on
the launching stream, a barrier and a device synchronise on both sides, the
max over ranks. Every step reads more than the 126 MB L2 (stated in config).

``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload instead (rank 0 only).

Multi-GPU (torchrun): each rank runs its own batch (different seed); there is
no collective on the data path (weak scaling); value = all ranks' work / the
slowest rank's time.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from dynamic_block_sparse_nsa_b200 import inputs  # noqa: E402

METRIC = "NSA decode KV GB/s & prefill TFLOP/s at 64k ctx; fraction of roofline"
DEFAULT_WORKLOAD = "nsa_decode_bf16_b32_l65536"
L2_BYTES = 126 * 2**20


# --------------------------------------------------------------------------
# peaks, clocks
# --------------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm=float(pk["hbm_gbs"]), bf16=float(pk["bf16_tflops"]),
                    bf16_sus=float(pk["bf16_tflops_sustained"]), src="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


_REASONS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, device_index, period_s=0.005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.err = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: clocks reported as unavailable
            self._nv = None
            self.err = f"nvml unavailable: {e}"
        self._t = None

    def _reasons(self):
        nv = self._nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return fn(self._h)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = self._reasons()
                self.samples.append((mhz, rs))
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0, "note": self.err or "no samples"}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        names = [n for b, n in _REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(mhz)}


# --------------------------------------------------------------------------
# algorithmic work (bytes for decode, flops for prefill)
# --------------------------------------------------------------------------

def n_cmp(T, l, s):
    return 0 if T < l else (T - l) // s + 1


def sel_tokens(sel, t, bs):
    """Tokens of the selected blocks up to position t (sel: int array, -1 padded)."""
    blk = sel[sel >= 0].astype(np.int64)
    return int(np.sum(np.minimum(blk * bs + bs - 1, t) - blk * bs + 1))


def decode_work(w, lens, sel_h):
    """Algorithmic bytes of one decode step: every branch's reads counted once,
    plus q/out/gate/selection traffic; and the union bytes (selected blocks and
    window deduplicated)."""
    d, Hkv, Hq, n, bs, win = w["d"], w["Hkv"], w["Hq"], w["top_n"], w["sel_block"], w["window"]
    esz = 2 if w["dtype"] == "bf16" else 4
    row = d * esz
    total = union = 0
    parts = dict(cmp=0, slc=0, win=0, io=0)
    for b, L in enumerate(lens):
        t = L - 1
        nv = n_cmp(L, w["cmp_block"], w["cmp_stride"])
        for g in range(Hkv):
            ks = sel_tokens(sel_h[b, g], t, bs)
            kw = min(win, L)
            parts["cmp"] += 2 * nv * row
            parts["slc"] += 2 * ks * row
            parts["win"] += 2 * kw * row
            toks = set()
            for j in sel_h[b, g][sel_h[b, g] >= 0]:
                toks.update(range(j * bs, min(j * bs + bs - 1, t) + 1))
            toks.update(range(t - kw + 1, t + 1))
            union += 2 * nv * row + 2 * len(toks) * row
        io = 2 * Hq * d * esz + d * 3 * 4 + 4 + Hkv * n * 4
        parts["io"] += io
        union += io
    total = sum(parts.values())
    return total, union, parts


def prefill_flops(w, sel_h):
    """Algorithmic flops (4 d per query head and attended key, causal exact)."""
    T, Hq, Hkv, d, bs, win = w["T"], w["Hq"], w["Hkv"], w["d"], w["sel_block"], w["window"]
    G = Hq // Hkv
    t = np.arange(T)
    nvis = np.where(t + 1 >= w["cmp_block"], (t + 1 - w["cmp_block"]) // w["cmp_stride"] + 1, 0)
    cmp_keys = int(nvis.sum()) * Hq
    win_keys = int(np.minimum(win, t + 1).sum()) * Hq
    sel = sel_h.reshape(-1, T, Hkv, sel_h.shape[-1]).astype(np.int64)
    tt = np.broadcast_to(t[None, :, None, None], sel.shape)
    ok = sel >= 0
    cnt = np.where(ok, np.minimum(sel * bs + bs - 1, tt) - sel * bs + 1, 0)
    slc_keys = int(cnt.sum()) * G
    f = 4 * d
    return dict(cmp=cmp_keys * f, slc=slc_keys * f, win=win_keys * f)


def moba_flops(w, sel_h):
    T, Hq, d, m = w["T"], w["Hq"], w["d"], w["block"]
    t = np.arange(T)
    sel = sel_h.reshape(-1, T, Hq, sel_h.shape[-1]).astype(np.int64)
    tt = np.broadcast_to(t[None, :, None, None], sel.shape)
    cnt = np.where(sel >= 0, np.minimum(sel * m + m - 1, tt) - sel * m + 1, 0)
    attn = int(cnt.sum()) * 4 * d
    own = int((t - (t // m) * m + 1).sum()) * Hq * sel.shape[0] * 4 * d
    gate = int((t // m).sum()) * Hq * 2 * d
    return dict(attn=attn, gate=gate, attn_own=own, attn_past=attn - own)


# --------------------------------------------------------------------------
# measured DRAM traffic (ncu) recorded under profiles/
# --------------------------------------------------------------------------

def kernel_traffic(name, workload):
    """DRAM bytes per launch from profiles/dram_traffic.txt, if recorded for this
    kernel and workload and the kernel's source has not changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        f = line.split()
        if len(f) != 5 or f[0].startswith("#"):
            continue
        kname, wl, src, sha, nbytes = f
        if kname != name or wl != workload:
            continue
        sp = os.path.join(ROOT, "dynamic_block_sparse_nsa_b200", "csrc", src)
        if not os.path.exists(sp):
            return None
        cur = hashlib.sha256(open(sp, "rb").read()).hexdigest()[:16]
        return float(nbytes) if cur == sha else None
    return None


# --------------------------------------------------------------------------
# distributed helpers
# --------------------------------------------------------------------------

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _dist_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def reduce_max(x, ws):
    """Max over ranks (the step time every rank waits for)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, ws):
    """Sum over ranks (the work of the whole job)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=_dist_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# --------------------------------------------------------------------------
# the timed loops
# --------------------------------------------------------------------------

def _run_steps(step, K, graph, trace_only=None, trace_all=False, sampler=None):
    """Run K steps (optionally as one CUDA graph) between CUDA events on the
    launching stream; returns (ms, trace records, launches, clock summary)."""
    from dynamic_block_sparse_nsa_b200 import nsa
    tracing = trace_all or trace_only is not None
    g = None
    if graph:
        if tracing:
            nsa.trace_enable(True, capacity=K * 8 + 64, only=trace_only)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(K):
                step()
        g.replay()  # untimed: uploads the graph
        torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if tracing and not graph:
        nsa.trace_enable(True, capacity=K * 8 + 64, only=trace_only)
    clk = ClockSampler(sampler) if sampler is not None else None
    if clk:
        clk.__enter__()
    e0.record(s)
    if graph:
        g.replay()
    else:
        for _ in range(K):
            step()
    e1.record(s)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__()
    ms = e0.elapsed_time(e1)
    recs, launches = [], 0
    if tracing:
        recs, launches = nsa.trace_records()
        nsa.trace_enable(False)  # (graph: launches counted at capture = one replay)
    del g
    return ms, recs, launches, (clk.summary() if clk else None)


def timed(step, K, W, ws, device_index, graph=False):
    """W warm-up steps; a short traced pass names the dominant kernel; then two
    timed regions of exactly K steps, each between a barrier and a device
    synchronise: (A) uninstrumented -- the step time and clocks; (B) events
    around every launch of the dominant kernel only -- its mean duration.
    Event-record nodes between kernels delay the next launch, hence (A)."""
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    _, recs0, _, _ = _run_steps(step, min(K, 50), graph, trace_all=True)
    table0 = kernel_table(recs0, min(K, 50))
    dom = max(table0, key=lambda n: table0[n]["total_ms"]) if table0 else None
    barrier(ws)
    torch.cuda.synchronize()
    ms, _, _, clk = _run_steps(step, K, graph, sampler=device_index)
    barrier(ws)
    torch.cuda.synchronize()
    msb, recs, launches, _ = _run_steps(step, K, graph, trace_only=dom or "")
    barrier(ws)
    return dict(ms=ms, ms_traced=msb, recs=recs, launches=launches, clk=clk, table0=table0,
                dom=dom)


def kernel_table(recs, K):
    tab = {}
    for name, ms in recs:
        e = tab.setdefault(name, dict(launches=0, total_ms=0.0))
        e["launches"] += 1
        e["total_ms"] += ms
    tot = sum(e["total_ms"] for e in tab.values()) or 1.0
    for e in tab.values():
        e["mean_us"] = 1000.0 * e["total_ms"] / max(1, e["launches"])
        e["share"] = e["total_ms"] / tot
    return tab


def run_decode(w, K, W, ws, rank, local, e2e=True, use_graph=True):
    from dynamic_block_sparse_nsa_b200 import nsa
    inp = inputs.make_decode(w, seed=w["seed"] + rank, device="cuda")
    p = nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], cmp_block=w["cmp_block"],
                   cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                   window=w["window"], dtype=inputs.DTYPES[w["dtype"]])
    kc, vc = nsa.nsa_compress_kv(p, inp["k"], inp["v"], inp["w_cmp"])
    ws_buf = nsa.workspace(p, nsa.OP_DECODE)
    out = torch.empty(w["B"], w["Hq"], w["d"], dtype=inputs.DTYPES[w["dtype"]], device="cuda")
    sel = torch.empty(w["B"], w["Hkv"], w["top_n"], dtype=torch.int32, device="cuda")
    q, lens = inp["q"], inp["seq_lens"]

    def step():
        nsa.nsa_decode(p, q, inp["k"], inp["v"], lens, kc, vc, inp["w_gate"], out=out,
                       sel_idx=sel, ws=ws_buf)

    step()
    nsa.nsa_check()
    res = timed(step, K, W, ws, local, graph=use_graph)
    nsa.nsa_check()
    sel_h = sel.cpu().numpy()
    lens_l = lens.cpu().tolist()
    step_bytes, union_bytes, parts = decode_work(w, lens_l, sel_h)
    res.update(work=step_bytes, union=union_bytes, parts=parts)
    if e2e:
        res.update(decode_e2e(p, inp, kc, vc, ws_buf, q, lens, out, sel, K, ws, use_graph))
    return res


def decode_e2e(p, inp, kc, vc, ws_buf, q, lens, out, sel, K, ws, use_graph):
    """End to end through the public call with host buffers, as a serving loop
    runs it: every step copies its query and lengths from pinned host memory
    and reads its output and selection back; the KV caches are device-resident
    state, not per-step inputs. Query and output buffers are double-buffered so
    the H2D of step i + 1 (one copy stream) and the D2H of step i - 1 (another)
    overlap the decode of step i; every copy of the K steps is inside the timed
    region. Captured as one CUDA graph (streams forked and joined with events)."""
    from dynamic_block_sparse_nsa_b200 import nsa
    q_h = q.cpu().pin_memory()
    lens_h = lens.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    sel_h = torch.empty(sel.shape, dtype=sel.dtype).pin_memory()
    qd = [q, torch.empty_like(q)]
    ld = [lens, torch.empty_like(lens)]
    od = [out, torch.empty_like(out)]
    sd = [sel, torch.empty_like(sel)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run(nsteps):
        main = torch.cuda.current_stream()  # the capture stream while capturing
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_done = [torch.cuda.Event() for _ in range(nsteps)]
        ev_read = [torch.cuda.Event() for _ in range(nsteps)]
        start = torch.cuda.Event()
        start.record(main)
        s_in.wait_event(start)
        s_out.wait_event(start)

        def h2d(i):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_done[i - 2])  # buffer i % 2 no longer read
                qd[i % 2].copy_(q_h, non_blocking=True)
                ld[i % 2].copy_(lens_h, non_blocking=True)
                ev_in[i].record(s_in)

        h2d(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                h2d(i + 1)
            main.wait_event(ev_in[i])
            if i >= 2:
                main.wait_event(ev_read[i - 2])  # output buffer i % 2 read back
            nsa.nsa_decode(p, qd[i % 2], inp["k"], inp["v"], ld[i % 2], kc, vc, inp["w_gate"],
                           out=od[i % 2], sel_idx=sd[i % 2], ws=ws_buf)
            ev_done[i].record(main)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                out_h.copy_(od[i % 2], non_blocking=True)
                sel_h.copy_(sd[i % 2], non_blocking=True)
                ev_read[i].record(s_out)
        main.wait_event(ev_read[nsteps - 1])
        main.wait_stream(s_in)

    run(4)
    torch.cuda.synchronize()
    g = None
    if use_graph:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run(K)
        g.replay()
        torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    if g is not None:
        g.replay()
    else:
        run(K)
    e1.record()
    torch.cuda.synchronize()
    barrier(ws)
    ms = e0.elapsed_time(e1)
    del g
    # the last step's output read back equals the device-only run's
    if not torch.equal(out_h, out.cpu()):
        raise RuntimeError("decode end-to-end output differs from the device-resident run")
    return {"e2e_ms": ms,
            "e2e_how": ("K steps of (H2D query + lengths from pinned memory, nsa_decode, D2H "
                        "output + selection), double-buffered: the H2D of step i + 1 and the D2H "
                        "of step i - 1 on two copy streams overlap the decode of step i; "
                        + ("one CUDA graph" if use_graph else "eager launches")),
            "h2d": q_h.numel() * q_h.element_size() + lens_h.numel() * 4,
            "d2h": out_h.numel() * out_h.element_size() + sel_h.numel() * 4}


def run_prefill(w, K, W, ws, rank, local, e2e=True):
    from dynamic_block_sparse_nsa_b200 import nsa
    inp = inputs.make_prefill(w, seed=w["seed"] + rank, device="cuda")
    dt = inputs.DTYPES[w["dtype"]]
    p = nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], cmp_block=w["cmp_block"],
                   cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                   window=w["window"], dtype=dt, sel_mode=w.get("sel_mode", 0),
                   top_p=w.get("top_p", 0.0))
    Nc = nsa.num_cmp_blocks(w["T"], w["cmp_block"], w["cmp_stride"])
    kc = torch.empty(w["B"], Nc, w["Hkv"], w["d"], dtype=dt, device="cuda")
    vc = torch.empty_like(kc)
    ws_buf = nsa.workspace(p, nsa.OP_PREFILL)
    out = torch.empty_like(inp["q"])
    sel = torch.empty(w["B"], w["T"], w["Hkv"], w["top_n"], dtype=torch.int32, device="cuda")

    def step():
        nsa.nsa_compress_kv(p, inp["k"], inp["v"], inp["w_cmp"], kc, vc)
        nsa.nsa_prefill(p, inp["q"], inp["k"], inp["v"], kc, vc, inp["w_gate"], out=out,
                        sel_idx=sel, ws=ws_buf)

    step()
    nsa.nsa_check()
    res = timed(step, K, W, ws, local)
    nsa.nsa_check()
    fl = prefill_flops(w, sel.cpu().numpy())
    res.update(work=sum(fl.values()), parts=fl)
    if e2e:
        hq = inp["q"].cpu().pin_memory()
        hk = inp["k"].cpu().pin_memory()
        hv = inp["v"].cpu().pin_memory()
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            inp["q"].copy_(hq, non_blocking=True)
            inp["k"].copy_(hk, non_blocking=True)
            inp["v"].copy_(hv, non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        res["e2e_ms"] = _run_steps(e2e_step, K, False)[0]
        barrier(ws)
        res["h2d"] = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        res["d2h"] = ho.numel() * ho.element_size()
    return res


def run_moba(w, K, W, ws, rank, local, e2e=True):
    from dynamic_block_sparse_nsa_b200 import nsa
    inp = inputs.make_prefill(w, seed=w["seed"] + rank, device="cuda")
    p = nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], sel_block=w["block"],
                   top_n=w["top_k"], dtype=inputs.DTYPES[w["dtype"]])
    ws_buf = nsa.workspace(p, nsa.OP_MOBA_PREFILL)
    out = torch.empty_like(inp["q"])
    sel = torch.empty(w["B"], w["T"], w["Hq"], w["top_k"], dtype=torch.int32, device="cuda")

    def step():
        nsa.moba_prefill(p, inp["q"], inp["k"], inp["v"], out=out, sel_idx=sel, ws=ws_buf)

    step()
    nsa.nsa_check()
    res = timed(step, K, W, ws, local)
    nsa.nsa_check()
    fl = moba_flops(w, sel.cpu().numpy())
    res.update(work=fl["attn"] + fl["gate"], parts=fl)
    if e2e:
        hq, hk, hv = (inp[x].cpu().pin_memory() for x in ("q", "k", "v"))
        ho = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def e2e_step():
            inp["q"].copy_(hq, non_blocking=True)
            inp["k"].copy_(hk, non_blocking=True)
            inp["v"].copy_(hv, non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        res["e2e_ms"] = _run_steps(e2e_step, K, False)[0]
        barrier(ws)
        res["h2d"] = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
        res["d2h"] = ho.numel() * ho.element_size()
    return res


# --------------------------------------------------------------------------
# dominant kernel: algorithmic work per launch
# --------------------------------------------------------------------------

def kernel_work(kind, name, res, w):
    """Algorithmic bytes (decode) or flops (prefill) of one launch of `name`,
    and whether it is bandwidth ('hbm') or tensor ('tensor') bound."""
    if kind == "decode":
        p = res["parts"]
        per = {
            "nsa_rows_simt": p["cmp"] + p["slc"] + p["win"] + p["io"],
            "dec_cmp_partial": p["cmp"],
            "dec_sel_win": p["slc"] + p["win"],
        }
        return per.get(name), "hbm"
    if kind == "prefill":
        p = res["parts"]
        per = {
            "nsa_rows_simt": p["cmp"] + p["slc"] + p["win"],
            "pf_cmp_win": p["cmp"] + p["win"],
            "pf_slc_attn": p["slc"],
        }
        return per.get(name), "tensor"
    p = res["parts"]
    per = {"moba_rows_simt": p["attn"] + p["gate"], "moba_own": p["attn_own"],
           "moba_blk": p["attn_past"]}
    return per.get(name), "tensor"


# --------------------------------------------------------------------------
# CPU oracle (baseline leg and reference arm)
# --------------------------------------------------------------------------

def oracle_sample(w, budget_s):
    """Time the fp64 oracle on a bounded sample of the workload: returns
    (work units of the sample in the metric's unit numerator, seconds, cores,
    description)."""
    import oracle
    cores = os.cpu_count() or 1
    kind = w["kind"]
    if kind == "decode":
        # unit: one query row (the G heads of a KV group) against one KV
        # group's 65536-token cache and its compressed cache; `cores` units run
        # in parallel per oracle call (OpenMP over rows).
        one = dict(w, B=1)
        inp = inputs.make_decode(one, seed=w["seed"] + 1000)
        G = w["Hq"] // w["Hkv"]
        op = dict(B=1, T=w["T"], Hq=G, Hkv=1, d=w["d"], cmp_block=w["cmp_block"],
                  cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                  window=w["window"], scale=0.0, gate_mode=0, store=w["dtype"], score_mode=0)
        kg = np.ascontiguousarray(inp["k"][:, :, 0:1].double().numpy())
        vg = np.ascontiguousarray(inp["v"][:, :, 0:1].double().numpy())
        kc, vc = oracle.compress(op, kg, vg, inp["w_cmp"].double().numpy())
        q = inp["q"][0, 0:G].double().numpy()
        qrows = np.ascontiguousarray(np.broadcast_to(q, (cores, G, w["d"])))
        wg = inp["w_gate"].double().numpy()
        L = w["T"]
        byt, secs, done = 0, 0.0, 0
        while True:
            t0 = time.perf_counter()
            res = oracle.nsa_rows(op, [0] * cores, [L - 1] * cores, qrows, kg, vg, kc, vc, wg)
            secs += time.perf_counter() - t0
            for i in range(cores):
                byt += decode_work(dict(w, Hkv=1, Hq=G), [L], res["sel"][i:i + 1])[0]
            done += cores
            if secs >= budget_s:
                break
        return byt, secs, cores, (f"{done} (query row, KV head) units of the 65536-token "
                                  f"decode ({w['B'] * w['Hkv']} units make one step)")
    if kind == "prefill":
        inp = inputs.make_prefill(w, seed=w["seed"] + 1000)
        op = dict(B=w["B"], T=w["T"], Hq=w["Hq"], Hkv=w["Hkv"], d=w["d"],
                  cmp_block=w["cmp_block"], cmp_stride=w["cmp_stride"],
                  sel_block=w["sel_block"], top_n=w["top_n"], window=w["window"], scale=0.0,
                  gate_mode=0, store=w["dtype"], score_mode=0)
        k64, v64 = inp["k"].double().numpy(), inp["v"].double().numpy()
        kc, vc = oracle.compress(op, k64, v64, inp["w_cmp"].double().numpy())
        wg64 = inp["w_gate"].double().numpy()
        rng = np.random.default_rng(0)
        fl, t_used, done = 0, 0.0, 0
        while t_used < budget_s:
            rows = np.sort(rng.integers(0, w["T"], cores))
            q_rows = np.ascontiguousarray(inp["q"][0, torch.from_numpy(rows)].double().numpy())
            t0 = time.perf_counter()
            res = oracle.nsa_rows(op, [0] * len(rows), rows, q_rows, k64, v64, kc, vc, wg64)
            t_used += time.perf_counter() - t0
            for i, t in enumerate(rows):
                nv = n_cmp(t + 1, w["cmp_block"], w["cmp_stride"])
                ks = sum(sel_tokens(res["sel"][i, g], t, w["sel_block"]) for g in range(w["Hkv"]))
                fl += 4 * w["d"] * (nv * w["Hq"] + ks * (w["Hq"] // w["Hkv"])
                                    + min(w["window"], t + 1) * w["Hq"])
            done += len(rows)
        return fl, t_used, cores, f"{done} uniformly sampled query rows (all heads)"
    # moba
    inp = inputs.make_prefill(dict(w, Hq=4, Hkv=4), seed=w["seed"] + 1000)
    op = dict(B=1, T=w["T"], Hq=4, Hkv=4, d=w["d"], block=w["block"], top_k=w["top_k"],
              scale=0.0)
    k64, v64, q64 = (inp[x].double().numpy() for x in ("k", "v", "q"))
    kbar = oracle.moba_block_means(op, k64)
    rng = np.random.default_rng(0)
    fl, t_used, done = 0, 0.0, 0
    while t_used < budget_s:
        rows = np.sort(rng.integers(0, w["T"], cores))
        t0 = time.perf_counter()
        res = oracle.moba_rows(op, [0] * len(rows), rows, q64[0, rows], k64, v64, kbar)
        t_used += time.perf_counter() - t0
        for i, t in enumerate(rows):
            for h in range(4):
                fl += 4 * w["d"] * sel_tokens(res["sel"][i, h], t, w["block"])
                fl += 2 * w["d"] * (t // w["block"])
        done += len(rows)
    return fl, t_used, cores, f"{done} sampled query rows x 4 heads"


def unit_of(kind):
    return ("GB/s", 1e9) if kind == "decode" else ("TFLOP/s", 1e12)


def run_reference(args, w):
    """The oracle, as it stands, timed on the host cores: K steps of a bounded
    sample each, sized so the whole run stays within a few minutes."""
    kind = w["kind"]
    unit, scale = unit_of(kind)
    per_step = max(0.02, args.ref_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, per_step)
    work = secs = 0.0
    cores, desc = 1, ""
    for _ in range(args.steps):
        wk, dt, cores, desc = oracle_sample(w, per_step)
        work += wk
        secs += dt
    value = work / secs / scale
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * secs / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, **config_of(w),
                   **({"overrides": args.set} if args.set else {})},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {desc}"},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w):
    keys = [k for k in ("B", "T", "Hq", "Hkv", "d", "cmp_block", "cmp_stride", "sel_block",
                        "top_n", "window", "block", "top_k", "dtype") if k in w]
    c = {k: w[k] for k in keys}
    return c


# --------------------------------------------------------------------------

def run_dense(w, K, W, rank):
    """Dense causal attention of the prefill's shape, with this library: nsa_prefill
    with gates fixed to (0, 0, 1) and a window covering the sequence (the
    closed form in which NSA is dense attention; the zero-gated branches are
    skipped). Returns (ms per step, algorithmic flops per step)."""
    from dynamic_block_sparse_nsa_b200 import nsa
    inp = inputs.make_prefill(w, seed=w["seed"] + rank, device="cuda")
    dt = inputs.DTYPES[w["dtype"]]
    p = nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], cmp_block=w["cmp_block"],
                   cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                   window=w["T"], dtype=dt, gate_mode=1, fixed_gates=(0.0, 0.0, 1.0))
    Nc = nsa.num_cmp_blocks(w["T"], w["cmp_block"], w["cmp_stride"])
    kc = torch.zeros(w["B"], Nc, w["Hkv"], w["d"], dtype=dt, device="cuda")
    vc = torch.zeros_like(kc)
    ws_buf = nsa.workspace(p, nsa.OP_PREFILL)
    out = torch.empty_like(inp["q"])

    def step():
        nsa.nsa_prefill(p, inp["q"], inp["k"], inp["v"], kc, vc, None, out=out, ws=ws_buf,
                        want_sel=False)

    for _ in range(W):
        step()
    nsa.nsa_check()
    ms = _run_steps(step, K, False)[0] / K
    nsa.nsa_check()
    T = w["T"]
    flops = w["B"] * (T * (T + 1) // 2) * w["Hq"] * 4 * w["d"]
    return ms, flops


def kernel_entries(kind, res, w, K, peaks, wname):
    """Every traced kernel of a prefill-like step against the bf16 peak
    (burst, and sustained beside it), from the first timed region's events."""
    per = {}
    for n, e in res["table0"].items():
        wk, _ = kernel_work(kind, n, res, w)
        if wk is None or not e["launches"]:
            continue
        per_launch = wk / (e["launches"] / min(K, 50))
        mean_s = e["total_ms"] / e["launches"] / 1000.0
        ach = per_launch / mean_s / 1e12
        ent = {"tflops": ach, "frac": ach / peaks["bf16"], "peak": peaks["bf16"],
               "frac_sustained": ach / peaks["bf16_sus"], "mean_launch_us": 1e6 * mean_s,
               "flops_per_launch": per_launch}
        tr = kernel_traffic(n, wname)
        if tr is not None:
            ent["traffic"] = tr  # DRAM bytes per launch (ncu), while the source is unchanged
        g = gather_bytes(kind, n, res, w)
        if g is not None:
            ent["gathered_bytes_per_launch"] = g
            ent["gather_gbs"] = g / mean_s / 1e9
        per[n] = ent
    return per


def gather_bytes(kind, name, res, w):
    """Bytes a kernel moves into shared memory per launch by design (not its
    DRAM traffic): the selected-branch prefill kernel reads every selected
    block's K and V once per (token, KV head), so this is its ingest figure."""
    if kind == "prefill" and name == "pf_slc_attn":
        return res["parts"]["slc"] / (4 * w["d"]) / (w["Hq"] // w["Hkv"]) * 2 * w["d"] * 2
    return None


def side_summary(name, ws, rank, local, peaks, K, W, cpu_budget, dense=False, e2e=True):
    """One more workload timed like the main line (prefill or MoBA): whole-step
    TFLOP/s, every kernel against the bf16 peak, the end-to-end figure with
    host copies, and the oracle timed on a bounded sample (rank 0, one GPU)."""
    w = inputs.workload(name)
    kind = w["kind"]
    runner = {"prefill": run_prefill, "moba": run_moba}[kind]
    res = runner(w, K, W, ws, rank, local, e2e=e2e)
    ms_max = reduce_max(res["ms"], ws)
    work_all = reduce_sum(res["work"] * K, ws)
    out = {"workload": name, "config": config_of(w), "value": work_all / (ms_max / 1000.0) / 1e12,
           "unit": "TFLOP/s", "ms_per_step": ms_max / K, "steps": K, "warmup": W,
           "flops_per_step": res["parts"],
           "kernel_tflops": kernel_entries(kind, res, w, K, peaks, name),
           "peak_source": peaks["src"], "clocks": res["clk"]}
    out["value_frac"] = out["value"] / peaks["bf16"]
    if "e2e_ms" in res:
        e_ms = reduce_max(res["e2e_ms"], ws)
        out["e2e"] = {"value": work_all / (e_ms / 1000.0) / 1e12, "unit": "TFLOP/s",
                      "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
                      "ms_per_step": e_ms / K,
                      "how": "H2D of q, k, v from pinned memory, the call(s), D2H of the "
                             "output, every step"}
    if dense:
        dms, dfl = run_dense(w, 2, 1, rank)
        dms = reduce_max(dms, ws)
        out["dense_causal"] = {
            "ms_per_step": dms, "tflops": dfl / (dms / 1000.0) / 1e12, "flops_per_step": dfl,
            "frac": dfl / (dms / 1000.0) / 1e12 / peaks["bf16"],
            "nsa_speedup": dms / (ms_max / K),
            "how": "nsa_prefill with gates fixed to (0, 0, 1) and window = T (dense causal "
                   "attention, same shape), 2 timed steps after 1 warm-up"}
    if rank == 0 and ws == 1 and cpu_budget > 0:
        wk, secs, cores, desc = oracle_sample(w, cpu_budget)
        out["cpu_baseline"] = {"value": wk / secs / 1e12, "unit": "TFLOP/s", "cores": cores,
                               "kind": "oracle", "sample": desc, "seconds": secs}
    if kind == "prefill":
        out["note"] = ("algorithmic flops (4 d per query head and attended key); a step is "
                       "nsa_compress_kv + nsa_prefill on device-resident inputs")
    else:
        out["note"] = ("algorithmic flops: 4 d per (query head, attended key) plus the gate's "
                       "2 d per (query head, earlier block); a step is one moba_prefill")
    return out


def backward_oracle_sample(budget_s=6.0):
    """The fp64 backward oracle, as it stands, on the host: whole backward
    passes of a bounded sample with the benchmark's heads and head dim (bf16
    values, 64 / 4 heads, d = 128, top-16, window 512) and fewer tokens,
    repeated until the budget is spent. Returns a cpu_baseline dict in the
    bench's flop count (10 d per query head and attended key)."""
    import oracle
    from oracle import backward as obwd
    T = 128
    w = inputs.workload("nsa_prefill_bf16_t8192", T=T)
    inp = inputs.make_prefill(w, seed=5)
    op = dict(B=1, T=T, Hq=w["Hq"], Hkv=w["Hkv"], d=w["d"], cmp_block=w["cmp_block"],
              cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
              window=w["window"], scale=0.0, gate_mode=0, fixed_gates=(0.0, 0.0, 0.0),
              store="bf16", score_mode=0, top_p=0.0)
    f64 = {k_: v_.double().numpy() for k_, v_ in inp.items()}
    fwd = oracle.nsa_prefill(op, f64["q"], f64["k"], f64["v"], f64["w_cmp"], f64["w_gate"])
    sel = fwd["sel"].reshape(1, T, w["Hkv"], w["top_n"])
    dout = np.random.default_rng(6).standard_normal(f64["q"].shape)
    bs, l, s_ = w["sel_block"], w["cmp_block"], w["cmp_stride"]
    t = np.arange(T)
    tt = t[None, :, None, None]
    ok = (sel >= 0) & (sel <= tt // bs)
    nslc = np.where(ok, np.minimum(bs, tt + 1 - sel * bs), 0).sum()
    keys = nslc + w["Hkv"] * (np.where(t + 1 >= l, (t + 1 - l) // s_ + 1, 0).sum() +
                              np.minimum(w["window"], t + 1).sum())
    flops_per = 10.0 * w["d"] * (w["Hq"] // w["Hkv"]) * float(keys)
    done, used = 0, 0.0
    while used < budget_s:
        t0 = time.perf_counter()
        obwd.nsa_prefill_backward(op, f64["q"], f64["k"], f64["v"], f64["w_cmp"], f64["w_gate"],
                                  dout, sel, kc=fwd["k_cmp"], vc=fwd["v_cmp"])
        used += time.perf_counter() - t0
        done += 1
    return {"value": done * flops_per / used / 1e12, "unit": "TFLOP/s", "cores": 1,
            "kind": "oracle", "seconds": used,
            "sample": f"{done} whole backward passes of a {T}-token sequence (64 / 4 heads, "
                      f"d = 128, top-16, window 512)"}


def backward_summary(ws, rank, peaks, clk_max_mhz, K=2, W=1):
    """The prefill backward at 8192 tokens (64 / 4 heads, d = 128, bf16):
    forward once for the selection, then K timed backward steps. Algorithmic
    flops: 10 d per (query head, attended key) over the three branches (the
    logits again, dO . v, and the dq, dk, dv products). The path runs on CUDA
    cores in fp32, so its roofline is the fp32 FMA rate: SMs x 128 lanes x 2
    flops x the maximum SM clock."""
    from dynamic_block_sparse_nsa_b200 import nsa
    name = "nsa_prefill_bf16_t8192"
    w = inputs.workload(name)
    inp = inputs.make_prefill(w, seed=w["seed"] + rank, device="cuda")
    dt = inputs.DTYPES[w["dtype"]]
    p = nsa.params(w["B"], w["T"], w["Hq"], w["Hkv"], w["d"], cmp_block=w["cmp_block"],
                   cmp_stride=w["cmp_stride"], sel_block=w["sel_block"], top_n=w["top_n"],
                   window=w["window"], dtype=dt)
    kc, vc = nsa.nsa_compress_kv(p, inp["k"], inp["v"], inp["w_cmp"])
    _, sel = nsa.nsa_prefill(p, inp["q"], inp["k"], inp["v"], kc, vc, inp["w_gate"])
    gen = torch.Generator(device="cuda").manual_seed(w["seed"] + 7 + rank)
    dout = torch.randn(inp["q"].shape, generator=gen, device="cuda").to(dt)
    ws_buf = nsa.workspace(p, nsa.OP_PREFILL_BACKWARD)

    def step():
        nsa.nsa_prefill_backward(p, inp["q"], inp["k"], inp["v"], kc, vc, inp["w_cmp"],
                                 inp["w_gate"], sel, dout, ws=ws_buf)

    for _ in range(W):
        step()
    nsa.nsa_check()
    ms = reduce_max(_run_steps(step, K, False)[0] / K, ws)
    nsa.nsa_check()
    # attended keys per (token, KV head): visible compressed blocks, selected
    # tokens up to t, window
    T, bs, l, s_ = w["T"], w["sel_block"], w["cmp_block"], w["cmp_stride"]
    t = np.arange(T)
    nvis = np.where(t + 1 >= l, (t + 1 - l) // s_ + 1, 0)
    sl = sel.cpu().numpy().astype(np.int64)  # [B, T, Hkv, n]
    tt = t[None, :, None, None]
    ok = (sl >= 0) & (sl <= tt // bs)
    nslc = np.where(ok, np.minimum(bs, tt + 1 - sl * bs), 0).sum(axis=-1)  # [B, T, Hkv]
    nwin = np.minimum(w["window"], t + 1)
    keys = nslc.sum() + w["B"] * w["Hkv"] * (nvis.sum() + nwin.sum())
    G = w["Hq"] // w["Hkv"]
    flops = 10.0 * w["d"] * G * float(keys)
    tflops = flops / (ms / 1000.0) / 1e12
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    peak = sms * 128 * 2 * clk_max_mhz * 1e6 / 1e12
    cpu = backward_oracle_sample() if rank == 0 else None
    return {"workload": name, "value": tflops, "unit": "TFLOP/s", "ms_per_step": ms,
            "steps": K, "warmup": W, "flops_per_step": flops, "cpu_baseline": cpu,
            "roofline": {"bound": "alu", "achieved": tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": tflops / peak,
                         "peak_from": f"{sms} SMs x 128 fp32 lanes x 2 flops x {clk_max_mhz} MHz"},
            "note": "nsa_prefill_backward (CUDA-core fp32 path): dq, dk, dv, dw_cmp, dw_gate "
                    "of sum(dout * out), selection from the forward"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--side-cpu-budget", type=float, default=8.0,
                    help="host seconds of oracle timing for each workload beside the main one")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="host seconds the reference arm spends over all its steps")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill, MoBA and backward workloads measured beside the "
                         "default decode line")
    ap.add_argument("--only-backward", action="store_true",
                    help="time only the 8192-token prefill backward (for profiling it)")
    ap.add_argument("--no-graph", action="store_true",
                    help="time decode steps as separate launches instead of one CUDA graph")
    ap.add_argument("--set", action="append", default=[], metavar="KEY=VALUE",
                    help="override a workload field (smaller cases for profiling)")
    args = ap.parse_args()
    w = inputs.workload(args.workload)
    for kv in args.set:
        key, val = kv.split("=", 1)
        w[key] = type(w[key])(val) if key in w else int(val)
    kind = w["kind"]
    if args.set and args.impl == "ours":
        args.no_cpu_baseline = True
    if args.steps is None:
        args.steps = {"decode": 2000, "prefill": 20, "moba": 10}[kind]
    if args.warmup is None:
        args.warmup = {"decode": 20, "prefill": 3, "moba": 3}[kind]
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank == 0:
            run_reference(args, w)
        return

    ws, rank, local = dist_setup()
    import dynamic_block_sparse_nsa_b200.nsa  # noqa: F401  (fails loudly if unbuilt)
    if args.only_backward:
        bw = backward_summary(ws, rank, load_peaks(), 1965)
        if rank == 0:
            print(json.dumps({"prefill_backward_8k": bw}), flush=True)
        return
    runner = {"decode": run_decode, "prefill": run_prefill, "moba": run_moba}[kind]
    kw = {"use_graph": not args.no_graph} if kind == "decode" else {}
    res = runner(w, args.steps, args.warmup, ws, rank, local, e2e=not args.no_e2e, **kw)

    K = args.steps
    ms_max = reduce_max(res["ms"], ws)
    work_all = reduce_sum(res["work"] * K, ws)
    unit, scale = unit_of(kind)
    value = work_all / (ms_max / 1000.0) / scale
    e2e = None
    if "e2e_ms" in res:
        e_ms = reduce_max(res["e2e_ms"], ws)
        e2e = {"value": work_all / (e_ms / 1000.0) / scale, "unit": unit,
               "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"],
               "ms_per_step": e_ms / K}
        if "e2e_how" in res:
            e2e["how"] = res["e2e_how"]

    tab = kernel_table(res["recs"], K)
    peaks = load_peaks()
    roof = None
    dom = res["dom"]
    if dom and dom in tab:
        wk, bound = kernel_work(kind, dom, res, w)
        mean_s = tab[dom]["total_ms"] / tab[dom]["launches"] / 1000.0
        mean_s = reduce_max(mean_s, ws)
        if wk is not None:
            per_launch = wk / (tab[dom]["launches"] / K)
            if bound == "hbm":
                ach = per_launch / mean_s / 1e9
                pk, u = peaks["hbm"], "GB/s"
            else:
                ach = per_launch / mean_s / 1e12
                pk, u = peaks["bf16"], "TFLOP/s"
            roof = {"scope": "kernel", "kernel": dom, "bound": bound, "achieved": ach, "peak": pk,
                    "unit": u, "frac": ach / pk, "peak_source": peaks["src"],
                    "traffic": kernel_traffic(dom, args.workload),
                    "algorithmic_per_launch": per_launch,
                    "mean_launch_us": mean_s * 1e6,
                    "timing": "events around each launch of this kernel over a second "
                              "timed region of the same K steps",
                    # the whole step against the same peak (the line's value)
                    "step": {"achieved": value, "frac": value / pk,
                             **({"frac_nominal_8tbs": value / 8000.0} if bound == "hbm" else {})}}

    sides = {}
    if kind == "decode" and not args.set and not args.no_prefill and args.workload == DEFAULT_WORKLOAD:
        cb = 0.0 if args.no_cpu_baseline else args.side_cpu_budget
        sides["prefill_64k"] = side_summary("nsa_prefill_bf16_t65536", ws, rank, local, peaks,
                                            K=5, W=3, cpu_budget=cb, dense=True,
                                            e2e=not args.no_e2e)
        sides["prefill_8k"] = side_summary("nsa_prefill_bf16_t8192", ws, rank, local, peaks,
                                           K=20, W=3, cpu_budget=cb, e2e=not args.no_e2e)
        sides["moba_128k"] = side_summary("moba_prefill_bf16_t131072", ws, rank, local, peaks,
                                          K=5, W=3, cpu_budget=cb, e2e=not args.no_e2e)
        clk_max = (res.get("clk") or {}).get("sm_max_mhz") or 1965
        sides["prefill_backward_8k"] = backward_summary(ws, rank, peaks, clk_max)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        wk, secs, cores, desc = oracle_sample(w, args.cpu_budget)
        cpu = {"value": wk / secs / scale, "unit": unit, "cores": cores, "kind": "oracle",
               "sample": desc, "seconds": secs}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": unit, "n_gpus": ws, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
            "config": {"workload": args.workload, **config_of(w),
                       **({"overrides": args.set} if args.set else {}),
                       "l2": "inputs larger than L2 every step "
                             f"({res['work'] / 1e6:.0f} MB read per step)" if kind == "decode"
                       else "inputs larger than L2 every step"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": res["launches"],
            "timing": "cuda_graph" if (kind == "decode" and not args.no_graph) else "stream",
            "clocks": res["clk"],
            "kernels_event_bracketed": {
                n: {k: (round(v, 4) if isinstance(v, float) else v) for k, v in e.items()}
                for n, e in res["table0"].items()},
        }
        if kind == "decode":
            line["decode_bytes"] = {"per_step": res["work"], "union_per_step": res["union"],
                                    **{k: v for k, v in res["parts"].items()}}
            line["hbm_frac_nominal_8tbs"] = value / 8000.0
        else:
            line["flops_per_step"] = {k: v for k, v in res["parts"].items()}
            # every traced kernel against the bf16 peak (first timed region's events)
            per = kernel_entries(kind, res, w, K, peaks, args.workload)
            line["kernel_tflops"] = per
        line.update(sides)
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
