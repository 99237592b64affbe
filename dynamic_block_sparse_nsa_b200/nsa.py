"""Thin Python binding of ``libnsa_b200.so`` (argument marshalling only).

Every step of the computation runs in the library's CUDA kernels; this module
turns torch tensors into device pointers, passes the current CUDA stream and
raises :class:`NsaError` on a non-OK status. If the library has not been built
the import fails loudly -- there is no fallback.

Names mirror the C ABI in ``include/nsa.h``: ``nsa_compress_kv``,
``nsa_prefill``, ``nsa_decode``, ``moba_prefill``, ``nsa_check``.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnsa_b200.so")

NSA_OK = 0
STATUS = {
    0: "NSA_OK", 1: "NSA_ERR_INVALID_ARGUMENT", 2: "NSA_ERR_UNSUPPORTED",
    3: "NSA_ERR_WORKSPACE_TOO_SMALL", 4: "NSA_ERR_CUDA", 5: "NSA_ERR_DEVICE_TIMEOUT",
}
OP_COMPRESS, OP_PREFILL, OP_DECODE, OP_MOBA_PREFILL, OP_PREFILL_BACKWARD = 0, 1, 2, 3, 4
DTYPE_F32, DTYPE_BF16 = 0, 1
_TORCH_DTYPE = {DTYPE_F32: torch.float32, DTYPE_BF16: torch.bfloat16}

# Every symbol include/nsa.h declares.
EXPORTS = (
    "nsa_workspace_size", "nsa_num_cmp_blocks", "nsa_compress_kv", "nsa_prefill",
    "nsa_prefill_backward", "nsa_decode",
    "moba_prefill", "nsa_decode_noalloc", "nsa_append_kv", "nsa_block_bounds",
    "nsa_append_bounds", "nsa_decode_quest", "nsa_check", "nsa_debug_bounded_wait", "nsa_status_string",
    "nsa_last_error_detail", "nsa_trace_enable", "nsa_trace_set_filter", "nsa_trace_count",
    "nsa_trace_timed", "nsa_trace_get",
)


class NsaError(RuntimeError):
    def __init__(self, status, detail):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {detail}")


class NsaParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("T", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("d", ctypes.c_int), ("cmp_block", ctypes.c_int), ("cmp_stride", ctypes.c_int),
        ("sel_block", ctypes.c_int), ("top_n", ctypes.c_int), ("window", ctypes.c_int),
        ("softmax_scale", ctypes.c_float), ("gate_mode", ctypes.c_int),
        ("fixed_gates", ctypes.c_float * 3), ("dtype", ctypes.c_int), ("top_p", ctypes.c_float),
        ("sel_mode", ctypes.c_int),
    ]

    @property
    def torch_dtype(self):
        return _TORCH_DTYPE[self.dtype]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with dynamic_block_sparse_nsa_b200.build.build()")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(NsaParams)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "nsa_workspace_size": [P, ctypes.c_int, ctypes.POINTER(sz)],
        "nsa_num_cmp_blocks": [ctypes.c_int] * 3,
        "nsa_compress_kv": [P, vp, vp, vp, vp, vp, vp],
        "nsa_prefill": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "nsa_decode": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "nsa_prefill_backward": [P] + [vp] * 15 + [sz, vp],
        "moba_prefill": [P, vp, vp, vp, vp, vp, vp, sz, vp],
        "nsa_decode_noalloc": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "nsa_append_kv": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "nsa_block_bounds": [P, vp, vp, vp, vp],
        "nsa_append_bounds": [P, vp, vp, vp, vp],
        "nsa_decode_quest": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "nsa_check": [vp],
        "nsa_debug_bounded_wait": [vp, ctypes.c_int, vp],
        "nsa_status_string": [ctypes.c_int],
        "nsa_last_error_detail": [],
        "nsa_trace_enable": [ctypes.c_int, ctypes.c_int],
        "nsa_trace_count": [],
        "nsa_trace_timed": [],
        "nsa_trace_set_filter": [ctypes.c_char_p],
        "nsa_trace_get": [ctypes.c_int, ctypes.POINTER(ctypes.c_char_p),
                          ctypes.POINTER(ctypes.c_float)],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.nsa_status_string.restype = ctypes.c_char_p
    lib.nsa_last_error_detail.restype = ctypes.c_char_p
    return lib


LIB = _load()


def _raise(st):
    if st != NSA_OK:
        raise NsaError(st, LIB.nsa_last_error_detail().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    """The stream to enqueue on: `stream`, else the current stream of `device`
    (of the current device when None). A given stream must live on `device`."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != torch.device(device):
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _dev(t, name, dtype=None, device=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device} (all tensors of a call "
                         f"must share one device)")


class _on:
    """Makes the tensors' device current for the call: the library reads the
    current device for its per-device state (error word, cached tensor maps,
    the no-allocation scratch), so it must be the device the data lives on."""

    def __init__(self, device):
        self.ctx = torch.cuda.device(device)

    def __enter__(self):
        self.ctx.__enter__()

    def __exit__(self, *a):
        self.ctx.__exit__(*a)


def params(B, T, Hq, Hkv, d, cmp_block=32, cmp_stride=16, sel_block=64, top_n=16, window=512,
           softmax_scale=0.0, gate_mode=0, fixed_gates=(0.0, 0.0, 0.0), dtype=torch.bfloat16,
           top_p=0.0, sel_mode=0):
    p = NsaParams()
    p.B, p.T, p.Hq, p.Hkv, p.d = B, T, Hq, Hkv, d
    p.cmp_block, p.cmp_stride, p.sel_block, p.top_n, p.window = (
        cmp_block, cmp_stride, sel_block, top_n, window)
    p.softmax_scale = softmax_scale
    p.gate_mode = gate_mode
    for i in range(3):
        p.fixed_gates[i] = fixed_gates[i]
    p.dtype = DTYPE_BF16 if dtype == torch.bfloat16 else DTYPE_F32
    p.top_p = top_p
    p.sel_mode = sel_mode
    return p


def num_cmp_blocks(T, l, s):
    return LIB.nsa_num_cmp_blocks(T, l, s)


def workspace_size(p, op):
    n = ctypes.c_size_t(0)
    _raise(LIB.nsa_workspace_size(ctypes.byref(p), op, ctypes.byref(n)))
    return n.value


def workspace(p, op, device="cuda"):
    n = workspace_size(p, op)
    return torch.empty(max(n, 1), dtype=torch.uint8, device=device) if n else None


def nsa_compress_kv(p, k, v, w_cmp, k_cmp=None, v_cmp=None, stream=None):
    dt = p.torch_dtype
    _dev(k, "k", dt)
    dev = k.device
    _dev(v, "v", dt, dev)
    _dev(w_cmp, "w_cmp", torch.float32, dev)
    Nc = num_cmp_blocks(p.T, p.cmp_block, p.cmp_stride)
    shape = (p.B, Nc, p.Hkv, p.d)
    if k_cmp is None:
        k_cmp = torch.empty(shape, dtype=dt, device=dev)
    if v_cmp is None:
        v_cmp = torch.empty(shape, dtype=dt, device=dev)
    _dev(k_cmp, "k_cmp", dt, dev)
    _dev(v_cmp, "v_cmp", dt, dev)
    with _on(dev):
        _raise(LIB.nsa_compress_kv(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(w_cmp), _ptr(k_cmp),
                                   _ptr(v_cmp), _stream(stream, dev)))
    return k_cmp, v_cmp


def nsa_prefill(p, q, k, v, k_cmp, v_cmp, w_gate=None, out=None, sel_idx=None, ws=None,
                stream=None, want_sel=True):
    dt = p.torch_dtype
    _dev(q, "q", dt)
    dev = q.device
    for t, nm in ((k, "k"), (v, "v"), (k_cmp, "k_cmp"), (v_cmp, "v_cmp")):
        _dev(t, nm, dt, dev)
    _dev(w_gate, "w_gate", torch.float32, dev)
    if out is None:
        out = torch.empty(p.B, p.T, p.Hq, p.d, dtype=dt, device=dev)
    if sel_idx is None and want_sel:
        sel_idx = torch.empty(p.B, p.T, p.Hkv, p.top_n, dtype=torch.int32, device=dev)
    _dev(out, "out", dt, dev)
    _dev(sel_idx, "sel_idx", torch.int32, dev)
    if ws is None:
        ws = workspace(p, OP_PREFILL, dev)
    _dev(ws, "ws", None, dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    with _on(dev):
        _raise(LIB.nsa_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(k_cmp),
                               _ptr(v_cmp), _ptr(w_gate), _ptr(out), _ptr(sel_idx), _ptr(ws),
                               nbytes, _stream(stream, dev)))
    return out, sel_idx


def nsa_prefill_backward(p, q, k, v, k_cmp, v_cmp, w_cmp, w_gate, sel_idx, dout, ws=None,
                         stream=None):
    """Gradients of sum(dout * out) of nsa_prefill: (dq, dk, dv, dw_cmp, dw_gate), fp32."""
    dt = p.torch_dtype
    _dev(q, "q", dt)
    dev = q.device
    for t, nm in ((k, "k"), (v, "v"), (k_cmp, "k_cmp"), (v_cmp, "v_cmp"), (dout, "dout")):
        _dev(t, nm, dt, dev)
    _dev(w_cmp, "w_cmp", torch.float32, dev)
    _dev(w_gate, "w_gate", torch.float32, dev)
    _dev(sel_idx, "sel_idx", torch.int32, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    dq = torch.empty(p.B, p.T, p.Hq, p.d, **f32)
    dk = torch.empty(p.B, p.T, p.Hkv, p.d, **f32)
    dv = torch.empty(p.B, p.T, p.Hkv, p.d, **f32)
    dw_cmp = torch.empty(p.cmp_block, **f32)
    dw_gate = torch.empty(p.d, 3, **f32)
    if ws is None:
        ws = workspace(p, OP_PREFILL_BACKWARD, dev)
    _dev(ws, "ws", None, dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    with _on(dev):
        _raise(LIB.nsa_prefill_backward(
            ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(k_cmp), _ptr(v_cmp), _ptr(w_cmp),
            _ptr(w_gate), _ptr(sel_idx), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dw_cmp),
            _ptr(dw_gate), _ptr(ws), nbytes, _stream(stream, dev)))
    return dq, dk, dv, dw_cmp, dw_gate


def _decode_args(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out, sel_idx,
                 want_sel):
    """Checks of the decode arguments (one device for all); allocates the
    outputs that are not given."""
    dt = p.torch_dtype
    _dev(q, "q", dt)
    dev = q.device
    for t, nm in ((k_cache, "k_cache"), (v_cache, "v_cache"), (k_cmp, "k_cmp"),
                  (v_cmp, "v_cmp")):
        _dev(t, nm, dt, dev)
    _dev(seq_lens, "seq_lens", torch.int32, dev)
    _dev(w_gate, "w_gate", torch.float32, dev)
    if out is None:
        out = torch.empty(p.B, p.Hq, p.d, dtype=dt, device=dev)
    if sel_idx is None and want_sel:
        sel_idx = torch.empty(p.B, p.Hkv, p.top_n, dtype=torch.int32, device=dev)
    _dev(out, "out", dt, dev)
    _dev(sel_idx, "sel_idx", torch.int32, dev)
    return out, sel_idx


def nsa_decode(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate=None, out=None,
               sel_idx=None, ws=None, stream=None, want_sel=True):
    out, sel_idx = _decode_args(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out,
                                sel_idx, want_sel)
    dev = q.device
    if ws is None:
        ws = workspace(p, OP_DECODE, dev)
    _dev(ws, "ws", None, dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    with _on(dev):
        _raise(LIB.nsa_decode(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                              _ptr(seq_lens), _ptr(k_cmp), _ptr(v_cmp), _ptr(w_gate), _ptr(out),
                              _ptr(sel_idx), _ptr(ws), nbytes, _stream(stream, dev)))
    return out, sel_idx


def nsa_decode_noalloc(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate=None, out=None,
                       sel_idx=None, stream=None, want_sel=True):
    """nsa_decode with the library's static scratch instead of a workspace, for
    callers that cannot allocate device memory (include/nsa.h gives the limits;
    calls must not overlap on the GPU). The C call allocates nothing; this
    wrapper allocates `out` / `sel_idx` only when they are not given."""
    out, sel_idx = _decode_args(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out,
                                sel_idx, want_sel)
    dev = q.device
    # the device current during the call selects which GPU's static scratch is used
    with _on(dev):
        _raise(LIB.nsa_decode_noalloc(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                      _ptr(seq_lens), _ptr(k_cmp), _ptr(v_cmp), _ptr(w_gate),
                                      _ptr(out), _ptr(sel_idx), _stream(stream, dev)))
    return out, sel_idx


def nsa_append_kv(p, k_new, v_new, pos, k_cache, v_cache, w_cmp, k_cmp, v_cmp, stream=None):
    """Write one token per sequence at pos[b] into the caches; complete
    compressed blocks are written into k_cmp / v_cmp (see include/nsa.h)."""
    dt = p.torch_dtype
    _dev(k_new, "k_new", dt)
    dev = k_new.device
    for t, nm in ((v_new, "v_new"), (k_cache, "k_cache"), (v_cache, "v_cache"),
                  (k_cmp, "k_cmp"), (v_cmp, "v_cmp")):
        _dev(t, nm, dt, dev)
    _dev(pos, "pos", torch.int32, dev)
    _dev(w_cmp, "w_cmp", torch.float32, dev)
    with _on(dev):
        _raise(LIB.nsa_append_kv(ctypes.byref(p), _ptr(k_new), _ptr(v_new), _ptr(pos),
                                 _ptr(k_cache), _ptr(v_cache), _ptr(w_cmp), _ptr(k_cmp),
                                 _ptr(v_cmp), _stream(stream, dev)))


def nsa_block_bounds(p, k_cache, seq_lens, k_bounds=None, stream=None):
    """Per selection block of the cache, the element-wise max and min of its
    keys among the first seq_lens[b] tokens: [B, nblk, Hkv, 2, d]."""
    dt = p.torch_dtype
    _dev(k_cache, "k_cache", dt)
    dev = k_cache.device
    _dev(seq_lens, "seq_lens", torch.int32, dev)
    nblk = -(-p.T // p.sel_block)
    if k_bounds is None:
        k_bounds = torch.empty(p.B, nblk, p.Hkv, 2, p.d, dtype=dt, device=dev)
    _dev(k_bounds, "k_bounds", dt, dev)
    with _on(dev):
        _raise(LIB.nsa_block_bounds(ctypes.byref(p), _ptr(k_cache), _ptr(seq_lens), _ptr(k_bounds),
                                    _stream(stream, dev)))
    return k_bounds


def nsa_append_bounds(p, k_new, pos, k_bounds, stream=None):
    """Fold the keys appended at pos[b] into their blocks' bounds."""
    dt = p.torch_dtype
    _dev(k_new, "k_new", dt)
    dev = k_new.device
    _dev(pos, "pos", torch.int32, dev)
    _dev(k_bounds, "k_bounds", dt, dev)
    with _on(dev):
        _raise(LIB.nsa_append_bounds(ctypes.byref(p), _ptr(k_new), _ptr(pos), _ptr(k_bounds),
                                     _stream(stream, dev)))


def nsa_decode_quest(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, k_bounds, w_gate=None,
                     out=None, sel_idx=None, ws=None, stream=None, want_sel=True):
    """nsa_decode ranking blocks by the Quest-style bound from k_bounds
    (p.sel_mode must be 1)."""
    out, sel_idx = _decode_args(p, q, k_cache, v_cache, seq_lens, k_cmp, v_cmp, w_gate, out,
                                sel_idx, want_sel)
    dev = q.device
    _dev(k_bounds, "k_bounds", p.torch_dtype, dev)
    if ws is None:
        ws = workspace(p, OP_DECODE, dev)
    _dev(ws, "ws", None, dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    with _on(dev):
        _raise(LIB.nsa_decode_quest(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _ptr(seq_lens), _ptr(k_cmp), _ptr(v_cmp), _ptr(k_bounds),
                                    _ptr(w_gate), _ptr(out), _ptr(sel_idx), _ptr(ws), nbytes,
                                    _stream(stream, dev)))
    return out, sel_idx


def moba_prefill(p, q, k, v, out=None, sel_idx=None, ws=None, stream=None, want_sel=True):
    dt = p.torch_dtype
    _dev(q, "q", dt)
    dev = q.device
    _dev(k, "k", dt, dev)
    _dev(v, "v", dt, dev)
    if out is None:
        out = torch.empty(p.B, p.T, p.Hq, p.d, dtype=dt, device=dev)
    if sel_idx is None and want_sel:
        sel_idx = torch.empty(p.B, p.T, p.Hq, p.top_n, dtype=torch.int32, device=dev)
    _dev(out, "out", dt, dev)
    _dev(sel_idx, "sel_idx", torch.int32, dev)
    if ws is None:
        ws = workspace(p, OP_MOBA_PREFILL, dev)
    _dev(ws, "ws", None, dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    with _on(dev):
        _raise(LIB.moba_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                _ptr(sel_idx), _ptr(ws), nbytes, _stream(stream, dev)))
    return out, sel_idx


def nsa_check(stream=None):
    _raise(LIB.nsa_check(_stream(stream)))


def status_of_check(stream=None):
    return LIB.nsa_check(_stream(stream))


def trace_enable(on=True, capacity=4096, only=None):
    """Bracket launches with CUDA events; `only`: a kernel-name prefix to time."""
    _raise(LIB.nsa_trace_set_filter(only.encode() if only else None))
    _raise(LIB.nsa_trace_enable(1 if on else 0, capacity))


def trace_records():
    """([(kernel name, device ms)] of the timed launches, count of all launches)
    since trace_enable."""
    out = []
    n = LIB.nsa_trace_count()
    for i in range(LIB.nsa_trace_timed()):
        name, ms = ctypes.c_char_p(), ctypes.c_float()
        if LIB.nsa_trace_get(i, ctypes.byref(name), ctypes.byref(ms)) != NSA_OK:
            break
        out.append((name.value.decode(), ms.value))
    return out, n
