"""Python binding of libmoba (C ABI in include/moba.h): argument marshalling only.

Every step of the MoBA prefill forward runs in libmoba's CUDA kernels; this
module only passes torch tensors' device pointers, sizes and the current
stream through ctypes.  There is no fallback: if libmoba.so is missing or no
CUDA device is present the calls raise.

    import block_sparse_long_07_b200 as moba
    o, lse = moba.forward(q, k, v, block_size=4096, top_k=12)          # [b,N,H,d]
    o, lse = moba.forward_varlen(q, k, v, cu_seqlens, block_size=512, top_k=8)
    o, lse = moba.full_causal(q, k, v)
    sel = moba.gate(q, k, block_size=..., top_k=...)
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoba.so")

MOBA_OK = 0
_STATUS = {0: "MOBA_OK", 1: "MOBA_ERR_INVALID_ARG", 2: "MOBA_ERR_UNSUPPORTED",
           3: "MOBA_ERR_WORKSPACE", 4: "MOBA_ERR_CUDA", 5: "MOBA_ERR_TIMEOUT",
           6: "MOBA_ERR_DEVICE_CHECK"}

EXPORTS = ("moba_workspace_size", "moba_workspace_size_varlen", "moba_gate", "moba_gate_varlen",
           "moba_gate_noalloc", "moba_gate_noalloc_status",
           "moba_forward", "moba_forward_varlen", "moba_full_causal_workspace_size",
           "moba_full_causal", "moba_full_causal_varlen", "moba_last_device_status",
           "moba_status_string", "moba_version", "moba_last_error_string", "moba_profile_enable", "moba_profile_reset",
           "moba_profile_read", "moba_selftest_wait_timeout", "moba_decode_workspace_size",
           "moba_kbar_cache_size", "moba_kbar_cache_update", "moba_decode",
           "moba_static_selection", "moba_gate_minmax", "moba_forward_selected",
           "moba_forward_minmax", "moba_backward_workspace_size", "moba_backward",
           "moba_forward_host_buffer_size", "moba_forward_host",
           "moba_static_selection_varlen", "moba_gate_minmax_varlen",
           "moba_forward_selected_varlen", "moba_forward_minmax_varlen",
           "moba_backward_workspace_size_varlen", "moba_backward_varlen",
           "moba_forward_host_buffer_size_varlen", "moba_forward_host_varlen")

ROUTE_WINDOW, ROUTE_SINK = 0, 1


class MobaError(RuntimeError):
    def __init__(self, code, what, detail=""):
        self.code = code
        msg = "%s failed: %s" % (what, _STATUS.get(code, str(code)))
        super().__init__(msg + (" (%s)" % detail if detail else ""))


class MobaParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("seqlen", ctypes.c_int),
                ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int),
                ("top_k", ctypes.c_int), ("softmax_scale", ctypes.c_float)]


class MobaDecodeParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("cache_len", ctypes.c_int),
                ("num_q_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int),
                ("top_k", ctypes.c_int), ("softmax_scale", ctypes.c_float)]


class KernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 24), ("launches", ctypes.c_int),
                ("total_ms", ctypes.c_double)]


_lib = None


def load_library(path=None):
    """Load libmoba.so (raises OSError if it is missing: no fallback exists)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError("libmoba.so not built at %s (run python -m block_sparse_long_07_b200.build)" % p)
    lib = ctypes.CDLL(p)
    vp, sz, i32, i64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_int64
    pp = ctypes.POINTER(MobaParams)
    lib.moba_workspace_size.restype = sz
    lib.moba_workspace_size.argtypes = [pp, i32]
    lib.moba_workspace_size_varlen.restype = sz
    lib.moba_workspace_size_varlen.argtypes = [pp, i64, i32, i32]
    lib.moba_gate.restype = i32
    lib.moba_gate.argtypes = [vp, vp, vp, pp, vp, sz, vp]
    lib.moba_gate_varlen.restype = i32
    lib.moba_gate_varlen.argtypes = [vp, vp, vp, i32, i64, vp, pp, vp, sz, vp]
    lib.moba_gate_noalloc.restype = i32
    lib.moba_gate_noalloc.argtypes = [vp, vp, vp, pp, vp]
    lib.moba_gate_noalloc_status.restype = i32
    lib.moba_gate_noalloc_status.argtypes = [vp]
    lib.moba_forward.restype = i32
    lib.moba_forward.argtypes = [vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_forward_varlen.restype = i32
    lib.moba_forward_varlen.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_full_causal_workspace_size.restype = sz
    lib.moba_full_causal_workspace_size.argtypes = [i64, i32]
    lib.moba_full_causal.restype = i32
    lib.moba_full_causal.argtypes = [vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_full_causal_varlen.restype = i32
    lib.moba_full_causal_varlen.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, pp, vp, sz, vp]
    lib.moba_last_device_status.restype = i32
    lib.moba_last_device_status.argtypes = [vp, vp]
    lib.moba_status_string.restype = ctypes.c_char_p
    lib.moba_status_string.argtypes = [i32]
    lib.moba_version.restype = i32
    lib.moba_version.argtypes = []
    lib.moba_last_error_string.restype = ctypes.c_char_p
    lib.moba_last_error_string.argtypes = []
    lib.moba_profile_enable.restype = None
    lib.moba_profile_enable.argtypes = [i32]
    lib.moba_profile_reset.restype = None
    lib.moba_profile_reset.argtypes = []
    lib.moba_selftest_wait_timeout.restype = i32
    lib.moba_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_longlong, vp]
    lib.moba_profile_read.restype = i32
    lib.moba_profile_read.argtypes = [ctypes.POINTER(KernelTime), i32]
    lib.moba_static_selection.restype = i32
    lib.moba_static_selection.argtypes = [vp, i32, pp, vp]
    lib.moba_gate_minmax.restype = i32
    lib.moba_gate_minmax.argtypes = [vp, vp, vp, pp, vp, sz, vp]
    lib.moba_forward_selected.restype = i32
    lib.moba_forward_selected.argtypes = [vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_forward_minmax.restype = i32
    lib.moba_forward_minmax.argtypes = [vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_forward_host_buffer_size.restype = sz
    lib.moba_forward_host_buffer_size.argtypes = [pp, i32]
    lib.moba_forward_host.restype = i32
    lib.moba_forward_host.argtypes = [vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_backward_workspace_size.restype = sz
    lib.moba_backward_workspace_size.argtypes = [pp, i32]
    lib.moba_backward.restype = i32
    lib.moba_backward.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, pp, vp, sz, vp]
    lib.moba_static_selection_varlen.restype = i32
    lib.moba_static_selection_varlen.argtypes = [vp, i32, vp, i32, i64, pp, vp]
    lib.moba_gate_minmax_varlen.restype = i32
    lib.moba_gate_minmax_varlen.argtypes = [vp, vp, vp, i32, i64, vp, pp, vp, sz, vp]
    lib.moba_forward_selected_varlen.restype = i32
    lib.moba_forward_selected_varlen.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, vp, pp, vp,
                                                 sz, vp]
    lib.moba_forward_minmax_varlen.restype = i32
    lib.moba_forward_minmax_varlen.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, vp, pp, vp,
                                               sz, vp]
    lib.moba_backward_workspace_size_varlen.restype = sz
    lib.moba_backward_workspace_size_varlen.argtypes = [pp, i64, i32, i32]
    lib.moba_backward_varlen.restype = i32
    lib.moba_backward_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp,
                                         pp, vp, sz, vp]
    lib.moba_forward_host_buffer_size_varlen.restype = sz
    lib.moba_forward_host_buffer_size_varlen.argtypes = [pp, i64, i32, i32]
    lib.moba_forward_host_varlen.restype = i32
    lib.moba_forward_host_varlen.argtypes = [vp, vp, vp, vp, i32, i64, vp, vp, vp, pp, vp, sz,
                                             vp]
    dp = ctypes.POINTER(MobaDecodeParams)
    lib.moba_decode_workspace_size.restype = sz
    lib.moba_decode_workspace_size.argtypes = [dp]
    lib.moba_kbar_cache_size.restype = sz
    lib.moba_kbar_cache_size.argtypes = [dp]
    lib.moba_kbar_cache_update.restype = i32
    lib.moba_kbar_cache_update.argtypes = [vp, vp, vp, i32, dp, vp, sz, vp]
    lib.moba_decode.restype = i32
    lib.moba_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, dp, vp, sz, vp]
    if path is None:
        _lib = lib
    return lib


def _torch():
    import torch
    return torch


def _check(code, what):
    if code != MOBA_OK:
        detail = ""
        if code == 4:
            detail = load_library().moba_last_error_string().decode()
        raise MobaError(code, what, detail)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr() if t is not None else 0)


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_params(batch, seqlen, Hq, Hkv, d, block_size=128, top_k=1, softmax_scale=0.0):
    return MobaParams(int(batch), int(seqlen), int(Hq), int(Hkv), int(d), int(block_size),
                      int(top_k), float(softmax_scale))


def _require_cuda_bf16(*ts):
    torch = _torch()
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()):
            raise ValueError("expected contiguous bf16 CUDA tensors")


def workspace_size(params, heads_per_pass=0):
    return int(load_library().moba_workspace_size(ctypes.byref(params), int(heads_per_pass)))


def workspace_size_varlen(params, total_tokens, num_seqs, heads_per_pass=0):
    return int(load_library().moba_workspace_size_varlen(ctypes.byref(params), int(total_tokens),
                                                         int(num_seqs), int(heads_per_pass)))


def full_causal_workspace_size(total_tokens, num_seqs):
    return int(load_library().moba_full_causal_workspace_size(int(total_tokens), int(num_seqs)))


DEFAULT_WS_BUDGET = 32 << 30  # bytes a forward call may take for its workspace by default


def pick_heads_per_pass(size_fn, num_kv_heads, budget=DEFAULT_WS_BUDGET):
    """Largest number of kv heads per pass whose workspace fits `budget` (at least 1)."""
    for hp in range(num_kv_heads, 0, -1):
        if size_fn(hp) <= budget:
            return hp
    return 1


def alloc_workspace(nbytes, device=None):
    """A workspace of nbytes whose status word (first 256 bytes) starts at zero,
    as the library requires of a workspace's first use."""
    torch = _torch()
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")
    ws[:256].zero_()
    return ws


def profile_enable(on=True):
    """Bracket every library kernel launch with CUDA events (see moba.h)."""
    lib = load_library()
    lib.moba_profile_reset()
    lib.moba_profile_enable(1 if on else 0)


def profile_read():
    """{kernel class: (launches, total device ms)} since profile_enable."""
    arr = (KernelTime * 32)()
    n = load_library().moba_profile_read(arr, 32)
    return {arr[i].name.decode(): (arr[i].launches, arr[i].total_ms) for i in range(n)}


def last_device_status(ws, stream=None):
    """Synchronises and returns the device status latched in `ws` (0 = ok)."""
    return int(load_library().moba_last_device_status(_ptr(ws), _stream(stream)))


def gate(q, k, block_size, top_k, softmax_scale=0.0, ws=None, sel=None, stream=None):
    """Selection sel [b, Hq, N, top_k] int32 for q [b,N,Hq,d], k [b,N,Hkv,d]."""
    torch = _torch()
    _require_cuda_bf16(q, k)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(b, N, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if sel is None:
        sel = torch.empty(b, Hq, N, top_k, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = alloc_workspace(workspace_size(p, 1), q.device)
    _check(load_library().moba_gate(_ptr(q), _ptr(k), _ptr(sel), ctypes.byref(p), _ptr(ws),
                                    ws.numel(), _stream(stream)), "moba_gate")
    return sel


def gate_varlen(q, k, cu_seqlens, block_size, top_k, softmax_scale=0.0, ws=None, sel=None,
                stream=None):
    """Selection sel [Hq, T, top_k] for packed q [T,Hq,d], k [T,Hkv,d]."""
    torch = _torch()
    _require_cuda_bf16(q, k)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if sel is None:
        sel = torch.empty(Hq, T, top_k, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = alloc_workspace(workspace_size_varlen(p, T, nseq, 1), q.device)
    _check(load_library().moba_gate_varlen(_ptr(q), _ptr(k), _ptr(cu_seqlens), nseq, T,
                                           _ptr(sel), ctypes.byref(p), _ptr(ws), ws.numel(),
                                           _stream(stream)), "moba_gate_varlen")
    return sel


def forward(q, k, v, block_size, top_k, softmax_scale=0.0, ws=None, out=None, lse=None,
            sel_out=None, stream=None):
    """MoBA prefill forward for q [b,N,Hq,d], k/v [b,N,Hkv,d]: (o, lse)."""
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(b, N, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(b, Hq, N, dtype=torch.float32, device=q.device)
    if ws is None:
        hp = pick_heads_per_pass(lambda n: workspace_size(p, n), Hkv)
        ws = alloc_workspace(workspace_size(p, hp), q.device)
    _check(load_library().moba_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                       _ptr(sel_out), ctypes.byref(p), _ptr(ws), ws.numel(),
                                       _stream(stream)), "moba_forward")
    return out, lse


def forward_varlen(q, k, v, cu_seqlens, block_size, top_k, softmax_scale=0.0, ws=None,
                   out=None, lse=None, sel_out=None, stream=None):
    """MoBA prefill forward on packed sequences q [T,Hq,d], k/v [T,Hkv,d]: (o, lse [Hq,T])."""
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, T, dtype=torch.float32, device=q.device)
    if ws is None:
        hp = pick_heads_per_pass(lambda n: workspace_size_varlen(p, T, nseq, n), Hkv)
        ws = alloc_workspace(workspace_size_varlen(p, T, nseq, hp), q.device)
    _check(load_library().moba_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq,
                                              T, _ptr(out), _ptr(lse), _ptr(sel_out),
                                              ctypes.byref(p), _ptr(ws), ws.numel(),
                                              _stream(stream)), "moba_forward_varlen")
    return out, lse


def full_causal(q, k, v, softmax_scale=0.0, ws=None, out=None, lse=None, stream=None):
    """Dense causal attention (the k = n comparator) for q [b,N,Hq,d]: (o, lse)."""
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(b, N, Hq, Hkv, d, 128, 1, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(b, Hq, N, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(full_causal_workspace_size(b * N, b), q.device)
    _check(load_library().moba_full_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                           ctypes.byref(p), _ptr(ws), ws.numel(),
                                           _stream(stream)), "moba_full_causal")
    return out, lse


def full_causal_varlen(q, k, v, cu_seqlens, softmax_scale=0.0, ws=None, out=None, lse=None,
                       stream=None):
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hkv, d, 128, 1, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, T, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(full_causal_workspace_size(T, nseq), q.device)
    _check(load_library().moba_full_causal_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                                  nseq, T, _ptr(out), _ptr(lse), ctypes.byref(p),
                                                  _ptr(ws), ws.numel(), _stream(stream)),
           "moba_full_causal_varlen")
    return out, lse


# ---------------------------------------------------------------- decode
def make_decode_params(batch, cache_len, Hq, Hkv, d, block_size, top_k, softmax_scale=0.0):
    return MobaDecodeParams(int(batch), int(cache_len), int(Hq), int(Hkv), int(d),
                            int(block_size), int(top_k), float(softmax_scale))


def decode_workspace_size(params):
    return int(load_library().moba_decode_workspace_size(ctypes.byref(params)))


def kbar_cache_size(params):
    return int(load_library().moba_kbar_cache_size(ctypes.byref(params)))


def _decode_params(k_cache, q_heads, block_size, top_k, softmax_scale):
    b, cap, Hkv, d = k_cache.shape
    return make_decode_params(b, cap, q_heads, Hkv, d, block_size, top_k, softmax_scale)


def alloc_kbar_cache(k_cache, block_size):
    """Zeroed fp32 block-mean cache [b, Hkv, ceil(cap / B), d] for k_cache [b, cap, Hkv, d]."""
    torch = _torch()
    b, cap, Hkv, d = k_cache.shape
    return torch.zeros(b, Hkv, (cap + block_size - 1) // block_size, d, dtype=torch.float32,
                       device=k_cache.device)


def kbar_cache_update(k_cache, seqlens, kbar, block_size, only_last=False, ws=None, stream=None):
    """Block means of the complete cache blocks (all, or the one the newest token completed)."""
    _require_cuda_bf16(k_cache)
    p = _decode_params(k_cache, k_cache.shape[2], block_size, 1, 0.0)
    if ws is None:
        ws = alloc_workspace(decode_workspace_size(p), k_cache.device)
    _check(load_library().moba_kbar_cache_update(_ptr(k_cache), _ptr(seqlens), _ptr(kbar),
                                                 1 if only_last else 0, ctypes.byref(p),
                                                 _ptr(ws), ws.numel(), _stream(stream)),
           "moba_kbar_cache_update")
    return kbar


def decode(q, k_cache, v_cache, seqlens, kbar, block_size, top_k, softmax_scale=0.0, ws=None,
           out=None, lse=None, sel_out=None, stream=None):
    """One decode step for q [b, Hq, d] against k/v caches [b, cap, Hkv, d]: (o, lse [b, Hq])."""
    torch = _torch()
    _require_cuda_bf16(q, k_cache, v_cache)
    b, Hq, d = q.shape
    p = _decode_params(k_cache, Hq, block_size, top_k, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(b, Hq, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = alloc_workspace(decode_workspace_size(p), q.device)
    _check(load_library().moba_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seqlens),
                                      _ptr(kbar), _ptr(out), _ptr(lse), _ptr(sel_out),
                                      ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)),
           "moba_decode")
    return out, lse


# ---------------------------------------------------------------- routing variants
def static_selection(batch, seqlen, Hq, block_size, top_k, mode, device=None, sel=None,
                     stream=None):
    """Window (mode ROUTE_WINDOW) or sink (ROUTE_SINK) selection
    sel [batch, Hq, seqlen, top_k]."""
    torch = _torch()
    p = make_params(batch, seqlen, Hq, Hq, 128, block_size, top_k)
    if sel is None:
        sel = torch.empty(batch, Hq, seqlen, top_k, dtype=torch.int32, device=device or "cuda")
    _check(load_library().moba_static_selection(_ptr(sel), int(mode), ctypes.byref(p),
                                                _stream(stream)), "moba_static_selection")
    return sel


def gate_minmax(q, k, block_size, top_k, softmax_scale=0.0, ws=None, sel=None, stream=None):
    """Min/max-pooled gate: sel [b, Hq, N, top_k] for q [b,N,Hq,d], k [b,N,Hkv,d]."""
    torch = _torch()
    _require_cuda_bf16(q, k)
    b, N, Hq, d = q.shape
    p = make_params(b, N, Hq, k.shape[2], d, block_size, top_k, softmax_scale)
    if sel is None:
        sel = torch.empty(b, Hq, N, top_k, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = alloc_workspace(workspace_size(p, 1), q.device)
    _check(load_library().moba_gate_minmax(_ptr(q), _ptr(k), _ptr(sel), ctypes.byref(p),
                                           _ptr(ws), ws.numel(), _stream(stream)),
           "moba_gate_minmax")
    return sel


def _forward_common(q, k, v, block_size, top_k, softmax_scale, ws, out, lse):
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(b, N, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(b, Hq, N, dtype=torch.float32, device=q.device)
    if ws is None:
        hp = pick_heads_per_pass(lambda n: workspace_size(p, n), Hkv)
        ws = alloc_workspace(workspace_size(p, hp), q.device)
    return p, out, lse, ws


def forward_selected(q, k, v, sel, block_size, top_k, softmax_scale=0.0, ws=None, out=None,
                     lse=None, stream=None):
    """MoBA forward over a given selection sel [b, Hq, N, top_k] (gate format)."""
    p, out, lse, ws = _forward_common(q, k, v, block_size, top_k, softmax_scale, ws, out, lse)
    _check(load_library().moba_forward_selected(_ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                                _ptr(lse), _ptr(sel), ctypes.byref(p),
                                                _ptr(ws), ws.numel(), _stream(stream)),
           "moba_forward_selected")
    return out, lse


def forward_minmax(q, k, v, block_size, top_k, softmax_scale=0.0, ws=None, out=None, lse=None,
                   sel_out=None, stream=None):
    """MoBA forward with the min/max-pooled gate: (o, lse)."""
    p, out, lse, ws = _forward_common(q, k, v, block_size, top_k, softmax_scale, ws, out, lse)
    _check(load_library().moba_forward_minmax(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                              _ptr(sel_out), ctypes.byref(p), _ptr(ws),
                                              ws.numel(), _stream(stream)),
           "moba_forward_minmax")
    return out, lse


def static_selection_varlen(cu_seqlens, total_tokens, Hq, block_size, top_k, mode, sel=None,
                            stream=None):
    """Window / sink selection sel [Hq, T, top_k] for packed sequences."""
    torch = _torch()
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hq, 128, block_size, top_k)
    if sel is None:
        sel = torch.empty(Hq, total_tokens, top_k, dtype=torch.int32, device=cu_seqlens.device)
    _check(load_library().moba_static_selection_varlen(_ptr(sel), int(mode), _ptr(cu_seqlens),
                                                       nseq, int(total_tokens), ctypes.byref(p),
                                                       _stream(stream)),
           "moba_static_selection_varlen")
    return sel


def _varlen_common(q, k, v, cu_seqlens, block_size, top_k, softmax_scale, ws, out, lse):
    torch = _torch()
    _require_cuda_bf16(q, k, v)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hkv, d, block_size, top_k, softmax_scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, T, dtype=torch.float32, device=q.device)
    if ws is None:
        hp = pick_heads_per_pass(lambda n: workspace_size_varlen(p, T, nseq, n), Hkv)
        ws = alloc_workspace(workspace_size_varlen(p, T, nseq, hp), q.device)
    return p, nseq, T, out, lse, ws


def gate_minmax_varlen(q, k, cu_seqlens, block_size, top_k, softmax_scale=0.0, ws=None,
                       sel=None, stream=None):
    """Min/max-pooled gate on packed sequences: sel [Hq, T, top_k]."""
    torch = _torch()
    _require_cuda_bf16(q, k)
    T, Hq, d = q.shape
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, k.shape[1], d, block_size, top_k, softmax_scale)
    if sel is None:
        sel = torch.empty(Hq, T, top_k, dtype=torch.int32, device=q.device)
    if ws is None:
        ws = alloc_workspace(workspace_size_varlen(p, T, nseq, 1), q.device)
    _check(load_library().moba_gate_minmax_varlen(_ptr(q), _ptr(k), _ptr(cu_seqlens), nseq, T,
                                                  _ptr(sel), ctypes.byref(p), _ptr(ws),
                                                  ws.numel(), _stream(stream)),
           "moba_gate_minmax_varlen")
    return sel


def forward_selected_varlen(q, k, v, cu_seqlens, sel, block_size, top_k, softmax_scale=0.0,
                            ws=None, out=None, lse=None, stream=None):
    """Forward over a given selection sel [Hq, T, top_k] on packed sequences: (o, lse)."""
    p, nseq, T, out, lse, ws = _varlen_common(q, k, v, cu_seqlens, block_size, top_k,
                                              softmax_scale, ws, out, lse)
    _check(load_library().moba_forward_selected_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, _ptr(out), _ptr(lse), _ptr(sel),
        ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)), "moba_forward_selected_varlen")
    return out, lse


def forward_minmax_varlen(q, k, v, cu_seqlens, block_size, top_k, softmax_scale=0.0, ws=None,
                          out=None, lse=None, sel_out=None, stream=None):
    """Min/max-gate forward on packed sequences: (o, lse [Hq, T])."""
    p, nseq, T, out, lse, ws = _varlen_common(q, k, v, cu_seqlens, block_size, top_k,
                                              softmax_scale, ws, out, lse)
    _check(load_library().moba_forward_minmax_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, _ptr(out), _ptr(lse),
        _ptr(sel_out), ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)),
        "moba_forward_minmax_varlen")
    return out, lse


# ---------------------------------------------------------------- backward
def backward_workspace_size_varlen(params, total_tokens, num_seqs, heads_per_pass=0):
    return int(load_library().moba_backward_workspace_size_varlen(
        ctypes.byref(params), int(total_tokens), int(num_seqs), int(heads_per_pass)))


def backward_varlen(q, k, v, o, lse, dO, sel, cu_seqlens, block_size, top_k, softmax_scale=0.0,
                    ws=None, dq=None, dk=None, dv=None, stream=None):
    """Gradients (dq, dk, dv) for packed sequences: q, o, dO [T, Hq, d], k, v
    [T, Hkv, d], lse [Hq, T] and sel [Hq, T, top_k] as forward_varlen wrote them."""
    torch = _torch()
    _require_cuda_bf16(q, k, v, o, dO)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, Hkv, d, block_size, top_k, softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        hp = pick_heads_per_pass(lambda n: backward_workspace_size_varlen(p, T, nseq, n), Hkv)
        ws = alloc_workspace(backward_workspace_size_varlen(p, T, nseq, hp), q.device)
    _check(load_library().moba_backward_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO), _ptr(sel), _ptr(cu_seqlens),
        nseq, T, _ptr(dq), _ptr(dk), _ptr(dv), ctypes.byref(p), _ptr(ws), ws.numel(),
        _stream(stream)), "moba_backward_varlen")
    return dq, dk, dv


# ---------------------------------------------------------------- backward
def backward_workspace_size(params, heads_per_pass=0):
    return int(load_library().moba_backward_workspace_size(ctypes.byref(params),
                                                           int(heads_per_pass)))


def backward(q, k, v, o, lse, dO, sel, block_size, top_k, softmax_scale=0.0, ws=None,
             dq=None, dk=None, dv=None, stream=None):
    """Gradients (dq, dk, dv) of the forward's attention over its selection
    sel [b, Hq, N, top_k], for the output gradient dO [b, N, Hq, d]."""
    torch = _torch()
    _require_cuda_bf16(q, k, v, o, dO)
    b, N, Hq, d = q.shape
    Hkv = k.shape[2]
    p = make_params(b, N, Hq, Hkv, d, block_size, top_k, softmax_scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if ws is None:
        hp = pick_heads_per_pass(lambda n: backward_workspace_size(p, n), Hkv)
        ws = alloc_workspace(backward_workspace_size(p, hp), q.device)
    _check(load_library().moba_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dO),
                                        _ptr(sel), _ptr(dq), _ptr(dk), _ptr(dv),
                                        ctypes.byref(p), _ptr(ws), ws.numel(), _stream(stream)),
           "moba_backward")
    return dq, dk, dv


# ---------------------------------------------------------------- host-buffer forward
def forward_host_buffer_size(params, heads_per_pass=0):
    return int(load_library().moba_forward_host_buffer_size(ctypes.byref(params),
                                                            int(heads_per_pass)))


def forward_host(q, k, v, block_size, top_k, out, lse, dev_buf=None, heads_per_pass=0,
                 softmax_scale=0.0, sel_out=None, stream=None):
    """MoBA forward on host (preferably pinned) tensors q [b,N,Hq,d], k/v
    [b,N,Hkv,d]; writes the host tensors out [b,N,Hq,d] and lse [b,Hq,N].
    The copies run inside the call, overlapped with the work of other kv-head
    groups; synchronise the stream before reading out."""
    torch = _torch()
    for t in (q, k, v, out):
        if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
            raise ValueError("expected contiguous bf16 host tensors")
    b, N, Hq, d = q.shape
    p = make_params(b, N, Hq, k.shape[2], d, block_size, top_k, softmax_scale)
    if dev_buf is None:
        dev_buf = alloc_workspace(forward_host_buffer_size(p, heads_per_pass))
    _check(load_library().moba_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse),
                                            _ptr(sel_out), ctypes.byref(p), _ptr(dev_buf),
                                            dev_buf.numel(), _stream(stream)),
           "moba_forward_host")
    return out, lse


def forward_host_buffer_size_varlen(params, total_tokens, num_seqs, heads_per_pass=0):
    return int(load_library().moba_forward_host_buffer_size_varlen(
        ctypes.byref(params), int(total_tokens), int(num_seqs), int(heads_per_pass)))


def forward_host_varlen(q, k, v, cu_seqlens, block_size, top_k, out, lse, dev_buf=None,
                        heads_per_pass=0, softmax_scale=0.0, sel_out=None, stream=None):
    """forward_host for packed sequences: host tensors q [T,Hq,d], k/v [T,Hkv,d],
    cu_seqlens (int32, host), out [T,Hq,d], lse [Hq,T] (and sel_out [Hq,T,k])."""
    torch = _torch()
    for t in (q, k, v, out, cu_seqlens):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("expected contiguous host tensors")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    T, Hq, d = q.shape
    nseq = cu_seqlens.numel() - 1
    p = make_params(1, 0, Hq, k.shape[1], d, block_size, top_k, softmax_scale)
    if dev_buf is None:
        dev_buf = alloc_workspace(forward_host_buffer_size_varlen(p, T, nseq, heads_per_pass))
    _check(load_library().moba_forward_host_varlen(
        _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, _ptr(out), _ptr(lse),
        _ptr(sel_out), ctypes.byref(p), _ptr(dev_buf), dev_buf.numel(), _stream(stream)),
        "moba_forward_host_varlen")
    return out, lse
