"""Sep-Attention and the four-block SepCache on B200 (sm_100a).

Thin Python binding of the C ABI in include/sepattn.h (libsepattn.so, built
in-tree by `python streaming_kv_cache_sep_b200/build.py`).  It only
marshals arguments: every step of the path runs in the CUDA library.
PyTorch supplies device memory and the current CUDA stream.  There is no
CPU fallback: if the library is missing, importing this package fails.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsepattn.so")

SEP_OK = 0
SEP_F32 = 0
SEP_BF16 = 1

# every symbol include/sepattn.h declares
ABI_SYMBOLS = (
    "sep_strerror", "sep_version", "sep_flags_from_ids", "sep_build_index",
    "sep_build_index_from_ids", "sep_count_pairs",
    "sep_attn_prefill_workspace", "sep_attn_prefill", "sepcache_bytes", "sepcache_carve",
    "sepcache_init", "sepcache_append", "sepcache_compact", "sep_attn_decode_workspace",
    "sep_attn_decode", "sepcache_status", "sep_device_status", "sep_attn_decode_noalloc",
    "sep_attn_decode_step", "sepcache_ingest", "sepcache_set_rope",
    "sep_attn_decode_masked_workspace", "sep_attn_decode_masked",
    "sep_attn_backward_workspace", "sep_attn_backward",
)


class SepError(RuntimeError):
    def __init__(self, fn: str, status: int):
        msg = _lib.sep_strerror(status).decode() if _lib is not None else str(status)
        super().__init__("%s failed: %s (%d)" % (fn, msg, status))
        self.status = status


class SepCacheCfg(ctypes.Structure):
    _fields_ = [("a", ctypes.c_int32), ("s", ctypes.c_int32), ("past", ctypes.c_int32),
                ("w", ctypes.c_int32), ("mode", ctypes.c_int32)]


# variant bits of SepCacheCfg.mode (the KV manager's switches)
NO_ACCUMULATION = 1   # a flush keeps only the flushed past window's separators
UNBOUNDED_SEPS = 2    # separators are never evicted; more than s sets CACHE_ESEPS
TOTAL_TRIGGER = 4     # flush when the whole cache exceeds a+s+past+w
CACHE_EOVERFLOW, CACHE_ESTATE, CACHE_ESEPS = 1, 2, 4  # cache status bits


class _SepCacheC(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("pos", ctypes.c_void_p),
                ("flag", ctypes.c_void_p), ("counts", ctypes.c_void_p), ("plan", ctypes.c_void_p),
                ("step", ctypes.c_void_p), ("status", ctypes.c_void_p), ("rope", ctypes.c_void_p), ("layers", ctypes.c_int32),
                ("B", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("cap", ctypes.c_int32), ("cfg", SepCacheCfg),
                ("rope_theta", ctypes.c_float), ("rope_rows", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libsepattn.so is not built; run `python streaming_kv_cache_sep_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
    L.sep_strerror.argtypes = [i32]
    L.sep_strerror.restype = ctypes.c_char_p
    L.sep_version.argtypes = []
    L.sep_flags_from_ids.argtypes = [P, i64, P, i32, P, P]
    L.sep_build_index.argtypes = [P, i32, i32, P, P, P, P]
    L.sep_build_index_from_ids.argtypes = [P, i32, i32, P, i32, P, P, P, P, P]
    L.sep_count_pairs.argtypes = [P, i32, i32, i32, i32, P, P]
    L.sep_attn_prefill_workspace.argtypes = [i32, i32, i32, i32, i32, i32]
    L.sep_attn_prefill_workspace.restype = sz
    L.sep_attn_prefill.argtypes = [P, P, P, i32, P, P, P, i32, i32, i32, i32, i32, i32, i32, f32,
                                   P, P, P, sz, P]
    L.sepcache_bytes.argtypes = [SepCacheCfg, i32, i32, i32, i32, i32]
    L.sepcache_bytes.restype = sz
    L.sepcache_carve.argtypes = [ctypes.POINTER(_SepCacheC), P, sz, SepCacheCfg, i32, i32, i32,
                                 i32, i32]
    L.sepcache_init.argtypes = [ctypes.POINTER(_SepCacheC), P]
    L.sepcache_append.argtypes = [ctypes.POINTER(_SepCacheC), i32, P, P, P, P]
    L.sepcache_compact.argtypes = [ctypes.POINTER(_SepCacheC), i32, P]
    L.sepcache_ingest.argtypes = [ctypes.POINTER(_SepCacheC), i32, P, P, P, P, P, i32, P]
    L.sepcache_set_rope.argtypes = [ctypes.POINTER(_SepCacheC), f32, P]
    L.sep_attn_backward_workspace.argtypes = [i32, i32, i32, i32, i32]
    L.sep_attn_backward_workspace.restype = sz
    L.sep_attn_backward.argtypes = [P, P, P, P, P, P, i32, P, P, P, i32, i32, i32, i32, i32, i32,
                                    i32, f32, P, P, P, P, sz, P]
    L.sep_attn_decode_masked_workspace.argtypes = [i32, i32, i32, i32, i32]
    L.sep_attn_decode_masked_workspace.restype = sz
    L.sep_attn_decode_masked.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32, i32, i32, i32,
                                         i32, f32, P, P, P, sz, P]
    L.sep_attn_decode_workspace.argtypes = [ctypes.POINTER(_SepCacheC), i32]
    L.sep_attn_decode_workspace.restype = sz
    L.sep_attn_decode.argtypes = [ctypes.POINTER(_SepCacheC), i32, P, i32, f32, P, P, P, sz, P]
    L.sep_attn_decode_step.argtypes = [ctypes.POINTER(_SepCacheC), i32, P, P, P, P, i32, f32, P, P,
                                       P, sz, P]
    L.sep_attn_decode_noalloc.argtypes = [ctypes.POINTER(_SepCacheC), i32, P, i32, f32, P, P, P]
    L.sepcache_status.argtypes = [ctypes.POINTER(_SepCacheC), ctypes.POINTER(ctypes.c_int32), P]
    L.sep_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), i32, P]
    for name in ABI_SYMBOLS:
        fn = getattr(L, name)
        if name not in ("sep_strerror", "sep_attn_prefill_workspace", "sepcache_bytes",
                        "sep_attn_decode_workspace", "sep_attn_decode_masked_workspace",
                        "sep_attn_backward_workspace"):
            fn.restype = ctypes.c_int
    return L


_lib = _load()


def lib():
    """The loaded ctypes handle of libsepattn.so."""
    return _lib


def _check(fn: str, rc: int):
    if rc != SEP_OK:
        raise SepError(fn, rc)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SEP_BF16
    if t.dtype == torch.float32:
        return SEP_F32
    raise TypeError("unsupported dtype %s" % t.dtype)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("expected contiguous CUDA tensors")
    dev = next((t.device for t in ts if t is not None), None)
    for t in ts:
        if t is not None and t.device != dev:
            raise ValueError("expected every tensor on %s, got one on %s" % (dev, t.device))


def _expect(t, name, dtype, shape):
    """The C calls take bare pointers and trust the sizes they are given, so
    the binding checks each tensor's dtype and shape against the layout the
    call documents (None: an optional tensor that was not passed)."""
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError("%s: expected %s, got %s" % (name, dtype, t.dtype))
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _dims(t, name, n):
    if t.dim() != n:
        raise ValueError("%s: expected %d dimensions, got shape %s" % (name, n, tuple(t.shape)))
    return tuple(t.shape)


def _nbytes(t) -> int:
    return 0 if t is None else t.numel() * t.element_size()


# ------------------------------------------------------------------ index


def flags_from_ids(ids: torch.Tensor, sep_ids, stream=None) -> torch.Tensor:
    """uint8 flags: 1 where ids is one of sep_ids (a host list, <= 32 ids)."""
    _expect(ids, "ids", torch.int32, ids.shape)
    _need_cuda(ids)
    out = torch.empty(ids.shape, dtype=torch.uint8, device=ids.device)
    arr = (ctypes.c_int32 * len(sep_ids))(*[int(x) for x in sep_ids])
    _check("sep_flags_from_ids", _lib.sep_flags_from_ids(
        _ptr(ids), ids.numel(), ctypes.cast(arr, ctypes.c_void_p), len(sep_ids), _ptr(out),
        _stream(stream)))
    return out


def build_index(is_sep: torch.Tensor, out=None, stream=None):
    """(prefix [B,S+1], idx [B,S] (-1 padded), count [B]) int32 on the device."""
    B, S = _dims(is_sep, "is_sep", 2)
    _expect(is_sep, "is_sep", torch.uint8, (B, S))
    if out is None:
        _need_cuda(is_sep)
        dev = is_sep.device
        out = (torch.empty((B, S + 1), dtype=torch.int32, device=dev),
               torch.empty((B, S), dtype=torch.int32, device=dev),
               torch.empty((B,), dtype=torch.int32, device=dev))
    prefix, idx, count = out
    _expect(prefix, "prefix", torch.int32, (B, S + 1))
    _expect(idx, "idx", torch.int32, (B, S))
    _expect(count, "count", torch.int32, (B,))
    _need_cuda(is_sep, prefix, idx, count)
    _check("sep_build_index", _lib.sep_build_index(_ptr(is_sep), B, S, _ptr(prefix), _ptr(idx),
                                                   _ptr(count), _stream(stream)))
    return prefix, idx, count


def build_index_from_ids(ids: torch.Tensor, sep_ids, out=None, stream=None):
    """flags_from_ids then build_index in one launch: ids int32 [B,S] ->
    (is_sep uint8 [B,S], prefix [B,S+1], idx [B,S], count [B]) on the device."""
    B, S = _dims(ids, "ids", 2)
    _expect(ids, "ids", torch.int32, (B, S))
    if out is None:
        _need_cuda(ids)
        dev = ids.device
        out = (torch.empty((B, S), dtype=torch.uint8, device=dev),
               torch.empty((B, S + 1), dtype=torch.int32, device=dev),
               torch.empty((B, S), dtype=torch.int32, device=dev),
               torch.empty((B,), dtype=torch.int32, device=dev))
    is_sep, prefix, idx, count = out
    _expect(is_sep, "is_sep", torch.uint8, (B, S))
    _expect(prefix, "prefix", torch.int32, (B, S + 1))
    _expect(idx, "idx", torch.int32, (B, S))
    _expect(count, "count", torch.int32, (B,))
    _need_cuda(ids, is_sep, prefix, idx, count)
    arr = (ctypes.c_int32 * len(sep_ids))(*[int(x) for x in sep_ids])
    _check("sep_build_index_from_ids", _lib.sep_build_index_from_ids(
        _ptr(ids), B, S, ctypes.cast(arr, ctypes.c_void_p), len(sep_ids), _ptr(is_sep),
        _ptr(prefix), _ptr(idx), _ptr(count), _stream(stream)))
    return is_sep, prefix, idx, count


def count_pairs(prefix: torch.Tensor, a: int, n: int, out=None, stream=None) -> torch.Tensor:
    """Kept (query, key) pairs per sequence for one head, int64 [B]."""
    B, S1 = _dims(prefix, "prefix", 2)
    _expect(prefix, "prefix", torch.int32, (B, S1))
    _expect(out, "out", torch.int64, (B,))
    _need_cuda(prefix, out)
    out = out if out is not None else torch.empty((B,), dtype=torch.int64, device=prefix.device)
    _check("sep_count_pairs", _lib.sep_count_pairs(_ptr(prefix), B, S1 - 1, a, n, _ptr(out),
                                                   _stream(stream)))
    return out


# ------------------------------------------------------------------ prefill


def prefill_workspace_bytes(B, Hq, Hkv, S, D, dtype) -> int:
    return int(_lib.sep_attn_prefill_workspace(B, Hq, Hkv, S, D, dtype))


def prefill(q, k, v, is_sep, prefix, idx, a: int, n: int, scale: float = 0.0, out=None,
            lse=None, workspace=None, want_lse: bool = True, stream=None):
    """Sep-Attention over whole sequences.  q [B,Hq,S,D], k/v [B,Hkv,S,D]
    (bf16 -> tcgen05 path, fp32 -> exact FMA path).  Returns (out, lse)."""
    B, Hq, S, D = _dims(q, "q", 4)
    dt = _dtype_code(q)
    Hkv = _dims(k, "k", 4)[1]
    _expect(k, "k", q.dtype, (B, Hkv, S, D))
    _expect(v, "v", q.dtype, (B, Hkv, S, D))
    _expect(is_sep, "is_sep", torch.uint8, (B, S))
    _expect(prefix, "prefix", torch.int32, (B, S + 1))
    _expect(idx, "idx", torch.int32, (B, S))
    _expect(out, "out", q.dtype, (B, Hq, S, D))
    _expect(lse, "lse", torch.float32, (B, Hq, S))
    _need_cuda(q, k, v, is_sep, prefix, idx, out, lse, workspace)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, S), dtype=torch.float32, device=q.device)
    need = prefill_workspace_bytes(B, Hq, Hkv, S, D, dt)
    if workspace is None or _nbytes(workspace) < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check("sep_attn_prefill", _lib.sep_attn_prefill(
        _ptr(q), _ptr(k), _ptr(v), dt, _ptr(is_sep), _ptr(prefix), _ptr(idx), B, Hq, Hkv, S, D,
        a, n, float(scale), _ptr(out), _ptr(lse), _ptr(workspace), _nbytes(workspace),
        _stream(stream)))
    return out, lse


def backward(q, k, v, out, lse, dout, is_sep, prefix, idx, a: int, n: int, scale: float = 0.0,
             dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of sum(out * dout) through Sep-Attention: q/out/dout
    [B,Hq,S,D], k/v [B,Hkv,S,D] bf16, lse [B,Hq,S] from prefill.
    Returns (dq, dk, dv)."""
    B, Hq, S, D = _dims(q, "q", 4)
    dt = _dtype_code(q)
    Hkv = _dims(k, "k", 4)[1]
    _expect(k, "k", q.dtype, (B, Hkv, S, D))
    _expect(v, "v", q.dtype, (B, Hkv, S, D))
    _expect(out, "out", q.dtype, (B, Hq, S, D))
    _expect(lse, "lse", torch.float32, (B, Hq, S))
    _expect(dout, "dout", q.dtype, (B, Hq, S, D))
    _expect(is_sep, "is_sep", torch.uint8, (B, S))
    _expect(prefix, "prefix", torch.int32, (B, S + 1))
    _expect(idx, "idx", torch.int32, (B, S))
    _expect(dq, "dq", q.dtype, (B, Hq, S, D))
    _expect(dk, "dk", q.dtype, (B, Hkv, S, D))
    _expect(dv, "dv", q.dtype, (B, Hkv, S, D))
    _need_cuda(q, k, v, out, lse, dout, is_sep, prefix, idx, dq, dk, dv, workspace)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = int(_lib.sep_attn_backward_workspace(B, Hq, Hkv, S, D))
    if workspace is None or _nbytes(workspace) < need:
        workspace = torch.empty((need,), dtype=torch.uint8, device=q.device)
    _check("sep_attn_backward", _lib.sep_attn_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), dt, _ptr(is_sep),
        _ptr(prefix), _ptr(idx), B, Hq, Hkv, S, D, a, n, float(scale), _ptr(dq), _ptr(dk),
        _ptr(dv), _ptr(workspace), _nbytes(workspace), _stream(stream)))
    return dq, dk, dv


_masked_ws = {}


def decode_masked(q, k, v, prefix, idx, T: int, a: int, n: int, scale: float = 0.0, out=None,
                  lse=None, want_lse: bool = True, workspace=None, stream=None):
    """Mask-based generation over a full history: q [B,Hq,D] (token T-1)
    attends over k/v [B,Hkv,S,D] rows 0..T-1 with the Sep-Attention kept set
    of its row; prefix/idx from build_index of the flags [B,S].
    Returns (out [B,Hq,D], lse [B,Hq])."""
    B, Hq, D = _dims(q, "q", 3)
    dt = _dtype_code(q)
    _, Hkv, S, _ = _dims(k, "k", 4)
    _expect(k, "k", q.dtype, (B, Hkv, S, D))
    _expect(v, "v", q.dtype, (B, Hkv, S, D))
    _expect(prefix, "prefix", torch.int32, (B, S + 1))
    _expect(idx, "idx", torch.int32, (B, S))
    _expect(out, "out", q.dtype, (B, Hq, D))
    _expect(lse, "lse", torch.float32, (B, Hq))
    _need_cuda(q, k, v, prefix, idx, out, lse, workspace)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
    wsb = 0
    if dt == SEP_F32:
        need = int(_lib.sep_attn_decode_masked_workspace(B, Hq, Hkv, S, D))
        if workspace is None:
            key = (q.device, B, Hq, Hkv, S, D)
            workspace = _masked_ws.get(key)
            if workspace is None:
                workspace = torch.zeros((need,), dtype=torch.uint8, device=q.device)
                _masked_ws[key] = workspace
        wsb = _nbytes(workspace)
    _check("sep_attn_decode_masked", _lib.sep_attn_decode_masked(
        _ptr(q), _ptr(k), _ptr(v), dt, _ptr(prefix), _ptr(idx), B, Hq, Hkv, S, int(T), D, a, n,
        float(scale), _ptr(out), _ptr(lse), _ptr(workspace), wsb, _stream(stream)))
    return out, lse


def device_status(clear: bool = True, stream=None) -> int:
    """Synchronise and return the library's device error bits (0 = none)."""
    bits = ctypes.c_int32(0)
    _lib.sep_device_status(ctypes.byref(bits), 1 if clear else 0, _stream(stream))
    return bits.value


# ------------------------------------------------------------------ SepCache


class SepCache:
    """The four-block KV cache of `layers` layers for B sequences, in one
    device buffer.  Sizes: a initial, s separator, past window, w local."""

    def __init__(self, a: int, s: int, past: int, w: int, layers: int, B: int, Hkv: int, D: int,
                 dtype=torch.bfloat16, device="cuda", stream=None, mode: int = 0):
        self.cfg = SepCacheCfg(a, s, past, w, mode)
        self.dt = SEP_BF16 if dtype == torch.bfloat16 else SEP_F32
        nbytes = int(_lib.sepcache_bytes(self.cfg, layers, B, Hkv, D, self.dt))
        if nbytes == 0:
            raise SepError("sepcache_bytes", -1)
        self.buffer = torch.empty((nbytes,), dtype=torch.uint8, device=device)
        self.c = _SepCacheC()
        _check("sepcache_carve", _lib.sepcache_carve(ctypes.byref(self.c), _ptr(self.buffer),
                                                     nbytes, self.cfg, layers, B, Hkv, D, self.dt))
        self.layers, self.B, self.Hkv, self.D, self.cap = layers, B, Hkv, D, self.c.cap
        self.dtype = dtype
        self._ws = {}
        self.init(stream)

    def _view(self, addr, shape, dtype):
        base = self.buffer.data_ptr()
        off = addr - base
        esz = torch.tensor([], dtype=dtype).element_size()
        n = 1
        for d in shape:
            n *= d
        return self.buffer[off: off + n * esz].view(dtype).view(*shape)

    # device views of the cache state
    @property
    def k(self):
        return self._view(self.c.k, (self.layers, self.B, self.Hkv, self.cap, self.D), self.dtype)

    @property
    def v(self):
        return self._view(self.c.v, (self.layers, self.B, self.Hkv, self.cap, self.D), self.dtype)

    @property
    def pos(self):
        return self._view(self.c.pos, (self.B, self.cap), torch.int32)

    @property
    def flag(self):
        return self._view(self.c.flag, (self.B, self.cap), torch.uint8)

    @property
    def counts(self):
        return self._view(self.c.counts, (self.B, 4), torch.int32)

    @property
    def step(self):
        return self._view(self.c.step, (self.B,), torch.int64)

    def init(self, stream=None):
        _check("sepcache_init", _lib.sepcache_init(ctypes.byref(self.c), _stream(stream)))

    def set_rope(self, theta: float, stream=None):
        """Positional-encoding shifting: with theta > 0 the cache holds keys
        before their rotary encoding and every decode encodes each retained
        key at its slot in the cache and q at the newest slot; 0 switches it
        off (keys stored encoded)."""
        _check("sepcache_set_rope", _lib.sepcache_set_rope(ctypes.byref(self.c), float(theta),
                                                           _stream(stream)))

    @property
    def rope_theta(self) -> float:
        return float(self.c.rope_theta)

    # layout checks of the per-token tensors (the library reads B * Hkv rows
    # of D elements in the cache dtype, B flags and B * Hq query rows)
    def _check_new(self, k_new, v_new, is_sep_new):
        shape = (self.B, self.Hkv, self.D)
        _expect(k_new, "k_new", self.dtype, shape)
        _expect(v_new, "v_new", self.dtype, shape)
        _expect(is_sep_new, "is_sep_new", torch.uint8, (self.B,))

    def _check_query(self, q, out, lse) -> int:
        Hq = _dims(q, "q", 3)[1]
        _expect(q, "q", self.dtype, (self.B, Hq, self.D))
        _expect(out, "out", self.dtype, (self.B, Hq, self.D))
        _expect(lse, "lse", torch.float32, (self.B, Hq))
        return Hq

    def append(self, layer: int, k_new, v_new, is_sep_new=None, stream=None):
        self._check_new(k_new, v_new, is_sep_new)
        _need_cuda(k_new, v_new, is_sep_new, self.buffer)
        _check("sepcache_append", _lib.sepcache_append(
            ctypes.byref(self.c), layer, _ptr(k_new), _ptr(v_new), _ptr(is_sep_new),
            _stream(stream)))

    def compact(self, layer: int, stream=None):
        _check("sepcache_compact", _lib.sepcache_compact(ctypes.byref(self.c), layer,
                                                         _stream(stream)))

    def ingest(self, layer: int, k, v, is_sep=None, prefix=None, idx=None, stream=None):
        """Put a prompt's T tokens into this (empty) cache at `layer`: k, v
        [B, Hkv, T, D]; is_sep [B, T], prefix [B, T+1], idx [B, T] from
        build_index (read at layer 0).  Same result as T appends."""
        T = _dims(k, "k", 4)[2]
        _expect(k, "k", self.dtype, (self.B, self.Hkv, T, self.D))
        _expect(v, "v", self.dtype, (self.B, self.Hkv, T, self.D))
        _expect(is_sep, "is_sep", torch.uint8, (self.B, T))
        _expect(prefix, "prefix", torch.int32, (self.B, T + 1))
        _expect(idx, "idx", torch.int32, (self.B, T))
        _need_cuda(k, v, is_sep, prefix, idx, self.buffer)
        _check("sepcache_ingest", _lib.sepcache_ingest(
            ctypes.byref(self.c), layer, _ptr(k), _ptr(v), _ptr(is_sep), _ptr(prefix), _ptr(idx), T,
            _stream(stream)))

    def workspace(self, Hq: int):
        ws = self._ws.get(Hq)
        if ws is None:
            nbytes = int(_lib.sep_attn_decode_workspace(ctypes.byref(self.c), Hq))
            ws = torch.zeros((nbytes,), dtype=torch.uint8, device=self.buffer.device)
            self._ws[Hq] = ws
        return ws

    def decode(self, layer: int, q, scale: float = 0.0, out=None, lse=None, want_lse=True,
               stream=None):
        Hq = self._check_query(q, out, lse)
        _need_cuda(q, out, lse, self.buffer)
        B = self.B
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        ws = self.workspace(Hq)
        _check("sep_attn_decode", _lib.sep_attn_decode(
            ctypes.byref(self.c), layer, _ptr(q), Hq, float(scale), _ptr(out), _ptr(lse),
            _ptr(ws), ws.numel(), _stream(stream)))
        return out, lse

    def decode_step(self, layer: int, q, k_new, v_new, is_sep_new=None, scale: float = 0.0,
                    out=None, lse=None, want_lse=True, stream=None):
        """append + compact + decode of one layer in one launch (plus the
        layer-0 bookkeeping launch)."""
        Hq = self._check_query(q, out, lse)
        self._check_new(k_new, v_new, is_sep_new)
        _need_cuda(q, k_new, v_new, is_sep_new, out, lse, self.buffer)
        B = self.B
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        ws = self.workspace(Hq)
        _check("sep_attn_decode_step", _lib.sep_attn_decode_step(
            ctypes.byref(self.c), layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(is_sep_new), Hq,
            float(scale), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
        return out, lse

    def decode_noalloc(self, layer: int, q, scale: float = 0.0, out=None, lse=None,
                       want_lse=True, stream=None):
        """decode() for callers that cannot allocate: no workspace; the
        library's fixed scratch holds the partials (see the header)."""
        Hq = self._check_query(q, out, lse)
        _need_cuda(q, out, lse, self.buffer)
        B = self.B
        if out is None:
            out = torch.empty_like(q)
        if lse is None and want_lse:
            lse = torch.empty((B, Hq), dtype=torch.float32, device=q.device)
        _check("sep_attn_decode_noalloc", _lib.sep_attn_decode_noalloc(
            ctypes.byref(self.c), layer, _ptr(q), Hq, float(scale), _ptr(out), _ptr(lse),
            _stream(stream)))
        return out, lse

    def status(self, stream=None) -> int:
        v = ctypes.c_int32(0)
        _lib.sepcache_status(ctypes.byref(self.c), ctypes.byref(v), _stream(stream))
        return v.value
