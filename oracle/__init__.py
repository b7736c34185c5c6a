"""CPU oracle for Sep-Attention and the four-block SepCache (fp64).

TEST INFRASTRUCTURE ONLY: only the tests, the smoke check and the bench's
CPU-baseline leg may import this package.  It shares no code with the CUDA
library and never imports it.  The arithmetic lives in `sep_oracle.c`; this
file only marshals numpy arrays into it.

Every routine cites the passage of the pages it follows in `sep_oracle.c`.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        _LIB = ctypes.CDLL(_build.build())
        L = _LIB
        P = ctypes.c_void_p
        i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.oracle_flags_from_ids.argtypes = [P, i64, P, i32, P]
        L.oracle_build_index.argtypes = [P, i32, i32, P, P, P]
        L.oracle_count_pairs.argtypes = [P, i32, i32, i32, i32, P, i32]
        L.oracle_prefill_rows.argtypes = [P, P, P, i32, P, i32, i32, i32, i32, i32, i32, i32,
                                          dbl, P, i64, P, P, i32]
        L.oracle_attend.argtypes = [P, P, P, i32, i32, i32, i32, i32, dbl, P, P]
        L.oracle_sepcache_simulate.argtypes = [P, i32, i64, i32, i32, i32, i32, P, i32, i32,
                                               P, P, P, P, i32, P]
        L.oracle_rope.argtypes = [P, i32, i64, i32, P, dbl, P]
        L.oracle_prefill_backward.argtypes = [P, P, P, i32, P, i32, P, i32, i32, i32, i32, i32,
                                              i32, i32, dbl, P, P, P, i32]
        for f in (L.oracle_flags_from_ids, L.oracle_build_index, L.oracle_count_pairs,
                  L.oracle_prefill_rows, L.oracle_attend, L.oracle_sepcache_simulate,
                  L.oracle_rope, L.oracle_prefill_backward):
            f.restype = ctypes.c_int
    return _LIB


def nthreads() -> int:
    """Host threads the oracle uses: the cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _elems(x):
    """(contiguous numpy array of raw element bits, dtype code): fp32 -> 0,
    bf16 bit patterns (uint16) -> 1, fp64 -> 2.  Accepts numpy arrays or CPU
    tensors."""
    if hasattr(x, "numpy"):  # a torch tensor
        import torch
        x = x.detach().cpu().contiguous()
        if x.dtype == torch.bfloat16:
            return x.view(torch.int16).numpy().view(np.uint16), 1
        if x.dtype == torch.float32:
            return x.numpy(), 0
        if x.dtype == torch.float64:
            return x.numpy(), 2
        raise TypeError(x.dtype)
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, 0
    if x.dtype == np.float64:
        return x, 2
    if x.dtype == np.uint16:
        return x, 1
    raise TypeError(x.dtype)


def _shape(name, a, shape):
    """The C routines take bare pointers: every array must have the layout
    its sizes imply."""
    if tuple(a.shape) != tuple(shape):
        raise ValueError("%s: expected shape %s, got %s" % (name, tuple(shape), tuple(a.shape)))


def flags_from_ids(ids: np.ndarray, sep_ids) -> np.ndarray:
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    sep = np.ascontiguousarray(np.asarray(sep_ids, dtype=np.int32))
    out = np.zeros(ids.shape, dtype=np.uint8)
    _lib().oracle_flags_from_ids(_ptr(ids), ids.size, _ptr(sep), sep.size, _ptr(out))
    return out


def build_index(is_sep: np.ndarray):
    """(prefix [B,S+1], idx [B,S] (-1 padded), count [B]) as int32."""
    f = np.ascontiguousarray(is_sep, dtype=np.uint8)
    B, S = f.shape
    prefix = np.zeros((B, S + 1), dtype=np.int32)
    idx = np.zeros((B, S), dtype=np.int32)
    count = np.zeros((B,), dtype=np.int32)
    _lib().oracle_build_index(_ptr(f), B, S, _ptr(prefix), _ptr(idx), _ptr(count))
    return prefix, idx, count


def count_pairs(is_sep: np.ndarray, a: int, n: int, threads: int | None = None) -> np.ndarray:
    """Kept (query, key) pairs per sequence, for one head, int64 [B]."""
    f = np.ascontiguousarray(is_sep, dtype=np.uint8)
    B, S = f.shape
    out = np.zeros((B,), dtype=np.int64)
    _lib().oracle_count_pairs(_ptr(f), B, S, a, n, _ptr(out), threads or nthreads())
    return out


def prefill_rows(q, k, v, is_sep, a: int, n: int, rows=None, scale: float = 0.0,
                 threads: int | None = None):
    """Sep-Attention of the selected query rows, in fp64.

    q [B,Hq,S,D], k/v [B,Hkv,S,D] (fp32 arrays, bf16 bit patterns as uint16,
    or CPU tensors of either dtype); is_sep uint8 [B,S].  `rows` holds flat
    row ids (b*Hq + h)*S + i; None means every row.  Returns
    (out [nrows, D] float64, lse [nrows] float64)."""
    qa, dq = _elems(q)
    ka, dk = _elems(k)
    va, dv = _elems(v)
    assert dq == dk == dv
    B, Hq, S, D = qa.shape
    Hkv = ka.shape[1]
    f = np.ascontiguousarray(is_sep, dtype=np.uint8)
    _shape("k", ka, (B, Hkv, S, D))
    _shape("v", va, (B, Hkv, S, D))
    _shape("is_sep", f, (B, S))
    if rows is None:
        rows = np.arange(B * Hq * S, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, D), dtype=np.float64)
    lse = np.zeros((rows.size,), dtype=np.float64)
    rc = _lib().oracle_prefill_rows(_ptr(qa), _ptr(ka), _ptr(va), dq, _ptr(f), B, Hq, Hkv, S, D,
                                    a, n, float(scale), _ptr(rows), rows.size, _ptr(out),
                                    _ptr(lse), threads or nthreads())
    if rc != 0:
        raise ValueError("oracle_prefill_rows rejected its arguments")
    return out, lse


def prefill(q, k, v, is_sep, a: int, n: int, scale: float = 0.0, threads: int | None = None):
    """Every row: (out [B,Hq,S,D] float64, lse [B,Hq,S] float64)."""
    qa, _ = _elems(q)
    B, Hq, S, D = qa.shape
    out, lse = prefill_rows(q, k, v, is_sep, a, n, None, scale, threads)
    return out.reshape(B, Hq, S, D), lse.reshape(B, Hq, S)


def attend(q, k, v, scale: float = 0.0):
    """Attention of q [Hq,D] over every row of k/v [Hkv,L,D]; fp64
    (out [Hq,D], lse [Hq])."""
    qa, dq = _elems(q)
    ka, dk = _elems(k)
    va, dv = _elems(v)
    assert dq == dk == dv
    Hq, D = qa.shape
    Hkv, L, _ = ka.shape
    _shape("k", ka, (Hkv, L, D))
    _shape("v", va, (Hkv, L, D))
    out = np.zeros((Hq, D), dtype=np.float64)
    lse = np.zeros((Hq,), dtype=np.float64)
    rc = _lib().oracle_attend(_ptr(qa), _ptr(ka), _ptr(va), dq, Hq, Hkv, L, D, float(scale),
                              _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attend rejected its arguments")
    return out, lse


NO_ACCUMULATION = 1   # a flush keeps only the flushed past window's separators
UNBOUNDED_SEPS = 2    # separators are never evicted (overflow past s is flagged)
TOTAL_TRIGGER = 4     # flush when the whole cache exceeds a+s+past+w


def sepcache_simulate(flags: np.ndarray, a: int, s: int, past: int, w: int, snap_steps,
                      cap: int | None = None, want_flushed: bool = False, mode: int = 0):
    """Run the four-block cache over flags [T,B].

    Returns dict(pos [nsnap,B,cap] int32 (-1 padded), flag [nsnap,B,cap] uint8,
    counts [nsnap,B,4] int32 = (|I|,|S|,|P|,|L|), flushed [T,B] uint8 or None,
    overflowed [B] uint8), the cache being read after the token of each snap
    step.  mode: a sum of NO_ACCUMULATION, UNBOUNDED_SEPS, TOTAL_TRIGGER."""
    f = np.ascontiguousarray(flags, dtype=np.uint8)
    T, B = f.shape
    snaps = np.ascontiguousarray(np.asarray(snap_steps, dtype=np.int64))
    assert np.all(np.diff(snaps) > 0), "snap steps must ascend"
    cap = cap or (a + s + past + w + 1)
    pos = np.zeros((snaps.size, B, cap), dtype=np.int32)
    flg = np.zeros((snaps.size, B, cap), dtype=np.uint8)
    cnt = np.zeros((snaps.size, B, 4), dtype=np.int32)
    flushed = np.zeros((T, B), dtype=np.uint8) if want_flushed else None
    overflowed = np.zeros((B,), dtype=np.uint8)
    rc = _lib().oracle_sepcache_simulate(
        _ptr(f), B, T, a, s, past, w, _ptr(snaps), snaps.size, cap, _ptr(pos), _ptr(flg),
        _ptr(cnt), _ptr(flushed) if flushed is not None else None, int(mode), _ptr(overflowed))
    if rc == -2:
        raise AssertionError("cache exceeded a+s+past+w")
    if rc != 0:
        raise ValueError("oracle_sepcache_simulate failed (%d)" % rc)
    return dict(pos=pos, flag=flg, counts=cnt, flushed=flushed, overflowed=overflowed)


def rope(x, positions, theta: float) -> np.ndarray:
    """Rotary position encoding of the rows of x [..., D] at `positions`
    (one per row, broadcast over the leading dims), rotate-half pairing:
    the pair (x_i, x_{i+D/2}) turns by pos * theta^(-2i/D).  fp64 out."""
    xa, dt = _elems(x)
    D = xa.shape[-1]
    rows = xa.size // D
    pos = np.ascontiguousarray(np.broadcast_to(np.asarray(positions, dtype=np.int64),
                                               xa.shape[:-1]).reshape(-1))
    out = np.zeros(xa.shape, dtype=np.float64)
    rc = _lib().oracle_rope(_ptr(xa), dt, rows, D, _ptr(pos), float(theta), _ptr(out))
    if rc != 0:
        raise ValueError("oracle_rope rejected its arguments")
    return out


def decode_shifted(q, k, v, theta: float, scale: float = 0.0):
    """Decode over a cache whose keys are stored before the position is
    encoded: the retained rows k/v [Hkv,L,D] (cache order) take the positions
    0..L-1 they hold inside the cache, the query q [Hq,D] (the newest token,
    the last row) takes L-1.  fp64 (out [Hq,D], lse [Hq])."""
    ka, _ = _elems(k)
    L = ka.shape[1]
    kr = rope(k, np.arange(L, dtype=np.int64)[None, :], theta)
    qr = rope(q, L - 1, theta)
    va, dv = _elems(v)
    return attend(qr, kr, va.astype(np.float64) if dv == 0 else _bf16_to_f64(va), scale)


def _bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact values of bf16 bit patterns (uint16)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def decode_masked(q, k, v, is_sep, T: int, a: int, n: int, scale: float = 0.0):
    """Mask-based generation: q [B,Hq,D] is the query of token T-1, which
    attends over k/v [B,Hkv,S,D] with its row's kept set -- the prefill rule
    for that one row (the generate mask applies the prefill mask's rule to a
    query of length 1).  fp64 (out [B,Hq,D], lse [B,Hq])."""
    qa, dq = _elems(q)
    ka, _ = _elems(k)
    va, _ = _elems(v)
    B, Hq, D = qa.shape
    S = ka.shape[2]
    qfull = np.zeros((B, Hq, T, D), dtype=qa.dtype)
    qfull[:, :, T - 1, :] = qa
    kT = np.ascontiguousarray(ka[:, :, :T, :])
    vT = np.ascontiguousarray(va[:, :, :T, :])
    f = np.ascontiguousarray(np.asarray(is_sep, dtype=np.uint8)[:, :T])
    rows = np.array([(b * Hq + h) * T + (T - 1) for b in range(B) for h in range(Hq)], dtype=np.int64)
    out, lse = prefill_rows(qfull, kT, vT, f, a, n, rows, scale)
    return out.reshape(B, Hq, D), lse.reshape(B, Hq)


def prefill_backward(q, k, v, dout, is_sep, a: int, n: int, scale: float = 0.0,
                     threads: int | None = None):
    """Gradients (dq [B,Hq,S,D], dk, dv [B,Hkv,S,D], fp64) of
    sum(out * dout) through Sep-Attention, out recomputed in fp64."""
    qa, dq_ = _elems(q)
    ka, dk_ = _elems(k)
    va, dv_ = _elems(v)
    oa, do_ = _elems(dout)
    assert dq_ == dk_ == dv_
    B, Hq, S, D = qa.shape
    Hkv = ka.shape[1]
    f = np.ascontiguousarray(is_sep, dtype=np.uint8)
    _shape("k", ka, (B, Hkv, S, D))
    _shape("v", va, (B, Hkv, S, D))
    _shape("dout", oa, (B, Hq, S, D))
    _shape("is_sep", f, (B, S))
    gq = np.zeros((B, Hq, S, D), dtype=np.float64)
    gk = np.zeros((B, Hkv, S, D), dtype=np.float64)
    gv = np.zeros((B, Hkv, S, D), dtype=np.float64)
    rc = _lib().oracle_prefill_backward(_ptr(qa), _ptr(ka), _ptr(va), dq_, _ptr(oa), do_, _ptr(f),
                                        B, Hq, Hkv, S, D, a, n, float(scale), _ptr(gq), _ptr(gk),
                                        _ptr(gv), threads or nthreads())
    if rc != 0:
        raise ValueError("oracle_prefill_backward rejected its arguments")
    return gq, gk, gv
