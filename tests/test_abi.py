"""The C-ABI library loads, exports every symbol include/sepattn.h declares,
and rejects invalid arguments on the host (no GPU needed: every case here
fails validation before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_symbols():
    txt = open(os.path.join(ROOT, "include", "sepattn.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    names = set(re.findall(r"\b((?:sep|sepcache)_[a-z0-9_]+)\s*\(", txt))
    return sorted(names)


@pytest.fixture(scope="module")
def sl():
    import streaming_kv_cache_sep_b200 as m
    return m


def test_header_symbols_exported(sl):
    names = _header_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(sl.lib(), n), n
    assert set(names) == set(sl.ABI_SYMBOLS)


def test_strerror_and_version(sl):
    L = sl.lib()
    assert L.sep_strerror(0) == b"ok"
    assert b"invalid" in L.sep_strerror(-1)
    assert L.sep_version() >= 100


FAKE = ctypes.c_void_p(4096)  # never dereferenced: validation fails first


def test_prefill_rejects_bad_arguments(sl):
    L = sl.lib()
    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, is_sep=FAKE, prefix=FAKE, idx=FAKE, B=1, Hq=4,
                 Hkv=2, S=16, D=64, a=4, n=8, scale=0.0, out=FAKE, lse=None, ws=FAKE, wsb=1 << 30)
        a.update(kw)
        return L.sep_attn_prefill(a["q"], a["k"], a["v"], a["dtype"], a["is_sep"], a["prefix"],
                                  a["idx"], a["B"], a["Hq"], a["Hkv"], a["S"], a["D"], a["a"],
                                  a["n"], a["scale"], a["out"], a["lse"], a["ws"], a["wsb"], None)
    assert call(n=0) == -1
    assert call(a=-1) == -1
    assert call(S=0) == -1
    assert call(Hq=3, Hkv=2) == -1
    assert call(D=96) == -2
    assert call(dtype=7) == -2
    assert call(dtype=0, D=256) == -2
    assert call(q=None) == -6
    assert call(q=ctypes.c_void_p(4100)) == -3
    assert call(ws=ctypes.c_void_p(4096 + 16)) == -3
    assert call(wsb=16) == -1


def test_index_rejects_bad_arguments(sl):
    L = sl.lib()
    assert L.sep_build_index(FAKE, 0, 10, FAKE, FAKE, FAKE, None) == -1
    assert L.sep_build_index(FAKE, 1, 0, FAKE, FAKE, FAKE, None) == -1
    assert L.sep_build_index(None, 1, 10, FAKE, FAKE, FAKE, None) == -6
    assert L.sep_count_pairs(FAKE, 1, 10, -1, 4, FAKE, None) == -1
    assert L.sep_count_pairs(FAKE, 1, 10, 0, 0, FAKE, None) == -1
    ids = (ctypes.c_int32 * 40)(*range(40))
    assert L.sep_flags_from_ids(FAKE, 10, ids, 33, FAKE, None) == -1
    assert L.sep_flags_from_ids(FAKE, 10, ids, 0, FAKE, None) == -1
    assert L.sep_flags_from_ids(FAKE, -1, ids, 3, FAKE, None) == -1
    assert L.sep_flags_from_ids(None, 0, ids, 3, None, None) == 0  # empty is a no-op
    F = FAKE
    assert L.sep_build_index_from_ids(F, 0, 10, ids, 3, F, F, F, F, None) == -1
    assert L.sep_build_index_from_ids(F, 1, 0, ids, 3, F, F, F, F, None) == -1
    assert L.sep_build_index_from_ids(F, 1, 10, ids, 0, F, F, F, F, None) == -1
    assert L.sep_build_index_from_ids(F, 1, 10, ids, 33, F, F, F, F, None) == -1
    assert L.sep_build_index_from_ids(F, 1, 10, None, 3, F, F, F, F, None) == -6
    assert L.sep_build_index_from_ids(None, 1, 10, ids, 3, F, F, F, F, None) == -6
    assert L.sep_build_index_from_ids(F, 1, 10, ids, 3, F, F, None, F, None) == -6


def test_cache_layout_and_validation(sl):
    L = sl.lib()
    cfg = sl.SepCacheCfg(4, 64, 128, 256)
    nb = L.sepcache_bytes(cfg, 32, 16, 8, 128, 1)
    cap = 4 + 64 + 128 + 256 + 1
    kv = 32 * 16 * 8 * cap * 128 * 2
    # K and V, one buffer each (flushes compact in place); the metadata and
    # the rotary table are small
    assert nb >= 2 * kv and nb < 2 * kv + 512 * 1024
    assert L.sepcache_bytes(sl.SepCacheCfg(4, 64, 128, 0), 1, 1, 1, 128, 1) == 0  # w >= 1
    assert L.sepcache_bytes(sl.SepCacheCfg(-1, 64, 128, 4), 1, 1, 1, 128, 1) == 0
    assert L.sepcache_bytes(cfg, 1, 1, 1, 96, 1) == 0
    c = sl._SepCacheC()
    base = ctypes.c_void_p(1 << 20)
    assert L.sepcache_carve(ctypes.byref(c), base, nb, cfg, 32, 16, 8, 128, 1) == 0
    assert c.cap == cap and c.k == (1 << 20) and c.v - c.k >= kv
    assert all(getattr(c, f) % 256 == 0
               for f in ("pos", "flag", "counts", "plan", "step", "status", "rope"))
    # rotary table: max(cap, 65) rows of D/2 (cos, sin) pairs, at the end
    assert c.rope_rows == cap and c.rope_theta == 0.0
    assert c.rope + cap * 128 * 4 <= (1 << 20) + nb
    # positional-encoding shifting: theta 0 (off) enqueues nothing; negative
    # or (0, 1] is refused before anything is enqueued
    assert L.sepcache_set_rope(ctypes.byref(c), 0.0, None) == 0 and c.rope_theta == 0.0
    assert L.sepcache_set_rope(ctypes.byref(c), -5.0, None) == -1
    assert L.sepcache_set_rope(ctypes.byref(c), 1.0, None) == -1
    assert L.sepcache_set_rope(ctypes.byref(c), float("nan"), None) == -1
    assert L.sepcache_set_rope(None, 10000.0, None) == -6
    small = sl._SepCacheC()
    cfg_s = sl.SepCacheCfg(1, 1, 1, 1)
    assert L.sepcache_carve(ctypes.byref(small), base, L.sepcache_bytes(cfg_s, 1, 1, 1, 64, 1),
                            cfg_s, 1, 1, 1, 64, 1) == 0
    assert small.rope_rows == 65  # the turns by 8 and 64 slots are always in the table
    assert L.sepcache_carve(ctypes.byref(c), ctypes.c_void_p((1 << 20) + 16), nb, cfg, 32, 16, 8,
                            128, 1) == -3
    assert L.sepcache_carve(ctypes.byref(c), base, nb - 1, cfg, 32, 16, 8, 128, 1) == -1
    assert L.sepcache_carve(ctypes.byref(c), base, nb, cfg, 32, 16, 8, 128, 5) == -2
    # the StreamingLLM special case (s = 0, past = 0) is a valid cache
    assert L.sepcache_bytes(sl.SepCacheCfg(4, 0, 0, 252), 1, 1, 1, 128, 1) > 0
    # append / compact / decode check the layer index and pointers first
    assert L.sepcache_carve(ctypes.byref(c), base, nb, cfg, 32, 16, 8, 128, 1) == 0
    assert L.sepcache_append(ctypes.byref(c), 32, FAKE, FAKE, FAKE, None) == -1
    assert L.sepcache_append(ctypes.byref(c), 0, FAKE, FAKE, None, None) == -6
    assert L.sepcache_append(ctypes.byref(c), 1, ctypes.c_void_p(4100), FAKE, None, None) == -3
    assert L.sepcache_compact(ctypes.byref(c), -1, None) == -1
    ws = L.sep_attn_decode_workspace(ctypes.byref(c), 32)
    assert ws > 0
    assert L.sep_attn_decode(ctypes.byref(c), 0, FAKE, 30, 0.0, FAKE, None, FAKE, ws, None) == -1
    assert L.sep_attn_decode(ctypes.byref(c), 0, FAKE, 8 * 16, 0.0, FAKE, None, FAKE, ws, None) == -1
    assert L.sep_attn_decode(ctypes.byref(c), 0, FAKE, 32, 0.0, FAKE, None, FAKE, ws - 1, None) == -1
    assert L.sep_attn_decode(ctypes.byref(c), 0, None, 32, 0.0, FAKE, None, FAKE, ws, None) == -6


def test_backward_rejects_bad_arguments(sl):
    L = sl.lib()
    need = L.sep_attn_backward_workspace(1, 4, 2, 16, 64)
    assert need > 0
    assert L.sep_attn_backward_workspace(1, 4, 2, 16, 96) == 0
    assert L.sep_attn_backward_workspace(1, 3, 2, 16, 64) == 0
    assert L.sep_attn_backward_workspace(0, 4, 2, 16, 64) == 0
    assert L.sep_attn_backward_workspace(1, 4, 2, 0, 64) == 0
    # grows with the sequence (fp32 dK/dV sums, compact rows, the item list)
    assert L.sep_attn_backward_workspace(1, 4, 2, 4096, 128) > L.sep_attn_backward_workspace(1, 4, 2, 16, 128)
    order = ("q", "k", "v", "out", "lse", "dout", "dtype", "is_sep", "prefix", "idx", "B", "Hq",
             "Hkv", "S", "D", "a", "n", "scale", "dq", "dk", "dv", "ws", "wsb")

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, out=FAKE, lse=FAKE, dout=FAKE, dtype=1, is_sep=FAKE,
                 prefix=FAKE, idx=FAKE, B=1, Hq=4, Hkv=2, S=16, D=64, a=4, n=8, scale=0.0,
                 dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, wsb=need)
        a.update(kw)
        return L.sep_attn_backward(*[a[x] for x in order], None)

    assert call(dtype=0) == -2  # bf16 only
    assert call(D=96) == -2
    for bad in (dict(B=0), dict(S=0), dict(Hq=3), dict(a=-1), dict(n=0), dict(B=70000)):
        assert call(**bad) == -1, bad
    for name in ("q", "k", "v", "out", "lse", "dout", "is_sep", "prefix", "idx", "dq", "dk", "dv",
                 "ws"):
        assert call(**{name: None}) == -6, name
    for name in ("q", "k", "v", "out", "dout", "dq", "dk", "dv"):
        assert call(**{name: ctypes.c_void_p(4100)}) == -3, name
    assert call(ws=ctypes.c_void_p(4096 + 16)) == -3  # the workspace is 256-byte aligned
    assert call(wsb=need - 1) == -1


def test_masked_generation_rejects_bad_arguments(sl):
    L = sl.lib()
    need = L.sep_attn_decode_masked_workspace(2, 8, 2, 64, 128)
    assert need > 0
    assert L.sep_attn_decode_masked_workspace(2, 8, 2, 64, 96) == 0
    assert L.sep_attn_decode_masked_workspace(2, 6, 2, 64, 128) == 0  # 3 query heads per kv head
    order = ("q", "k", "v", "dtype", "prefix", "idx", "B", "Hq", "Hkv", "S", "T", "D", "a", "n",
             "scale", "out", "lse", "ws", "wsb")

    def call(**kw):
        a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, prefix=FAKE, idx=FAKE, B=2, Hq=8, Hkv=2, S=64,
                 T=40, D=128, a=4, n=16, scale=0.0, out=FAKE, lse=None, ws=None, wsb=0)
        a.update(kw)
        return L.sep_attn_decode_masked(*[a[x] for x in order], None)

    assert call(dtype=2) == -2
    assert call(D=96) == -2
    for bad in (dict(T=0), dict(T=65), dict(Hq=6), dict(Hq=32), dict(Hq=7), dict(a=-1), dict(n=0),
                dict(B=0), dict(S=0, T=0)):
        assert call(**bad) == -1, bad
    for name in ("q", "k", "v", "prefix", "idx", "out"):
        assert call(**{name: None}) == -6, name
    for name in ("q", "k", "v", "out"):
        assert call(**{name: ctypes.c_void_p(4100)}) == -3, name
    # fp32 merges its splits through the caller's workspace
    assert call(dtype=0) == -6
    assert call(dtype=0, ws=ctypes.c_void_p(4100), wsb=need) == -3
    assert call(dtype=0, ws=FAKE, wsb=16) == -1


def _carved(sl, cfg, layers, B, Hkv, D, dtype):
    L = sl.lib()
    nb = L.sepcache_bytes(cfg, layers, B, Hkv, D, dtype)
    assert nb > 0
    c = sl._SepCacheC()
    assert L.sepcache_carve(ctypes.byref(c), ctypes.c_void_p(1 << 20), nb, cfg, layers, B, Hkv, D,
                            dtype) == 0
    return c


def test_ingest_and_decode_step_reject_bad_arguments(sl):
    L = sl.lib()
    c = _carved(sl, sl.SepCacheCfg(4, 64, 128, 256), 32, 16, 8, 128, 1)
    cp = ctypes.byref(c)
    F = FAKE
    # ingestion: cache, layer and T first, then pointers, then alignment
    assert L.sepcache_ingest(None, 0, F, F, F, F, F, 10, None) == -6
    assert L.sepcache_ingest(cp, 32, F, F, F, F, F, 10, None) == -1
    assert L.sepcache_ingest(cp, -1, F, F, F, F, F, 10, None) == -1
    assert L.sepcache_ingest(cp, 0, F, F, F, F, F, 0, None) == -1
    assert L.sepcache_ingest(cp, 0, None, F, F, F, F, 10, None) == -6
    assert L.sepcache_ingest(cp, 0, F, F, None, F, F, 10, None) == -6  # layer 0 reads the index
    assert L.sepcache_ingest(cp, 1, ctypes.c_void_p(4100), F, None, None, None, 10, None) == -3
    assert L.sepcache_ingest(cp, 1, F, F, None, None, None, 1 << 24, None) == -1  # B Hkv T >= 2^31
    # a cache whose fields do not agree is refused by every call
    bad = _carved(sl, sl.SepCacheCfg(4, 64, 128, 256), 32, 16, 8, 128, 1)
    bad.cap += 1
    assert L.sepcache_ingest(ctypes.byref(bad), 1, F, F, None, None, None, 10, None) == -1
    assert L.sepcache_append(ctypes.byref(bad), 1, F, F, None, None) == -1
    assert L.sep_attn_decode_workspace(ctypes.byref(bad), 32) == 0
    # the fused step: layer, head grouping, pointers, alignment, workspace size
    ws = L.sep_attn_decode_workspace(cp, 32)
    assert ws > 0

    def step(layer=1, q=F, kn=F, vn=F, is_sep=None, Hq=32, out=F, w=F, wb=ws, cache=cp):
        return L.sep_attn_decode_step(cache, layer, q, kn, vn, is_sep, Hq, 0.0, out, None, w, wb,
                                      None)

    assert step(cache=None) == -6
    assert step(cache=ctypes.byref(bad)) == -1
    assert step(layer=32) == -1
    assert step(Hq=24) == -1   # 3 query heads per kv head
    assert step(Hq=128) == -1  # 16 query heads per kv head
    assert step(Hq=30) == -1   # not a multiple of Hkv
    assert step(layer=0) == -6  # layer 0 advances the cache from is_sep_new
    for kw in (dict(q=None), dict(kn=None), dict(vn=None), dict(out=None), dict(w=None)):
        assert step(**kw) == -6, kw
    for kw in (dict(q=ctypes.c_void_p(4100)), dict(kn=ctypes.c_void_p(4104)),
               dict(vn=ctypes.c_void_p(4108)), dict(out=ctypes.c_void_p(4100)),
               dict(w=ctypes.c_void_p(4100))):
        assert step(**kw) == -3, kw
    assert step(wb=ws - 1) == -1


def test_noalloc_decode_rejects_bad_arguments(sl):
    L = sl.lib()
    c = _carved(sl, sl.SepCacheCfg(4, 64, 128, 256), 2, 2, 2, 64, 1)
    cp = ctypes.byref(c)
    assert L.sep_attn_decode_noalloc(None, 0, FAKE, 4, 0.0, FAKE, None, None) == -6
    assert L.sep_attn_decode_noalloc(cp, 2, FAKE, 4, 0.0, FAKE, None, None) == -1
    assert L.sep_attn_decode_noalloc(cp, 0, FAKE, 6, 0.0, FAKE, None, None) == -1
    assert L.sep_attn_decode_noalloc(cp, 0, FAKE, 3, 0.0, FAKE, None, None) == -1
    assert L.sep_attn_decode_noalloc(cp, 0, None, 4, 0.0, FAKE, None, None) == -6
    assert L.sep_attn_decode_noalloc(cp, 0, FAKE, 4, 0.0, None, None, None) == -6
    assert L.sep_attn_decode_noalloc(cp, 0, ctypes.c_void_p(4100), 4, 0.0, FAKE, None, None) == -3
    # an fp32 cache of more than 512 rows merges through the fixed scratch:
    # B * Hq * ceil(cap / 64) partials beyond its 8192 slots are refused
    # before anything is enqueued
    big = _carved(sl, sl.SepCacheCfg(4, 300, 200, 100), 1, 64, 8, 64, 0)
    assert big.cap == 605
    assert L.sep_attn_decode_noalloc(ctypes.byref(big), 0, FAKE, 64, 0.0, FAKE, None, None) == -7


def test_binding_checks_layouts_before_the_device(sl):
    """The Python binding checks each tensor's dtype and shape against the
    documented layout before it hands bare pointers to the library (CPU
    tensors here: a correct layout gets as far as the device check)."""
    import torch
    bf, f32, u8, i32 = torch.bfloat16, torch.float32, torch.uint8, torch.int32
    B, Hq, Hkv, S, D = 2, 4, 2, 40, 64
    q = torch.zeros((B, Hq, S, D), dtype=bf)
    k = torch.zeros((B, Hkv, S, D), dtype=bf)
    v = torch.zeros((B, Hkv, S, D), dtype=bf)
    fl = torch.zeros((B, S), dtype=u8)
    pre = torch.zeros((B, S + 1), dtype=i32)
    idx = torch.zeros((B, S), dtype=i32)
    cuda_msg = "expected contiguous CUDA tensors"

    with pytest.raises(ValueError, match=cuda_msg):
        sl.prefill(q, k, v, fl, pre, idx, 4, 8)
    with pytest.raises(TypeError, match="k:"):
        sl.prefill(q, k.float(), v, fl, pre, idx, 4, 8)
    with pytest.raises(ValueError, match="v: expected shape"):
        sl.prefill(q, k, v[:, :, :S - 1].contiguous(), fl, pre, idx, 4, 8)
    with pytest.raises(TypeError, match="is_sep:"):
        sl.prefill(q, k, v, fl.bool(), pre, idx, 4, 8)
    with pytest.raises(TypeError, match="prefix:"):
        sl.prefill(q, k, v, fl, pre.long(), idx, 4, 8)
    with pytest.raises(ValueError, match="prefix: expected shape"):
        sl.prefill(q, k, v, fl, pre[:, :S].contiguous(), idx, 4, 8)
    with pytest.raises(ValueError, match="idx: expected shape"):
        sl.prefill(q, k, v, fl, pre, idx[:1].contiguous(), 4, 8)
    with pytest.raises(TypeError, match="lse:"):
        sl.prefill(q, k, v, fl, pre, idx, 4, 8, lse=torch.zeros((B, Hq, S), dtype=bf))
    with pytest.raises(ValueError, match="out: expected shape"):
        sl.prefill(q, k, v, fl, pre, idx, 4, 8, out=torch.zeros((B, Hq, S, 2 * D), dtype=bf))
    with pytest.raises(ValueError, match="q: expected 4"):
        sl.prefill(q[0], k, v, fl, pre, idx, 4, 8)
    with pytest.raises(TypeError, match="unsupported dtype"):
        sl.prefill(q.half(), k.half(), v.half(), fl, pre, idx, 4, 8)

    lse = torch.zeros((B, Hq, S), dtype=f32)
    with pytest.raises(ValueError, match=cuda_msg):
        sl.backward(q, k, v, q, lse, q, fl, pre, idx, 4, 8)
    with pytest.raises(ValueError, match="dout: expected shape"):
        sl.backward(q, k, v, q, lse, q[:, :2].contiguous(), fl, pre, idx, 4, 8)
    with pytest.raises(ValueError, match="lse: expected shape"):
        sl.backward(q, k, v, q, lse[:, :, :4].contiguous(), q, fl, pre, idx, 4, 8)
    with pytest.raises(ValueError, match="dk: expected shape"):
        sl.backward(q, k, v, q, lse, q, fl, pre, idx, 4, 8, dk=torch.zeros_like(q))

    qd = torch.zeros((B, Hq, D), dtype=bf)
    with pytest.raises(ValueError, match=cuda_msg):
        sl.decode_masked(qd, k, v, pre, idx, S, 4, 8)
    with pytest.raises(ValueError, match="k: expected shape"):
        sl.decode_masked(qd, k[:, :, :, :32].contiguous(), v, pre, idx, S, 4, 8)
    with pytest.raises(ValueError, match="lse: expected shape"):
        sl.decode_masked(qd, k, v, pre, idx, S, 4, 8, lse=torch.zeros((B, Hq, 1), dtype=f32))

    with pytest.raises(ValueError, match=cuda_msg):
        sl.build_index(fl)
    with pytest.raises(TypeError, match="is_sep:"):
        sl.build_index(fl.int())
    with pytest.raises(ValueError, match="is_sep: expected 2"):
        sl.build_index(fl[0])
    with pytest.raises(ValueError, match="prefix: expected shape"):
        sl.build_index(fl, out=(idx, idx, torch.zeros((B,), dtype=i32)))
    ids = torch.zeros((B, S), dtype=i32)
    with pytest.raises(TypeError, match="ids:"):
        sl.flags_from_ids(ids.long(), [1, 2])
    with pytest.raises(TypeError, match="ids:"):
        sl.build_index_from_ids(ids.long(), [1, 2])
    with pytest.raises(ValueError, match=cuda_msg):
        sl.build_index_from_ids(ids, [1, 2])
    with pytest.raises(TypeError, match="prefix:"):
        sl.count_pairs(pre.long(), 4, 8)
    with pytest.raises(TypeError, match="out:"):
        sl.count_pairs(pre, 4, 8, out=torch.zeros((B,), dtype=i32))
