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
