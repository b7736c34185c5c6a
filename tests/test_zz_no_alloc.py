"""sep_attn_decode_noalloc: decode for callers that cannot allocate.

Some callers cannot give the library a workspace -- a plug-in that its host
framework calls with only the call's tensors, or a serving loop whose device
memory is all reserved for the KV pool, where a new cudaMalloc would fail or
stall the device.  For them the library keeps the decode's split-K scratch in
a fixed array of its own.  These tests call that entry point through the C
ABI, on two calls in a row, and check it against the workspace-taking
sep_attn_decode (within the tolerance the decode tests use) and, for the fp32
cache whose splits merge through the scratch array, against the oracle's
attention over the oracle's retained rows.  This file is collected last so
that a run stopping at its first failure has already run every other test;
it also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_RMS = 2e-2, 2e-3
F32_MAX = 1e-5


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


RING = 13  # distinct per-token inputs, cycled by step


def _fill_cache(sl, cfg, T, layers, seed, dtype=torch.bfloat16):
    dt = "bf16" if dtype == torch.bfloat16 else "f32"
    wl = dict(Hq=cfg["Hq"], Hkv=cfg["Hkv"], D=cfg["D"], dtype=dt, qkv_std=1.0, B=cfg["B"])
    flags = synth.bernoulli_flags(synth.rng((seed, 10)), (T, cfg["B"]), 0.1)
    cache = sl.SepCache(cfg["a"], cfg["s"], cfg["past"], cfg["w"], layers, cfg["B"], cfg["Hkv"],
                        cfg["D"], dtype=dtype)
    # ring[l][r] = (q, k, v) of layer l for every token t with t % RING == r
    ring = [[synth.decode_step_qkv(wl, seed, r, l) for r in range(RING)] for l in range(layers)]
    dring = [[(q.cuda(), k.cuda(), v.cuda()) for q, k, v in rl] for rl in ring]
    dflags = torch.from_numpy(flags).cuda()
    for t in range(T):
        for l in range(layers):
            _, k, v = dring[l][t % RING]
            cache.append(l, k, v, dflags[t] if l == 0 else None)
            cache.compact(l)
    torch.cuda.synchronize()
    return cache, ring, dring, flags


def _close(a, b):
    d = a.double() - b.double()
    return float(d.abs().max()) <= BF16_MAX and float(d.pow(2).mean().sqrt()) <= BF16_RMS


@pytest.mark.parametrize("T", [20, 700])  # one split (<= 64 rows) and several splits
def test_noalloc_matches_workspace_decode_twice(sl, T):
    cfg = dict(synth.WORKLOADS["decode_llama3_8b_b16_l32_t65536_d128_bf16"])
    cache, _, dring, _ = _fill_cache(sl, cfg, T, layers=2, seed=1234 + T)
    for call in range(2):  # two calls in a row, different queries and layers
        layer = call % 2
        q = dring[layer][call + 1][0]
        want, want_lse = cache.decode(layer, q)
        got, got_lse = cache.decode_noalloc(layer, q)
        torch.cuda.synchronize()
        assert _close(got, want), "call %d" % call
        assert float((got_lse - want_lse).abs().max()) <= 2e-2
    assert sl.device_status() == 0


def test_noalloc_fp32_scratch_merge_matches_oracle_twice(sl):
    """An fp32 cache of more than 512 rows: its splits merge through the
    library's scratch array (partials, then the last CTA by atomic ticket).
    Two calls in a row on different layers and queries; each must equal the
    oracle's attention over the rows the oracle's own state machine retains,
    and the workspace decode, within the fp32 tolerance.  The first call also
    finds the tickets the previous test file may have left, and the second
    the ones the first left."""
    cfg = dict(a=4, s=300, past=100, w=420, B=3, Hq=8, Hkv=2, D=64)
    T = 1000  # five flushes; every sequence then retains more than 512 rows
    cache, ring, dring, flags = _fill_cache(sl, cfg, T, layers=2, seed=4321, dtype=torch.float32)
    cap = cfg["a"] + cfg["s"] + cfg["past"] + cfg["w"] + 1
    assert (cap + 63) // 64 > 8  # more splits than one cluster: the scratch path
    snap = oracle.sepcache_simulate(flags, cfg["a"], cfg["s"], cfg["past"], cfg["w"], [T - 1])
    np.testing.assert_array_equal(cache.counts.cpu().numpy(), snap["counts"][0])
    np.testing.assert_array_equal(cache.pos.cpu().numpy(), snap["pos"][0])
    assert int(snap["counts"][0].sum(1).max()) > 512
    for call, (layer, r) in enumerate([(1, 3), (0, 7)]):
        q = dring[layer][r][0]
        got, got_lse = cache.decode_noalloc(layer, q)
        want_ws, want_ws_lse = cache.decode(layer, q)
        torch.cuda.synchronize()
        assert float((got - want_ws).abs().max()) <= F32_MAX, "call %d" % call
        assert float((got_lse - want_ws_lse).abs().max()) <= F32_MAX, "call %d" % call
        g = got.double().cpu().numpy()
        gl = got_lse.double().cpu().numpy()
        for b in range(cfg["B"]):
            n = int(snap["counts"][0, b].sum())
            pos = snap["pos"][0, b, :n]
            k = torch.stack([ring[layer][p % RING][1][b] for p in pos], 1)  # [Hkv, n, D]
            v = torch.stack([ring[layer][p % RING][2][b] for p in pos], 1)
            want, want_lse = oracle.attend(ring[layer][r][0][b], k, v)
            assert np.abs(g[b] - want).max() <= F32_MAX, (call, b)
            assert np.abs(gl[b] - want_lse).max() <= F32_MAX, (call, b)
    assert sl.device_status() == 0


def test_noalloc_through_raw_c_abi(sl):
    """The exported C symbol itself, with raw pointers and the current stream."""
    cfg = dict(a=2, s=8, past=6, w=20, B=3, Hq=8, Hkv=2, D=64)
    cache, _, dring, _ = _fill_cache(sl, cfg, 120, layers=1, seed=77)
    L = sl.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        q = dring[0][call][0]
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device="cuda")
        rc = L.sep_attn_decode_noalloc(ctypes.byref(cache.c), 0, ctypes.c_void_p(q.data_ptr()),
                                       cfg["Hq"], ctypes.c_float(0.0),
                                       ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(lse.data_ptr()), stream)
        assert rc == 0
        want, want_lse = cache.decode(0, q)
        torch.cuda.synchronize()
        assert _close(out, want)
        assert float((lse - want_lse).abs().max()) <= 2e-2


def test_noalloc_rejects_sizes_beyond_its_scratch(sl):
    # fp32, more than 8 splits: B * Hq * ceil(cap / 64) = 16 * 64 * 10 > 8192 partials
    cache = sl.SepCache(4, 200, 128, 256, 1, 16, 8, 64, dtype=torch.float32)
    q = torch.zeros((16, 64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(sl.SepError) as e:
        cache.decode_noalloc(0, q)
    assert e.value.status == -7
    assert b"scratch" in sl.lib().sep_strerror(-7)


def test_noalloc_bf16_needs_no_scratch(sl):
    """bf16 caches merge inside a thread-block cluster and never use the
    scratch array, so sizes beyond its limits are accepted and give the
    workspace decode's result."""
    cfg = dict(a=4, s=64, past=128, w=256, B=64, Hq=32, Hkv=8, D=128)
    cache, _, dring, _ = _fill_cache(sl, cfg, 500, layers=1, seed=99)
    q = dring[0][5][0]
    got, got_lse = cache.decode_noalloc(0, q)
    want, want_lse = cache.decode(0, q)
    torch.cuda.synchronize()
    assert _close(got, want)
    assert float((got_lse - want_lse).abs().max()) <= 2e-2
