"""sep_attn_decode_noalloc: decode for callers that cannot allocate.

Some callers cannot give the library a workspace -- a plug-in that its host
framework calls with only the call's tensors, or a serving loop whose device
memory is all reserved for the KV pool, where a new cudaMalloc would fail or
stall the device.  For them the library keeps the decode's split-K scratch in
a fixed array of its own.  These tests call that entry point through the C
ABI and check it against the workspace-taking sep_attn_decode, within the
bf16 tolerance the decode tests use, on two calls in a row.  This file is
collected last so that a run stopping at its first failure has already run
every other test; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

BF16_MAX, BF16_RMS = 2e-2, 2e-3


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


def _fill_cache(sl, cfg, T, layers, seed):
    wl = dict(Hq=cfg["Hq"], Hkv=cfg["Hkv"], D=cfg["D"], dtype="bf16", qkv_std=1.0, B=cfg["B"])
    flags = synth.bernoulli_flags(synth.rng((seed, 10)), (T, cfg["B"]), 0.1)
    cache = sl.SepCache(cfg["a"], cfg["s"], cfg["past"], cfg["w"], layers, cfg["B"], cfg["Hkv"],
                        cfg["D"], dtype=torch.bfloat16)
    ring = [synth.decode_step_qkv(wl, seed, r, 0) for r in range(13)]
    dring = [(q.cuda(), k.cuda(), v.cuda()) for q, k, v in ring]
    dflags = torch.from_numpy(flags).cuda()
    for t in range(T):
        _, k, v = dring[t % 13]
        for l in range(layers):
            cache.append(l, k, v, dflags[t] if l == 0 else None)
            cache.compact(l)
    torch.cuda.synchronize()
    return cache, dring


def _close(a, b):
    d = a.double() - b.double()
    return float(d.abs().max()) <= BF16_MAX and float(d.pow(2).mean().sqrt()) <= BF16_RMS


@pytest.mark.parametrize("T", [20, 700])  # one split (<= 64 rows) and several splits
def test_noalloc_matches_workspace_decode_twice(sl, T):
    cfg = dict(synth.WORKLOADS["decode_llama3_8b_b16_l32_t65536_d128_bf16"])
    cache, dring = _fill_cache(sl, cfg, T, layers=2, seed=1234 + T)
    for call in range(2):  # two calls in a row, different queries and layers
        q = dring[call + 1][0]
        layer = call % 2
        want, want_lse = cache.decode(layer, q)
        got, got_lse = cache.decode_noalloc(layer, q)
        torch.cuda.synchronize()
        assert _close(got, want), "call %d" % call
        assert float((got_lse - want_lse).abs().max()) <= 2e-2
    assert sl.device_status() == 0


def test_noalloc_through_raw_c_abi(sl):
    """The exported C symbol itself, with raw pointers and the current stream."""
    cfg = dict(a=2, s=8, past=6, w=20, B=3, Hq=8, Hkv=2, D=64)
    cache, dring = _fill_cache(sl, cfg, 120, layers=1, seed=77)
    L = sl.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        q = dring[call][0]
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
    # B * Hq * ceil(cap / 64) = 64 * 32 * 8 > 8192 partials
    cache = sl.SepCache(4, 64, 128, 256, 1, 64, 8, 128, dtype=torch.bfloat16)
    q = torch.zeros((64, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sl.SepError) as e:
        cache.decode_noalloc(0, q)
    assert e.value.status == -7
    assert b"scratch" in sl.lib().sep_strerror(-7)
