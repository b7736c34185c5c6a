"""GPU parity of the SepCache variants against the oracle.

The KV manager's switches ("HKUDS047: SepLLM ..." study, section "KV Cache
Manager"): no separator accumulation, no maximum on the separator cache
(an eviction is then flagged in the cache status word), and compression
when the whole cache exceeds its budget.  Each variant is streamed through
sepcache_append / _compact / sep_attn_decode and through the fused
sep_attn_decode_step, and prompts are ingested with sepcache_ingest: block
sizes, positions, flags and K/V bytes bit-exact against the oracle's state
machine run with the same mode, decode outputs within the bf16 (max|d| <=
2e-2, RMS <= 2e-3) or fp32 (max|d| <= 1e-5) tolerance, and the overflow
flag equal to the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from test_gpu_cache import Stream, _check_decode, _check_kv, _check_meta
from test_gpu_ingest import _check_state, _flags, _prompt

pytestmark = pytest.mark.gpu

MODES = [1, 2, 3, 4, 5, 6, 7]


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


SHAPES = [
    # a, s, past, w, B, Hkv, Hq, D, dtype
    (4, 8, 6, 10, 3, 2, 4, 64, torch.bfloat16),
    (1, 3, 2, 2, 2, 1, 2, 128, torch.float32),
    (3, 40, 100, 30, 2, 2, 8, 128, torch.bfloat16),  # more than 64 rows: split decode
]


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "_".join(map(str, s[:8])))
def test_variant_streams(sl, shape, mode, fused):
    a, s, past, w, B, Hkv, Hq, D, dtype = shape
    T = 420
    st = Stream(sl, a, s, past, w, B, Hkv, Hq, D, 2, dtype, seed=31 * mode + a + s + past + w,
                T=T, fused=fused, mode=mode)
    sim = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T), mode=mode)
    for t in range(T):
        dec = (0, 1) if (t < 30 or t % 3 == 0) else ()
        outs = st.step(decode_layers=dec)
        _check_meta(st, sim, t)
        if t % 13 == 0 or t > T - 5:
            _check_kv(st, sim, t)
        if dec:
            _check_decode(st, sim, t, outs, t)
    want = sl.CACHE_ESEPS if sim["overflowed"].any() else 0
    assert st.cache.status() == want
    assert sl.device_status() == 0


INGEST = [
    # a, s, past, w, B, Hkv, Hq, D, dtype, prompt lengths
    (4, 8, 6, 10, 3, 2, 4, 64, torch.bfloat16, [1, 14, 15, 20, 21, 22, 29, 30, 36, 200]),
    (1, 2, 2, 2, 2, 1, 2, 128, torch.bfloat16, [3, 5, 6, 7, 8, 9, 10, 40]),
    (2, 3, 0, 5, 3, 2, 2, 64, torch.float32, [7, 8, 9, 10, 11, 50]),
    (3, 40, 100, 30, 2, 2, 4, 128, torch.bfloat16, [133, 134, 174, 175, 300, 700]),
]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("case", INGEST, ids=lambda c: "_".join(map(str, c[:8])))
def test_variant_ingest(sl, case, mode):
    a, s, past, w, B, Hkv, Hq, D, dtype, lengths = case
    layers = 2
    seed = 3 * mode + a * 1000 + s * 100 + past * 10 + w
    Tmax = max(lengths)
    flags = _flags(seed, B, Tmax, p=0.3)
    kp, vp = _prompt(seed, layers, B, Hkv, Tmax, D, dtype)
    for T in lengths:
        sim = oracle.sepcache_simulate(np.ascontiguousarray(flags[:, :T].T), a, s, past, w,
                                       [T - 1], mode=mode)
        cache = sl.SepCache(a, s, past, w, layers, B, Hkv, D, dtype=dtype, mode=mode)
        is_sep = torch.from_numpy(np.ascontiguousarray(flags[:, :T])).cuda()
        prefix, idx, _ = sl.build_index(is_sep)
        k = kp[:, :, :, :T].contiguous().cuda()
        v = vp[:, :, :, :T].contiguous().cuda()
        for l in range(layers):
            cache.ingest(l, k[l], v[l], is_sep, prefix, idx)

        def kv_of(l, b, pos):
            return kp[l, b][:, pos].contiguous(), vp[l, b][:, pos].contiguous()

        _check_state(cache, sim, 0, B, layers, kv_of)
        want = sl.CACHE_ESEPS if sim["overflowed"].any() else 0
        assert cache.status() == want, T
