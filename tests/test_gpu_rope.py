"""GPU parity of positional-encoding shifting in streaming decode.

The streaming setting needs positional-encoding shifting (HKUDS047 SepLLM
study, section on the three versions; section "Streaming-SepLLM": the Llama
positional-encoding-shifting module).  With a rotary base set on the cache,
keys are cached un-encoded, and each decode encodes retained key r at its
slot r inside the cache and the query at the newest slot.  The CUDA path
(sepcache_set_rope + the decode calls) is compared with the oracle's
decode_shifted, which encodes in fp64, over the retained rows that the
oracle's own state machine lists.  Tolerances: bf16 max|d| <= 2e-2 and RMS
<= 2e-3 (the encoded q and keys are rounded to bf16 for the tensor cores,
as the unencoded ones already are); fp32 max|d| <= 1e-5."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from test_gpu_cache import RING, SMALL, Stream, _check_kv, _check_meta

pytestmark = pytest.mark.gpu

THETA = {64: 10000.0, 128: 500000.0}  # Llama-2 and Llama-3 rotary bases


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


def _check_shifted(st, snap, k, outs, t, theta):
    r = t % RING
    for l, (out, lse) in outs.items():
        got = out.double().cpu().numpy()
        got_lse = lse.double().cpu().numpy()
        for b in range(st.B):
            n = int(snap["counts"][k, b].sum())
            kr, vr = st.kv_rows(l, snap["pos"][k, b, :n], b)
            want, want_lse = oracle.decode_shifted(st.ring_q[l][r, b], kr, vr, theta)
            d = got[b] - want
            if st.dt == "f32":
                assert np.abs(d).max() <= 1e-5, (t, l, b)
                assert np.abs(got_lse[b] - want_lse).max() <= 1e-5
            else:
                assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3, (t, l, b)
                assert np.abs(got_lse[b] - want_lse).max() <= 2e-2


ROPE_CASES = SMALL + [
    (4, 32, 64, 64, 2, 2, 8, 64, torch.bfloat16),    # > 128 rows: several chunks per CTA
    (4, 24, 40, 100, 2, 1, 1, 128, torch.bfloat16),  # G = 1, several chunks
]


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("shape", ROPE_CASES, ids=lambda s: "_".join(map(str, s[:8])))
def test_rope_small_caches(sl, shape, fused):
    a, s, past, w, B, Hkv, Hq, D, dtype = shape
    theta = THETA[D]
    T = 330
    st = Stream(sl, a, s, past, w, B, Hkv, Hq, D, 2, dtype, seed=7 + a * 100 + s + past + w, T=T,
                fused=fused)
    st.cache.set_rope(theta)
    assert st.cache.rope_theta == theta
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T))
    for t in range(T):
        dec = (0, 1) if (t < 24 or t % 5 == 0 or t > T - 40) else ()
        outs = st.step(decode_layers=dec)
        _check_meta(st, snap, t)
        if t % 41 == 0:
            _check_kv(st, snap, t)  # the cache keeps the un-encoded keys
        if dec:
            _check_shifted(st, snap, t, outs, t, theta)
    assert st.cache.status() == 0
    assert sl.device_status() == 0


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_rope_llama3_8b_shape(sl, fused):
    name = "decode_llama3_8b_b16_l32_t65536_d128_bf16"
    cfg = synth.WORKLOADS[name]
    a, s, past, w = cfg["a"], cfg["s"], cfg["past"], cfg["w"]
    T = 1300
    st = Stream(sl, a, s, past, w, cfg["B"], cfg["Hkv"], cfg["Hq"], cfg["D"], 2, torch.bfloat16,
                seed=synth.WORKLOAD_SEED[name] + 2, T=T, fused=fused)
    st.cache.set_rope(500000.0)
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T))
    flushes = {a + w + k * (past + 1) - 1 for k in range(1, 10)}
    near = {t + d for t in flushes for d in (-1, 0, 1)}
    for t in range(T):
        dec = (0, 1) if (t in near or t % 113 == 0 or t < 4 or t == T - 1) else ()
        outs = st.step(decode_layers=dec)
        if dec:
            _check_meta(st, snap, t)
            _check_shifted(st, snap, t, outs, t, 500000.0)
    assert st.cache.status() == 0


def test_rope_noalloc_and_switch_off(sl):
    a, s, past, w, B, Hkv, Hq, D = 4, 16, 32, 48, 2, 2, 8, 128
    T = 150
    st = Stream(sl, a, s, past, w, B, Hkv, Hq, D, 1, torch.bfloat16, seed=99, T=T)
    st.cache.set_rope(500000.0)
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, [T - 1])
    for _ in range(T):
        st.step()
    r = (T - 1) % RING
    q = st.dq[0][r]
    o1, l1 = st.cache.decode(0, q)
    o2, l2 = st.cache.decode_noalloc(0, q)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    _check_shifted(st, snap, 0, {0: (o1, l1)}, T - 1, 500000.0)
    # switched off, the same rows are read as already encoded
    st.cache.set_rope(0.0)
    o3, l3 = st.cache.decode(0, q)
    for b in range(B):
        n = int(snap["counts"][0, b].sum())
        kr, vr = st.kv_rows(0, snap["pos"][0, b, :n], b)
        want, _ = oracle.attend(st.ring_q[0][r, b], kr, vr)
        d = o3[b].double().cpu().numpy() - want
        assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3


@pytest.mark.parametrize("D", [64, 128])
def test_rope_table(sl, D):
    c = sl.SepCache(4, 8, 8, 8, 1, 1, 1, D)
    theta = THETA[D]
    c.set_rope(theta)
    rows = c.c.rope_rows
    tab = c._view(c.c.rope, (rows, D // 2, 2), torch.float32).double().cpu().numpy()
    # (cos, sin) of r * theta^(-2i/D), rounded to fp32 from fp64
    i = np.arange(D // 2)
    phi = np.arange(rows)[:, None] * np.power(float(theta), -2.0 * i / D)[None, :]
    np.testing.assert_allclose(tab[..., 0], np.cos(phi), atol=2 ** -24)
    np.testing.assert_allclose(tab[..., 1], np.sin(phi), atol=2 ** -24)
    assert rows == 65 and math.isclose(c.rope_theta, theta)
