"""GPU parity of prompt ingestion (sepcache_ingest) against the oracle.

Ingesting a T-token prompt into an empty cache must leave exactly the state
T sequential appends leave: the oracle's four-block state machine run over
the prompt's flags gives the retained positions, flags and block sizes
(compared bit-exactly), and every retained K/V row must hold the prompt's
row at its position.  Streaming then continues with fused decode steps,
checked like the cache tests (state bit-exact, outputs within the bf16 /
fp32 tolerance against fp64 oracle attention)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


def _flags(seed, B, T, p=0.15):
    return synth.bernoulli_flags(synth.rng((seed, 21)), (B, T), p)


def _prompt(seed, layers, B, Hkv, T, D, dtype):
    dt = "bf16" if dtype == torch.bfloat16 else "f32"
    g = synth.rng((seed, 22))
    k = torch.stack([synth.normal(g, (B, Hkv, T, D), 1.0, dt) for _ in range(layers)])
    v = torch.stack([synth.normal(g, (B, Hkv, T, D), 1.0, dt) for _ in range(layers)])
    return k, v


def _check_state(cache, snap, k_snap, B, layers, kv_of):
    np.testing.assert_array_equal(cache.counts.cpu().numpy(), snap["counts"][k_snap])
    np.testing.assert_array_equal(cache.pos.cpu().numpy(), snap["pos"][k_snap])
    np.testing.assert_array_equal(cache.flag.cpu().numpy(), snap["flag"][k_snap])
    K, V = cache.k.cpu(), cache.v.cpu()
    for b in range(B):
        n = int(snap["counts"][k_snap, b].sum())
        pos = snap["pos"][k_snap, b, :n]
        for l in range(layers):
            kr, vr = kv_of(l, b, pos)
            assert torch.equal(K[l, b, :, :n], kr), (b, l)
            assert torch.equal(V[l, b, :, :n], vr), (b, l)


CASES = [
    # a, s, past, w, B, Hkv, Hq, D, dtype, prompt lengths
    (4, 8, 6, 10, 3, 2, 4, 64, torch.bfloat16, [1, 3, 4, 5, 14, 15, 20, 21, 22, 27, 28, 29, 200]),
    (1, 2, 2, 2, 2, 1, 2, 128, torch.bfloat16, [1, 2, 3, 5, 6, 7, 40]),
    (0, 5, 3, 4, 2, 2, 2, 64, torch.float32, [1, 4, 5, 8, 9, 60]),
    (4, 0, 0, 16, 2, 1, 8, 128, torch.bfloat16, [3, 20, 21, 100]),     # StreamingLLM case
    (2, 3, 0, 5, 3, 2, 2, 64, torch.bfloat16, [7, 8, 9, 50]),          # flush on every slide
    (3, 40, 100, 30, 2, 2, 4, 128, torch.float32, [133, 134, 300]),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "_".join(map(str, c[:8])))
def test_ingest_equals_sequential_appends(sl, case):
    a, s, past, w, B, Hkv, Hq, D, dtype, lengths = case
    layers = 2
    seed = a * 1000 + s * 100 + past * 10 + w
    Tmax = max(lengths)
    flags = _flags(seed, B, Tmax)
    kp, vp = _prompt(seed, layers, B, Hkv, Tmax, D, dtype)
    snap = oracle.sepcache_simulate(flags.T.copy(), a, s, past, w, np.asarray(lengths) - 1)
    for i, T in enumerate(lengths):
        cache = sl.SepCache(a, s, past, w, layers, B, Hkv, D, dtype=dtype)
        is_sep = torch.from_numpy(np.ascontiguousarray(flags[:, :T])).cuda()
        prefix, idx, _ = sl.build_index(is_sep)
        k = kp[:, :, :, :T].contiguous().cuda()
        v = vp[:, :, :, :T].contiguous().cuda()
        for l in range(layers):
            cache.ingest(l, k[l], v[l], is_sep, prefix, idx)
        assert int(cache.step.min()) == T and int(cache.step.max()) == T

        def kv_of(l, b, pos):
            return kp[l, b][:, pos].contiguous(), vp[l, b][:, pos].contiguous()

        _check_state(cache, snap, i, B, layers, kv_of)
        assert cache.status() == 0


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("case", [CASES[0], CASES[3], CASES[5]], ids=lambda c: "_".join(map(str, c[:8])))
def test_ingest_then_stream(sl, case, fused):
    """Ingest a prompt, then decode N more tokens: the state follows the
    oracle's sequential run over prompt + new tokens, and the decode output
    matches fp64 attention over the retained rows."""
    a, s, past, w, B, Hkv, Hq, D, dtype, lengths = case
    layers, T, N = 2, lengths[-1], 3 * (past + 1) + 7
    seed = 7 + a + s + past + w
    flags = _flags(seed, B, T + N)
    kp, vp = _prompt(seed, layers, B, Hkv, T, D, dtype)
    dt = "bf16" if dtype == torch.bfloat16 else "f32"
    wl = dict(Hq=Hq, Hkv=Hkv, D=D, dtype=dt, qkv_std=1.0, B=B)
    new = [[synth.decode_step_qkv(wl, seed, t, l) for l in range(layers)] for t in range(N)]
    snap = oracle.sepcache_simulate(flags.T.copy(), a, s, past, w, np.arange(T - 1, T + N))
    cache = sl.SepCache(a, s, past, w, layers, B, Hkv, D, dtype=dtype)
    is_sep = torch.from_numpy(np.ascontiguousarray(flags[:, :T])).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    k, v = kp[:, :, :, :T].contiguous().cuda(), vp[:, :, :, :T].contiguous().cuda()
    for l in range(layers):
        cache.ingest(l, k[l], v[l], is_sep, prefix, idx)

    def kv_of(l, b, pos):
        ks, vs = [], []
        for p in pos:
            if p < T:
                ks.append(kp[l, b, :, p])
                vs.append(vp[l, b, :, p])
            else:
                ks.append(new[p - T][l][1][b])
                vs.append(new[p - T][l][2][b])
        return torch.stack(ks, 1), torch.stack(vs, 1)

    _check_state(cache, snap, 0, B, layers, kv_of)
    dflags = torch.from_numpy(np.ascontiguousarray(flags.T)).cuda()
    for t in range(N):
        outs = {}
        for l in range(layers):
            q, kn, vn = (x.cuda() for x in new[t][l])
            f = dflags[T + t] if l == 0 else None
            if fused:
                outs[l] = cache.decode_step(l, q, kn, vn, f)
            else:
                cache.append(l, kn, vn, f)
                cache.compact(l)
                outs[l] = cache.decode(l, q)
        _check_state(cache, snap, t + 1, B, layers, kv_of)
        for l, (out, lse) in outs.items():
            got = out.double().cpu().numpy()
            for b in range(B):
                n = int(snap["counts"][t + 1, b].sum())
                kr, vr = kv_of(l, b, snap["pos"][t + 1, b, :n])
                want, want_lse = oracle.attend(new[t][l][0][b], kr, vr)
                d = got[b] - want
                if dt == "f32":
                    assert np.abs(d).max() <= 1e-5
                else:
                    assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3, (t, l, b)
                assert np.abs(lse.double().cpu().numpy()[b] - want_lse).max() <= (
                    1e-5 if dt == "f32" else 2e-2)
    assert cache.status() == 0


def test_ingest_llama3_8b_shape(sl):
    """The decode workload's cache sizes (a=4, s=64, past=128, w=256; B=16,
    8 kv heads, D=128): a 6000-token prompt (dozens of flushes, the
    separator cache full) ingested at 2 layers."""
    cfg = synth.WORKLOADS["decode_llama3_8b_b16_l32_t65536_d128_bf16"]
    a, s, past, w = cfg["a"], cfg["s"], cfg["past"], cfg["w"]
    B, Hkv, D, layers, T = cfg["B"], cfg["Hkv"], cfg["D"], 2, 6000
    seed = synth.WORKLOAD_SEED["decode_llama3_8b_b16_l32_t65536_d128_bf16"] + 3
    flags = synth.bernoulli_flags(synth.rng((seed, 21)), (B, T), 0.1)
    kp, vp = _prompt(seed, layers, B, Hkv, T, D, torch.bfloat16)
    snap = oracle.sepcache_simulate(flags.T.copy(), a, s, past, w, [T - 1])
    cache = sl.SepCache(a, s, past, w, layers, B, Hkv, D, dtype=torch.bfloat16)
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    k, v = kp.cuda(), vp.cuda()
    for l in range(layers):
        cache.ingest(l, k[l], v[l], is_sep, prefix, idx)

    def kv_of(l, b, pos):
        return kp[l, b][:, pos].contiguous(), vp[l, b][:, pos].contiguous()

    _check_state(cache, snap, 0, B, layers, kv_of)
    assert int(cache.counts[:, 1].min()) == s  # the separator cache is full
    assert cache.status() == 0


def test_ingest_refuses_a_non_empty_cache(sl):
    a, s, past, w, B, Hkv, D = 2, 3, 2, 4, 2, 1, 64
    cache = sl.SepCache(a, s, past, w, 1, B, Hkv, D, dtype=torch.bfloat16)
    kn = torch.zeros((B, Hkv, D), dtype=torch.bfloat16, device="cuda")
    cache.append(0, kn, kn, torch.ones((B,), dtype=torch.uint8, device="cuda"))
    before = (cache.counts.clone(), cache.pos.clone(), cache.step.clone())
    T = 10
    is_sep = torch.ones((B, T), dtype=torch.uint8, device="cuda")
    prefix, idx, _ = sl.build_index(is_sep)
    k = torch.ones((B, Hkv, T, D), dtype=torch.bfloat16, device="cuda")
    cache.ingest(0, k, k, is_sep, prefix, idx)
    assert torch.equal(cache.counts, before[0]) and torch.equal(cache.pos, before[1])
    assert torch.equal(cache.step, before[2])
    assert cache.status() != 0
