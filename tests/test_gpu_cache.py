"""GPU parity of the streaming SepCache (append / compact / decode) against
the CPU oracle's four-block state machine and fp64 attention.

Cache contents are compared bit-exactly: the positions, flags and block
sizes after every checked step, and the K/V bytes of every retained row
(each row must hold the K/V of the token at its position).  Decode outputs
must meet the bf16 tolerance (max|d| <= 2e-2, RMS <= 2e-3) or the fp32 one
(max|d| <= 1e-5) against oracle attention over the retained positions the
oracle itself computes."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

RING = 97  # distinct per-step inputs, cycled by step


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


class Stream:
    """Drive a SepCache through the C ABI with ring-cycled synthetic inputs."""

    def __init__(self, sl, a, s, past, w, B, Hkv, Hq, D, layers, dtype, seed, T, fused=False,
                 mode=0):
        self.fused = fused
        self.sl = sl
        self.cfg = dict(a=a, s=s, past=past, w=w)
        self.B, self.Hkv, self.Hq, self.D, self.layers = B, Hkv, Hq, D, layers
        self.dt = "bf16" if dtype == torch.bfloat16 else "f32"
        wl = dict(Hq=Hq, Hkv=Hkv, D=D, dtype=self.dt, qkv_std=1.0, B=B)
        self.ring_q, self.ring_k, self.ring_v = [], [], []
        for l in range(layers):
            qs, ks, vs = zip(*[synth.decode_step_qkv(wl, seed, r, l) for r in range(RING)])
            self.ring_q.append(torch.stack(qs))
            self.ring_k.append(torch.stack(ks))
            self.ring_v.append(torch.stack(vs))
        self.dq = [x.cuda() for x in self.ring_q]
        self.dk = [x.cuda() for x in self.ring_k]
        self.dv = [x.cuda() for x in self.ring_v]
        self.flags = synth.bernoulli_flags(synth.rng((seed, 10)), (T, B), 0.1)
        self.dflags = torch.from_numpy(self.flags).cuda()
        self.cache = sl.SepCache(a, s, past, w, layers, B, Hkv, D, dtype=dtype, mode=mode)
        self.t = 0

    def step(self, decode_layers=()):
        t, r = self.t, self.t % RING
        outs = {}
        for l in range(self.layers):
            f = self.dflags[t] if l == 0 else None
            if self.fused:  # one launch per layer: append + compact + decode
                o = self.cache.decode_step(l, self.dq[l][r], self.dk[l][r], self.dv[l][r], f)
                if l in decode_layers:
                    outs[l] = o
                continue
            self.cache.append(l, self.dk[l][r], self.dv[l][r], f)
            self.cache.compact(l)
            if l in decode_layers:
                outs[l] = self.cache.decode(l, self.dq[l][r])
        self.t += 1
        return outs

    def kv_rows(self, l, positions, b):
        """K/V of the tokens at `positions` for sequence b: [Hkv, n, D]."""
        idx = torch.as_tensor(positions % RING, dtype=torch.long)
        k = self.ring_k[l][idx, b]  # [n, Hkv, D]
        v = self.ring_v[l][idx, b]
        return k.transpose(0, 1).contiguous(), v.transpose(0, 1).contiguous()


def _check_meta(st, snap, k):
    c = st.cache
    cnt = c.counts.cpu().numpy()
    np.testing.assert_array_equal(cnt, snap["counts"][k])
    np.testing.assert_array_equal(c.pos.cpu().numpy(), snap["pos"][k])
    np.testing.assert_array_equal(c.flag.cpu().numpy(), snap["flag"][k])
    return cnt


def _check_kv(st, snap, k):
    c = st.cache
    K, V = c.k.cpu(), c.v.cpu()
    for b in range(st.B):
        n = int(snap["counts"][k, b].sum())
        pos = snap["pos"][k, b, :n]
        for l in range(st.layers):
            kr, vr = st.kv_rows(l, pos, b)
            assert torch.equal(K[l, b, :, :n], kr), (k, b, l)
            assert torch.equal(V[l, b, :, :n], vr), (k, b, l)


def _check_decode(st, snap, k, outs, t):
    r = t % RING
    for l, (out, lse) in outs.items():
        got = out.double().cpu().numpy()
        got_lse = lse.double().cpu().numpy()
        for b in range(st.B):
            n = int(snap["counts"][k, b].sum())
            kr, vr = st.kv_rows(l, snap["pos"][k, b, :n], b)
            want, want_lse = oracle.attend(st.ring_q[l][r, b], kr, vr)
            d = got[b] - want
            if st.dt == "f32":
                assert np.abs(d).max() <= 1e-5
                assert np.abs(got_lse[b] - want_lse).max() <= 1e-5
            else:
                assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3, (t, l, b)
                assert np.abs(got_lse[b] - want_lse).max() <= 2e-2


SMALL = [
    # a, s, past, w, B, Hkv, Hq, D, dtype
    (4, 8, 6, 10, 3, 2, 4, 64, torch.bfloat16),
    (1, 2, 2, 2, 2, 1, 2, 128, torch.bfloat16),
    (0, 5, 3, 4, 2, 2, 2, 64, torch.float32),
    (4, 0, 0, 16, 2, 1, 8, 128, torch.bfloat16),   # StreamingLLM special case
    (2, 3, 0, 5, 3, 2, 2, 64, torch.bfloat16),     # flush on every slide
    (3, 40, 100, 30, 2, 2, 4, 128, torch.float32),  # more than 64 rows: split decode
]


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "_".join(map(str, s[:8])))
def test_small_caches_every_step(sl, shape, fused):
    a, s, past, w, B, Hkv, Hq, D, dtype = shape
    T = 400
    st = Stream(sl, a, s, past, w, B, Hkv, Hq, D, 2, dtype, seed=a * 100 + s + past + w, T=T,
                fused=fused)
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T))
    for t in range(T):
        outs = st.step(decode_layers=(0, 1))
        _check_meta(st, snap, t)
        if t % 7 == 0 or t < 40:
            _check_kv(st, snap, t)
        _check_decode(st, snap, t, outs, t)
    assert st.cache.status() == 0
    assert sl.device_status() == 0


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_fp32_more_than_eight_splits_every_step(sl, fused):
    """An exact (fp32) cache of up to 643 rows: ten 64-row splits, merged
    through the workspace by the last split to finish; on flush steps the
    fused step's rows move in place only after every split has read its
    sources.  Late in the stream the sequences retain more than 512 rows."""
    a, s, past, w, B, Hkv, Hq, D = 2, 160, 40, 440, 2, 1, 2, 64
    T = 1300
    st = Stream(sl, a, s, past, w, B, Hkv, Hq, D, 2, torch.float32, seed=7777, T=T, fused=fused)
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T))
    flushes = {a + w + k * (past + 1) - 1 for k in range(1, 40)}
    for t in range(T):
        dec = (0, 1) if (t % 7 == 0 or t in flushes or t + 1 in flushes) else ()
        outs = st.step(decode_layers=dec)
        _check_meta(st, snap, t)
        if t % 13 == 0 or t in flushes:
            _check_kv(st, snap, t)
        if dec:
            _check_decode(st, snap, t, outs, t)
    assert int(snap["counts"][T - 1].sum(1).min()) > 8 * 64
    assert st.cache.status() == 0
    assert sl.device_status() == 0


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_llama3_8b_shape_first_2000_steps(sl, fused):
    cfg = synth.WORKLOADS["decode_llama3_8b_b16_l32_t65536_d128_bf16"]
    a, s, past, w = cfg["a"], cfg["s"], cfg["past"], cfg["w"]
    T = 2000
    st = Stream(sl, a, s, past, w, cfg["B"], cfg["Hkv"], cfg["Hq"], cfg["D"], 2, torch.bfloat16,
                seed=synth.WORKLOAD_SEED["decode_llama3_8b_b16_l32_t65536_d128_bf16"], T=T,
                fused=fused)
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, np.arange(T))
    flushes = {a + w + k * (past + 1) - 1 for k in range(1, 20)}
    near_flush = {t + d for t in flushes for d in (-2, -1, 0, 1, 2)}
    for t in range(T):
        dec = (0, 1) if (t in near_flush or t % 97 == 0 or t < 8) else ()
        outs = st.step(decode_layers=dec)
        _check_meta(st, snap, t)
        if t in near_flush or t % 251 == 0:
            _check_kv(st, snap, t)
        if dec:
            _check_decode(st, snap, t, outs, t)
    assert st.cache.status() == 0


def test_llama3_8b_shape_full_stream_checkpoints(sl):
    cfg = synth.WORKLOADS["decode_llama3_8b_b16_l32_t65536_d128_bf16"]
    a, s, past, w, T = cfg["a"], cfg["s"], cfg["past"], cfg["w"], cfg["T"]
    st = Stream(sl, a, s, past, w, cfg["B"], cfg["Hkv"], cfg["Hq"], cfg["D"], 2, torch.bfloat16,
                seed=synth.WORKLOAD_SEED["decode_llama3_8b_b16_l32_t65536_d128_bf16"] + 1, T=T,
                fused=True)
    checks = sorted(set([1000, 4095, 4096, 10000, 32767, 40000, 65534, T - 1] +
                        [a + w + k * (past + 1) - 1 for k in (100, 300, 505)]))
    snap = oracle.sepcache_simulate(st.flags, a, s, past, w, checks)
    k = 0
    for t in range(T):
        want_check = k < len(checks) and checks[k] == t
        outs = st.step(decode_layers=(0, 1) if want_check else ())
        if want_check:
            _check_meta(st, snap, k)
            _check_kv(st, snap, k)
            _check_decode(st, snap, k, outs, t)
            k += 1
    assert k == len(checks)
    assert st.cache.status() == 0
    # retained length never exceeds a+s+past+w and stays near the simulated mean
    assert int(st.cache.counts.sum(1).max()) <= a + s + past + w
