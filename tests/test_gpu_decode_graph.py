"""The decode step exactly as the bench times it: the per-ring-slot CUDA graphs
of bench.DecodeWorkload (one fused sep_attn_decode_step launch per layer, the
layer-0 call also launching the step's bookkeeping), replayed token after
token over all 32 layers of the Llama-3-8B-shaped streaming workload
(B16, 32 query / 8 kv heads, D128, a4 s64 past128 w256), across three flushes
of the past window.

At checkpoints every layer's out and lse are compared with the oracle's fp64
attention over the rows the oracle's own four-block state machine retains
(K/V rebuilt on the host from the seeded per-token inputs), and the cache's
positions, flags, block sizes and K/V bytes with the oracle's, bit-exactly.
The per-token inputs come from the seeded host generator (a ring of 13, so
that a row at the wrong position holds different values), copied into the
workload's device ring before the graphs are captured."""
import numpy as np
import pytest
import torch

import bench
import oracle
import synth

pytestmark = pytest.mark.gpu

NAME = "decode_llama3_8b_b16_l32_t65536_d128_bf16"


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


class RingWorkload(bench.DecodeWorkload):
    RING = 13


def test_graph_replayed_decode_step_matches_oracle(sl):
    cfg = synth.WORKLOADS[NAME]
    a, s, past, w = cfg["a"], cfg["s"], cfg["past"], cfg["w"]
    seed = synth.WORKLOAD_SEED[NAME] + 17
    wl = RingWorkload(sl, NAME, seed)
    R, L, B, Hkv = wl.RING, wl.L, wl.B, wl.Hkv
    assert L == 32
    gen = dict(Hq=wl.Hq, Hkv=Hkv, D=wl.D, dtype="bf16", qkv_std=1.0, B=B)
    hq = torch.empty(tuple(wl.q.shape), dtype=torch.bfloat16)
    hk = torch.empty(tuple(wl.k.shape), dtype=torch.bfloat16)
    hv = torch.empty(tuple(wl.v.shape), dtype=torch.bfloat16)
    for r in range(R):
        for l in range(L):
            hq[r, l], hk[r, l], hv[r, l] = synth.decode_step_qkv(gen, seed, r, l)
    wl.q.copy_(hq)
    wl.k.copy_(hk)
    wl.v.copy_(hv)

    flushes = [a + w + k * (past + 1) - 1 for k in (1, 2, 3)]  # 388, 517, 646
    checks = sorted({40, 41} | {t + d for t in flushes for d in (-1, 0, 1)} | {700})
    T = checks[-1] + 1
    flags = wl.flags_host[:T]
    snap = oracle.sepcache_simulate(flags, a, s, past, w, checks)

    for _ in range(40):  # eager steps, then the graphs the bench replays
        wl.eager_step()
    wl.capture()
    k = 0
    kv_layers = (0, 13, L - 1)
    while wl.t < T:
        t = wl.t
        wl.graph_step()
        if t != checks[k]:
            continue
        torch.cuda.synchronize()
        c = wl.cache
        np.testing.assert_array_equal(c.counts.cpu().numpy(), snap["counts"][k], err_msg=str(t))
        np.testing.assert_array_equal(c.pos.cpu().numpy(), snap["pos"][k], err_msg=str(t))
        np.testing.assert_array_equal(c.flag.cpu().numpy(), snap["flag"][k], err_msg=str(t))
        out = wl.out.double().cpu().numpy()
        lse = wl.lse.double().cpu().numpy()
        r = t % R
        for b in range(B):
            n = int(snap["counts"][k, b].sum())
            pos = snap["pos"][k, b, :n]
            ring_idx = torch.as_tensor(pos % R, dtype=torch.long)
            for l in range(L):
                kr = hk[ring_idx, l, b].transpose(0, 1).contiguous()  # [Hkv, n, D]
                vr = hv[ring_idx, l, b].transpose(0, 1).contiguous()
                if l in kv_layers:
                    assert torch.equal(c.k[l, b, :, :n].cpu(), kr), (t, l, b)
                    assert torch.equal(c.v[l, b, :, :n].cpu(), vr), (t, l, b)
                want, want_lse = oracle.attend(hq[r, l, b], kr, vr)
                d = out[l, b] - want
                assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3, (t, l, b)
                assert np.abs(lse[l, b] - want_lse).max() <= 2e-2, (t, l, b)
        k += 1
    assert k == len(checks)
    assert wl.cache.status() == 0
    assert sl.device_status() == 0
    del wl.graphs
