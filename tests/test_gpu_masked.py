"""GPU parity of mask-based generation (sep_attn_decode_masked) against the
oracle: the newest token attends over the full KV history with the kept set
of its row (the study's generate mask, section "SepAttention": the prefill
mask's rule for a query of length 1).  Outputs within the bf16 (max|d| <=
2e-2, RMS <= 2e-3) or fp32 (max|d| <= 1e-5) tolerance of the fp64 oracle;
lse within 2e-2 / 1e-5."""
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


def _inputs(seed, B, Hq, Hkv, S, D, dtype, p_sep):
    dt = "bf16" if dtype == torch.bfloat16 else "f32"
    g = synth.rng((seed, 41))
    q = synth.normal(g, (B, Hq, D), 1.0, dt)
    k = synth.normal(g, (B, Hkv, S, D), 1.0, dt)
    v = synth.normal(g, (B, Hkv, S, D), 1.0, dt)
    flags = synth.bernoulli_flags(synth.rng((seed, 42)), (B, S), p_sep)
    return q, k, v, flags


def _check(got, want, got_lse, want_lse, dtype, ctx):
    d = got.double().cpu().numpy() - want
    dl = got_lse.double().cpu().numpy() - want_lse
    if dtype == torch.float32:
        assert np.abs(d).max() <= 1e-5 and np.abs(dl).max() <= 1e-5, ctx
    else:
        assert np.abs(d).max() <= 2e-2 and np.sqrt((d * d).mean()) <= 2e-3, ctx
        assert np.abs(dl).max() <= 2e-2, ctx


CASES = [
    # B, Hq, Hkv, S, D, dtype, a, n, p_sep, history lengths T
    (3, 4, 2, 300, 64, torch.bfloat16, 4, 32, 0.1, [1, 2, 4, 5, 31, 32, 33, 36, 37, 100, 299, 300]),
    (2, 8, 1, 700, 128, torch.bfloat16, 0, 1, 0.2, [1, 2, 64, 65, 128, 129, 700]),
    (2, 4, 4, 200, 128, torch.bfloat16, 3, 200, 0.1, [1, 50, 199, 200]),  # window covers all
    (2, 2, 1, 500, 64, torch.bfloat16, 4, 16, 1.0, [17, 300, 500]),       # every token a separator
    (2, 8, 2, 333, 128, torch.float32, 4, 40, 0.15, [1, 5, 45, 46, 200, 333]),
    (1, 2, 2, 900, 64, torch.float32, 2, 8, 0.3, [9, 10, 600, 900]),      # > 8 splits: workspace merge
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "_".join(map(str, c[:8])))
def test_masked_generate(sl, case):
    B, Hq, Hkv, S, D, dtype, a, n, p_sep, lengths = case
    seed = B * 1000 + Hq * 100 + S + D
    q, k, v, flags = _inputs(seed, B, Hq, Hkv, S, D, dtype, p_sep)
    dq, dk, dv = q.cuda(), k.cuda(), v.cuda()
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    for T in lengths:
        out, lse = sl.decode_masked(dq, dk, dv, prefix, idx, T, a, n)
        want, want_lse = oracle.decode_masked(q, k, v, flags, T, a, n)
        _check(out, want, lse, want_lse, dtype, (T,))
    assert sl.device_status() == 0


def test_masked_equals_prefill_last_row(sl):
    # the same kept set, two independent kernels: the tensor-core prefill's
    # row T-1 and the gather decode
    B, Hq, Hkv, S, D = 2, 8, 2, 640, 128
    q, k, v, flags = _inputs(5, B, Hq, Hkv, S, D, torch.bfloat16, 0.1)
    T = S
    qf = torch.zeros((B, Hq, S, D), dtype=torch.bfloat16)
    qf[:, :, T - 1] = q
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    o1, l1 = sl.prefill(qf.cuda(), k.cuda(), v.cuda(), is_sep, prefix, idx, 4, 64)
    o2, l2 = sl.decode_masked(q.cuda(), k.cuda(), v.cuda(), prefix, idx, T, 4, 64)
    d = (o1[:, :, T - 1].float() - o2.float()).abs().max().item()
    assert d <= 2e-2
    assert (l1[:, :, T - 1] - l2).abs().max().item() <= 1e-2


def test_masked_llama3_8b_shape(sl):
    # 16 sequences with 8k-token histories, 32 q / 8 kv heads: sampled
    # sequences against the oracle
    B, Hq, Hkv, S, D, a, n = 16, 32, 8, 8192, 128, 4, 256
    q, k, v, flags = _inputs(11, B, Hq, Hkv, S, D, torch.bfloat16, 0.1)
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    dk, dv = k.cuda(), v.cuda()
    for T in (8192, 5000):
        out, lse = sl.decode_masked(q.cuda(), dk, dv, prefix, idx, T, a, n)
        for b in (0, 7, 15):
            want, want_lse = oracle.decode_masked(q[b:b + 1], k[b:b + 1], v[b:b + 1],
                                                  flags[b:b + 1], T, a, n)
            _check(out[b:b + 1], want, lse[b:b + 1], want_lse, torch.bfloat16, (T, b))
