"""GPU parity of the Sep-Attention backward (sep_attn_backward) against the
fp64 oracle (gradients of sum(out * dout), out recomputed in fp64).

Tolerance (derived from the arithmetic; the pages state none for gradients):
the inputs are bf16 and read exactly; the kernel rounds P and dS to bf16 for
the tensor-core products (2^-9 relative each) and takes delta from the bf16
forward output, and every gradient element is a sum of many such terms with
fp32 accumulation.  So each gradient tensor X must satisfy
  RMS(X_gpu - X_ref) <= 1e-2 * RMS(X_ref)  and
  max|X_gpu - X_ref| <= 5e-2 * max|X_ref|
(about five times the bf16 rounding of one term)."""
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


def _run(sl, B, Hq, Hkv, S, D, a, n, p_sep, seed, std=1.0):
    g = synth.rng((seed, 61))
    q = synth.normal(g, (B, Hq, S, D), std, "bf16")
    k = synth.normal(g, (B, Hkv, S, D), std, "bf16")
    v = synth.normal(g, (B, Hkv, S, D), 1.0, "bf16")
    dout = synth.normal(g, (B, Hq, S, D), 1.0, "bf16")
    flags = synth.bernoulli_flags(synth.rng((seed, 62)), (B, S), p_sep)
    dq_, dk_, dv_ = q.cuda(), k.cuda(), v.cuda()
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    out, lse = sl.prefill(dq_, dk_, dv_, is_sep, prefix, idx, a, n)
    gq, gk, gv = sl.backward(dq_, dk_, dv_, out, lse, dout.cuda(), is_sep, prefix, idx, a, n)
    torch.cuda.synchronize()
    assert sl.device_status() == 0
    ref = oracle.prefill_backward(q, k, v, dout, flags, a, n)
    return (gq, gk, gv), ref


def _check(got, ref, ctx):
    worst = []
    for name, x, r in zip("qkv", got, ref):
        d = x.double().cpu().numpy() - r
        rms_ref = np.sqrt((r * r).mean())
        rms = np.sqrt((d * d).mean())
        mx = np.abs(d).max()
        worst.append((name, rms / max(rms_ref, 1e-30), mx / max(np.abs(r).max(), 1e-30)))
        assert rms <= 1e-2 * rms_ref + 1e-6, (ctx, name, rms, rms_ref)
        assert mx <= 5e-2 * np.abs(r).max() + 1e-5, (ctx, name, mx, np.abs(r).max())
    return worst


CASES = [
    # B, Hq, Hkv, S, D, a, n, p_sep
    (1, 1, 1, 64, 64, 4, 16, 0.1),
    (2, 4, 2, 200, 64, 4, 32, 0.1),      # ragged tail, GQA
    (2, 8, 2, 333, 128, 3, 40, 0.15),
    (1, 4, 4, 257, 128, 0, 1, 0.3),      # window of the query alone
    (1, 2, 1, 300, 64, 4, 300, 0.1),     # dense causal (n >= S)
    (1, 2, 2, 190, 64, 2, 8, 1.0),       # every token a separator
    (1, 4, 1, 600, 128, 4, 64, 0.0),     # no separators: sinks + window
    (2, 8, 8, 700, 64, 4, 100, 0.08),    # many chunks of global keys
    (1, 8, 2, 430, 128, 4, 48, 0.12),    # GQA, short window, last tile under 64 rows
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "_".join(map(str, c)))
def test_backward_small(sl, case):
    B, Hq, Hkv, S, D, a, n, p = case
    got, ref = _run(sl, B, Hq, Hkv, S, D, a, n, p, seed=S + D + n)
    print(case, _check(got, ref, case))


def test_backward_pythia160m_shape(sl):
    # B8, 12 heads (MHA), D64, S2048, a=4, n=64, 8 % separators, data / 8
    got, ref = _run(sl, 8, 12, 12, 2048, 64, 4, 64, 0.08, seed=1002, std=1.0 / 8.0)
    print(_check(got, ref, "pythia"))


def test_backward_llama3_8b_shape(sl):
    # the bench's Llama-3-8B shape: B1, 32 query / 8 kv heads, D128, S8192,
    # a=4, n=256, 10 % separators; every element of dq, dk and dv checked
    got, ref = _run(sl, 1, 32, 8, 8192, 128, 4, 256, 0.1, seed=1003)
    print(_check(got, ref, "llama3-8k"))
