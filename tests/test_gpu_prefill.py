"""GPU parity of the index and prefill path against the CPU oracle.

Every call goes through the C ABI (libsepattn.so via the thin binding).
Integer results (flags, prefix, idx, count, kept pairs) must match the
oracle bit-exactly; outputs must meet the stated tolerances against the
fp64 oracle: max|d| <= 1e-5 for fp32, max|d| <= 2e-2 and RMS <= 2e-3 for
bf16 (fp32 accumulation)."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

F32_MAX = 1e-5
BF16_MAX, BF16_RMS = 2e-2, 2e-3
LSE_MAX = 2e-2


@pytest.fixture(scope="module")
def sl():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    import streaming_kv_cache_sep_b200 as m
    return m


def _cuda(x):
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    return x.contiguous().cuda()


def _assert_close(got, want, dtype, what=""):
    got = got.double().cpu().numpy()
    d = got - want
    mx = float(np.abs(d).max()) if d.size else 0.0
    if dtype == "f32":
        assert mx <= F32_MAX, "%s max|d| %.3g" % (what, mx)
    else:
        rms = float(np.sqrt(np.mean(d * d))) if d.size else 0.0
        assert mx <= BF16_MAX and rms <= BF16_RMS, "%s max|d| %.3g rms %.3g" % (what, mx, rms)
    return mx


def _run_prefill(sl, inp, a=None, n=None):
    a = inp["a"] if a is None else a
    n = inp["n"] if n is None else n
    q, k, v = _cuda(inp["q"]), _cuda(inp["k"]), _cuda(inp["v"])
    is_sep = _cuda(inp["is_sep"])
    prefix, idx, count = sl.build_index(is_sep)
    out, lse = sl.prefill(q, k, v, is_sep, prefix, idx, a, n)
    torch.cuda.synchronize()
    assert sl.device_status() == 0
    return out, lse


# ------------------------------------------------------------------ index


def _index_cases():
    rng = np.random.default_rng(7)
    cases = []
    for name, cfg in synth.WORKLOADS.items():
        if cfg["kind"] != "prefill":
            continue
        inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name], S=min(cfg["S"], 20000))
        cases.append((name, inp["is_sep"]))
    for B, S, p in [(1, 1, 1.0), (1, 1, 0.0), (3, 16384, 0.5), (2, 16385, 0.1), (2, 40000, 0.02),
                    (1, 100, 0.0), (1, 100, 1.0)]:
        cases.append(("rand_%d_%d_%g" % (B, S, p), (rng.random((B, S)) < p).astype(np.uint8)))
    alt = np.zeros((2, 33000), np.uint8)
    alt[0, ::2] = 1
    alt[1, 16383:16386] = 1  # a run across the 16384-position chunk edge
    cases.append(("alternating_and_edge_run", alt))
    # several chunks with flag bytes other than 1 (any nonzero byte is a
    # separator): rows 16-byte aligned (S % 16 == 0) and not (S odd)
    for S in (40000, 40001):
        f = rng.choice(np.array([0, 0, 0, 0, 1, 2, 127, 128, 255], np.uint8), size=(2, S))
        cases.append(("nonzero_bytes_%d" % S, f))
    return cases


@pytest.mark.parametrize("case", _index_cases(), ids=lambda c: c[0])
def test_build_index_bit_exact(sl, case):
    _, flags = case
    prefix, idx, count = sl.build_index(_cuda(flags))
    p0, i0, c0 = oracle.build_index(flags)
    np.testing.assert_array_equal(prefix.cpu().numpy(), p0)
    np.testing.assert_array_equal(idx.cpu().numpy(), i0)
    np.testing.assert_array_equal(count.cpu().numpy(), c0)


@pytest.mark.parametrize("B,S,n_ids", [(8, 2048, 9), (1, 256, 9), (2, 16385, 3), (1, 40000, 32),
                                        (3, 1, 1), (2, 777, 5)])
def test_build_index_from_ids_bit_exact(sl, B, S, n_ids):
    """One-launch flags + index from token ids against the oracle's two steps."""
    g = np.random.default_rng(B * 100003 + S + n_ids)
    sep_ids = [int(x) for x in g.choice(1000, size=n_ids, replace=False)]
    ids = g.integers(0, 60, size=(B, S)).astype(np.int32)  # dense hits among ids < 60
    ids[:, ::7] = sep_ids[-1]
    flags, prefix, idx, count = sl.build_index_from_ids(_cuda(ids), sep_ids)
    want_flags = oracle.flags_from_ids(ids, sep_ids)
    p0, i0, c0 = oracle.build_index(want_flags)
    np.testing.assert_array_equal(flags.cpu().numpy(), want_flags)
    np.testing.assert_array_equal(prefix.cpu().numpy(), p0)
    np.testing.assert_array_equal(idx.cpu().numpy(), i0)
    np.testing.assert_array_equal(count.cpu().numpy(), c0)


def test_build_index_from_ids_workload(sl):
    name = "prefill_pythia160m_b8h12_s2048_d64_bf16"
    inp = synth.prefill_inputs(synth.WORKLOADS[name], synth.WORKLOAD_SEED[name])
    flags, prefix, idx, count = sl.build_index_from_ids(_cuda(inp["ids"]), list(inp["sep_ids"]))
    p0, i0, c0 = oracle.build_index(inp["is_sep"])
    np.testing.assert_array_equal(flags.cpu().numpy(), inp["is_sep"])
    np.testing.assert_array_equal(prefix.cpu().numpy(), p0)
    np.testing.assert_array_equal(idx.cpu().numpy(), i0)
    np.testing.assert_array_equal(count.cpu().numpy(), c0)


def test_flags_from_ids_bit_exact(sl):
    for name in ("prefill_tiny_b1h1_s256_d64_f32", "prefill_pythia160m_b8h12_s2048_d64_bf16"):
        cfg = synth.WORKLOADS[name]
        inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name])
        got = sl.flags_from_ids(_cuda(inp["ids"]), list(inp["sep_ids"]))
        want = oracle.flags_from_ids(inp["ids"], inp["sep_ids"])
        np.testing.assert_array_equal(got.cpu().numpy(), want)
        np.testing.assert_array_equal(want, inp["is_sep"])


@pytest.mark.parametrize("a,n", [(4, 32), (4, 64), (4, 256), (0, 1), (7, 1024), (5000, 3)])
def test_count_pairs_bit_exact(sl, a, n):
    flags = (np.random.default_rng(a + n).random((3, 3000)) < 0.1).astype(np.uint8)
    prefix, _, _ = sl.build_index(_cuda(flags))
    got = sl.count_pairs(prefix, a, n).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.count_pairs(flags, a, n))


def test_count_pairs_workloads(sl):
    for name, cfg in synth.WORKLOADS.items():
        if cfg["kind"] != "prefill" or cfg["S"] > 10000:
            continue
        inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name])
        prefix, _, _ = sl.build_index(_cuda(inp["is_sep"]))
        got = sl.count_pairs(prefix, cfg["a"], cfg["n"]).cpu().numpy()
        np.testing.assert_array_equal(got, oracle.count_pairs(inp["is_sep"], cfg["a"], cfg["n"]))


# ------------------------------------------------------------------ prefill fp32


@pytest.mark.parametrize("seed_off", [0, 1, 2])
def test_prefill_tiny_f32_full(sl, seed_off):
    name = "prefill_tiny_b1h1_s256_d64_f32"
    cfg = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name] + 100 * seed_off)
    out, lse = _run_prefill(sl, inp)
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], cfg["a"], cfg["n"])
    _assert_close(out, want, "f32", "out")
    assert float(np.abs(lse.double().cpu().numpy() - want_lse).max()) <= F32_MAX


@pytest.mark.parametrize("B,Hq,Hkv,S,D,a,n,p", [
    (2, 4, 2, 300, 64, 4, 32, 0.1), (1, 2, 1, 517, 128, 3, 100, 0.2), (1, 1, 1, 1, 32, 4, 1, 0.5),
    (1, 1, 1, 40, 64, 0, 1, 0.0), (1, 2, 2, 90, 128, 9, 200, 1.0)])
def test_prefill_f32_shapes(sl, B, Hq, Hkv, S, D, a, n, p):
    g = np.random.default_rng(S + D)
    inp = dict(q=torch.from_numpy(g.standard_normal((B, Hq, S, D), dtype=np.float32)),
               k=torch.from_numpy(g.standard_normal((B, Hkv, S, D), dtype=np.float32)),
               v=torch.from_numpy(g.standard_normal((B, Hkv, S, D), dtype=np.float32)),
               is_sep=(g.random((B, S)) < p).astype(np.uint8), a=a, n=n)
    out, lse = _run_prefill(sl, inp)
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], a, n)
    _assert_close(out, want, "f32")
    assert float(np.abs(lse.double().cpu().numpy() - want_lse).max()) <= F32_MAX


# ------------------------------------------------------------------ prefill bf16 (tcgen05)


def _bf16_case(B, Hq, Hkv, S, D, a, n, p, seed, std=1.0, flags=None):
    g = np.random.default_rng(seed)
    mk = lambda shape, k: synth.normal(synth.rng((seed, k)), shape, std, "bf16")
    is_sep = flags if flags is not None else (g.random((B, S)) < p).astype(np.uint8)
    return dict(q=mk((B, Hq, S, D), 1), k=mk((B, Hkv, S, D), 2), v=mk((B, Hkv, S, D), 3),
                is_sep=is_sep, a=a, n=n)


BF16_SHAPES = [
    # several tiles, ragged tail, GQA, both head dims
    (2, 4, 2, 300, 64, 4, 32, 0.1),
    (1, 4, 1, 1000, 128, 4, 256, 0.1),
    (1, 2, 2, 777, 128, 3, 64, 0.3),
    (2, 3, 3, 640, 64, 4, 64, 0.08),
    # degenerate cases
    (1, 1, 1, 1, 64, 4, 1, 0.5),        # one token
    (1, 2, 1, 129, 128, 0, 1, 0.0),     # each row keeps only itself
    (1, 2, 1, 400, 64, 4, 1000, 0.1),   # n >= S: dense causal
    (1, 2, 1, 400, 64, 0, 8, 1.0),      # all separators: dense causal
    (1, 2, 1, 500, 128, 4, 16, 0.0),    # no separators: sink + sliding window
    (1, 2, 2, 300, 64, 1000, 5, 0.1),   # a > S: every key is initial
    (1, 1, 1, 2000, 128, 4, 128, 0.15),  # many gathered blocks
]


@pytest.mark.parametrize("shape", BF16_SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_prefill_bf16_shapes(sl, shape):
    B, Hq, Hkv, S, D, a, n, p = shape
    inp = _bf16_case(B, Hq, Hkv, S, D, a, n, p, seed=S * 7 + D)
    out, lse = _run_prefill(sl, inp)
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], a, n)
    _assert_close(out, want, "bf16", "out")
    assert float(np.abs(lse.double().cpu().numpy() - want_lse).max()) <= LSE_MAX


def test_prefill_bf16_runs_of_separators(sl):
    name = "prefill_long_b1_s131072_d128_bf16"
    cfg = synth.WORKLOADS[name]
    g = synth.rng(5)
    flags = synth.run_flags(g, 1, 3000, cfg["p_single"], cfg["p_run_start"], cfg["run_len"])
    inp = _bf16_case(1, 4, 1, 3000, 128, 4, 300, 0.0, seed=11, flags=flags)
    out, lse = _run_prefill(sl, inp)
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], 4, 300)
    _assert_close(out, want, "bf16")


def test_prefill_pythia160m_full(sl):
    name = "prefill_pythia160m_b8h12_s2048_d64_bf16"
    cfg = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name])
    is_sep = sl.flags_from_ids(_cuda(inp["ids"]), list(inp["sep_ids"]))
    prefix, idx, _ = sl.build_index(is_sep)
    out, lse = sl.prefill(_cuda(inp["q"]), _cuda(inp["k"]), _cuda(inp["v"]), is_sep, prefix, idx,
                          cfg["a"], cfg["n"])
    torch.cuda.synchronize()
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], cfg["a"], cfg["n"])
    _assert_close(out, want, "bf16", "out")
    assert float(np.abs(lse.double().cpu().numpy() - want_lse).max()) <= LSE_MAX


def test_prefill_llama3_8k_full(sl):
    name = "prefill_llama3_8b_b1_s8192_d128_bf16"
    cfg = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name])
    out, lse = _run_prefill(sl, inp)
    want, want_lse = oracle.prefill(inp["q"], inp["k"], inp["v"], inp["is_sep"], cfg["a"], cfg["n"])
    _assert_close(out, want, "bf16", "out")
    assert float(np.abs(lse.double().cpu().numpy() - want_lse).max()) <= LSE_MAX


def _long_rows(S, Hq, rng):
    """Sampled query rows of the long workload: 96 random rows per head, every
    row of the first and last 128-row tiles of heads 0 and Hq-1, and whole
    tiles that straddle separator runs (chosen by the caller)."""
    rows = set()
    for h in range(Hq):
        for i in rng.choice(S, size=96, replace=False):
            rows.add(h * S + int(i))
    for h in (0, Hq - 1):
        for i in list(range(128)) + list(range(S - 128, S)):
            rows.add(h * S + i)
    return rows


def test_prefill_long_131k_sampled(sl):
    name = "prefill_long_b1_s131072_d128_bf16"
    cfg = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(cfg, synth.WORKLOAD_SEED[name])
    S, Hq = cfg["S"], cfg["Hq"]
    out, lse = _run_prefill(sl, inp)
    rng = np.random.default_rng(3)
    rows = _long_rows(S, Hq, rng)
    # two tiles that hold a run of 3 separators, in heads 5 and 17
    f = inp["is_sep"][0]
    runs = np.flatnonzero(f[:-2] & f[1:-1] & f[2:])
    for h, r in ((5, runs[len(runs) // 3]), (17, runs[2 * len(runs) // 3])):
        t0 = (int(r) // 128) * 128
        for i in range(t0, t0 + 128):
            rows.add(h * S + i)
    rows = np.array(sorted(rows), dtype=np.int64)
    want, want_lse = oracle.prefill_rows(inp["q"], inp["k"], inp["v"], inp["is_sep"], cfg["a"],
                                         cfg["n"], rows=rows)
    got = out.view(-1, cfg["D"])[torch.from_numpy(rows).cuda()]
    _assert_close(got, want, "bf16", "sampled rows")
    got_lse = lse.view(-1)[torch.from_numpy(rows).cuda()].double().cpu().numpy()
    assert float(np.abs(got_lse - want_lse).max()) <= LSE_MAX
    # every row is finite (a property that holds at any size)
    assert torch.isfinite(out.float()).all()


def test_prefill_repeatable_and_workspace_reuse(sl):
    inp = _bf16_case(1, 4, 2, 1500, 128, 4, 200, 0.1, seed=99)
    q, k, v = _cuda(inp["q"]), _cuda(inp["k"]), _cuda(inp["v"])
    is_sep = _cuda(inp["is_sep"])
    prefix, idx, _ = sl.build_index(is_sep)
    ws = torch.full((sl.prefill_workspace_bytes(1, 4, 2, 1500, 128, 1),), 255, dtype=torch.uint8,
                    device="cuda")  # NaN bit patterns everywhere
    o1, l1 = sl.prefill(q, k, v, is_sep, prefix, idx, 4, 200, workspace=ws)
    o2, l2 = sl.prefill(q, k, v, is_sep, prefix, idx, 4, 200, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.isfinite(o1.float()).all()
