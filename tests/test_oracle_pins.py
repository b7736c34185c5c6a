"""Pins of the CPU oracle to facts fixed outside it (run without a GPU).

Each test checks the oracle against something it does not share code with:
hand-worked fixtures, library routines (torch's fp64 attention and softmax,
numpy's cumsum / flatnonzero / isin), closed forms, special cases that
reduce to known methods (dense causal attention; attention sinks plus a
sliding window) and brute force on tiny inputs.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(size=shape).astype(np.float32)


def _torch_attention(q, k, v, mask, scale):
    """fp64 softmax attention through torch, GQA by repeating kv heads.
    mask: bool [S,S] (True = attend) or None for plain causal."""
    q = torch.from_numpy(q).double()
    k = torch.from_numpy(k).double()
    v = torch.from_numpy(v).double()
    G = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(G, dim=1)
    v = v.repeat_interleave(G, dim=1)
    if mask is None:
        out = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=scale)
        S = q.shape[2]
        mask = torch.ones(S, S, dtype=torch.bool).tril()
    else:
        out = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=scale)
    scores = (q @ k.transpose(-1, -2)) * scale
    lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1)
    return out.numpy(), lse.numpy()


def _page_mask(flags_row, a, n):
    """Mask built the way the pages describe build_prefill_mask: start empty,
    set the separator columns, set the first a columns, add the local
    triangular band of width n, then AND with the lower-triangular causal
    mask (HKUDS047 SepLLM study, section "SepAttention")."""
    S = flags_row.shape[0]
    m = torch.zeros(S, S, dtype=torch.bool)
    m[:, torch.from_numpy(flags_row.astype(bool))] = True
    m[:, :a] = True
    ones = torch.ones(S, S, dtype=torch.bool)
    band = ones.tril(0) & ~ones.tril(-n)
    m |= band
    return m & ones.tril(0)


# ---------------------------------------------------------------- golden


def _read_mask_golden():
    rows, meta = [], {}
    with open(os.path.join(GOLD, "mask_s10_a2_n3.txt")) as fh:
        for line in fh:
            line = line.strip()
            if line.startswith("# a="):
                for kv in line[2:].split():
                    k_, v_ = kv.split("=")
                    meta[k_] = v_
            elif line and not line.startswith("#"):
                rows.append([int(c) for c in line])
    return np.array(rows, dtype=np.int64), meta


def test_golden_mask_readback():
    """Q = 0 and V = identity read the kept set back: out[i,j] = 1/|K_i| on
    kept keys, 0 elsewhere, and lse_i = ln |K_i| (hand-worked fixture)."""
    want, meta = _read_mask_golden()
    S, a, n = int(meta["S"]), int(meta["a"]), int(meta["n"])
    flags = np.zeros((1, S), dtype=np.uint8)
    for p in meta["seps"].split(","):
        flags[0, int(p)] = 1
    D = 16
    q = np.zeros((1, 1, S, D), np.float32)
    k = _rand((1, 1, S, D), 1)
    v = np.zeros((1, 1, S, D), np.float32)
    for j in range(S):
        v[0, 0, j, j] = 1.0
    out, lse = oracle.prefill(q, k, v, flags, a, n)
    cnt = want.sum(1)
    np.testing.assert_array_equal(out[0, 0, :, :S] > 0, want.astype(bool))
    np.testing.assert_allclose(out[0, 0, :, :S], want / cnt[:, None], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[0, 0], np.log(cnt), rtol=0, atol=1e-14)
    # the same fixture through the page-order mask construction
    np.testing.assert_array_equal(_page_mask(flags[0], a, n).numpy().astype(np.int64), want)


def test_golden_pair_count():
    want, meta = _read_mask_golden()
    S, a, n = int(meta["S"]), int(meta["a"]), int(meta["n"])
    flags = np.zeros((1, S), dtype=np.uint8)
    for p in meta["seps"].split(","):
        flags[0, int(p)] = 1
    assert oracle.count_pairs(flags, a, n)[0] == want.sum() == 43


# ---------------------------------------------------------------- limits


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dense_limit(seed):
    """n >= S: every causal pair is kept, so the oracle equals dense causal
    attention (torch fp64 scaled_dot_product_attention)."""
    B, Hq, Hkv, S, D = 2, 4, 2, 37, 16
    rng = np.random.default_rng(seed)
    q, k, v = _rand((B, Hq, S, D), seed), _rand((B, Hkv, S, D), seed + 10), _rand((B, Hkv, S, D), seed + 20)
    flags = (rng.random((B, S)) < 0.3).astype(np.uint8)
    a = int(rng.integers(0, 5))
    for n in (S, S + 5):
        out, lse = oracle.prefill(q, k, v, flags, a, n)
        ref, ref_lse = _torch_attention(q, k, v, None, 1.0 / math.sqrt(D))
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_all_separators_is_dense():
    B, Hq, Hkv, S, D = 1, 2, 1, 29, 8
    q, k, v = _rand((B, Hq, S, D), 3), _rand((B, Hkv, S, D), 4), _rand((B, Hkv, S, D), 5)
    flags = np.ones((B, S), np.uint8)
    out, lse = oracle.prefill(q, k, v, flags, 0, 1)
    ref, ref_lse = _torch_attention(q, k, v, None, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("a,n", [(0, 1), (4, 5), (3, 16), (0, 40)])
def test_no_separators_is_sink_plus_sliding_window(a, n):
    """No separators: SepLLM reduces to StreamingLLM-style attention, i.e.
    attention sinks (the first a tokens) plus a sliding window of n
    (HKUDS047 study, section "SepLLM and StreamingLLM").  The reference mask
    is a band matrix plus sink columns, through torch fp64 attention."""
    B, Hq, Hkv, S, D = 1, 2, 2, 50, 8
    q, k, v = _rand((B, Hq, S, D), 6), _rand((B, Hkv, S, D), 7), _rand((B, Hkv, S, D), 8)
    flags = np.zeros((B, S), np.uint8)
    ones = torch.ones(S, S, dtype=torch.bool)
    sink = torch.zeros(S, S, dtype=torch.bool)
    sink[:, :a] = True
    mask = (ones.tril(0) & ~ones.tril(-n)) | (sink & ones.tril(0))
    out, lse = oracle.prefill(q, k, v, flags, a, n)
    ref, ref_lse = _torch_attention(q, k, v, mask, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_single_key_closed_form():
    """n = 1, a = 0, no separators: each query keeps only itself, so
    out_i = v_i exactly and lse_i = scale * q_i . k_i."""
    B, Hq, Hkv, S, D = 1, 4, 2, 20, 32
    q, k, v = _rand((B, Hq, S, D), 9), _rand((B, Hkv, S, D), 10), _rand((B, Hkv, S, D), 11)
    flags = np.zeros((B, S), np.uint8)
    scale = 0.37
    out, lse = oracle.prefill(q, k, v, flags, 0, 1, scale=scale)
    for h in range(Hq):
        g = h // 2
        np.testing.assert_array_equal(out[0, h], v[0, g].astype(np.float64))
        dots = np.einsum("sd,sd->s", q[0, h].astype(np.float64), k[0, g].astype(np.float64))
        np.testing.assert_allclose(lse[0, h], scale * dots, rtol=0, atol=1e-12)


def test_gqa_head_mapping():
    """Query head h reads kv head h // (Hq/Hkv): swapping kv heads swaps the
    outputs of exactly those query-head groups."""
    B, Hq, Hkv, S, D = 1, 6, 3, 12, 8
    q, k, v = _rand((B, Hq, S, D), 12), _rand((B, Hkv, S, D), 13), _rand((B, Hkv, S, D), 14)
    flags = (np.random.default_rng(0).random((B, S)) < 0.3).astype(np.uint8)
    out, _ = oracle.prefill(q, k, v, flags, 1, 3)
    k2, v2 = k[:, [1, 0, 2]].copy(), v[:, [1, 0, 2]].copy()
    q2 = q[:, [2, 3, 0, 1, 4, 5]].copy()
    out2, _ = oracle.prefill(q2, k2, v2, flags, 1, 3)
    np.testing.assert_array_equal(out2, out[:, [2, 3, 0, 1, 4, 5]])


# ---------------------------------------------------------------- brute force


def test_brute_force_tiny():
    """S <= 6: every flag pattern, a in [0,3], n in [1,S], against a full
    S x S softmax with an additive -inf mask (torch fp64)."""
    D = 4
    rng = np.random.default_rng(5)
    for S in range(1, 7):
        q, k, v = _rand((1, 1, S, D), 100 + S), _rand((1, 1, S, D), 200 + S), _rand((1, 1, S, D), 300 + S)
        qt, kt, vt = (torch.from_numpy(x[0, 0]).double() for x in (q, k, v))
        scores = (qt @ kt.T) / math.sqrt(D)
        for bits in itertools.product([0, 1], repeat=S):
            flags = np.array([bits], dtype=np.uint8)
            for a in range(4):
                for n in range(1, S + 1):
                    m = _page_mask(flags[0], a, n)
                    add = torch.zeros(S, S, dtype=torch.float64).masked_fill(~m, float("-inf"))
                    p = torch.softmax(scores + add, dim=-1)
                    ref = (p @ vt).numpy()
                    ref_lse = torch.logsumexp(scores + add, dim=-1).numpy()
                    out, lse = oracle.prefill(q, k, v, flags, a, n)
                    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-13)
                    np.testing.assert_allclose(lse[0, 0], ref_lse, rtol=0, atol=1e-13)
    assert rng is not None


# ---------------------------------------------------------------- invariants


def test_softmax_rows_sum_to_one_and_convexity():
    B, Hq, Hkv, S, D = 1, 2, 1, 48, 48
    rng = np.random.default_rng(21)
    flags = (rng.random((B, S)) < 0.15).astype(np.uint8)
    q, k = _rand((B, Hq, S, D), 22) * 3, _rand((B, Hkv, S, D), 23) * 3
    eye = np.zeros((B, Hkv, S, D), np.float32)
    eye[0, 0, np.arange(S), np.arange(S)] = 1
    probs, _ = oracle.prefill(q, k, eye, flags, 4, 7)
    np.testing.assert_allclose(probs.sum(-1), 1.0, rtol=0, atol=1e-12)
    assert (probs >= 0).all()
    # outputs lie inside the range of the kept v rows
    v = _rand((B, Hkv, S, D), 24)
    out, _ = oracle.prefill(q, k, v, flags, 4, 7)
    kept = probs[0] > 0  # [Hq, S, S]
    for h in range(Hq):
        for i in range(S):
            rows = v[0, 0][kept[h, i]]
            assert (out[0, h, i] >= rows.min(0) - 1e-12).all()
            assert (out[0, h, i] <= rows.max(0) + 1e-12).all()
    # constant v gives constant output
    c = np.full((B, Hkv, S, D), 0.625, np.float32)
    outc, _ = oracle.prefill(q, k, c, flags, 4, 7)
    np.testing.assert_allclose(outc, 0.625, rtol=0, atol=1e-14)


def test_bf16_inputs_read_exactly():
    """bf16 inputs are read as exactly the values torch gives them: the same
    values passed as fp32 give bit-identical oracle outputs."""
    B, Hq, Hkv, S, D = 1, 2, 1, 33, 16
    rng = np.random.default_rng(30)
    flags = (rng.random((B, S)) < 0.2).astype(np.uint8)
    qb = torch.from_numpy(_rand((B, Hq, S, D), 31)).to(torch.bfloat16)
    kb = torch.from_numpy(_rand((B, Hkv, S, D), 32)).to(torch.bfloat16)
    vb = torch.from_numpy(_rand((B, Hkv, S, D), 33)).to(torch.bfloat16)
    o1, l1 = oracle.prefill(qb, kb, vb, flags, 2, 5)
    o2, l2 = oracle.prefill(qb.float(), kb.float(), vb.float(), flags, 2, 5)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


# ---------------------------------------------------------------- counts and index


@pytest.mark.parametrize("a,n", [(0, 1), (4, 32), (4, 300), (7, 3), (400, 5)])
def test_pair_count_closed_form(a, n):
    """kept_i = (i - lo + 1) + min(a, lo) + (C[max(lo, a)] - C[a]) with
    lo = max(0, i - n + 1) and C the separator prefix count: the window, the
    initial tokens left of it, and the separators in [a, lo)."""
    S = 300
    flags = (np.random.default_rng(a * 1000 + n).random((2, S)) < 0.12).astype(np.uint8)
    got = oracle.count_pairs(flags, a, n)
    for b in range(2):
        C = np.concatenate([[0], np.cumsum(flags[b])])
        tot = 0
        for i in range(S):
            lo = max(0, i - n + 1)
            aa = min(a, S)
            tot += (i - lo + 1) + min(a, lo) + (C[max(lo, aa)] - C[aa])
        assert got[b] == tot


def test_build_index_pins():
    rng = np.random.default_rng(40)
    for B, S, p in [(3, 1, 0.5), (2, 257, 0.1), (1, 1000, 0.0), (1, 999, 1.0), (4, 4096, 0.3)]:
        flags = (rng.random((B, S)) < p).astype(np.uint8)
        prefix, idx, count = oracle.build_index(flags)
        for b in range(B):
            np.testing.assert_array_equal(prefix[b], np.concatenate([[0], np.cumsum(flags[b])]))
            nz = np.flatnonzero(flags[b])
            assert count[b] == int(flags[b].sum()) == nz.size
            np.testing.assert_array_equal(idx[b, : nz.size], nz)
            assert (idx[b, nz.size:] == -1).all()
            assert (np.diff(idx[b, : nz.size]) > 0).all()
            assert (flags[b, idx[b, : nz.size]] == 1).all()


def test_flags_from_ids():
    rng = np.random.default_rng(41)
    sep = np.array([15, 13, 32, 2, 28, 27, 209, 186, 187], np.int32)
    ids = rng.integers(0, 300, size=(3, 500)).astype(np.int32)
    np.testing.assert_array_equal(oracle.flags_from_ids(ids, sep), np.isin(ids, sep).astype(np.uint8))


# ---------------------------------------------------------------- SepCache


def _read_trace(name="sepcache_trace_a1_s2_p2_w2.txt"):
    meta, steps = {"mode": 0}, []
    with open(os.path.join(GOLD, name)) as fh:
        for line in fh:
            line = line.strip()
            if line.startswith("# a="):
                for kv in line[2:].split():
                    k_, v_ = kv.split("=")
                    meta[k_] = int(v_)
            elif line and not line.startswith("#"):
                parts = [p.strip() for p in line.split("|")]
                t, f = (int(x) for x in parts[0].split())
                last = parts[4].split()
                flushed = last[-1] == "F"
                if flushed:
                    last = last[:-1]
                blocks = [[] if p == "-" else [int(x) for x in p.split()] for p in parts[1:4]]
                blocks.append([] if last == ["-"] else [int(x) for x in last])
                steps.append((t, f, blocks, flushed))
    return meta, steps


@pytest.mark.parametrize("name", ["sepcache_trace_a1_s2_p2_w2.txt",
                                  "sepcache_trace_a1_s2_p2_w2_noacc.txt",
                                  "sepcache_trace_a1_s2_p2_w2_total.txt"])
def test_sepcache_golden_trace(name):
    meta, steps = _read_trace(name)
    T = len(steps)
    flags = np.array([[f] for (_, f, _, _) in steps], dtype=np.uint8)
    sim = oracle.sepcache_simulate(flags, meta["a"], meta["s"], meta["past"], meta["w"],
                                   np.arange(T), want_flushed=True, mode=meta["mode"])
    for k, (t, f, blocks, flushed) in enumerate(steps):
        cnt = sim["counts"][k, 0]
        assert list(cnt) == [len(x) for x in blocks], t
        want = [p for blk in blocks for p in blk]
        got = sim["pos"][k, 0]
        assert list(got[: len(want)]) == want, t
        assert (got[len(want):] == -1).all()
        assert bool(sim["flushed"][t, 0]) == flushed, t


@pytest.mark.parametrize("a,s,past,w", [(4, 64, 128, 256), (1, 3, 4, 5), (0, 8, 2, 3), (3, 0, 5, 4),
                                        (2, 5, 0, 3)])
def test_sepcache_invariants_and_flush_schedule(a, s, past, w):
    T, B = 3000, 3
    flags = (np.random.default_rng(a + s + past + w).random((T, B)) < 0.1).astype(np.uint8)
    snaps = np.arange(T)
    sim = oracle.sepcache_simulate(flags, a, s, past, w, snaps, want_flushed=True)
    # flush schedule: token t_k = a + w + k(past+1) - 1, k >= 1, every sequence
    want_flush = np.zeros(T, bool)
    k = 1
    while a + w + k * (past + 1) - 1 < T:
        want_flush[a + w + k * (past + 1) - 1] = True
        k += 1
    for b in range(B):
        np.testing.assert_array_equal(sim["flushed"][:, b].astype(bool), want_flush)
    for t in range(T):
        for b in range(B):
            nI, nS, nP, nL = sim["counts"][t, b]
            assert nI <= a and nS <= s and nP <= past and nL <= w
            assert nI + nS + nP + nL <= a + s + past + w
            tot = nI + nS + nP + nL
            pos = sim["pos"][t, b, :tot]
            fl = sim["flag"][t, b, :tot]
            assert (np.diff(pos) > 0).all()
            np.testing.assert_array_equal(pos[:nI], np.arange(min(a, t + 1)))
            assert (fl[nI: nI + nS] == 1).all()
            np.testing.assert_array_equal(pos[nI + nS:], np.arange(t - nP - nL + 1, t + 1))
            np.testing.assert_array_equal(fl, flags[pos, b])


def test_sepcache_streamingllm_special_case():
    """s = 0 and past = 0: the cache is the initial tokens plus the last w
    tokens, i.e. StreamingLLM (HKUDS047 study, section "SepLLM and
    StreamingLLM"; the StreamingLLM budget rule local = cache - init)."""
    a, w, T = 4, 16, 500
    flags = (np.random.default_rng(3).random((T, 2)) < 0.3).astype(np.uint8)
    sim = oracle.sepcache_simulate(flags, a, 0, 0, w, np.arange(T))
    for t in range(T):
        want = sorted(set(range(min(a, t + 1))) | set(range(max(0, t - w + 1), t + 1)))
        for b in range(2):
            tot = sim["counts"][t, b].sum()
            assert list(sim["pos"][t, b, :tot]) == want


def test_sepcache_holds_everything_before_first_flush():
    a, s, past, w = 4, 64, 128, 256
    T = a + w + past  # the first flush is at token a + w + past
    flags = (np.random.default_rng(4).random((T, 2)) < 0.1).astype(np.uint8)
    sim = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T))
    for t in range(T):
        for b in range(2):
            tot = sim["counts"][t, b].sum()
            assert list(sim["pos"][t, b, :tot]) == list(range(t + 1))


def test_sepcache_retained_set_equals_prefill_kept_set():
    """Before any separator is evicted (s large), the cache after token t
    holds exactly the prefill kept set of row t with window n_t = |P|+|L|:
    the four-block cache and the Sep-Attention mask agree (cross-check of
    the two oracle parts through the Q=0, V=I readback)."""
    a, s, past, w, T = 2, 1000, 5, 7, 60
    flags = (np.random.default_rng(8).random((T, 1)) < 0.25).astype(np.uint8)
    sim = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T))
    D = 64
    q = np.zeros((1, 1, T, D), np.float32)
    k = _rand((1, 1, T, D), 9)
    v = np.zeros((1, 1, T, D), np.float32)
    v[0, 0, np.arange(T), np.arange(T)] = 1
    for t in range(T):
        nI, nS, nP, nL = sim["counts"][t, 0]
        n_t = int(nP + nL) if nP + nL > 0 else 1
        out, _ = oracle.prefill_rows(q, k, v, flags.T.copy(), a, n_t, rows=np.array([t]))
        kept = set(np.flatnonzero(out[0] > 0).tolist())
        tot = int(sim["counts"][t, 0].sum())
        assert kept == set(sim["pos"][t, 0, :tot].tolist()), t


def test_attend_equals_prefill_row_on_same_set():
    """Decode attention over a listed set of rows equals the prefill row whose
    kept set is that list."""
    S, D, a, n = 40, 16, 3, 6
    flags = (np.random.default_rng(11).random((1, S)) < 0.2).astype(np.uint8)
    q, k, v = _rand((1, 4, S, D), 12), _rand((1, 2, S, D), 13), _rand((1, 2, S, D), 14)
    i = S - 1
    out, lse = oracle.prefill_rows(q, k, v, flags, a, n, rows=np.arange(4) * S + i)
    keep = [j for j in range(i + 1) if j < a or flags[0, j] or i - j < n]
    kq = np.ascontiguousarray(k[0][:, keep])
    vq = np.ascontiguousarray(v[0][:, keep])
    o2, l2 = oracle.attend(np.ascontiguousarray(q[0, :, i]), kq, vq)
    np.testing.assert_array_equal(out, o2)
    np.testing.assert_array_equal(lse, l2)


# ---------------------------------------------------------------------------
# rotary position encoding and the position-shifted decode.  Streaming needs
# positional-encoding shifting: keys are cached before the encoding and take
# their position inside the cache at each step (HKUDS047 SepLLM study,
# section on the three versions and section "Streaming-SepLLM").  The
# encoding is read as the rotate-half rotary form of Llama models.

def test_rope_direction_and_pairing():
    # the pair (x_i, x_{i+D/2}) is the complex number x_i + j x_{i+D/2},
    # turned counter-clockwise: e_0 at angle 1 -> (cos 1, 0, sin 1, 0), and
    # e_2 (the partner of e_0) -> (-sin 1, 0, cos 1, 0)
    c1, s1 = math.cos(1.0), math.sin(1.0)
    x = np.eye(4)
    out = oracle.rope(x, [1, 1, 1, 1], 10000.0)
    np.testing.assert_allclose(out[0], [c1, 0, s1, 0], atol=1e-15)
    np.testing.assert_allclose(out[2], [-s1, 0, c1, 0], atol=1e-15)
    # D = 4, theta = 10^4: the second frequency is 10^4^(-1/2) = 0.01, so
    # e_1 at position 100 also turns by 1 rad, into the pair (1, 3)
    out = oracle.rope(x[1:2], [100], 10000.0)
    np.testing.assert_allclose(out[0], [0, c1, 0, s1], atol=1e-13)
    # position 0 is the identity
    r = _rand((5, 64), 70)
    np.testing.assert_array_equal(oracle.rope(r, 0, 500000.0), r.astype(np.float64))


def test_rope_frequencies():
    # D = 8, theta = 256: frequency i is 256^(-2i/8) = 4^(-i), so e_i at
    # position 4^i turns by exactly 1 rad for every i < 4
    c1, s1 = math.cos(1.0), math.sin(1.0)
    for i in range(4):
        x = np.zeros((1, 8))
        x[0, i] = 1.0
        out = oracle.rope(x, [4 ** i], 256.0)[0]
        want = np.zeros(8)
        want[i], want[i + 4] = c1, s1
        np.testing.assert_allclose(out, want, atol=1e-13)


def test_rope_is_a_rotation_group():
    rng = np.random.default_rng(71)
    x = rng.standard_normal((16, 128))
    m = rng.integers(0, 5000, size=16)
    n = rng.integers(0, 5000, size=16)
    rm = oracle.rope(x, m, 500000.0)
    # norms are kept, and turning by m then by n is turning by m + n
    np.testing.assert_allclose(np.linalg.norm(rm, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(oracle.rope(rm, n, 500000.0), oracle.rope(x, m + n, 500000.0),
                               atol=1e-10)
    # turning back by -m restores x
    np.testing.assert_allclose(oracle.rope(rm, -m, 500000.0), x, atol=1e-11)


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(72)
    q = rng.standard_normal((1, 64))
    k = rng.standard_normal((1, 64))
    for m, n, t in [(10, 3, 7), (452, 0, 1000), (5, 5, 123456)]:
        a = oracle.rope(q, m, 10000.0) @ oracle.rope(k, n, 10000.0).T
        b = oracle.rope(q, m + t, 10000.0) @ oracle.rope(k, n + t, 10000.0).T
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_decode_shifted_is_attention_over_cache_positions(theta):
    # keys at their cache slots 0..L-1, the query (the newest row) at L-1:
    # torch fp64 attention over the encoded rows gives the same result
    Hq, Hkv, L, D = 8, 2, 37, 64
    q = _rand((Hq, D), 73)
    k = _rand((Hkv, L, D), 74)
    v = _rand((Hkv, L, D), 75)
    out, lse = oracle.decode_shifted(q, k, v, theta)
    qr = oracle.rope(q, L - 1, theta)
    kr = oracle.rope(k, np.arange(L)[None, :], theta)
    ref_o, ref_l = _torch_attention(qr[None, :, None, :], kr[None], v[None].astype(np.float64),
                                    torch.ones(1, L, dtype=torch.bool), 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out, ref_o[0, :, 0], atol=1e-12)
    np.testing.assert_allclose(lse, ref_l[0, :, 0], atol=1e-12)
    # the same scores from the relative offsets alone: q unrotated, key j
    # turned by j - (L-1)
    G = Hq // Hkv
    for h in (0, Hq - 1):
        krel = oracle.rope(k[h // G], np.arange(L) - (L - 1), theta)
        s = (krel @ q[h].astype(np.float64)) / math.sqrt(D)
        np.testing.assert_allclose(lse[h], np.log(np.exp(s - s.max()).sum()) + s.max(), atol=1e-12)


def test_decode_shifted_single_row_returns_its_value():
    q = _rand((4, 128), 76)
    k = _rand((1, 1, 128), 77)
    v = _rand((1, 1, 128), 78)
    out, lse = oracle.decode_shifted(q, k, v, 500000.0)
    np.testing.assert_allclose(out, np.repeat(v[0].astype(np.float64), 4, axis=0), atol=1e-15)
    # one row at slot 0 and the query at slot 0: no turn at all
    np.testing.assert_allclose(lse, q.astype(np.float64) @ k[0, 0].astype(np.float64) / math.sqrt(128),
                               atol=1e-12)


# ---------------------------------------------------------------------------
# cache variants.  The KV manager's compression step, read off the study's
# pseudocode ("HKUDS047: SepLLM ..." study, section "KV Cache Manager") and
# written here as a whole-cache recomputation per token -- a different
# formulation from the oracle's block state machine: when the cache is over
# its budget, initial = first a tokens, local = last w, past window = the
# tokens between the separator block and the local window; new separators =
# the flagged tokens of the past window; seps = old + new (accumulation) or
# new; seps = last s of them (maximum on; with the maximum off, more than s
# is the flagged overflow and the newest s stay).


def _pseudocode_cache(flags, a, s, past, w, mode):
    acc = not (mode & oracle.NO_ACCUMULATION)
    use_max = not (mode & oracle.UNBOUNDED_SEPS)
    total_trigger = bool(mode & oracle.TOTAL_TRIGGER)
    init, seps, rest = [], [], []  # rest = past window + local window, in order
    states, overflow = [], False
    for t, f in enumerate(flags):
        if len(init) < a:
            init.append(t)
        else:
            rest.append(t)
        n_past = max(0, len(rest) - w)
        size = len(init) + len(seps) + len(rest)
        over = size > a + s + past + w if total_trigger else n_past > past
        if over:
            past_window, local = rest[:n_past], rest[n_past:]
            new = [p for p in past_window if flags[p]]
            seps = (seps + new) if acc else new
            if len(seps) > s:
                overflow = overflow or not use_max
                seps = seps[len(seps) - s:]
            rest = local
        n_past = max(0, len(rest) - w)
        states.append((list(init), list(seps), rest[:n_past], rest[n_past:]))
    return states, overflow


@pytest.mark.parametrize("mode", range(8))
@pytest.mark.parametrize("a,s,past,w", [(1, 2, 2, 2), (3, 5, 4, 6), (0, 3, 0, 2), (2, 1, 3, 1)])
def test_sepcache_variants_match_pseudocode(mode, a, s, past, w):
    T, B = 400, 3
    rng = np.random.default_rng(1000 + 17 * mode + a + s + past + w)
    flags = (rng.random((T, B)) < 0.3).astype(np.uint8)
    sim = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T), mode=mode)
    for b in range(B):
        states, overflow = _pseudocode_cache(flags[:, b], a, s, past, w, mode)
        for t in range(T):
            I, S, P, L = states[t]
            assert list(sim["counts"][t, b]) == [len(I), len(S), len(P), len(L)], (mode, b, t)
            want = I + S + P + L
            assert list(sim["pos"][t, b, : len(want)]) == want, (mode, b, t)
        assert bool(sim["overflowed"][b]) == overflow, (mode, b)


def test_sepcache_variant_special_cases():
    T, B = 2000, 4
    flags = (np.random.default_rng(91).random((T, B)) < 0.1).astype(np.uint8)
    a, s, past, w = 4, 64, 128, 256
    base = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T))
    # with no maximum the cache is the default one until the first eviction,
    # which is flagged
    unb = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T), mode=oracle.UNBOUNDED_SEPS)
    np.testing.assert_array_equal(unb["pos"], base["pos"])
    big = oracle.sepcache_simulate(flags, a, 4096, past, w, [T - 1], mode=oracle.UNBOUNDED_SEPS)
    assert not big["overflowed"].any()
    n_flushed_seps = big["counts"][0, :, 1]
    assert (unb["overflowed"] == (n_flushed_seps > s)).all()
    # without accumulation every separator of the cache came from the last
    # flushed past window, which spans past + 1 positions
    noacc = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T), mode=oracle.NO_ACCUMULATION)
    for t in range(T):
        for b in range(B):
            nI, nS, nP, nL = noacc["counts"][t, b]
            S = noacc["pos"][t, b, nI:nI + nS]
            if nS:
                assert S[-1] - S[0] <= past and flags[S, b].all()
    # the total-length trigger never lets the cache exceed a+s+past+w and
    # flushes exactly when it would; once S is full it flushes like the
    # past-window trigger
    tot = oracle.sepcache_simulate(flags, a, s, past, w, np.arange(T), mode=oracle.TOTAL_TRIGGER,
                                   want_flushed=True)
    sizes = tot["counts"].sum(-1)
    assert sizes.max() <= a + s + past + w
    for t in range(1, T):
        for b in range(B):
            if tot["flushed"][t, b]:
                assert sizes[t - 1, b] == a + s + past + w
            if tot["counts"][t - 1, b, 1] == s and tot["flushed"][t, b]:
                assert tot["counts"][t - 1, b, 2] == past


def test_decode_masked_limits():
    # the generate mask is the prefill rule for the last row: with n >= T it
    # is dense attention of token T-1; with no separators, sinks + window
    B, Hq, Hkv, S, D, T = 2, 4, 2, 40, 64, 33
    q = _rand((B, Hq, D), 80)
    k = _rand((B, Hkv, S, D), 81)
    v = _rand((B, Hkv, S, D), 82)
    flags = (np.random.default_rng(83).random((B, S)) < 0.3).astype(np.uint8)
    out, lse = oracle.decode_masked(q, k, v, flags, T, 2, T)
    qq = q[:, :, None, :]
    mask = torch.ones(1, T, dtype=torch.bool)
    ref_o, ref_l = _torch_attention(qq, k[:, :, :T], v[:, :, :T], mask, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out, ref_o[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(lse, ref_l[:, :, 0], atol=1e-12)
    a, n = 3, 5
    out, lse = oracle.decode_masked(q, k, v, np.zeros_like(flags), T, a, n)
    keep = torch.zeros(1, T, dtype=torch.bool)
    keep[0, :a] = True
    keep[0, T - n:] = True
    ref_o, ref_l = _torch_attention(qq, k[:, :, :T], v[:, :, :T], keep, 1.0 / math.sqrt(D))
    np.testing.assert_allclose(out, ref_o[:, :, 0], atol=1e-12)
    np.testing.assert_allclose(lse, ref_l[:, :, 0], atol=1e-12)


# ---------------------------------------------------------------------------
# backward: gradients of sum(out * dout) through Sep-Attention


def _loss(q, k, v, dout, flags, a, n):
    out, _ = oracle.prefill(q, k, v, flags, a, n)
    return float((out * dout).sum())


def test_backward_matches_finite_differences():
    # central differences of the (pinned) fp64 forward along random
    # directions: an independent route to the same derivative
    rng = np.random.default_rng(90)
    B, Hq, Hkv, S, D, a, n = 1, 4, 2, 23, 16, 2, 5
    q = rng.standard_normal((B, Hq, S, D))
    k = rng.standard_normal((B, Hkv, S, D))
    v = rng.standard_normal((B, Hkv, S, D))
    dout = rng.standard_normal((B, Hq, S, D))
    flags = (rng.random((B, S)) < 0.3).astype(np.uint8)
    gq, gk, gv = oracle.prefill_backward(q, k, v, dout, flags, a, n)
    eps = 1e-5
    for name, x, g in (("q", q, gq), ("k", k, gk), ("v", v, gv)):
        d = rng.standard_normal(x.shape)
        args = {"q": q, "k": k, "v": v}
        plus = dict(args, **{name: x + eps * d})
        minus = dict(args, **{name: x - eps * d})
        fd = (_loss(plus["q"], plus["k"], plus["v"], dout, flags, a, n) -
              _loss(minus["q"], minus["k"], minus["v"], dout, flags, a, n)) / (2 * eps)
        assert abs(fd - float((g * d).sum())) <= 1e-7 * max(1.0, abs(fd)), name


@pytest.mark.parametrize("a,n,p", [(4, 8, 0.2), (0, 1, 0.5), (3, 40, 0.0), (1, 3, 1.0)])
def test_backward_matches_torch_autograd(a, n, p):
    # torch fp64 autograd through a -inf-masked softmax attention (GQA by
    # repeating kv heads) with the kept set built the way the study builds
    # the prefill mask
    rng = np.random.default_rng(91 + a + n)
    B, Hq, Hkv, S, D = 2, 4, 2, 30, 8
    q = rng.standard_normal((B, Hq, S, D))
    k = rng.standard_normal((B, Hkv, S, D))
    v = rng.standard_normal((B, Hkv, S, D))
    dout = rng.standard_normal((B, Hq, S, D))
    flags = (rng.random((B, S)) < p).astype(np.uint8)
    gq, gk, gv = oracle.prefill_backward(q, k, v, dout, flags, a, n)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    G = Hq // Hkv
    outs = []
    for b in range(B):
        mask = _page_mask(flags[b], a, n)
        s = (tq[b] @ tk[b].repeat_interleave(G, 0).transpose(-1, -2)) / math.sqrt(D)
        pr = torch.softmax(s.masked_fill(~mask, float("-inf")), -1)
        outs.append(pr @ tv[b].repeat_interleave(G, 0))
    (torch.stack(outs) * torch.from_numpy(dout)).sum().backward()
    np.testing.assert_allclose(gq, tq.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gk, tk.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(gv, tv.grad.numpy(), atol=1e-11)


def test_backward_single_key_closed_form():
    # n = 1, a = 0, no separators: out_i = v_i, so dv = the summed dout of
    # the group's heads and dq = dk = 0
    rng = np.random.default_rng(92)
    B, Hq, Hkv, S, D = 1, 4, 2, 12, 8
    q, dout = rng.standard_normal((B, Hq, S, D)), rng.standard_normal((B, Hq, S, D))
    k, v = rng.standard_normal((B, Hkv, S, D)), rng.standard_normal((B, Hkv, S, D))
    gq, gk, gv = oracle.prefill_backward(q, k, v, dout, np.zeros((B, S), np.uint8), 0, 1)
    assert np.abs(gq).max() == 0 and np.abs(gk).max() == 0
    np.testing.assert_allclose(gv, dout.reshape(B, Hkv, 2, S, D).sum(2), atol=1e-14)
