"""Seeded synthetic inputs for the Sep-Attention and SepCache workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no masks, no scans, no softmax, no cache rules).  Both the
CUDA path's tests/bench and the CPU oracle take their inputs from here.

Workload shapes follow the pages' model settings:
  * separator-id lists: HKUDS047 SepLLM study, section "Separator Tokens"
    (Llama-3 and Pythia/GPT-NeoX id sets);
  * Llama-3-8B head layout 32 q / 8 kv, head_dim 128 and `layer_num=32`:
    HKUDS047 SepLLM study, section "SepCache" (the `SepCache(...)` demo call);
  * SepCache sizes a=4, s=64, past=128, w=256: the four-block table of the
    xugj520 article, section 3.3, and the streaming demo's `local_size=256`.

Every generator is a pure function of its seed.  Random draws use numpy's
PCG64; bf16 tensors are rounded from fp32 draws by torch's round-to-nearest-
even conversion.
"""
from __future__ import annotations

import numpy as np
import torch

# Separator token ids (HKUDS047 SepLLM study, section "Separator Tokens").
LLAMA3_SEP_IDS = (13, 11, 30, 0, 26, 25, 198, 220, 128000)
PYTHIA_SEP_IDS = (15, 13, 32, 2, 28, 27, 209, 186, 187)
# Tiny workload: ids 0..8 of a 1000-id vocabulary are the separators.
TINY_SEP_IDS = tuple(range(9))

# Workloads, named by what they are and their sizes.
WORKLOADS = {
    # B1 H1 D64 S256 fp32, ids over a 1000-id vocab, a=4 n=32
    "prefill_tiny_b1h1_s256_d64_f32": dict(
        kind="prefill", B=1, Hq=1, Hkv=1, S=256, D=64, dtype="f32", a=4, n=32,
        p_sep=0.1, ids="vocab1000", qkv_std=1.0),
    # Pythia-160M shape: B8 H12 (MHA) D64 S2048 bf16, a=4 n=64
    "prefill_pythia160m_b8h12_s2048_d64_bf16": dict(
        kind="prefill", B=8, Hq=12, Hkv=12, S=2048, D=64, dtype="bf16", a=4, n=64,
        p_sep=0.08, ids="pythia50k", qkv_std=1.0 / 8.0),
    # Llama-3-8B shape: B1 32q/8kv D128 S8192 bf16, a=4 n=256
    "prefill_llama3_8b_b1_s8192_d128_bf16": dict(
        kind="prefill", B=1, Hq=32, Hkv=8, S=8192, D=128, dtype="bf16", a=4, n=256,
        p_sep=0.1, ids=None, qkv_std=1.0),
    # Streaming decode over the four-block cache, Llama-3-8B shape, 32 layers
    "decode_llama3_8b_b16_l32_t65536_d128_bf16": dict(
        kind="decode", B=16, Hq=32, Hkv=8, D=128, dtype="bf16", layers=32, T=65536,
        a=4, s=64, past=128, w=256, p_sep=0.1, qkv_std=1.0),
    # Long context: B1 32q/8kv D128 S131072 bf16, flags with runs of 3, a=4 n=1024
    "prefill_long_b1_s131072_d128_bf16": dict(
        kind="prefill", B=1, Hq=32, Hkv=8, S=131072, D=128, dtype="bf16", a=4, n=1024,
        p_single=0.05, p_run_start=0.05 / 3.0, run_len=3, ids=None, qkv_std=1.0),
    # Prompt ingestion into the decode workload's cache: a 4096-token prompt
    # of 16 sequences, 8 kv heads, D128, 32 layers, a=4 s=64 past=128 w=256
    "ingest_llama3_8b_b16_l32_t4096_d128_bf16": dict(
        kind="ingest", B=16, Hq=32, Hkv=8, D=128, dtype="bf16", layers=32, T=4096,
        a=4, s=64, past=128, w=256, p_sep=0.1, qkv_std=1.0),
    # The decode workload with positional-encoding shifting: keys cached
    # un-encoded, rotary base 500000 (Llama-3), encoded at their cache slots
    "decode_rope_llama3_8b_b16_l32_t65536_d128_bf16": dict(
        kind="decode", B=16, Hq=32, Hkv=8, D=128, dtype="bf16", layers=32, T=65536,
        a=4, s=64, past=128, w=256, p_sep=0.1, qkv_std=1.0, rope_theta=500000.0),
    # Mask-based generation over full 8k-token histories (no eviction),
    # Llama-3-8B shape: 16 sequences, 32 q / 8 kv heads, D128, 32 layers,
    # a=4 n=256
    "generate_masked_llama3_8b_b16_s8192_d128_bf16": dict(
        kind="generate", B=16, Hq=32, Hkv=8, D=128, dtype="bf16", layers=32, S=8192,
        a=4, n=256, p_sep=0.1, qkv_std=1.0),
    # Backward of the prefill workloads (training): gradients of q, k, v
    "backward_llama3_8b_b1_s8192_d128_bf16": dict(
        kind="backward", B=1, Hq=32, Hkv=8, S=8192, D=128, dtype="bf16", a=4, n=256,
        p_sep=0.1, ids=None, qkv_std=1.0),
    "backward_pythia160m_b8h12_s2048_d64_bf16": dict(
        kind="backward", B=8, Hq=12, Hkv=12, S=2048, D=64, dtype="bf16", a=4, n=64,
        p_sep=0.08, ids="pythia50k", qkv_std=1.0 / 8.0),
    # The Llama-3-8B backward on 2k tokens: the size a full counter capture
    # of the D128 backward kernels takes
    "backward_llama3_8b_b1_s2048_d128_bf16": dict(
        kind="backward", B=1, Hq=32, Hkv=8, S=2048, D=128, dtype="bf16", a=4, n=256,
        p_sep=0.1, ids=None, qkv_std=1.0),
    # The long-context prefill on 32k tokens (same flags recipe and window):
    # the size a full counter capture of the D128 prefill kernel takes
    "prefill_long_b1_s32768_d128_bf16": dict(
        kind="prefill", B=1, Hq=32, Hkv=8, S=32768, D=128, dtype="bf16", a=4, n=1024,
        p_single=0.05, p_run_start=0.05 / 3.0, run_len=3, ids=None, qkv_std=1.0),
}

# Base seed per workload (1000 + index in the list above); parity tests add
# extra seeds on top.
WORKLOAD_SEED = {name: 1000 + i + 1 for i, name in enumerate(WORKLOADS)}


def rng(seed) -> np.random.Generator:
    """A PCG64 generator for `seed` (an int or a tuple of ints)."""
    return np.random.default_rng(seed)


def normal(g: np.random.Generator, shape, std: float, dtype: str) -> torch.Tensor:
    """N(0, std^2) draws as a CPU tensor of `dtype` ('f32' or 'bf16')."""
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    t = torch.from_numpy(x)
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def bernoulli_flags(g: np.random.Generator, shape, p: float) -> np.ndarray:
    """uint8 array of independent Bernoulli(p) draws."""
    return (g.random(size=shape) < p).astype(np.uint8)


def run_flags(g: np.random.Generator, B: int, S: int, p_single: float,
              p_run_start: float, run_len: int) -> np.ndarray:
    """Flags made of single separators (Bernoulli p_single) OR'ed with runs of
    `run_len` consecutive separators, a run starting at each position with
    probability p_run_start (runs are clipped at the sequence end)."""
    single = g.random(size=(B, S)) < p_single
    starts = g.random(size=(B, S)) < p_run_start
    run = np.zeros((B, S), dtype=bool)
    for r in range(run_len):
        run[:, r:] |= starts[:, : S - r]
    return (single | run).astype(np.uint8)


def token_ids(g: np.random.Generator, flags: np.ndarray, kind: str) -> np.ndarray:
    """int32 token ids whose separator-ness equals `flags`: a separator
    position draws uniformly from the separator-id set, any other position
    draws uniformly from the rest of the vocabulary."""
    if kind == "vocab1000":
        sep_ids, vocab = np.array(TINY_SEP_IDS), 1000
    elif kind == "pythia50k":
        sep_ids, vocab = np.array(PYTHIA_SEP_IDS), 50000
    else:
        raise ValueError(kind)
    non_sep = np.setdiff1d(np.arange(vocab), sep_ids)
    pick_sep = sep_ids[g.integers(0, len(sep_ids), size=flags.shape)]
    pick_non = non_sep[g.integers(0, len(non_sep), size=flags.shape)]
    return np.where(flags.astype(bool), pick_sep, pick_non).astype(np.int32)


def sep_id_set(kind):
    if kind == "vocab1000":
        return np.array(TINY_SEP_IDS, dtype=np.int32)
    if kind == "pythia50k":
        return np.array(PYTHIA_SEP_IDS, dtype=np.int32)
    return None


def prefill_inputs(cfg: dict, seed: int, S: int | None = None, B: int | None = None) -> dict:
    """Inputs of one prefill call: q [B,Hq,S,D], k/v [B,Hkv,S,D] (CPU tensors),
    is_sep uint8 [B,S] and, when the workload has them, int32 token ids [B,S]
    and the separator-id set.  `S`/`B` override the workload's sizes (used for
    small parity cases with the same distributions)."""
    B = cfg["B"] if B is None else B
    S = cfg["S"] if S is None else S
    Hq, Hkv, D, dt, std = cfg["Hq"], cfg["Hkv"], cfg["D"], cfg["dtype"], cfg["qkv_std"]
    g = rng((seed, 0))
    if "p_single" in cfg:
        flags = run_flags(g, B, S, cfg["p_single"], cfg["p_run_start"], cfg["run_len"])
    else:
        flags = bernoulli_flags(g, (B, S), cfg["p_sep"])
    out = dict(B=B, S=S, Hq=Hq, Hkv=Hkv, D=D, dtype=dt, a=cfg["a"], n=cfg["n"])
    if cfg.get("ids"):
        out["ids"] = token_ids(g, flags, cfg["ids"])
        out["sep_ids"] = sep_id_set(cfg["ids"])
    out["is_sep"] = flags
    out["q"] = normal(rng((seed, 1)), (B, Hq, S, D), std, dt)
    out["k"] = normal(rng((seed, 2)), (B, Hkv, S, D), std, dt)
    out["v"] = normal(rng((seed, 3)), (B, Hkv, S, D), std, dt)
    return out


def decode_flags(cfg: dict, seed: int, T: int | None = None, B: int | None = None) -> np.ndarray:
    """Separator flags of the decode stream, uint8 [T, B] (token t of every
    sequence is drawn independently)."""
    T = cfg["T"] if T is None else T
    B = cfg["B"] if B is None else B
    return bernoulli_flags(rng((seed, 10)), (T, B), cfg["p_sep"])


def decode_step_qkv(cfg: dict, seed: int, step: int, layer: int, B: int | None = None):
    """q [B,Hq,D], k_new/v_new [B,Hkv,D] of token `step` at `layer`.  Each
    (step, layer) has its own generator, so the K/V row of any past position
    can be regenerated on its own."""
    B = cfg["B"] if B is None else B
    g = rng((seed, 11, step, layer))
    dt, std = cfg["dtype"], cfg["qkv_std"]
    q = normal(g, (B, cfg["Hq"], cfg["D"]), std, dt)
    k = normal(g, (B, cfg["Hkv"], cfg["D"]), std, dt)
    v = normal(g, (B, cfg["Hkv"], cfg["D"]), std, dt)
    return q, k, v


def raw(t: torch.Tensor) -> np.ndarray:
    """The raw element bits of a CPU tensor as a contiguous numpy array
    (float32 stays float32; bf16 becomes uint16 bit patterns)."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.numpy()
    raise ValueError(t.dtype)
