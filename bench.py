#!/usr/bin/env python
"""Benchmark of the Sep-Attention hot path; prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Workloads (synthetic, seeded; see synth.WORKLOADS):
  prefill_* : one step = separator flags from token ids (when the workload has
              ids) -> separator index lists -> Sep-Attention prefill over the
              whole batch.  Metric: TFLOP/s on kept pairs (4*D FLOP per kept
              (query, key) pair and head).  L2 is flushed (256 MiB write)
              between timed steps; the flush is outside the timed events.
  decode_*  : one step = one token for every sequence through all layers:
              append (layer 0 also advances the block bookkeeping) ->
              compact -> decode, per layer, replayed as a CUDA graph.
              Metric: decode tokens/s.  The cache (~1 GB) is far larger than L2.

Multi-GPU (torchrun): every rank runs its own replica of the workload (weak
scaling, no data-path collective); the timing is the max over ranks.
--impl reference times the CPU oracle on this host's cores instead (the
reference arm), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402

# The default line is the largest single-GPU configuration: the 131,072-token
# long-context prefill (B1, 32 query / 8 kv heads, D128, a4, n1024).
DEFAULT_WORKLOAD = "prefill_long_b1_s131072_d128_bf16"
PREFILL_METRIC = "Sep-Attn prefill TFLOP/s on kept pairs"
DECODE_METRIC = "Sep-Attn decode tokens/s over the four-block SepCache"
INGEST_METRIC = "SepCache prompt ingestion tokens/s"
GENERATE_METRIC = "Sep-Attn mask-based generation tokens/s over full histories"
BACKWARD_METRIC = "Sep-Attn backward TFLOP/s on kept pairs"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant
# kernel, from one ncu capture each (summaries under profiles/).  A figure
# holds only for the kernel source it was taken on: when the hash of the
# kernel's files differs, the traffic is reported as unknown (null).  `per` is the unit the
# figure scales with: one launch, or one retained K/V row of one sequence
# (the capture ran a smaller cache than the bench; decode traffic grows in
# proportion to the retained rows).
TRAFFIC = {
    "decode_llama3_8b_b16_l32_t65536_d128_bf16": dict(
        bytes=(28617472 + 0) / (420.5 * 16), per="row", src=("decode.cu", "common.cuh"),
        sha1="15a13239d28cd65b3fab191c803aa3c5a4c49bee"),
    "decode_rope_llama3_8b_b16_l32_t65536_d128_bf16": dict(
        bytes=(28890368 + 0) / (421.19 * 16), per="row", src=("decode.cu", "common.cuh"),
        sha1="15a13239d28cd65b3fab191c803aa3c5a4c49bee"),
    "generate_masked_llama3_8b_b16_s8192_d128_bf16": dict(
        bytes=69489920 + 773120, per="launch", src=("decode.cu", "common.cuh"),
        sha1="15a13239d28cd65b3fab191c803aa3c5a4c49bee"),
    # one ingestion step: the state kernel and the 32 layers' row copies
    "ingest_llama3_8b_b16_l32_t4096_d128_bf16": dict(
        bytes=879904256 + 2625280, per="launch", src=("sepcache.cu", "common.cuh"),
        sha1="0d11d7ce0b1432ab13e322fbddf2eb9d687f9376"),
    "backward_llama3_8b_b1_s8192_d128_bf16": dict(
        bytes=433952512 + 67951872, per="launch", src=("backward.cu", "common.cuh"),
        sha1="0f3a298c018e77b40779bd9f5771a864484deb97"),
    "backward_pythia160m_b8h12_s2048_d64_bf16": dict(
        bytes=263013376 + 32558592, per="launch", src=("backward.cu", "common.cuh"),
        sha1="0f3a298c018e77b40779bd9f5771a864484deb97"),
    "prefill_llama3_8b_b1_s8192_d128_bf16": dict(
        bytes=104811776 + 20765440, per="launch", src=("prefill_tc.cu", "common.cuh"),
        sha1="0a11e6db6fab1045752f3db57e190bbd825b7948"),
    "prefill_pythia160m_b8h12_s2048_d64_bf16": dict(
        bytes=81602304 + 5924096, per="launch", src=("prefill_tc.cu", "common.cuh"),
        sha1="0a11e6db6fab1045752f3db57e190bbd825b7948"),
    "prefill_long_b1_s131072_d128_bf16": dict(
        bytes=2237840128 + 1067599872, per="launch", src=("prefill_tc.cu", "common.cuh"),
        sha1="0a11e6db6fab1045752f3db57e190bbd825b7948"),
}


def _src_sha1(fnames):
    import hashlib
    h = hashlib.sha1()
    for f in fnames:
        with open(os.path.join(ROOT, "streaming_kv_cache_sep_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def _traffic(name, units):
    t = TRAFFIC.get(name)
    if t is None:
        return None
    try:
        if _src_sha1(t["src"]) != t["sha1"]:
            return None
    except OSError:
        return None
    return int(round(t["bytes"] * (units if t["per"] == "row" else 1)))


# ---------------------------------------------------------------- clocks


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- distributed


def _dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- prefill


class PrefillWorkload:
    def __init__(self, sl, name, seed):
        self.sl = sl
        self.name = name
        self.cfg = cfg = synth.WORKLOADS[name]
        inp = synth.prefill_inputs(cfg, seed)
        self.host = inp
        self.q, self.k, self.v = inp["q"].cuda(), inp["k"].cuda(), inp["v"].cuda()
        self.has_ids = "ids" in inp
        if self.has_ids:
            self.ids = torch.from_numpy(inp["ids"]).cuda()
            self.sep_ids = [int(x) for x in inp["sep_ids"]]
            self.is_sep = torch.empty(self.ids.shape, dtype=torch.uint8, device="cuda")
        else:
            self.is_sep = torch.from_numpy(inp["is_sep"]).cuda()
        B, S = self.is_sep.shape
        self.B, self.S = B, S
        self.prefix = torch.empty((B, S + 1), dtype=torch.int32, device="cuda")
        self.idx = torch.empty((B, S), dtype=torch.int32, device="cuda")
        self.count = torch.empty((B,), dtype=torch.int32, device="cuda")
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.q.shape[:3], dtype=torch.float32, device="cuda")
        dt = 1 if self.q.dtype == torch.bfloat16 else 0
        self.ws = torch.empty((sl.prefill_workspace_bytes(B, cfg["Hq"], cfg["Hkv"], S, cfg["D"], dt),),
                              dtype=torch.uint8, device="cuda")
        # algorithmic work: 4*D FLOP per kept pair and head
        flags = torch.from_numpy(inp["is_sep"]).cuda()
        prefix, _, _ = sl.build_index(flags)
        kept = int(sl.count_pairs(prefix, cfg["a"], cfg["n"]).sum().item()) * cfg["Hq"]
        self.kept_pairs = kept
        self.flops = 4.0 * cfg["D"] * kept
        # front: one launch (flags and index from ids, or the index from
        # flags); sep_attn_prefill: the separator-row gather and attention
        self.launches_per_step = 1 + (2 if dt == 1 else 1)

    def front(self):
        if self.has_ids:
            self.sl.build_index_from_ids(self.ids, self.sep_ids,
                                         out=(self.is_sep, self.prefix, self.idx, self.count))
        else:
            self.sl.build_index(self.is_sep, out=(self.prefix, self.idx, self.count))

    def attn(self):
        c = self.cfg
        self.sl.prefill(self.q, self.k, self.v, self.is_sep, self.prefix, self.idx, c["a"], c["n"],
                        out=self.out, lse=self.lse, workspace=self.ws)

    def step(self):
        self.front()
        self.attn()


def bench_prefill(sl, args, world, rank):
    name = args.workload
    wl = PrefillWorkload(sl, name, synth.WORKLOAD_SEED[name] + 7919 * rank)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        flush.zero_()
        wl.step()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()  # untimed: evict L2 between steps
        ev[i][0].record()
        wl.front()
        ev[i][1].record()
        wl.attn()
        ev[i][2].record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(c) for a, b, c in ev]
    attn_ms = [b.elapsed_time(c) for a, b, c in ev]
    t_local = sum(step_ms) / 1e3
    t = _max_over_ranks(t_local, world)
    value = wl.flops * K * world / t / 1e12

    # end to end through the public API with host buffers: pinned host inputs
    # -> device, the whole step, output -> pinned host, all inside the events.
    # Two device buffer sets and three streams, as a serving loop would run
    # it: the inputs of step k+1 cross PCIe while step k computes and its
    # results come back (the link is full duplex); every step still copies
    # all its inputs in and its out and lse back.
    e2e = None
    if not args.skip_e2e:
        h = wl.host
        hq, hk, hv = (x.pin_memory() for x in (h["q"], h["k"], h["v"]))
        hin = torch.from_numpy(h["ids"]).pin_memory() if wl.has_ids else \
            torch.from_numpy(h["is_sep"]).pin_memory()
        hout = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
        hlse = torch.empty(wl.lse.shape, dtype=torch.float32).pin_memory()
        sets = [dict(q=torch.empty_like(wl.q), k=torch.empty_like(wl.k), v=torch.empty_like(wl.v),
                     inp=torch.empty(hin.shape, dtype=hin.dtype, device="cuda"),
                     out=torch.empty_like(wl.out), lse=torch.empty_like(wl.lse))
                for _ in range(2)]
        comp = torch.cuda.current_stream()
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = {(n, b): torch.cuda.Event() for n in ("in", "comp", "out") for b in range(2)}
        used = [False, False]
        c = wl.cfg

        def e2e_step(kstep):
            b = kstep % 2
            d = sets[b]
            with torch.cuda.stream(s_in):
                if used[b]:
                    s_in.wait_event(ev[("comp", b)])  # the step that last read set b is done
                d["q"].copy_(hq, non_blocking=True)
                d["k"].copy_(hk, non_blocking=True)
                d["v"].copy_(hv, non_blocking=True)
                d["inp"].copy_(hin, non_blocking=True)
                ev[("in", b)].record(s_in)
            comp.wait_event(ev[("in", b)])
            if used[b]:
                comp.wait_event(ev[("out", b)])  # set b's results have been read back
            if wl.has_ids:
                sl.build_index_from_ids(d["inp"], wl.sep_ids,
                                        out=(wl.is_sep, wl.prefix, wl.idx, wl.count))
                flags = wl.is_sep
            else:
                sl.build_index(d["inp"], out=(wl.prefix, wl.idx, wl.count))
                flags = d["inp"]
            sl.prefill(d["q"], d["k"], d["v"], flags, wl.prefix, wl.idx, c["a"], c["n"],
                       out=d["out"], lse=d["lse"], workspace=wl.ws)
            ev[("comp", b)].record(comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[("comp", b)])
                hout.copy_(d["out"], non_blocking=True)
                hlse.copy_(d["lse"], non_blocking=True)
                ev[("out", b)].record(s_out)
            used[b] = True

        for kk in range(2):
            e2e_step(kk)
        torch.cuda.synchronize()
        Ke = max(3, K // 2)
        _barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(comp)
        s_in.wait_stream(comp)  # the first copies start inside the timed region
        for kk in range(Ke):
            e2e_step(kk)
        comp.wait_stream(s_out)
        s1.record(comp)
        torch.cuda.synchronize()
        te = _max_over_ranks(s0.elapsed_time(s1) / 1e3, world)
        bi = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hin))
        bo = hout.numel() * hout.element_size() + hlse.numel() * 4
        e2e = {"value": wl.flops * Ke * world / te / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo)}

    pk = _peaks()
    attn_s = statistics.mean(attn_ms) / 1e3
    achieved = wl.flops / attn_s / 1e12
    c = wl.cfg
    # algorithmic bytes of one call: q, k, v read once, out and lse written
    esz = wl.q.element_size()
    alg_bytes = (wl.q.numel() + wl.k.numel() + wl.v.numel() + wl.out.numel()) * esz + wl.lse.numel() * 4
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16"],
                "unit": "TFLOP/s", "frac": round(achieved / pk["bf16"], 4),
                "traffic": _traffic(name, units=1),
                "bytes_per_launch": int(alg_bytes), "launch_us": round(attn_s * 1e6, 3),
                "kernel": "sep_attn_prefill (separator-row gather + tcgen05 attention)",
                "peak_source": pk["src"] + " bf16 dense burst",
                # the same call against HBM: below the ridge point (bf16 peak /
                # HBM bandwidth) the bytes bound the call before the FLOPs do
                "hbm_view": {"achieved": round(alg_bytes / attn_s / 1e9, 1), "peak": pk["hbm"],
                             "unit": "GB/s", "frac": round(alg_bytes / attn_s / 1e9 / pk["hbm"], 4),
                             "flop_per_byte": round(wl.flops / alg_bytes, 1),
                             "ridge_flop_per_byte": round(pk["bf16"] * 1e3 / pk["hbm"], 1)}}
    line = {
        "metric": PREFILL_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if wl.q.dtype == torch.bfloat16 else "f32", "data": "synthetic",
        "config": {"workload": name, "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "S": c["S"],
                   "D": c["D"], "a": c["a"], "n": c["n"], "kept_pairs": wl.kept_pairs,
                   "gflop_per_step": round(wl.flops / 1e9, 4),
                   "l2": "flushed between timed steps (256 MiB write, outside the events)",
                   "parallelism": "replica per GPU (weak)"},
        "roofline": roofline, "e2e": e2e, "clocks": clk,
        "gpu_launches": wl.launches_per_step * K,
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline_prefill(wl, budget_s=args.cpu_seconds)
    return line


def cpu_baseline_prefill(wl, budget_s=10.0):
    import oracle
    h, c = wl.host, wl.cfg
    rows, frac = _sample_rows(c, budget_hint=budget_s)
    kept = _kept_pairs_rows(h["is_sep"], c, rows)
    t0 = time.time()
    reps = 0
    while True:
        oracle.prefill_rows(h["q"], h["k"], h["v"], h["is_sep"], c["a"], c["n"], rows=rows)
        reps += 1
        if time.time() - t0 >= budget_s:
            break
    dt = time.time() - t0
    return {"value": round(4.0 * c["D"] * kept * reps / dt / 1e12, 6), "unit": "TFLOP/s",
            "cores": oracle.nthreads(), "kind": "oracle",
            "sample": "%d of %d query rows (%.3g of the workload), repeated %d times, %.1f s" % (
                rows.size, c["B"] * c["Hq"] * c["S"], frac, reps, dt)}


def _sample_rows(c, budget_hint=10.0):
    """A deterministic bounded sample of query rows: every row for workloads
    the oracle finishes in about a second, else an evenly strided subset."""
    total = c["B"] * c["Hq"] * c["S"]
    est = 4.0 * c["D"] * total * min(c["S"], c["n"] + 0.1 * c["S"] / 2 + c["a"]) / 1e10  # s, 8 cores
    stride = 1
    while est / stride > budget_hint / 4 and stride < total:
        stride *= 2
    rows = np.arange(0, total, stride, dtype=np.int64)
    return rows, rows.size / total


def _kept_pairs_rows(flags, c, rows):
    a, n, S = c["a"], c["n"], c["S"]
    C = np.concatenate([np.zeros((flags.shape[0], 1), np.int64), np.cumsum(flags, 1)], 1)
    i = rows % S
    b = rows // (S * c["Hq"])
    lo = np.maximum(0, i - n + 1)
    aa = min(a, S)
    kept = (i - lo + 1) + np.minimum(a, lo) + np.where(lo > aa, C[b, lo] - C[b, aa], 0)
    return int(kept.sum())


# ---------------------------------------------------------------- decode


class DecodeWorkload:
    RING = 4

    def __init__(self, sl, name, seed, layers=None):
        self.sl = sl
        self.cfg = c = dict(synth.WORKLOADS[name])
        if layers:
            c["layers"] = layers
        self.B, self.Hq, self.Hkv, self.D, self.L = c["B"], c["Hq"], c["Hkv"], c["D"], c["layers"]
        self.cache = sl.SepCache(c["a"], c["s"], c["past"], c["w"], self.L, self.B, self.Hkv, self.D,
                                 dtype=torch.bfloat16)
        self.rope_theta = c.get("rope_theta", 0.0)
        if self.rope_theta:
            self.cache.set_rope(self.rope_theta)  # keys cached un-encoded
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        R = self.RING
        self.q = torch.randn((R, self.L, self.B, self.Hq, self.D), generator=g, device="cuda").bfloat16()
        self.k = torch.randn((R, self.L, self.B, self.Hkv, self.D), generator=g, device="cuda").bfloat16()
        self.v = torch.randn((R, self.L, self.B, self.Hkv, self.D), generator=g, device="cuda").bfloat16()
        self.flags_host = synth.decode_flags(c, seed)
        self.flags = torch.from_numpy(self.flags_host).cuda()
        self.flag_buf = torch.zeros((self.B,), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((self.L, self.B, self.Hq, self.D), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty((self.L, self.B, self.Hq), dtype=torch.float32, device="cuda")
        self.cache.workspace(self.Hq)
        self.t = 0
        self.graphs = None

    def layer_ops(self, r, l):
        # append + compact + decode of the layer in one launch (layer 0 also
        # launches the block bookkeeping)
        self.cache.decode_step(l, self.q[r, l], self.k[r, l], self.v[r, l],
                               self.flag_buf if l == 0 else None, out=self.out[l], lse=self.lse[l])

    def eager_step(self):
        self.flag_buf.copy_(self.flags[self.t])
        r = self.t % self.RING
        for l in range(self.L):
            self.layer_ops(r, l)
        self.t += 1

    def capture(self):
        self.graphs = []
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for r in range(self.RING):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=s):
                    for l in range(self.L):
                        self.layer_ops(r, l)
                self.graphs.append(g)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()

    def graph_step(self):
        self.flag_buf.copy_(self.flags[self.t])
        self.graphs[self.t % self.RING].replay()
        self.t += 1


def bench_decode(sl, args, world, rank):
    name = args.workload
    c = synth.WORKLOADS[name]
    wl = DecodeWorkload(sl, name, synth.WORKLOAD_SEED[name] + 7919 * rank, layers=args.layers)
    c = wl.cfg
    fill = min(1000, c["T"] - args.steps - args.warmup)
    for _ in range(fill):  # reach the steady-state block sizes (untimed set-up)
        wl.eager_step()
    wl.capture()
    for _ in range(args.warmup):
        wl.graph_step()
    torch.cuda.synchronize()
    K = args.steps
    assert wl.t + K <= c["T"], "stream too short for the requested steps"
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(K):
        wl.graph_step()
    s1.record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    t = _max_over_ranks(s0.elapsed_time(s1) / 1e3, world)
    value = c["B"] * K * world / t
    # dominant kernel: decode, timed alone over every layer of the current state
    counts = wl.cache.counts.cpu().numpy()
    rows = int(counts.sum())
    kv_bytes = rows * wl.Hkv * wl.D * 2 * 2  # K and V, bf16, every sequence, one layer
    r = wl.t % wl.RING
    reps = 20
    # the dominant kernel as the timed step runs it: the fused decode step of
    # layers 1..L-1 (append + flush copy + attention, no bookkeeping launch),
    # replayed as one CUDA graph.  Without the layer-0 bookkeeping a replay
    # repeats the same plan: it rewrites the same new-token row, or copies the
    # same rows out of place again, so every replay does the step's work.
    gdec = torch.cuda.CUDAGraph()
    s_ = torch.cuda.Stream()
    s_.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_):
        with torch.cuda.graph(gdec, stream=s_):
            for l in range(1, wl.L):
                wl.layer_ops(r, l)
    torch.cuda.current_stream().wait_stream(s_)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        gdec.replay()
    torch.cuda.synchronize()
    d0.record()
    for _ in range(reps):
        gdec.replay()
    d1.record()
    torch.cuda.synchronize()
    dec_s = d0.elapsed_time(d1) / 1e3 / (reps * (wl.L - 1))
    # algorithmic bytes of one launch: the retained K/V rows read, the new
    # token's K/V row written, q read, out and lse written
    alg_bytes = kv_bytes + wl.B * (wl.Hkv * wl.D * 2 * 2 + wl.Hq * wl.D * 2 * 2 + wl.Hq * 4)
    achieved = alg_bytes / dec_s / 1e9
    traffic = _traffic(name, units=rows)
    pk = _peaks()
    # e2e: the step with its per-step inputs copied from pinned host memory
    # (q, k_new, v_new of every layer and the flags) and the outputs read back
    e2e = None
    if not args.skip_e2e:
        hq = wl.q[0].cpu().pin_memory()
        hk = wl.k[0].cpu().pin_memory()
        hv = wl.v[0].cpu().pin_memory()
        hf = torch.from_numpy(wl.flags_host).pin_memory()
        hout = torch.empty(wl.out.shape, dtype=wl.out.dtype).pin_memory()
        hlse = torch.empty(wl.lse.shape, dtype=torch.float32).pin_memory()
        Ke = min(200, c["T"] - wl.t)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(Ke):
            r = wl.t % wl.RING
            wl.q[r].copy_(hq, non_blocking=True)
            wl.k[r].copy_(hk, non_blocking=True)
            wl.v[r].copy_(hv, non_blocking=True)
            wl.flag_buf.copy_(hf[wl.t], non_blocking=True)
            wl.graphs[r].replay()
            wl.t += 1
            hout.copy_(wl.out, non_blocking=True)
            hlse.copy_(wl.lse, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        te = _max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
        bi = (hq.numel() + hk.numel() + hv.numel()) * 2 + wl.B
        bo = hout.numel() * 2 + hlse.numel() * 4
        e2e = {"value": round(c["B"] * Ke * world / te, 2), "unit": "tokens/s",
               "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo)}
    line = {
        "metric": DECODE_METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name, "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "D": c["D"],
                   "layers": c["layers"], "a": c["a"], "s": c["s"], "past": c["past"], "w": c["w"],
                   "rope_theta": c.get("rope_theta"),
                   "timed_tokens": [wl.t - K, wl.t] if e2e is None else None,
                   "mean_retained_rows": round(rows / wl.B, 2),
                   "l2": "working set (~1 GB of cache) far above L2",
                   "parallelism": "replica per GPU (weak)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4), "traffic": traffic,
                     "bytes_per_launch": int(alg_bytes), "launch_us": round(dec_s * 1e6, 3),
                     "kernel": "sep_attn_decode_step, layers 1..%d in one CUDA graph (fused append "
                               "+ flush copy + attention), per-launch mean" % (wl.L - 1),
                     "peak_source": pk["src"] + " HBM copy"},
        "e2e": e2e, "clocks": clk,
        "gpu_launches": (wl.L + 1) * K,
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        line["cpu_baseline"] = cpu_baseline_decode(wl, budget_s=args.cpu_seconds)
    return line


def cpu_baseline_decode(wl, budget_s=10.0):
    """The oracle's decode path on host cores: the four-block state machine
    over the token stream (per-token cost) plus fp64 attention of every
    query head over the retained rows (per-layer cost), combined into
    tokens/s for all layers."""
    import oracle
    c = wl.cfg
    T0 = 1000
    flags = wl.flags_host
    t0 = time.time()
    sim = oracle.sepcache_simulate(flags[: T0 + 1], c["a"], c["s"], c["past"], c["w"], [T0])
    state_s = (time.time() - t0) / ((T0 + 1) * wl.B)  # per token and sequence
    q = wl.q[0, 0].float().cpu()
    k = wl.k[0, 0].float().cpu()
    v = wl.v[0, 0].float().cpu()
    t0 = time.time()
    reps = 0
    while True:
        for b in range(wl.B):
            n = int(sim["counts"][0, b].sum())
            kk = k[b].unsqueeze(1).expand(wl.Hkv, n, wl.D).contiguous()
            vv = v[b].unsqueeze(1).expand(wl.Hkv, n, wl.D).contiguous()
            if wl.rope_theta:
                oracle.decode_shifted(q[b], kk, vv, wl.rope_theta)
            else:
                oracle.attend(q[b], kk, vv)
        reps += 1
        if time.time() - t0 >= budget_s:
            break
    attn_s = (time.time() - t0) / (reps * wl.B)  # per layer, token and sequence
    tok_s = 1.0 / (state_s + wl.L * attn_s)
    return {"value": round(tok_s, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": "state machine over %d tokens x %d sequences; fp64 attention of all %d heads "
                      "at token %d, %d repetitions of %d sequences, scaled to %d layers" % (
                          T0 + 1, wl.B, wl.Hq, T0, reps, wl.B, wl.L)}


# ---------------------------------------------------------------- prompt ingestion


def bench_ingest(sl, args, world, rank):
    """Prompt ingestion: every step resets the cache and ingests a T-token
    prompt at all layers (sepcache_ingest); value = prompt tokens of all
    sequences per second.  Each layer has its own prompt K/V, so the
    retained rows come from HBM, and L2 is flushed between steps."""
    name = args.workload
    c = dict(synth.WORKLOADS[name])
    if args.layers:
        c["layers"] = args.layers
    seed = synth.WORKLOAD_SEED[name] + 7919 * rank
    B, Hkv, D, L, T = c["B"], c["Hkv"], c["D"], c["layers"], c["T"]
    cache = sl.SepCache(c["a"], c["s"], c["past"], c["w"], L, B, Hkv, D, dtype=torch.bfloat16)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    kp = torch.randn((L, B, Hkv, T, D), generator=g, device="cuda").bfloat16()
    vp = torch.randn((L, B, Hkv, T, D), generator=g, device="cuda").bfloat16()
    flags = synth.bernoulli_flags(synth.rng((seed, 31)), (B, T), c["p_sep"])
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    flush = torch.empty((256 << 20,), dtype=torch.uint8, device="cuda")

    def step():
        cache.init()
        for l in range(L):
            cache.ingest(l, kp[l], vp[l], is_sep, prefix, idx)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()  # untimed: evict L2 between steps
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    ms = [a.elapsed_time(b) for a, b in ev]
    t = _max_over_ranks(sum(ms) / 1e3, world)
    value = B * T * K * world / t
    rows = int(cache.counts.sum())
    # algorithmic bytes of a step: every retained K/V row read from the prompt
    # and written to the cache at every layer, plus the block metadata
    row_bytes = Hkv * D * 2
    alg = L * rows * row_bytes * 2 * 2 + B * (cache.cap * 5 + 16 + 8)
    step_s = statistics.mean(ms) / 1e3
    pk = _peaks()
    achieved = alg / step_s / 1e9
    line = {
        "metric": INGEST_METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name, "B": B, "Hkv": Hkv, "D": D, "layers": L, "T": T,
                   "a": c["a"], "s": c["s"], "past": c["past"], "w": c["w"],
                   "retained_rows_per_sequence": round(rows / B, 2),
                   "l2": "flushed between timed steps (256 MiB write, outside the events)",
                   "parallelism": "replica per GPU (weak)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4),
                     "traffic": _traffic(name, units=1),
                     "bytes_per_launch": int(alg), "launch_us": round(step_s * 1e6, 3),
                     "kernel": "sepcache_ingest over %d layers (state at layer 0, row copies at "
                               "every layer)" % L,
                     "peak_source": pk["src"] + " HBM copy"},
        "e2e": None, "clocks": clk,
        "gpu_launches": (L + 1) * K,  # layer 0: state + rows; other layers: rows
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        ref = run_reference_ingest(argparse.Namespace(steps=3, warmup=1), 1, c, name)
        line["cpu_baseline"] = ref["cpu_baseline"]
    return line


# ---------------------------------------------------------------- backward


def bench_backward(sl, args, world, rank):
    """Backward of the prefill workload: the gradients of q, k, v for a
    seeded dout, given the forward's out and lse (computed once, untimed).
    value = 10 D FLOP per kept pair and head (the five products S, dP, dV,
    dK, dQ) / device time of sep_attn_backward.  L2 flushed between steps."""
    name = args.workload
    wl = PrefillWorkload(sl, name, synth.WORKLOAD_SEED[name] + 7919 * rank)
    c = wl.cfg
    B, Hq, Hkv, S, D = c["B"], c["Hq"], c["Hkv"], c["S"], c["D"]
    g = torch.Generator(device="cuda")
    g.manual_seed(synth.WORKLOAD_SEED[name] + 17 + 7919 * rank)
    dout = torch.randn(wl.q.shape, generator=g, device="cuda").bfloat16()
    wl.step()  # forward: index, out, lse
    dq, dk, dv = torch.empty_like(wl.q), torch.empty_like(wl.k), torch.empty_like(wl.v)
    ws = torch.empty((int(sl.lib().sep_attn_backward_workspace(B, Hq, Hkv, S, D)),),
                     dtype=torch.uint8, device="cuda")
    flops = 10.0 * D * wl.kept_pairs

    def bwd():
        sl.backward(wl.q, wl.k, wl.v, wl.out, wl.lse, dout, wl.is_sep, wl.prefix, wl.idx,
                    c["a"], c["n"], dq=dq, dk=dk, dv=dv, workspace=ws)

    flush = torch.empty((256 << 20,), dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        flush.zero_()
        bwd()
    torch.cuda.synchronize()
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    for i in range(K):
        flush.zero_()  # untimed: evict L2 between steps
        ev[i][0].record()
        bwd()
        ev[i][1].record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    ms = [a_.elapsed_time(b_) for a_, b_ in ev]
    t = _max_over_ranks(sum(ms) / 1e3, world)
    value = flops * K * world / t / 1e12
    step_s = statistics.mean(ms) / 1e3
    pk = _peaks()
    achieved = flops / step_s / 1e12
    e2e = None
    if not args.skip_e2e:
        h = wl.host
        hq, hk, hv = (x.pin_memory() for x in (h["q"], h["k"], h["v"]))
        hout, hdo = wl.out.cpu().pin_memory(), dout.cpu().pin_memory()
        hlse = wl.lse.cpu().pin_memory()
        hsep = torch.from_numpy(h["is_sep"]).pin_memory()
        gq_h = torch.empty(dq.shape, dtype=dq.dtype).pin_memory()
        gk_h = torch.empty(dk.shape, dtype=dk.dtype).pin_memory()
        gv_h = torch.empty(dv.shape, dtype=dv.dtype).pin_memory()
        dout_d, out_d, lse_d = torch.empty_like(dout), torch.empty_like(wl.out), torch.empty_like(wl.lse)

        def e2e_step():
            wl.q.copy_(hq, non_blocking=True)
            wl.k.copy_(hk, non_blocking=True)
            wl.v.copy_(hv, non_blocking=True)
            out_d.copy_(hout, non_blocking=True)
            lse_d.copy_(hlse, non_blocking=True)
            dout_d.copy_(hdo, non_blocking=True)
            wl.is_sep.copy_(hsep, non_blocking=True)
            sl.build_index(wl.is_sep, out=(wl.prefix, wl.idx, wl.count))
            sl.backward(wl.q, wl.k, wl.v, out_d, lse_d, dout_d, wl.is_sep, wl.prefix, wl.idx,
                        c["a"], c["n"], dq=dq, dk=dk, dv=dv, workspace=ws)
            gq_h.copy_(dq, non_blocking=True)
            gk_h.copy_(dk, non_blocking=True)
            gv_h.copy_(dv, non_blocking=True)
        e2e_step()
        torch.cuda.synchronize()
        Ke = max(3, K // 2)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record()
        for _ in range(Ke):
            e2e_step()
        s1.record()
        torch.cuda.synchronize()
        te = _max_over_ranks(s0.elapsed_time(s1) / 1e3, world)
        bi = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hout, hdo, hlse, hsep))
        bo = sum(x.numel() * x.element_size() for x in (gq_h, gk_h, gv_h))
        e2e = {"value": round(flops * Ke * world / te / 1e12, 3), "unit": "TFLOP/s",
               "h2d_bytes_per_step": int(bi), "d2h_bytes_per_step": int(bo)}
    line = {
        "metric": BACKWARD_METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name, "B": B, "Hq": Hq, "Hkv": Hkv, "S": S, "D": D, "a": c["a"],
                   "n": c["n"], "kept_pairs": wl.kept_pairs,
                   "gflop_per_step": round(flops / 1e9, 3),
                   "l2": "flushed between timed steps (256 MiB write, outside the events)",
                   "parallelism": "replica per GPU (weak)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16"],
                     "unit": "TFLOP/s", "frac": round(achieved / pk["bf16"], 4),
                     "traffic": _traffic(name, units=1), "launch_us": round(step_s * 1e6, 3),
                     "kernel": ("sep_attn_backward: separator-row gather, item plan, "
                                "k_bwd_q (dQ, delta) + k_bwd_kv (dK, dV) on tcgen05, "
                                "separator-key scatter; traffic = all five launches"),
                     "peak_source": pk["src"] + " bf16 dense burst"},
        "e2e": e2e, "clocks": clk,
        # gather, plan, two tcgen05 kernels, scatter
        "gpu_launches": 5 * K,
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        ref = run_reference_backward(argparse.Namespace(steps=1, warmup=0), 1, c, name)
        line["cpu_baseline"] = ref["cpu_baseline"]
    return line


def run_reference_backward(args, world, c, name):
    """The oracle's backward on host cores over a bounded sample: the first
    sequence's first S' tokens (S' <= 1024), all query heads; the kept pairs
    of the sample give its FLOPs (10 D per pair)."""
    import oracle
    inp = synth.prefill_inputs(c, synth.WORKLOAD_SEED[name])
    Sp = min(c["S"], 1024)
    q = np.ascontiguousarray(_bits(inp["q"])[:1, :, :Sp])
    k = np.ascontiguousarray(_bits(inp["k"])[:1, :, :Sp])
    v = np.ascontiguousarray(_bits(inp["v"])[:1, :, :Sp])
    dout = q.copy()
    flags = np.ascontiguousarray(inp["is_sep"][:1, :Sp])
    kept = int(oracle.count_pairs(flags, c["a"], c["n"]).sum()) * c["Hq"]
    for _ in range(args.warmup):
        oracle.prefill_backward(q, k, v, dout, flags, c["a"], c["n"])
    t0 = time.time()
    for _ in range(args.steps):
        oracle.prefill_backward(q, k, v, dout, flags, c["a"], c["n"])
    dt = (time.time() - t0) / args.steps
    value = 10.0 * c["D"] * kept / dt / 1e12
    sample = "sequence 0, tokens 0..%d, all %d query heads (%d kept pairs) per step" % (
        Sp - 1, c["Hq"], kept)
    return {"impl": "reference", "metric": BACKWARD_METRIC, "value": round(value, 6),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "S": c["S"],
                       "D": c["D"], "a": c["a"], "n": c["n"]},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": min(oracle.nthreads(), c["Hkv"]), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def _bits(t):
    """bf16 tensor -> raw bits (uint16) for the oracle; fp32 tensor as is."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return t.contiguous().numpy()


# ---------------------------------------------------------------- mask-based generation


def _kept_rows_last(flags, T, a, n):
    """Kept keys of query T-1 per sequence: window + initial + separators."""
    lo = max(0, T - n)
    a0 = min(a, lo)
    return (T - lo) + a0 + flags[:, a0:lo].astype(np.int64).sum(1)


def bench_generate(sl, args, world, rank):
    """Mask-based generation: one token of all sequences through every layer,
    each layer attending over its own full history of S tokens with the kept
    set of the newest row (sep_attn_decode_masked per layer, one CUDA graph
    per step).  value = tokens/s.  The kept rows of 32 layers (~2 GB) are far
    larger than L2."""
    name = args.workload
    c = dict(synth.WORKLOADS[name])
    if args.layers:
        c["layers"] = args.layers
    seed = synth.WORKLOAD_SEED[name] + 7919 * rank
    B, Hq, Hkv, D, L, S = c["B"], c["Hq"], c["Hkv"], c["D"], c["layers"], c["S"]
    a, n, T = c["a"], c["n"], S
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    k = torch.randn((L, B, Hkv, S, D), generator=g, device="cuda").bfloat16()
    v = torch.randn((L, B, Hkv, S, D), generator=g, device="cuda").bfloat16()
    q = torch.randn((L, B, Hq, D), generator=g, device="cuda").bfloat16()
    flags = synth.bernoulli_flags(synth.rng((seed, 51)), (B, S), c["p_sep"])
    is_sep = torch.from_numpy(flags).cuda()
    prefix, idx, _ = sl.build_index(is_sep)
    out = torch.empty((L, B, Hq, D), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((L, B, Hq), dtype=torch.float32, device="cuda")

    def layer(l):
        sl.decode_masked(q[l], k[l], v[l], prefix, idx, T, a, n, out=out[l], lse=lse[l])

    gstep = torch.cuda.CUDAGraph()
    s_ = torch.cuda.Stream()
    s_.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s_):
        for l in range(L):  # once eagerly, then captured
            layer(l)
        with torch.cuda.graph(gstep, stream=s_):
            for l in range(L):
                layer(l)
    torch.cuda.current_stream().wait_stream(s_)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        gstep.replay()
    torch.cuda.synchronize()
    K = args.steps
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    _barrier(world)
    torch.cuda.synchronize()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record()
    for _ in range(K):
        gstep.replay()
    s1.record()
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    local_s = s0.elapsed_time(s1) / 1e3
    t = _max_over_ranks(local_s, world)
    value = B * K * world / t
    # the dominant kernel: one layer's launch, the mean over this rank's graph
    per_launch = local_s / (K * L)
    kept = _kept_rows_last(flags, T, a, n)
    alg = int(kept.sum()) * Hkv * D * 2 * 2 + B * Hq * (D * 2 * 2 + 4)
    achieved = alg / per_launch / 1e9
    pk = _peaks()
    e2e = None
    if not args.skip_e2e:
        hq = q.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        Ke = min(K, 100)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(Ke):
            q.copy_(hq, non_blocking=True)
            gstep.replay()
            hout.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)
        e1.record()
        torch.cuda.synchronize()
        te = _max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
        e2e = {"value": round(B * Ke * world / te, 2), "unit": "tokens/s",
               "h2d_bytes_per_step": int(hq.numel() * 2),
               "d2h_bytes_per_step": int(hout.numel() * 2 + hlse.numel() * 4)}
    line = {
        "metric": GENERATE_METRIC, "value": round(value, 2), "unit": "tokens/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(t / K * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": name, "B": B, "Hq": Hq, "Hkv": Hkv, "D": D, "layers": L,
                   "history": T, "a": a, "n": n,
                   "mean_kept_rows": round(float(kept.mean()), 2),
                   "l2": "kept rows of all layers (~2 GB) far above L2",
                   "parallelism": "replica per GPU (weak)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm"], 4),
                     "traffic": _traffic(name, units=1),
                     "bytes_per_launch": alg, "launch_us": round(per_launch * 1e6, 3),
                     "kernel": "sep_attn_decode_masked of one layer (gathered kept rows), "
                               "per-launch mean over the step graph",
                     "peak_source": pk["src"] + " HBM copy"},
        "e2e": e2e, "clocks": clk,
        "gpu_launches": L * K,
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        ref = run_reference_generate(argparse.Namespace(steps=2, warmup=1), 1, c, name)
        line["cpu_baseline"] = ref["cpu_baseline"]
    return line


def run_reference_generate(args, world, c, name):
    """The oracle's mask-based generation on host cores: fp64 attention of
    every query head of one sequence over its kept set at one layer per step
    (the bounded sample); the step's time is scaled to all sequences and
    layers."""
    import oracle
    seed = synth.WORKLOAD_SEED[name]
    B, Hq, Hkv, D, L, S = c["B"], c["Hq"], c["Hkv"], c["D"], c["layers"], c["S"]
    g = synth.rng((seed, 52))
    flags = synth.bernoulli_flags(synth.rng((seed, 51)), (1, S), c["p_sep"])
    q = synth.normal(g, (1, Hq, D), 1.0, "bf16")
    k = synth.normal(g, (1, Hkv, S, D), 1.0, "bf16")
    v = synth.normal(g, (1, Hkv, S, D), 1.0, "bf16")
    for _ in range(args.warmup):
        oracle.decode_masked(q, k, v, flags, S, c["a"], c["n"])
    t0 = time.time()
    for _ in range(args.steps):
        oracle.decode_masked(q, k, v, flags, S, c["a"], c["n"])
    wall = time.time() - t0
    per_seq_layer = wall / args.steps
    per_step = per_seq_layer * B * L  # one token of every sequence through every layer
    value = B / per_step
    sample = ("fp64 attention of all %d query heads of 1 of %d sequences at 1 of %d layers per "
              "step, scaled to all" % (Hq, B, L))
    return {"impl": "reference", "metric": GENERATE_METRIC, "value": round(value, 3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "B": B, "Hq": Hq, "Hkv": Hkv, "D": D, "layers": L,
                       "history": S, "a": c["a"], "n": c["n"]},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s",
                             "cores": oracle.nthreads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- reference arm


def run_reference_decode(args, world, c, name):
    """The oracle's decode on host cores.  Set-up (untimed): the state machine
    over the first 1000 tokens.  A step: the state machine for one more token
    of every sequence, then fp64 attention of every query head of 2 of the
    sequences at one layer (the bounded sample); the step's time is scaled to
    all sequences and layers."""
    import oracle
    seed = synth.WORKLOAD_SEED[name]
    flags = synth.decode_flags(c, seed)
    B, L = c["B"], c["layers"]
    wl = dict(c, B=B)
    T0 = 1000
    nb = 2
    state_t, attn_t, n_rows = 0.0, 0.0, 0

    def one(t, timed):
        nonlocal state_t, attn_t, n_rows
        t0 = time.time()
        sim = oracle.sepcache_simulate(flags[: t + 1], c["a"], c["s"], c["past"], c["w"], [t])
        t1 = time.time()
        q, _, _ = synth.decode_step_qkv(wl, seed, t, 0)
        for b in range(nb):
            n = int(sim["counts"][0, b].sum())
            pos = sim["pos"][0, b, :n]
            ks = torch.stack([synth.decode_step_qkv(wl, seed, int(p2), 0)[1][b] for p2 in pos[:1]], 1)
            kk = ks.expand(c["Hkv"], n, c["D"]).contiguous()
            if c.get("rope_theta"):
                oracle.decode_shifted(q[b], kk, kk, c["rope_theta"])
            else:
                oracle.attend(q[b], kk, kk)
        t2 = time.time()
        if timed:
            # the simulation replays t+1 tokens; one token of the stream costs 1/(t+1) of it
            state_t += (t1 - t0) / (t + 1)
            attn_t += (t2 - t1) / nb
            n_rows += n
    for w in range(args.warmup):
        one(T0 + w, False)
    t0 = time.time()
    for k in range(args.steps):
        one(T0 + args.warmup + k, True)
    wall = time.time() - t0
    per_step = state_t / args.steps + L * B * attn_t / args.steps  # one token of all sequences
    value = B / per_step
    sample = ("state machine per token; fp64 attention of all %d query heads of %d of %d "
              "sequences at 1 of %d layers per step over the retained row count (one K/V row "
              "repeated: the cost depends on the count only), scaled to all" % (
                  c["Hq"], nb, B, L))
    return {"impl": "reference", "metric": DECODE_METRIC, "value": round(value, 3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "B": B, "Hq": c["Hq"], "Hkv": c["Hkv"], "D": c["D"],
                       "layers": L, "a": c["a"], "s": c["s"], "past": c["past"], "w": c["w"],
                       "rope_theta": c.get("rope_theta")},
            "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_reference_ingest(args, world, c, name):
    """The oracle's way to ingest a prompt: T sequential appends of the
    four-block state machine for every sequence, then the retained rows'
    K/V gathered from the prompt (numpy).  Bounded sample: one layer's rows
    per step, scaled to all layers."""
    import oracle
    seed = synth.WORKLOAD_SEED[name]
    B, Hkv, D, L, T = c["B"], c["Hkv"], c["D"], c["layers"], c["T"]
    flags = synth.bernoulli_flags(synth.rng((seed, 31)), (B, T), c["p_sep"])
    g = synth.rng((seed, 32))
    kp = g.standard_normal((B, Hkv, T, D), dtype=np.float32)
    vp = g.standard_normal((B, Hkv, T, D), dtype=np.float32)
    st_t, cp_t = 0.0, 0.0

    def one(timed):
        nonlocal st_t, cp_t
        t0 = time.time()
        sim = oracle.sepcache_simulate(flags.T.copy(), c["a"], c["s"], c["past"], c["w"], [T - 1])
        t1 = time.time()
        for b in range(B):
            n = int(sim["counts"][0, b].sum())
            pos = sim["pos"][0, b, :n]
            _ = kp[b][:, pos].copy(), vp[b][:, pos].copy()
        t2 = time.time()
        if timed:
            st_t += t1 - t0
            cp_t += t2 - t1
    for _ in range(args.warmup):
        one(False)
    t0 = time.time()
    for _ in range(args.steps):
        one(True)
    wall = time.time() - t0
    per_step = (st_t + L * cp_t) / args.steps
    value = B * T / per_step
    sample = ("state machine over %d tokens x %d sequences and the retained rows of 1 of %d "
              "layers per step, scaled to all layers" % (T, B, L))
    return {"impl": "reference", "metric": INGEST_METRIC, "value": round(value, 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(wall / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": name, "B": B, "Hkv": Hkv, "D": D, "layers": L, "T": T,
                       "a": c["a"], "s": c["s"], "past": c["past"], "w": c["w"]},
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle
    name = args.workload
    c = synth.WORKLOADS[name]
    if c["kind"] == "decode":
        return run_reference_decode(args, world, c, name)
    if c["kind"] == "ingest":
        return run_reference_ingest(args, world, c, name)
    if c["kind"] == "generate":
        return run_reference_generate(args, world, c, name)
    if c["kind"] == "backward":
        return run_reference_backward(args, world, c, name)
    inp = synth.prefill_inputs(c, synth.WORKLOAD_SEED[name])
    rows, frac = _sample_rows(c, budget_hint=4.0)
    kept = _kept_pairs_rows(inp["is_sep"], c, rows)
    flops = 4.0 * c["D"] * kept
    for _ in range(args.warmup):
        oracle.prefill_rows(inp["q"], inp["k"], inp["v"], inp["is_sep"], c["a"], c["n"], rows=rows)
    t0 = time.time()
    for _ in range(args.steps):
        oracle.prefill_rows(inp["q"], inp["k"], inp["v"], inp["is_sep"], c["a"], c["n"], rows=rows)
    dt = time.time() - t0
    value = flops * args.steps / dt / 1e12
    sample = "%d of %d query rows (%.3g of the workload) per step" % (
        rows.size, c["B"] * c["Hq"] * c["S"], frac)
    return {"impl": "reference", "metric": PREFILL_METRIC, "value": round(value, 6),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": name, "B": c["B"], "Hq": c["Hq"], "Hkv": c["Hkv"], "S": c["S"],
                       "D": c["D"], "a": c["a"], "n": c["n"]},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s",
                             "cores": oracle.nthreads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--skip-cpu", action="store_true", help="omit the cpu_baseline leg")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--layers", type=int, default=None,
                    help="decode: fewer layers than the workload (a small case for profilers); "
                         "the JSON line then names the count in config.layers")
    args = ap.parse_args()
    kind = synth.WORKLOADS[args.workload]["kind"]
    if args.steps is None:
        args.steps = {"prefill": 50, "ingest": 20, "generate": 200, "backward": 20}.get(kind, 2000)
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    world, rank, _ = _dist_setup(args.gpus)
    import streaming_kv_cache_sep_b200 as sl
    if kind == "prefill":
        line = bench_prefill(sl, args, world, rank)
    elif kind == "ingest":
        line = bench_ingest(sl, args, world, rank)
    elif kind == "generate":
        line = bench_generate(sl, args, world, rank)
    elif kind == "backward":
        line = bench_backward(sl, args, world, rank)
    else:
        line = bench_decode(sl, args, world, rank)
    status = sl.device_status()
    if status != 0:
        raise RuntimeError("device error bits set: %d" % status)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
