"""Benchmark of the RecSA hot path on B200 (one JSON line on stdout).

Headline: decode queries/s at a 1M-token context (B = 4 sequences, 32 query / 8 KV
heads, head_dim 128, b = 16, k = 8, one query per sequence), each step one
recsa_decode call over a tree built beforehand, L2 flushed between steps.  The same
line carries the roofline of the attend kernel, an end-to-end figure through host
buffers, a sweep of independent queries per sequence, causal prefill tokens/s
(524K + 8K chunk, and 1M + 8K), the 2M-token tree build in GB/s, 2M decode latency,
decode at 131K (B = 8), the decode loop (append + decode), per-sequence lengths, a paged
cache, and the fp64 oracle timed on the host cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--quick]

With --gpus N > 1 it runs under torchrun, one rank per GPU: every rank decodes its
own 4 sequences (weak scaling, no data-path collective); the timed region is
bracketed by barriers and the maximum over ranks is reported.
"""

from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

import recsa_inputs as I  # noqa: E402

METRIC = "RecSA decode queries/s & prefill tokens/s at 1M ctx; achieved HBM GB/s vs peak"
ROW = 256  # bytes of one bf16 row of 128
FLUSH_BYTES = 256 << 20  # > 126 MB L2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed work runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.idx = device_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        busy = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- timing

class Timer:
    """Per-step CUDA-event timing on the launching stream, L2 flushed before each step."""

    def __init__(self, dist_on: bool):
        self.dist_on = dist_on
        self.flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush(self):
        self.flush_buf.zero_()

    def barrier(self):
        if self.dist_on:
            import torch.distributed as dist
            dist.barrier()

    def run(self, fn, steps: int, warmup: int, flush: bool = True):
        for _ in range(warmup):
            if flush:
                self.flush()
            fn()
        stream = torch.cuda.current_stream()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        self.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for a, b in ev:
            if flush:
                self.flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        self.barrier()
        wall = time.perf_counter() - t0
        per = [a.elapsed_time(b) / 1e3 for a, b in ev]
        return per, wall


def max_over_ranks(x: float, dist_on: bool) -> float:
    """Largest value over all ranks (every rank gets it); identity on one process."""
    if not dist_on:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: int, steps: int, local_seconds: float, world: int, dist_on: bool):
    """Whole-job units/s of independent replicas: all ranks' units over the slowest rank's time."""
    slowest = max_over_ranks(local_seconds, dist_on)
    return world * units_per_rank_step * steps / slowest, slowest


def pct(xs, q):
    s = sorted(xs)
    return s[min(len(s) - 1, max(0, int(round(q * (len(s) - 1)))))]


# ----------------------------------------------------------------------------- legs

def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_sparse_attention_build_b200", "csrc")
    for f in ("recsa_attend.cu", "recsa_device.cuh", "recsa_internal.h"):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_profile(name: str):
    """Numeric fields of a committed ncu summary (profiles/<name>.txt, "key: value" lines),
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{name}.txt")
    try:
        kv = {k.strip(): v.strip() for k, v in (line.split(":", 1) for line in open(path) if ":" in line)}
        if kv.get("kernel_source_sha256", "") != kernel_source_sha():
            return None
        out = {}
        for k, v in kv.items():
            try:
                out[k] = float(v)
            except ValueError:
                out[k] = v
        return out
    except Exception:
        return None


def recorded_traffic(name: str, tiles: int):
    """DRAM bytes of a launch of `tiles` tiles from a committed ncu summary of smaller cases
    (a fixed part per launch plus a part per tile, fitted from two sizes), if it matches the
    current kernel source."""
    prof = recorded_profile(name)
    if prof is None:
        return None
    if "fixed_bytes" in prof and "bytes_per_tile" in prof:
        return prof["fixed_bytes"] + prof["bytes_per_tile"] * tiles
    if "dram_bytes_per_launch" in prof:
        return prof["dram_bytes_per_launch"] / prof.get("tiles", tiles) * tiles
    return None


def make_tree(R, p, inp, length, build=True):
    tree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], length)
    ws = R.Workspace(p, tree.capacity, "cuda")
    if build:
        R.build_tree(p, tree)
    return tree, ws


def decode_entries(R, p, tree, ws, q):
    B, Q, Hq, _ = q.shape
    tiles = B * p.num_kv_heads * Q
    ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")
    out = torch.empty(B, Q, Hq, 128, dtype=torch.bfloat16, device="cuda")
    R.decode(p, tree, q, out, ws, entries=ent)
    R.check_device_errors(ws)
    return int(ent.sum().item())


def leg_decode_1m(R, timer, args, dist_on, hbm_peak, peaks_src, heads=None):
    """The headline decode.  heads = (h0, h1): this rank's block of KV heads of every
    sequence (sharding by KV head); None: the whole batch (a replica)."""
    w = I.WORKLOADS["decode_1m"]
    if heads is not None:
        g = w.q_heads // w.kv_heads
        w = dataclasses.replace(w, kv_heads=heads[1] - heads[0], q_heads=g * (heads[1] - heads[0]))
    inp = I.decode_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    tree, ws = make_tree(R, p, inp, w.length)
    q = inp["q"]
    B, Q, Hq, _ = q.shape
    out = torch.empty(B, Q, Hq, 128, dtype=torch.bfloat16, device="cuda")
    rows = decode_entries(R, p, tree, ws, q)
    bytes_per_launch = rows * ROW + q.numel() * 2 + out.numel() * 2
    torch.cuda.synchronize()

    per, wall = timer.run(lambda: R.decode(p, tree, q, out, ws), args.steps, args.warmup)
    total = max_over_ranks(sum(per), dist_on)
    mean_s = total / args.steps
    res = dict(per_step_s=per, total_s=total, wall_s=wall, mean_s=mean_s, rows=rows,
               bytes_per_launch=bytes_per_launch, queries=B * Q)

    # end to end from host buffers, two ways, both inside the timed step: (mapped) the
    # host-buffer call with pinned buffers, which the kernel reads and writes across the
    # host link itself; (staged) one copy of the queries to the device, the decode call,
    # one copy of the output back (pinned buffers, cudaMemcpyAsync each way)
    q_host = q.cpu().pin_memory()
    out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    q_dev = torch.empty_like(q)

    def e2e_mapped():
        R.decode_host(p, tree, q_host, out_host, q_dev, out, ws)

    def e2e_staged():
        q_dev.copy_(q_host, non_blocking=True)
        R.decode(p, tree, q_dev, out, ws)
        out_host.copy_(out, non_blocking=True)

    per_m, _ = timer.run(e2e_mapped, args.steps, args.warmup)
    per_s, _ = timer.run(e2e_staged, args.steps, args.warmup)
    t_m = max_over_ranks(sum(per_m), dist_on)
    t_s = max_over_ranks(sum(per_s), dist_on)
    # breakdown of the staged step: each piece between its own events, L2 flushed first
    stream = torch.cuda.current_stream()
    pieces = {"h2d": [], "kernel": [], "d2h": []}
    for i in range(max(50, min(args.steps, 400))):
        timer.flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        q_dev.copy_(q_host, non_blocking=True)
        ev[1].record(stream)
        R.decode(p, tree, q_dev, out, ws)
        ev[2].record(stream)
        out_host.copy_(out, non_blocking=True)
        ev[3].record(stream)
        torch.cuda.synchronize()
        if i >= 5:
            for k, (a, b) in zip(pieces, ((0, 1), (1, 2), (2, 3))):
                pieces[k].append(ev[a].elapsed_time(ev[b]) * 1e3)
    res["e2e"] = {"mapped_us_per_step": t_m / args.steps * 1e6, "staged_us_per_step": t_s / args.steps * 1e6,
                  "path": "mapped" if t_m <= t_s else "staged",
                  "staged_breakdown_us_median": {k: statistics.median(v) for k, v in pieces.items()}}
    res["e2e_total_s"] = min(t_m, t_s)
    res["h2d"] = q_host.numel() * 2
    res["d2h"] = out_host.numel() * 2

    # independent decode queries per sequence (throughput regime), same caches
    sweep = []
    for nq in ([1, 4, 16, 64] if not args.quick else [1, 16]):
        g = torch.Generator(device="cuda").manual_seed(77 + nq)
        qs = torch.randn(B, nq, Hq, 128, generator=g, device="cuda").to(torch.bfloat16)
        outs = torch.empty(B, nq, Hq, 128, dtype=torch.bfloat16, device="cuda")
        r = decode_entries(R, p, tree, ws, qs)
        nb = r * ROW + qs.numel() * 2 + outs.numel() * 2
        st = max(20, args.steps // (4 * nq))
        per_s, _ = timer.run(lambda: R.decode(p, tree, qs, outs, ws), st, max(3, args.warmup // 4))
        t = max_over_ranks(sum(per_s), dist_on) / st
        sweep.append({"queries_per_seq": nq, "queries_per_s": B * nq / t, "us_per_call": t * 1e6,
                      "logical_GBps": nb / t / 1e9, "frac": nb / t / 1e9 / hbm_peak})
    res["sweep"] = sweep
    R.check_device_errors(ws)
    del tree, ws, inp, q, out
    torch.cuda.empty_cache()
    return res, w


def leg_prefill(R, timer, args, dist_on, hbm_peak, name, length):
    base = I.WORKLOADS["prefill_524k"]
    w = dataclasses.replace(base, name=name, length=length)
    inp = I.prefill_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    tree, ws = make_tree(R, p, inp, w.length)
    k_new, v_new, q = inp["k_new"], inp["v_new"], inp["q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    tiles = w.batch * w.kv_heads * w.chunk
    ent = torch.zeros(tiles, 2, dtype=torch.int32, device="cuda")

    def step(entries=None):
        tree.length = w.length  # the call appends at L; every step redoes the same chunk
        R.prefill_chunk(p, tree, k_new, v_new, q, out, ws, entries=entries)

    step(ent)
    R.check_device_errors(ws)
    rows = int(ent.sum().item())
    append_bytes = 2 * 2 * k_new.numel() * 2  # read chunk K/V, write into the caches
    nodes_touched = 0
    span = w.branching
    for _ in range(tree.levels):
        nodes_touched += -(-(w.length + w.chunk) // span) - w.length // span
        span *= w.branching
    ext_bytes = nodes_touched * w.kv_heads * w.batch * ROW * 2 * (w.branching + 1)
    logical = rows * ROW + q.numel() * 2 + out.numel() * 2 + append_bytes + ext_bytes
    steps = max(5, args.steps // 200) if not args.quick else 5
    per, _ = timer.run(step, steps, 2)
    t = max_over_ranks(sum(per), dist_on) / steps
    R.check_device_errors(ws)
    del tree, ws, inp
    torch.cuda.empty_cache()
    res = {"workload": f"{name}: B={w.batch}, L={w.length} cached + C={w.chunk} chunk, Hq={w.q_heads}, "
                       f"Hkv={w.kv_heads}, b={w.branching}, k={w.top_k}",
           "tokens_per_s": w.batch * w.chunk / t, "ms_per_chunk": t * 1e3,
           "rows_read": rows, "logical_bytes": logical, "logical_GBps": logical / t / 1e9,
           "logical_frac_of_hbm": logical / t / 1e9 / hbm_peak,
           "note": "append + extension build + causal attend per call; rows re-read by neighbouring "
                   "queries hit L2, so logical GB/s can exceed HBM bandwidth"}
    prof = recorded_profile("attend_warp_prefill_counters")
    if prof is not None:
        per_tile_dram = prof["dram_bytes_per_launch"] / prof["tiles"]
        per_tile_inst = prof["warp_inst_per_launch"] / prof["tiles"]
        dram = per_tile_dram * tiles
        inst = per_tile_inst * tiles
        peak_issue = prof["sms"] * 4 * prof["sm_hz"]  # one warp instruction per sub-partition per cycle
        res["dram"] = {"bytes_per_chunk": dram, "GBps": dram / t / 1e9, "frac_of_hbm": dram / t / 1e9 / hbm_peak,
                       "time": "the whole chunk call (append + extension + attend)",
                       "source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of the attend kernel on the "
                                 f"{prof['case']} case, per tile, times this call's {tiles} tiles"}
        res["issue"] = {"warp_inst_per_chunk": inst, "frac_of_peak_issue": inst / t / peak_issue,
                        "peak_issue_per_s": peak_issue,
                        "source": "ncu smsp__inst_executed.sum of the attend kernel on the same case, per tile; "
                                  "peak = SMs x 4 sub-partitions x SM clock"}
    return res


def leg_decode_loop(R, timer, args, dist_on):
    """Token-by-token decode at 1M (B = 4).  A decode-loop step appends the step's token to
    every sequence and updates the tree over it (recsa_append: the token slot and its
    ancestor path, one launch), then decodes that token's query over all tokens so far
    (recsa_decode).  Also timed: the same step as a causal chunk of one token
    (recsa_prefill_chunk with C = 1).  Each step grows the cache by one token."""
    w = I.WORKLOADS["decode_1m"]
    warmup, steps = 4, 64 if not args.quick else 16
    per_leg = warmup + steps
    inp = I.decode_inputs(w, device="cuda", capacity=w.length + 3 * per_leg + 8)
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    tree, ws = make_tree(R, p, inp, w.length)
    g = torch.Generator(device="cuda").manual_seed(91)
    B, Hkv, Hq = w.batch, w.kv_heads, w.q_heads
    toks = [tuple(torch.randn(B, 1, h, 128, generator=g, device="cuda").to(torch.bfloat16) for h in (Hkv, Hkv, Hq))
            for _ in range(3 * per_leg + 2)]
    out = torch.empty(B, 1, Hq, 128, dtype=torch.bfloat16, device="cuda")
    nxt = [0]

    def append_decode():
        kn, vn, qn = toks[nxt[0]]
        nxt[0] += 1
        R.append(p, tree, kn, vn)
        R.decode(p, tree, qn, out, ws)

    def chunk_of_one():
        kn, vn, qn = toks[nxt[0]]
        nxt[0] += 1
        R.prefill_chunk(p, tree, kn, vn, qn, out, ws)

    per, _ = timer.run(append_decode, steps, warmup)
    t = max_over_ranks(sum(per), dist_on) / steps
    per, _ = timer.run(chunk_of_one, steps, warmup)
    t_chunk = max_over_ranks(sum(per), dist_on) / steps
    R.check_device_errors(ws)

    # the same step as recsa_decode_step replayed from one CUDA graph: lengths on the device,
    # each step's token and query written into fixed buffers before the replay (untimed, as
    # the model would write them)
    seq_len = torch.full((B,), tree.length, dtype=torch.int64, device="cuda")
    gtree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], tree.length, k_node=tree.k_node,
                        v_node=tree.v_node, seq_len=seq_len)
    kbuf, vbuf, qbuf = (torch.empty(B, 1, h, 128, dtype=torch.bfloat16, device="cuda") for h in (Hkv, Hkv, Hq))

    def fill():
        kn, vn, qn = toks[nxt[0]]
        nxt[0] += 1
        kbuf.copy_(kn)
        vbuf.copy_(vn)
        qbuf.copy_(qn)

    fill()
    R.decode_step(p, gtree, kbuf, vbuf, qbuf, out, ws)  # first launches outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=side):
        R.decode_step(p, gtree, kbuf, vbuf, qbuf, out, ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(warmup + steps):
        fill()
        timer.flush()
        if i >= warmup:
            ev[i - warmup][0].record(stream)
        graph.replay()
        if i >= warmup:
            ev[i - warmup][1].record(stream)
    torch.cuda.synchronize()
    t_graph = max_over_ranks(sum(a.elapsed_time(b) / 1e3 for a, b in ev), dist_on) / steps
    R.check_device_errors(ws)
    del graph
    del tree, gtree, ws, inp
    torch.cuda.empty_cache()
    return {"workload": f"decode_loop_1m: B={B}, L={w.length} + 1 token per sequence per step, Hq={Hq}, "
                        f"Hkv={Hkv}, b={w.branching}, k={w.top_k}",
            "tokens_per_s": B / t, "us_per_step": t * 1e6, "launches_per_step": 2,
            "note": "recsa_append (token slot + ancestor path of every (sequence, KV head), one launch) + "
                    "recsa_decode of the new token's query; L2 flushed before each step",
            "graph_replay": {"us_per_step": t_graph * 1e6, "tokens_per_s": B / t_graph, "launches_per_step": 3,
                             "note": "recsa_decode_step (append, length advance, decode) captured once into a CUDA "
                                     "graph and replayed per step; L2 flushed before each replay (the eager calls "
                                     "above are queued while that flush runs, so their launch cost is hidden here "
                                     "too; the graph pays off when steps run back to back)"},
            "causal_chunk_of_1": {"us_per_step": t_chunk * 1e6, "launches_per_step": 2,
                                  "note": "recsa_prefill_chunk with C = 1: the same update, then the causal "
                                          "attend (the partial node on the query's path always expanded)"}}


def leg_decode_varlen(R, timer, args, dist_on):
    """Decode over a batch of unequal sequences: 8 sequences of 8/8, 7/8, ..., 1/8 of 1M tokens
    (the decode_1m head shape, b = 16, k = 8, one query each) in one call with per-sequence
    lengths, next to the same batch with every sequence at 1M."""
    w = dataclasses.replace(I.WORKLOADS["decode_1m"], batch=8)
    inp = I.decode_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    lens = [w.length * (w.batch - i) // w.batch for i in range(w.batch)]
    seq_len = torch.tensor(lens, dtype=torch.int64, device="cuda")
    q = inp["q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    steps = max(20, args.steps // 10) if not args.quick else 20
    res = {"workload": f"decode_varlen: B={w.batch}, lengths {lens[-1]}..{lens[0]} (step {lens[0] - lens[1]}), "
                       f"Hq={w.q_heads}, Hkv={w.kv_heads}, b={w.branching}, k={w.top_k}, 1 query per sequence"}
    for name, sl in (("per_sequence_lengths", seq_len), ("all_at_1m", None)):
        tree = R.RecsaTree(p, inp["k_tok"], inp["v_tok"], inp["pooler"], w.length, seq_len=sl)
        ws = R.Workspace(p, tree.capacity, "cuda")
        R.build_tree(p, tree)
        per, _ = timer.run(lambda: R.decode(p, tree, q, out, ws), steps, 3)
        t = max_over_ranks(sum(per), dist_on) / steps
        R.check_device_errors(ws)
        res[name] = {"queries_per_s": w.batch / t, "us_per_call": t * 1e6}
        del tree, ws
    del inp
    torch.cuda.empty_cache()
    return res


def leg_decode_paged(R, timer, args, dist_on):
    """The headline decode (1M, B = 4) over a paged token cache: pages of 64 tokens in a pool
    placed by a shuffled page table, next to the same caches stored contiguously."""
    w = I.WORKLOADS["decode_1m"]
    inp = I.decode_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    P = 64
    B, H, cap = w.batch, w.kv_heads, w.length
    pps = cap // P
    g = torch.Generator(device="cpu").manual_seed(17)
    perm = torch.randperm(B * pps, generator=g).to(torch.int32)
    table = perm.view(B, pps).contiguous().cuda()
    pools = []
    for x in (inp["k_tok"], inp["v_tok"]):
        pool = torch.empty(B * pps, H, P, 128, dtype=torch.bfloat16, device="cuda")
        pool[perm.long().cuda()] = x.view(B, H, pps, P, 128).permute(0, 2, 1, 3, 4).reshape(B * pps, H, P, 128)
        pools.append(pool)
    q = inp["q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    steps = max(20, args.steps // 10) if not args.quick else 20
    res = {"workload": f"decode_paged_1m: B={B}, L={w.length}, pages of {P} tokens, shuffled table, "
                       f"Hq={w.q_heads}, Hkv={H}, b={w.branching}, k={w.top_k}, 1 query per sequence"}
    del inp["k_tok"], inp["v_tok"]
    tree = R.RecsaTree(p, pools[0], pools[1], inp["pooler"], w.length, page_table=table)
    ws = R.Workspace(p, tree.capacity, "cuda")
    R.build_tree(p, tree)
    per, _ = timer.run(lambda: R.decode(p, tree, q, out, ws), steps, 3)
    t = max_over_ranks(sum(per), dist_on) / steps
    R.check_device_errors(ws)
    res["paged"] = {"queries_per_s": B / t, "us_per_call": t * 1e6}
    del tree, ws, pools, table
    torch.cuda.empty_cache()
    return res


def leg_decode_131k(R, timer, args, dist_on, hbm_peak):
    """Decode at 131K tokens, B = 8 (one query per sequence, per-(KV head, channel) scales on
    K and V): queries/s and the logical bytes against the HBM roofline."""
    w = I.WORKLOADS["decode_131k"]
    inp = I.decode_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    tree, ws = make_tree(R, p, inp, w.length)
    q = inp["q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    rows = decode_entries(R, p, tree, ws, q)
    nb = rows * ROW + q.numel() * 2 + out.numel() * 2
    steps = max(20, args.steps // 10) if not args.quick else 20
    per, _ = timer.run(lambda: R.decode(p, tree, q, out, ws), steps, 3)
    t = max_over_ranks(sum(per), dist_on) / steps
    R.check_device_errors(ws)
    del tree, ws, inp
    torch.cuda.empty_cache()
    return {"workload": f"decode_131k: B={w.batch}, L={w.length}, Hq={w.q_heads}, Hkv={w.kv_heads}, "
                        f"b={w.branching}, k={w.top_k}, 1 query per sequence",
            "queries_per_s": w.batch / t, "us_per_call": t * 1e6, "rows_read_per_call": rows,
            "logical_GBps": nb / t / 1e9, "frac": nb / t / 1e9 / hbm_peak}


def leg_build_2m(R, timer, args, dist_on, hbm_peak):
    w = I.WORKLOADS["build_decode_2m"]
    inp = I.decode_inputs(w, device="cuda")
    p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
    tree, ws = make_tree(R, p, inp, w.length, build=False)
    tok_bytes = 2 * inp["k_tok"].numel() * 2
    node_rows = 0
    n = w.length
    while n > w.branching:
        n = -(-n // w.branching)
        node_rows += n
    node_bytes = 2 * node_rows * w.kv_heads * w.batch * ROW
    algorithmic = tok_bytes + node_bytes  # every token read once, every node written once
    # the median of 10 builds (one launch per level): a single slow step moved a 5-step mean by 20%
    steps = max(10, args.steps // 200) if not args.quick else 3
    per, _ = timer.run(lambda: R.build_tree(p, tree), steps, 2)
    t_mean = max_over_ranks(sum(per), dist_on) / steps
    t = max_over_ranks(statistics.median(per), dist_on)
    q = inp["q"]
    out = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    rows = decode_entries(R, p, tree, ws, q)
    per_d, _ = timer.run(lambda: R.decode(p, tree, q, out, ws), max(50, args.steps // 4), args.warmup)
    R.check_device_errors(ws)
    del tree, ws, inp
    torch.cuda.empty_cache()
    return {"workload": f"build_decode_2m: B=1, L={w.length}, Hkv=8, b=16 (build); decode B=1, k=8",
            "build_ms": t * 1e3, "build_ms_mean": t_mean * 1e3, "build_steps": steps,
            "build_GBps": algorithmic / t / 1e9, "build_frac": algorithmic / t / 1e9 / hbm_peak,
            "build_bytes": algorithmic,
            "decode_latency_us": {"median": statistics.median(per_d) * 1e6, "p10": pct(per_d, 0.1) * 1e6,
                                  "p90": pct(per_d, 0.9) * 1e6},
            "decode_rows": rows}


# ----------------------------------------------------------------------------- oracle (CPU baseline)

class _NoBarrier:
    def wait(self):
        pass


_WORKER_BARRIER = None


def _oracle_pool_init(barrier):
    global _WORKER_BARRIER
    _WORKER_BARRIER = barrier


def oracle_sample(kind: str, budget_s: float, seed: int) -> dict:
    """One host worker of the oracle baseline: builds its own bounded sample of a workload
    (untimed), waits for the other workers, then times the oracle on it.

      decode:  one KV group of the decode_1m recipe (L = 2^20, b = 16, k = 8); tiles are
               decode queries of that group (the first from the recipe, the rest seeded
               N(0, 1) queries); a decode query of the workload is 8 tiles.
      prefill: one KV group of the prefill_524k recipe (L = 524288 cached + C = 8192), tree
               built over L + C; tiles are causal queries at p = L + i, i drawn from the
               chunk; a prefill token is 8 tiles.  The append and tree extension are not
               timed (the tree is built untimed).
      build:   recsa_build over one KV head of 2^18 tokens of the build_decode_2m recipe,
               repeated; bytes = token rows read + node rows written (K and V)."""
    import numpy as np
    from threadpoolctl import threadpool_limits

    from oracle import recsa_oracle as O

    barrier = _WORKER_BARRIER or _NoBarrier()
    with threadpool_limits(limits=1):
        if kind == "decode":
            w = dataclasses.replace(I.WORKLOADS["decode_1m"], batch=1, kv_heads=1, q_heads=4)
            inp = I.decode_inputs(w, device="cpu")
            tree = O.build_tree(O.bf16_bits_to_f64(I.bf16_bits(inp["k_tok"][0, 0])),
                                O.bf16_bits_to_f64(I.bf16_bits(inp["v_tok"][0, 0])), inp["pooler"].double().numpy(),
                                w.branching)
            q0 = O.bf16_bits_to_f64(I.bf16_bits(inp["q"][0, 0]))
            del inp
            rng = np.random.default_rng(seed)
            barrier.wait()
            tiles, t0 = 0, time.perf_counter()
            while True:
                O.attend(q0 if tiles == 0 else rng.standard_normal((4, 128)), tree, w.length, w.top_k)
                tiles += 1
                el = time.perf_counter() - t0
                if el >= budget_s:
                    break
            return {"units": tiles, "seconds": el}
        if kind == "prefill":
            w = dataclasses.replace(I.WORKLOADS["prefill_524k"], kv_heads=1, q_heads=4)
            inp = I.prefill_inputs(w, device="cpu")
            kb, vb = I.bf16_bits(inp["k_tok"][0, 0, :w.length]), I.bf16_bits(inp["v_tok"][0, 0, :w.length])
            kt = np.concatenate([O.bf16_bits_to_f64(kb), O.bf16_bits_to_f64(I.bf16_bits(inp["k_new"][0, :, 0]))])
            vt = np.concatenate([O.bf16_bits_to_f64(vb), O.bf16_bits_to_f64(I.bf16_bits(inp["v_new"][0, :, 0]))])
            tree = O.build_tree(kt, vt, inp["pooler"].double().numpy(), w.branching)
            qb = I.bf16_bits(inp["q"][0])
            del inp, kt, vt
            rng = np.random.default_rng(seed)
            barrier.wait()
            tiles, t0 = 0, time.perf_counter()
            while True:
                i = int(rng.integers(0, w.chunk))
                O.attend(O.bf16_bits_to_f64(qb[i]), tree, w.length + i, w.top_k, causal=True)
                tiles += 1
                el = time.perf_counter() - t0
                if el >= budget_s:
                    break
            return {"units": tiles, "seconds": el}
        if kind == "build":
            w = dataclasses.replace(I.WORKLOADS["build_decode_2m"], length=1 << 18, kv_heads=1, q_heads=4)
            inp = I.decode_inputs(w, device="cpu")
            kt = O.bf16_bits_to_f64(I.bf16_bits(inp["k_tok"][0, 0]))
            vt = O.bf16_bits_to_f64(I.bf16_bits(inp["v_tok"][0, 0]))
            W = inp["pooler"].double().numpy()
            del inp
            nodes = sum(O.level_counts(w.length, w.branching)[1:])
            per_build = (w.length + nodes) * 2 * ROW  # K and V: every token row read, every node row written
            barrier.wait()
            builds, t0 = 0, time.perf_counter()
            while True:
                O.build_tree(kt, vt, W, w.branching)
                builds += 1
                el = time.perf_counter() - t0
                if el >= budget_s:
                    break
            return {"units": builds, "seconds": el, "bytes_per_unit": per_build}
    raise ValueError(kind)


def oracle_workers_for_ram() -> int:
    """Host workers for the all-core oracle figures: every core, at most one worker per
    5 GB of available memory (a worker holds one fp64 tree of ~2-3 GB)."""
    import psutil

    cores = os.cpu_count() or 1
    avail = psutil.virtual_memory().available / 2 ** 30
    return max(1, min(cores, int((avail - 8) // 5), 64))


def oracle_baseline(budget_s: float) -> dict:
    """The fp64 oracle on the host cores: decode, prefill and build, each on one core and on
    `workers` spawned processes (one core each, numpy limited to one thread) that build
    their samples first and start timing together."""
    import multiprocessing as mp

    workers = oracle_workers_for_ram()
    out = {"cores_available": os.cpu_count(), "workers": workers}
    for kind in ("decode", "prefill", "build"):
        one = oracle_sample(kind, budget_s, seed=1)
        res = {"cores_1": one}
        if workers > 1:
            ctx = mp.get_context("spawn")
            barrier = ctx.Barrier(workers)
            with ctx.Pool(workers, initializer=_oracle_pool_init, initargs=(barrier,)) as pool:
                parts = pool.starmap(oracle_sample, [(kind, budget_s, 100 + i) for i in range(workers)])
            res["cores_all"] = {"units": sum(x["units"] for x in parts), "seconds": max(x["seconds"] for x in parts),
                                "bytes_per_unit": parts[0].get("bytes_per_unit")}
        out[kind] = res
    return out


def oracle_decode_rate(budget_s: float, device_inputs=None, max_tiles=None, warmup_tiles=0):
    """The fp64 oracle's decode rate on a bounded sample of the 1M workload.

    Sample: one sequence, two KV groups of the decode_1m recipe; their trees are built
    first (untimed, like the GPU leg, which decodes over a tree built beforehand), then
    the oracle attends as many query groups as fit in `budget_s`.  A decode query of the
    workload is 8 such tiles (one per KV group), so queries/s = tiles/s / 8."""
    from threadpoolctl import threadpool_limits

    from oracle import recsa_oracle as O

    w = I.WORKLOADS["decode_1m"]
    if device_inputs is not None:
        kb = I.bf16_bits(device_inputs["k_tok"][0, :2])
        vb = I.bf16_bits(device_inputs["v_tok"][0, :2])
        qb = I.bf16_bits(device_inputs["q"][0:1])
        W = device_inputs["pooler"].double().cpu().numpy()
        src = "slices of the GPU leg's seeded cache (sequence 0, KV heads 0-1)"
    else:
        small = dataclasses.replace(w, batch=1, kv_heads=2, q_heads=8)
        inp = I.decode_inputs(small, device="cpu")
        kb, vb, qb = I.bf16_bits(inp["k_tok"][0]), I.bf16_bits(inp["v_tok"][0]), I.bf16_bits(inp["q"])
        W = inp["pooler"].double().numpy()
        src = "the decode_1m recipe drawn on the CPU for 1 sequence x 2 KV heads"
    with threadpool_limits(limits=1):
        t_build = time.perf_counter()
        trees = [O.build_tree(O.bf16_bits_to_f64(kb[h, :w.length]), O.bf16_bits_to_f64(vb[h, :w.length]), W,
                              w.branching) for h in range(2)]
        t_build = time.perf_counter() - t_build
        g = torch.Generator().manual_seed(5)
        for i in range(warmup_tiles):  # untimed
            O.attend(torch.randn(4, 128, generator=g, dtype=torch.float64).numpy(), trees[i % 2], w.length, w.top_k)
        tiles = 0
        t0 = time.perf_counter()
        while True:
            h = tiles % 2
            if tiles < 2:
                q = O.bf16_bits_to_f64(qb[0, 0, h * 4:(h + 1) * 4])
            else:
                q = torch.randn(4, 128, generator=g, dtype=torch.float64).numpy()
            O.attend(q, trees[h], w.length, w.top_k)
            tiles += 1
            el = time.perf_counter() - t0
            if el >= budget_s or (max_tiles and tiles >= max_tiles):
                break
    return {"tiles": tiles, "seconds": el, "queries_per_s": tiles / 8 / el, "tree_build_s": t_build,
            "source": src}


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    # every step is one tile of the oracle on the host; K + W steps bounded to a few minutes
    steps, warmup = args.steps, args.warmup
    budget = None
    r = oracle_decode_rate(budget_s=1e9, max_tiles=steps, warmup_tiles=warmup) if steps + warmup <= 20000 else None
    if r is None:
        budget = 120.0
        r = oracle_decode_rate(budget_s=budget)
    value = r["queries_per_s"]
    w = I.WORKLOADS["decode_1m"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": warmup, "ms_per_step": r["seconds"] / max(r["tiles"], 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"decode_1m: B={w.batch}, L={w.length}, Hq={w.q_heads}, Hkv={w.kv_heads}, d=128, "
                               f"b={w.branching}, k={w.top_k}, Q=1", "batch": w.batch, "seq_len": w.length,
                   "parallelism": "none (host oracle)"},
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": 1, "kind": "oracle",
                         "sample": f"{r['tiles']} query-group tiles (1 step = 1 tile) over trees of 2 KV heads of "
                                   f"{r['source']}; trees built untimed in {r['tree_build_s']:.1f} s; "
                                   "queries/s = tiles/s / 8"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Small case of one kernel for an ncu capture (a few launches, a few GB on the device).

    decode: the 1M-context decode tile structure of the headline (b = 16, k = 8, needles)
    with 1 sequence and --profile-kv-heads KV groups (2 by default: 2 tiles per launch
    instead of 32, about 1 GB of caches)."""
    import hierarchical_sparse_attention_build_b200 as R

    torch.cuda.set_device(0)
    if args.profile == "decode":
        kvh = args.profile_kv_heads
        w = dataclasses.replace(I.WORKLOADS["decode_1m"], batch=1, kv_heads=kvh, q_heads=4 * kvh)
        inp = I.decode_inputs(w, device="cuda")
        p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
        tree, ws = make_tree(R, p, inp, w.length)
        out = torch.empty(inp["q"].shape, dtype=torch.bfloat16, device="cuda")
        flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        for _ in range(6):
            flush.zero_()
            R.decode(p, tree, inp["q"], out, ws)
        R.check_device_errors(ws)
        rows = decode_entries(R, p, tree, ws, inp["q"])
        print(json.dumps({"profile": "decode", "tiles": w.batch * w.kv_heads, "rows_per_launch": rows,
                          "kernel_source_sha256": kernel_source_sha()}))
    elif args.profile == "prefill":
        w = dataclasses.replace(I.WORKLOADS["prefill_524k"], length=65536, chunk=1024)
        inp = I.prefill_inputs(w, device="cuda")
        p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
        tree, ws = make_tree(R, p, inp, w.length)
        out = torch.empty(inp["q"].shape, dtype=torch.bfloat16, device="cuda")
        for _ in range(4):
            tree.length = w.length
            R.prefill_chunk(p, tree, inp["k_new"], inp["v_new"], inp["q"], out, ws)
        R.check_device_errors(ws)
        print(json.dumps({"profile": "prefill", "length": w.length, "chunk": w.chunk,
                          "tiles": w.batch * w.kv_heads * w.chunk, "kernel_source_sha256": kernel_source_sha()}))
    elif args.profile == "append":
        w = dataclasses.replace(I.WORKLOADS["decode_1m"], batch=1, kv_heads=4, q_heads=16)
        inp = I.decode_inputs(w, device="cuda", capacity=w.length + 64)
        p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
        tree, ws = make_tree(R, p, inp, w.length)
        g = torch.Generator(device="cuda").manual_seed(7)
        kn, vn = (torch.randn(1, 1, w.kv_heads, 128, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2))
        for _ in range(6):  # one token a step, the cache growing as in a decode loop
            R.append(p, tree, kn, vn)
        torch.cuda.synchronize()
        print(json.dumps({"profile": "append", "length": tree.length, "kv_heads": w.kv_heads}))
    elif args.profile == "decode_loop":
        w = I.WORKLOADS["decode_1m"]
        steps = 24
        inp = I.decode_inputs(w, device="cuda", capacity=w.length + steps + 8)
        p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
        tree, ws = make_tree(R, p, inp, w.length)
        g = torch.Generator(device="cuda").manual_seed(5)
        B, Hkv, Hq = w.batch, w.kv_heads, w.q_heads
        out = torch.empty(B, 1, Hq, 128, dtype=torch.bfloat16, device="cuda")
        flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        for _ in range(steps):  # append + decode per step, L2 flushed before each as in the bench
            kn, vn, qn = (torch.randn(B, 1, h, 128, generator=g, device="cuda").to(torch.bfloat16)
                          for h in (Hkv, Hkv, Hq))
            flush.zero_()
            R.append(p, tree, kn, vn)
            R.decode(p, tree, qn, out, ws)
        R.check_device_errors(ws)
        print(json.dumps({"profile": "decode_loop", "steps": steps, "length": tree.length}))
    elif args.profile == "build":
        w = dataclasses.replace(I.WORKLOADS["build_decode_2m"], length=1 << 19)
        inp = I.decode_inputs(w, device="cuda")
        p = R.params(num_kv_heads=w.kv_heads, num_q_heads=w.q_heads, branching=w.branching, top_k=w.top_k)
        tree, ws = make_tree(R, p, inp, w.length, build=False)
        for _ in range(4):
            R.build_tree(p, tree)
        torch.cuda.synchronize()
        print(json.dumps({"profile": "build", "length": w.length, "kv_heads": w.kv_heads}))
    torch.cuda.synchronize()


def run_gpu(args):
    import hierarchical_sparse_attention_build_b200 as R

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    hbm_peak, _, peaks_src = load_peaks()
    timer = Timer(dist_on)
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(visible.split(",")[local].strip() if visible else local)
    heads = None
    if args.shard == "heads":
        from hierarchical_sparse_attention_build_b200.sharding import kv_head_range
        heads = kv_head_range(I.WORKLOADS["decode_1m"].kv_heads, rank, world)
    dec, w = leg_decode_1m(R, timer, args, dist_on, hbm_peak, peaks_src, heads)
    extra = {}
    if not args.headline_only:
        extra["prefill"] = leg_prefill(R, timer, args, dist_on, hbm_peak, "prefill_524k", 524288)
        extra["prefill_1m"] = leg_prefill(R, timer, args, dist_on, hbm_peak, "prefill_1m", 1 << 20)
        extra["build_2m"] = leg_build_2m(R, timer, args, dist_on, hbm_peak)
        extra["decode_131k"] = leg_decode_131k(R, timer, args, dist_on, hbm_peak)
        extra["decode_loop_1m"] = leg_decode_loop(R, timer, args, dist_on)
        extra["decode_varlen"] = leg_decode_varlen(R, timer, args, dist_on)
        extra["decode_paged_1m"] = leg_decode_paged(R, timer, args, dist_on)
    clk = clocks.stop()
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ob = oracle_baseline(args.cpu_seconds)

        def rate(r, div=1.0):
            return None if r is None else r["units"] / r["seconds"] / div

        dec1, decn = ob["decode"]["cores_1"], ob["decode"].get("cores_all")
        pre1, pren = ob["prefill"]["cores_1"], ob["prefill"].get("cores_all")
        bld1, bldn = ob["build"]["cores_1"], ob["build"].get("cores_all")
        nw = ob["workers"]
        best = decn if decn is not None else dec1
        cpu = {"value": rate(best, 8.0), "unit": "queries/s", "cores": nw if decn is not None else 1,
               "kind": "oracle",
               "sample": f"decode_1m recipe, one KV group per worker (tree of 2^20 tokens built untimed), "
                         f"{best['units']} query-group tiles in {best['seconds']:.1f} s on {nw if decn else 1} worker "
                         "process(es), one core each (numpy limited to 1 thread); queries/s = tiles/s / 8 "
                         "(8 KV groups a query)",
               "cores_available": ob["cores_available"],
               "decode_queries_per_s": {"cores_1": rate(dec1, 8.0), "cores_all": rate(decn, 8.0)},
               "prefill_tokens_per_s": {"cores_1": rate(pre1, 8.0), "cores_all": rate(pren, 8.0),
                                        "sample": "prefill_524k recipe, one KV group per worker (tree over "
                                                  "524288 + 8192 tokens built untimed); causal attend of random "
                                                  "chunk queries; tokens/s = tiles/s / 8; the append and tree "
                                                  "extension are not timed"},
               "build_GBps": {"cores_1": None if bld1 is None else bld1["units"] * bld1["bytes_per_unit"] / bld1["seconds"] / 1e9,
                              "cores_all": None if bldn is None else bldn["units"] * bldn["bytes_per_unit"] / bldn["seconds"] / 1e9,
                              "sample": "build of one KV head of 2^18 tokens (b = 16) per worker, repeated; bytes = "
                                        "token rows read + node rows written, K and V"},
               "workers_note": "all-core figures: one spawned process per core, at most one per 5 GB of free "
                               "host memory"}
    if dist_on:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    B = w.batch
    n = world
    # total_s is already the max over ranks; replicas each decode their own batch, KV-head
    # shards together decode one batch
    shards = heads is not None
    job_queries = dec["queries"] if shards else n * dec["queries"]
    value = job_queries * args.steps / dec["total_s"]
    w_all = I.WORKLOADS["decode_1m"]
    mean_s = dec["mean_s"]
    achieved = dec["bytes_per_launch"] / mean_s / 1e9
    traffic = recorded_traffic("decode_1m_attend_traffic", B * w.kv_heads)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "queries/s",
        "n_gpus": n,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": mean_s * 1e3,
        "higher_is_better": True,
        "scaling": "strong" if shards else "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"decode_1m: B={B}, L={w.length}, Hq={w_all.q_heads}, Hkv={w_all.kv_heads}, d=128, "
                               f"b={w.branching}, k={w.top_k}, Q=1 query per sequence, needles=64 (bf16 K/V, "
                               "fp32 accumulation, bf16 output)",
                   "global_batch": B if shards else B * n, "seq_len": w.length,
                   "parallelism": (f"KV-head shards x{n}, {w.kv_heads} KV heads on rank 0 (no collective)" if shards
                                   else f"replicas x{n} (no collective)"),
                   "l2": "flushed between timed steps (256 MiB write, untimed)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "traffic": traffic,
                     "kernel": "attend_lean_kernel<4,4,2> (recsa_decode, 4-CTA clusters)",
                     "algorithmic_bytes_per_launch": dec["bytes_per_launch"],
                     "peak_source": f"{peaks_src} hbm_gbs (MEASURED_PEAKS.json)"},
        "e2e": {"value": job_queries * args.steps / dec["e2e_total_s"], "unit": "queries/s",
                "h2d_bytes_per_step": dec["h2d"], "d2h_bytes_per_step": dec["d2h"], **dec["e2e"]},
        "gpu_launches": args.steps,
        "clocks": clk,
        "decode": {"us_per_step_median": statistics.median(dec["per_step_s"]) * 1e6,
                   "us_per_step_p10": pct(dec["per_step_s"], 0.1) * 1e6,
                   "us_per_step_p90": pct(dec["per_step_s"], 0.9) * 1e6,
                   "rows_read_per_call": dec["rows"], "queries_per_seq_sweep": dec["sweep"]},
        "cpu_baseline": cpu,
    }
    line.update(extra)
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--quick", action="store_true", help="fewer sweep points and steps in the side legs")
    ap.add_argument("--headline-only", action="store_true", help="skip the prefill and build legs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=6.0)
    ap.add_argument("--shard", default="sequences", choices=["sequences", "heads"],
                    help="with N GPUs: N replicas of the batch (sequences, weak scaling) or the batch's "
                         "KV heads split over the N GPUs (heads, strong scaling)")
    ap.add_argument("--profile", choices=["decode", "prefill", "build", "append", "decode_loop"], help="run a small case of one kernel for ncu")
    ap.add_argument("--profile-kv-heads", type=int, default=2,
                    help="--profile decode: KV heads of the one 1M-token sequence (tiles per launch)")
    args = ap.parse_args()
    if args.profile:
        run_profile_case(args)
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
