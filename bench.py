#!/usr/bin/env python
"""Paged decode attention benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one decode step of the whole hot path over a batch whose K/V are
already in the paged cache: the cache write of each sequence's new token
(reshape_and_cache) followed by paged decode attention over the full context
(pass 1 + the partition merge).  The copy-on-write block copy has no pairs in
this batch (nothing is shared), so it issues no work.

Default workload: the Llama-3-8B-shaped GQA batch (256 sequences, 32 query /
8 kv heads, head_dim 128, bf16, block 16, log-normal contexts with median 512
clipped to [16, 4096], 65536-frame shuffled pool).  Inputs are seeded and
synthetic (``workloads.py``).  Timing: W warm-up steps, then K steps timed with
CUDA events on the launching stream, the L2 flushed before each timed step (a
256 MiB write, then a 256 MiB read of a second buffer, so only clean lines
remain), barrier + synchronize around the timed loop, max over ranks.

The line also carries a ``configs`` object: the other decode batches of the
method's workloads, each timed the same way (13B-shaped MHA at block sizes
8/16/32, on a contiguous cache and with sequential frames; shared-prefix
parallel sampling on logical and unique bytes; long contexts with the partition
merge timed on its own).

Every rank runs its own batch (seed + rank): the sequences of the job are
sharded across GPUs with no collective in the data path (weak scaling);
``value`` is the bytes all ranks processed over the slowest rank's time.
``--gpus N`` without a launcher starts the N ranks itself (torch.distributed.run).
``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

METRIC = "paged decode attn: HBM GB/s (% of B200 peak) and seqs/s; paged vs contiguous"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def l2_flush(buf, mode: str):
    """Evict the 126 MB L2 before a timed step by writing a 256 MiB buffer.

    `buf` holds two 256 MiB halves, zero-filled once when allocated.  The first
    half is written every time.  Mode "clean" then reads the second half, which
    is never written again, so the L2 ends up holding clean lines only and the
    timed step does not pay for writing the flush's dirty lines back to HBM;
    "dirty" leaves them (the write alone).  The read is a float32 sum: one
    reduction kernel, no temporary.
    """
    n = buf.numel() // 2
    buf[:n].zero_()
    if mode == "clean":
        buf[n:].view(torch.float32).sum()


# ------------------------------------------------------------------ helpers
def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--op", choices=["decode", "cache-ops", "prefill", "shared"], default="decode",
                    help="cache-ops: time reshape_and_cache and copy_blocks alone at HBM-bound sizes; "
                         "prefill: time the chunked-prefill batch alone; shared: the shared-prefix "
                         "decode batch alone")
    ap.add_argument("--workload", default="gqa8b", choices=["tiny", "mha13b", "gqa8b", "long"])
    ap.add_argument("--l2-flush", choices=["clean", "dirty"], default="clean",
                    help="L2 eviction before each timed step: 256 MiB write then read (clean) or write only")
    ap.add_argument("--block-size", type=int, default=0, help="override the workload's block size")
    ap.add_argument("--partition", type=int, default=0,
                    help="decode partition size; 0 (the library's default policy): 1024 tokens, balanced "
                         "per call for batches with fewer (sequence, kv head) pairs than decode CTAs")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="smaller batch of the same length law, pool sized to fit (profiling)")
    ap.add_argument("--no-contiguous", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads (13B MHA sweep, shared prefix, long context)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU baseline sample budget")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of CUDA-graph replays of the step")
    return ap.parse_args(argv)


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime

        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def aggregate(ms_total: float, bytes_total: float, seqs_total: float, device=None):
    """Max of the timed milliseconds and sums of the work over all ranks."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return ms_total, bytes_total, seqs_total
    t = torch.tensor([ms_total], dtype=torch.float64, device=device)
    w = torch.tensor([bytes_total, seqs_total], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(w, op=torch.distributed.ReduceOp.SUM)
    return float(t.item()), float(w[0].item()), float(w[1].item())


def job_throughput(step_ms, step_bytes: float, step_seqs: float, device=None):
    """Whole-job figures of K timed steps on every rank: the slowest rank's time
    per step, and the bytes and sequences of all ranks over that time (GB/s,
    sequences/s)."""
    K = len(step_ms)
    total_ms, total_bytes, total_seqs = aggregate(float(sum(step_ms)), step_bytes * K, step_seqs * K,
                                                  device)
    ms_per_step = total_ms / K
    return ms_per_step, total_bytes / (total_ms * 1e-3) / 1e9, total_seqs / (total_ms * 1e-3)


def barrier():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()


def measured_tensor_peak(sustained: bool = False):
    """Dense bf16 tensor-core TFLOP/s measured on this machine (MEASURED_PEAKS.json:
    the burst figure for a kernel timed alone, the sustained one for a kernel
    inside a long loop), else the recorded fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    try:
        with open(path) as f:
            return float(json.load(f)[key]), "measured"
    except Exception:
        return (1400.0 if sustained else 1590.0), "fallback"


def prefill_flops(inp: wl.PrefillInputs) -> int:
    """Algorithmic flops of causal prefill attention: each new token i of a
    sequence scores and weights p0 + i + 1 keys, 2 flops per multiply-add in
    q.K and in P.V, per query head and head dimension."""
    w = inp.w
    per_row_key = 4 * w.head_dim * w.num_heads
    total = 0
    for p0, T in zip(inp.cached.astype(np.int64), inp.chunk.astype(np.int64)):
        total += int(T * p0 + T * (T + 1) // 2)
    return per_row_key * total


def time_prefill(args, flush, device):
    """Chunked prefill over the paged cache (the prefill workload): every token's
    K/V written with the cache write, then the prefill call timed alone as a CUDA
    graph (events as graph nodes), the L2 flushed before each call."""
    from paged_kv_cache_419_b200 import binding as pkv

    inp = wl.make_prefill_inputs("prefill")
    w = inp.w
    td = torch.float16 if w.dtype == wl.F16 else torch.bfloat16

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(td).to(device)

    a = pkv.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    slots = np.concatenate([a.add_seq(s, int(inp.context_lens[s])) for s in range(w.num_seqs)])
    table, lens = a.block_table(np.arange(w.num_seqs, dtype=np.int32), w.max_blocks_per_seq)
    a.close()
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = torch.zeros(shape, dtype=td, device=device)
    vc = torch.zeros(shape, dtype=td, device=device)
    pkv.reshape_and_cache(dev(inp.k_stream), dev(inp.v_stream), kc, vc, torch.from_numpy(slots).to(device))
    q = dev(inp.q)
    out = torch.empty_like(q)
    tab_d, lens_d = torch.from_numpy(table).to(device), torch.from_numpy(lens).to(device)
    qs_d = torch.from_numpy(inp.query_start).to(device)
    max_q = int(inp.chunk.max())

    def call():
        pkv.paged_prefill(out, q, kc, vc, tab_d, qs_d, lens_d, w.scale, max_q)

    ms = graph_time_ms(call, flush, args.l2_flush, max(args.steps, 5))
    if pkv.device_error():
        raise RuntimeError("device error flags set by the prefill")
    flops = prefill_flops(inp)
    peak, kind = measured_tensor_peak()
    tflops = flops / (ms * 1e-3) / 1e12
    return {"ms": round(ms, 5), "tflops": round(tflops, 1), "flops": int(flops),
            "roofline": {"bound": "tensor", "achieved": round(tflops, 1), "peak": peak, "peak_kind": kind,
                         "unit": "TFLOP/s", "frac": round(tflops / peak, 4)},
            "workload": (f"{w.num_seqs} sequences, {w.num_heads}/{w.num_kv_heads} heads, D={w.head_dim}, "
                         f"B={w.block_size}, {wl.DTYPE_NAMES[w.dtype]}; chunks of "
                         f"{int(inp.chunk.min())}-{int(inp.chunk.max())} new tokens after "
                         f"{int(inp.cached.min())}-{int(inp.cached.max())} cached ones"),
            "new_tokens": int(inp.chunk.sum()), "context_tokens": int(inp.context_lens.sum())}


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


DECODE_SOURCES = ("decode.cuh", "decode_launch.cuh", "device.cuh")


def decode_sources_sha256() -> str:
    """Hash of the decode kernel's sources: the revision an ncu capture describes."""
    import hashlib

    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_419_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profile_traffic(algorithmic_bytes_per_launch: int):
    """DRAM bytes per decode launch from the committed ncu summary
    (profiles/decode_gqa8b64_traffic.json: read + write bytes over algorithmic bytes of the
    captured case, scaled to this launch).  None when there is no summary or when
    the decode sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "decode_gqa8b64_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        if t.get("sources_sha256") != decode_sources_sha256():
            return None
        return int(round(t["traffic_over_algorithmic"] * algorithmic_bytes_per_launch))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.remove(self.path)
        except Exception:
            return None
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")

        sm = [num(r[1]) for r in rows]
        smax = max(num(r[2]) for r in rows)
        loaded = [c for c in sm if c > 0.5 * smax] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(num(r[3]) for r in rows)}


# ------------------------------------------------------------------ workload
def workload(args):
    w = wl.WORKLOADS[args.workload]
    if args.block_size and args.block_size != w.block_size:
        w = w.with_block_size(args.block_size)
    if args.num_seqs:
        w = dataclasses.replace(w, num_seqs=args.num_seqs,
                                num_blocks=min(w.num_blocks, args.num_seqs * w.max_blocks_per_seq))
    return w


def algorithmic_bytes(w: wl.Workload, lens: np.ndarray) -> dict:
    """Bytes the step must move: K and V of every context token (read), q (read)
    and out (written); the cache write reads and writes one K and one V row per
    sequence and reads its slot.  Block tables and context lengths are listed
    apart (< 0.1 %)."""
    elt = w.elt_bytes
    S, Hq, Hkv, D = len(lens), w.num_heads, w.num_kv_heads, w.head_dim
    kv = int(lens.astype(np.int64).sum()) * Hkv * D * 2 * elt
    qo = 2 * S * Hq * D * elt
    write = 2 * S * Hkv * D * elt * 2 + 8 * S
    tables = 4 * int(np.sum((lens.astype(np.int64) + w.block_size - 1) // w.block_size)) + 4 * S
    return {"decode": kv + qo, "cache_write": write, "step": kv + qo + write, "tables": tables}


def build_gpu_batch(inp: wl.DecodeInputs, device):
    """Pool, prefill write of every sequence's cached context and the decode step's
    slots, all through the library (allocator + cache-write kernel)."""
    from paged_kv_cache_419_b200.binding import BlockAllocator, reshape_and_cache

    w = inp.w
    S = w.num_seqs
    td = torch.float16 if w.dtype == wl.F16 else torch.bfloat16

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(td).to(device)

    alloc = BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    pre = [alloc.add_seq(s, int(inp.context_lens[s]) - 1) for s in range(S)]
    new_slots, pairs = alloc.append_batch(np.arange(S, dtype=np.int32))
    table, lens = alloc.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    k_cache = torch.zeros(shape, dtype=td, device=device)
    v_cache = torch.zeros(shape, dtype=td, device=device)
    last = inp.offsets[1:] - 1
    keep = np.ones(inp.total_tokens, dtype=bool)
    keep[last] = False
    pre_slots = np.concatenate(pre)
    rows = np.nonzero(keep)[0]
    chunk = 1 << 16
    for lo in range(0, pre_slots.size, chunk):
        idx = rows[lo:lo + chunk]
        reshape_and_cache(dev(inp.k_stream[idx]), dev(inp.v_stream[idx]), k_cache, v_cache,
                          torch.from_numpy(pre_slots[lo:lo + chunk]).to(device))
    return {
        "q": dev(inp.q), "k_cache": k_cache, "v_cache": v_cache,
        "tables": torch.from_numpy(table).to(device), "lens": torch.from_numpy(lens).to(device),
        "new_k": dev(inp.k_stream[last]), "new_v": dev(inp.v_stream[last]),
        "slots": torch.from_numpy(new_slots.astype(np.int64)).to(device),
        "pairs": torch.from_numpy(pairs.astype(np.int64)).to(device),
        "out": torch.empty(S, w.num_heads, w.head_dim, dtype=td, device=device),
        "table_host": table, "lens_host": lens, "slots_host": new_slots,
    }


def build_contiguous(inp: wl.DecodeInputs, device):
    w = inp.w
    td = torch.float16 if w.dtype == wl.F16 else torch.bfloat16
    max_ctx = w.max_blocks_per_seq * w.block_size
    k = torch.zeros(w.num_seqs, w.num_kv_heads, max_ctx, w.head_dim, dtype=td, device=device)
    v = torch.zeros_like(k)
    ks = torch.from_numpy(inp.k_stream.view(np.int16)).view(td).to(device)
    vs = torch.from_numpy(inp.v_stream.view(np.int16)).view(td).to(device)
    for s in range(w.num_seqs):
        a, e = int(inp.offsets[s]), int(inp.offsets[s + 1])
        k[s, :, : e - a] = ks[a:e].transpose(0, 1)
        v[s, :, : e - a] = vs[a:e].transpose(0, 1)
    del ks, vs
    return k, v


# ------------------------------------------------------------------ timing
def graph_time_ms(fn, flush, flush_mode, K, warm=3):
    """Mean device time of `fn` (public-API calls on the current stream) over K
    CUDA-graph replays, the L2 flushed before each replay.  The timing events are
    nodes of the graph, recorded right before and after `fn`'s launches."""
    for _ in range(warm):
        l2_flush(flush, flush_mode)
        fn()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    with torch.cuda.graph(g, stream=side):
        ev[0].record()
        fn()
        ev[1].record()
    torch.cuda.current_stream().wait_stream(side)
    l2_flush(flush, flush_mode)
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(K):
        l2_flush(flush, flush_mode)
        g.replay()
        torch.cuda.synchronize()
        times.append(ev[0].elapsed_time(ev[1]))
    del g
    return statistics.mean(times)


def merge_alone_ms(call, K):
    """Pass 2 (the partition merge) on its own.  The decode call is captured with
    timing events around it; then the planning and decode kernel nodes are
    removed from the captured graph and the first event is made a dependency of
    the merge node, so a replay runs the merge alone.  It merges again what the
    earlier full calls left in the workspace (partials, statistics and complete
    publication counts, all of the same inputs), which sit in L2 as they do when
    the merge runs in the call.  Returns the mean device time over K replays."""
    from cuda.bindings import runtime as rt

    def ok(res):
        err = res[0] if isinstance(res, tuple) else res
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"CUDA graph edit failed: {err}")
        return res[1:] if isinstance(res, tuple) else None

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph(keep_graph=True)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
    with torch.cuda.graph(g, stream=side):
        ev[0].record()
        call()
        ev[1].record()
    torch.cuda.current_stream().wait_stream(side)
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    _, n = ok(rt.cudaGraphGetNodes(graph, 0))
    nodes, n = ok(rt.cudaGraphGetNodes(graph, n))
    kinds = [ok(rt.cudaGraphNodeGetType(nd))[0] for nd in nodes]
    kernels = [nd for nd, k in zip(nodes, kinds) if k == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel]
    records = [nd for nd, k in zip(nodes, kinds) if k == rt.cudaGraphNodeType.cudaGraphNodeTypeEventRecord]
    if len(kernels) != 3 or len(records) != 2:
        raise RuntimeError(f"expected plan, decode and merge kernels and two events, got "
                           f"{len(kernels)} kernels and {len(records)} events")

    def deps(nd):
        _, _, m = ok(rt.cudaGraphNodeGetDependencies_v2(nd, 0))
        if m == 0:
            return []
        found, _, m = ok(rt.cudaGraphNodeGetDependencies_v2(nd, m))
        return [int(x) for x in found[:m]]

    first = [r for r in records if not deps(r)]
    last = [r for r in records if deps(r)]
    if len(first) != 1 or len(last) != 1:
        raise RuntimeError("could not tell the two event nodes apart")
    merge = [k for k in kernels if int(k) in deps(last[0])]
    if len(merge) != 1:
        raise RuntimeError("could not find the merge node")
    for k in kernels:
        if int(k) != int(merge[0]):
            ok(rt.cudaGraphDestroyNode(k))
    ok(rt.cudaGraphAddDependencies(graph, [first[0]], [merge[0]], 1))
    g.instantiate()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(K):
        g.replay()
        torch.cuda.synchronize()
        times.append(ev[0].elapsed_time(ev[1]))
    del g
    return statistics.mean(times)


def relayout(inp: wl.DecodeInputs, w: wl.Workload, frame_order: np.ndarray) -> wl.DecodeInputs:
    """The same sequences, queries, keys and values on another pool (block size,
    frame count or frame order); only the layout changes."""
    return wl.DecodeInputs(w, inp.context_lens, frame_order.astype(np.int32), inp.q, inp.k_stream,
                           inp.v_stream, inp.offsets)


def decode_figures(nbytes: int, ms: float, peak: float, seqs: int) -> dict:
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms": round(ms, 5), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "pct_of_nominal_8tbs": round(100 * gbs / NOMINAL_HBM_GBS, 2),
            "seqs_per_s": round(seqs / (ms * 1e-3), 1), "bytes": int(nbytes)}


def time_paged_decode(args, inp, flush, device, peak, part, pass2=False):
    """Decode call alone (plan + decode + merge) over a batch whose whole context
    is in the paged cache, graph-timed with the L2 flushed before each call."""
    from paged_kv_cache_419_b200 import binding as pkv

    w = inp.w
    b = build_gpu_batch(inp, device)
    pkv.reshape_and_cache(b["new_k"], b["new_v"], b["k_cache"], b["v_cache"], b["slots"])
    ws = torch.empty(max(pkv.decode_workspace_bytes(w.num_seqs, w.num_heads, w.head_dim,
                                                    w.max_blocks_per_seq * w.block_size, part), 1),
                     dtype=torch.uint8, device=device)

    def call():
        pkv.paged_attention_decode(b["out"], b["q"], b["k_cache"], b["v_cache"], b["tables"], b["lens"],
                                   w.scale, partition_size=part, workspace=ws)

    K = max(args.steps, 5)
    ms = graph_time_ms(call, flush, args.l2_flush, K)
    res = decode_figures(algorithmic_bytes(w, inp.context_lens)["decode"], ms, peak, w.num_seqs)
    if pass2:
        try:
            res["pass2_alone_us"] = round(1e3 * merge_alone_ms(call, K), 2)
        except Exception as e:  # the figure never costs the line
            res["pass2_alone_us"] = None
            res["pass2_error"] = f"{type(e).__name__}: {e}"
    if pkv.device_error():
        raise RuntimeError(f"device error flags set by the {w.name} decode")
    return res, b, ws


def time_contiguous_decode(args, inp, b, ws, flush, device, peak, part):
    from paged_kv_cache_419_b200 import binding as pkv

    w = inp.w
    k, v = build_contiguous(inp, device)
    out_c = torch.empty_like(b["out"])

    def call():
        pkv.contiguous_attention_decode(out_c, b["q"], k, v, b["lens"], w.scale, partition_size=part,
                                        workspace=ws)

    ms = graph_time_ms(call, flush, args.l2_flush, max(args.steps, 5))
    res = decode_figures(algorithmic_bytes(w, inp.context_lens)["decode"], ms, peak, w.num_seqs)
    res["outputs_identical_to_paged"] = bool(torch.equal(out_c, b["out"]))
    del k, v
    return res


def build_shared_batch(device):
    """16 prompts x 4 samples through the library: each prompt written once and
    forked 3 times; every generated token goes allocator append -> copy_blocks
    (copy-on-write pairs) -> cache write, step by step."""
    from paged_kv_cache_419_b200 import binding as pkv

    inp = wl.make_shared_inputs()
    w = inp.w
    n, S = w.samples_per_prompt, w.num_seqs
    td = torch.bfloat16 if w.dtype == wl.BF16 else torch.float16

    def dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(td).to(device)

    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = torch.zeros(shape, dtype=td, device=device)
    vc = torch.zeros(shape, dtype=td, device=device)
    a = pkv.BlockAllocator(w.num_blocks, w.block_size, inp.frame_order)
    for p in range(w.num_prompts):
        slots = a.add_seq(p * n, inp.prompt_len)
        pkv.reshape_and_cache(dev(inp.prompt_k[p]), dev(inp.prompt_v[p]), kc, vc,
                              torch.from_numpy(slots).to(device))
        for c in range(1, n):
            a.fork(p * n, p * n + c)
    copies = 0
    for step in range(int(inp.gen_lens.max())):
        ids = np.nonzero(inp.gen_lens > step)[0].astype(np.int32)
        slots, pairs = a.append_batch(ids)
        if len(pairs):
            pkv.copy_blocks(kc, vc, torch.from_numpy(pairs).to(device))
            copies += len(pairs)
        rows = inp.gen_offsets[ids] + step
        pkv.reshape_and_cache(dev(inp.gen_k[rows]), dev(inp.gen_v[rows]), kc, vc,
                              torch.from_numpy(slots).to(device))
    table, lens = a.block_table(np.arange(S, dtype=np.int32), w.max_blocks_per_seq)
    a.close()
    return inp, kc, vc, table, lens, copies


def time_shared_decode(args, flush, device, peak, part):
    """Decode over the shared-prefix tables.  Logical bytes count every
    sequence's context as if it were private; unique bytes count each frame once,
    at the largest fill any table reads of it.  Most unique bytes are shared
    prompt frames that stay in L2 across the 4 samples, so the logical rate may
    exceed HBM bandwidth; the unique rate is the one that HBM bounds."""
    from paged_kv_cache_419_b200 import binding as pkv

    inp, kc, vc, table, lens, copies = build_shared_batch(device)
    w = inp.w
    S = w.num_seqs
    td = kc.dtype
    q = torch.from_numpy(np.ascontiguousarray(inp.q).view(np.int16)).view(td).to(device)
    out = torch.empty_like(q)
    tab_d = torch.from_numpy(table).to(device)
    lens_d = torch.from_numpy(lens).to(device)
    ws = torch.empty(pkv.decode_workspace_bytes(S, w.num_heads, w.head_dim,
                                                w.max_blocks_per_seq * w.block_size, part),
                     dtype=torch.uint8, device=device)

    def call():
        pkv.paged_attention_decode(out, q, kc, vc, tab_d, lens_d, w.scale, partition_size=part,
                                   workspace=ws)

    ms = graph_time_ms(call, flush, args.l2_flush, max(args.steps, 5))
    row = w.num_kv_heads * w.head_dim * 2 * w.elt_bytes   # K and V of one token
    qo = 2 * S * w.num_heads * w.head_dim * w.elt_bytes
    logical = int(lens.astype(np.int64).sum()) * row + qo
    fill = {}
    for s in range(S):
        for j in range(-(-int(lens[s]) // w.block_size)):
            f = int(table[s, j])
            fill[f] = max(fill.get(f, 0), min(w.block_size, int(lens[s]) - j * w.block_size))
    unique = sum(fill.values()) * row + qo
    res = decode_figures(logical, ms, peak, S)
    res["gbs_logical"] = res.pop("gbs")
    res["frac_logical"] = res.pop("frac")
    res.pop("pct_of_nominal_8tbs")
    res["bytes_logical"] = res.pop("bytes")
    u = decode_figures(unique, ms, peak, S)
    res.update({"gbs_unique": u["gbs"], "frac_unique": u["frac"], "bytes_unique": int(unique),
                "frames": len(fill), "cow_copies": copies})
    if pkv.device_error():
        raise RuntimeError("device error flags set by the shared-prefix decode")
    del kc, vc
    return res


def config_sweep(args, flush, device, peak):
    """The other decode batches of the workloads, each decode call timed alone
    (CUDA graph, events as graph nodes, L2 flushed before every call)."""
    part = args.partition
    res = {}
    base = wl.WORKLOADS["mha13b"]
    inp16 = wl.make_decode_inputs(base)
    for bs in (8, 16, 32):
        w = base if bs == 16 else base.with_block_size(bs)
        inp = inp16 if bs == 16 else relayout(
            inp16, w, np.random.default_rng(base.seed + 100 + bs).permutation(w.num_blocks))
        r, b, ws = time_paged_decode(args, inp, flush, device, peak, part)
        if bs == 16:
            r16, b16, ws16 = r, b, ws
        else:
            del b, ws
        res[f"mha13b_B{bs}"] = r
    seq = relayout(inp16, base, np.arange(base.num_blocks))
    r, b, ws = time_paged_decode(args, seq, flush, device, peak, part)
    r["outputs_identical_to_shuffled"] = bool(torch.equal(b["out"], b16["out"]))
    res["mha13b_B16_sequential_frames"] = r
    del b, ws
    res["mha13b_contiguous"] = time_contiguous_decode(args, inp16, b16, ws16, flush, device, peak, part)
    res["mha13b_overhead"] = {
        "paged_vs_contiguous": round(r16["ms"] / res["mha13b_contiguous"]["ms"] - 1.0, 4),
        "shuffled_vs_sequential_frames": round(r16["ms"] / r["ms"] - 1.0, 4),
    }
    del b16, ws16
    torch.cuda.empty_cache()
    res["shared_prefix"] = time_shared_decode(args, flush, device, peak, part)
    torch.cuda.empty_cache()
    r, b, ws = time_paged_decode(args, wl.make_decode_inputs("long"), flush, device, peak, part,
                                 pass2=True)
    res["long"] = r
    del b, ws
    torch.cuda.empty_cache()
    try:  # the prefill leg never costs the decode figures
        res["prefill"] = time_prefill(args, flush, device)
    except Exception as e:
        res["prefill"] = {"error": f"{type(e).__name__}: {e}"}
    torch.cuda.empty_cache()
    return res


# ------------------------------------------------------------------ our arm
def run_ours(args, world, rank, local):
    from paged_kv_cache_419_b200 import binding as pkv

    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    device = torch.device("cuda", local)
    w = workload(args)
    inp = wl.make_decode_inputs(w, seed=w.seed + rank)
    b = build_gpu_batch(inp, device)
    nbytes = algorithmic_bytes(w, inp.context_lens)
    part = args.partition
    ws_bytes = pkv.decode_workspace_bytes(w.num_seqs, w.num_heads, w.head_dim,
                                          w.max_blocks_per_seq * w.block_size, part)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    flush = torch.zeros(2 * L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    n_pairs = int(b["pairs"].shape[0])
    # the library launches the merge when the workspace holds more than one
    # partition per context; under the default policy it counts 512-token ones
    max_parts = math.ceil(w.max_blocks_per_seq * w.block_size / (part or 512))
    # cache write; plan + decode (+ partition merge when contexts can span partitions)
    decode_launches = 2 + (1 if max_parts > 1 else 0)
    launches_per_step = 1 + decode_launches + (1 if n_pairs else 0)

    def write_step():
        if n_pairs:
            pkv.copy_blocks(b["k_cache"], b["v_cache"], b["pairs"])
        pkv.reshape_and_cache(b["new_k"], b["new_v"], b["k_cache"], b["v_cache"], b["slots"])

    def decode_step():
        pkv.paged_attention_decode(b["out"], b["q"], b["k_cache"], b["v_cache"], b["tables"], b["lens"],
                                   w.scale, partition_size=part, workspace=ws)

    def timed_steps(run_write, run_decode, K):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
        barrier()
        torch.cuda.synchronize()
        for k in range(K):
            l2_flush(flush, args.l2_flush)
            evs[k][0].record()
            run_write()
            evs[k][1].record()
            run_decode()
            evs[k][2].record()
        torch.cuda.synchronize()
        barrier()
        return ([e[0].elapsed_time(e[2]) for e in evs], [e[1].elapsed_time(e[2]) for e in evs])

    for _ in range(max(args.warmup, 0)):
        l2_flush(flush, args.l2_flush)
        write_step()
        decode_step()
    torch.cuda.synchronize()
    if pkv.device_error():
        raise RuntimeError("device error flags set during warm-up")

    def timed_graphs(g_step, ev_step, g_call, ev_call, K):
        # Step k replays the whole step's graph, then the decode call's graph,
        # each after an L2 flush; the events are nodes of the graphs, read after
        # each replay (the host waits between replays, the GPU clock only runs
        # inside them).
        step, dec = [], []
        barrier()
        torch.cuda.synchronize()
        for _ in range(K):
            l2_flush(flush, args.l2_flush)
            g_step.replay()
            torch.cuda.synchronize()
            step.append(ev_step[0].elapsed_time(ev_step[1]))
            l2_flush(flush, args.l2_flush)
            g_call.replay()
            torch.cuda.synchronize()
            dec.append(ev_call[0].elapsed_time(ev_call[1]))
        barrier()
        return step, dec

    eager_step_ms, _ = timed_steps(write_step, decode_step, min(args.steps, 5))
    K = args.steps
    if args.eager:
        mode = "eager launches"
        run = lambda: timed_steps(write_step, decode_step, K)
    else:
        # A serving engine replays its whole decode step as one CUDA graph; so
        # does the bench: the cache write then the decode call, with timing
        # events recorded as nodes of the graph before and after.  The decode
        # call alone is a second graph, timed the same way.
        def capture(fn):
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
            with torch.cuda.graph(g, stream=side):
                ev[0].record()
                fn()
                ev[1].record()
            torch.cuda.current_stream().wait_stream(side)
            return g, ev

        g_step, ev_step = capture(lambda: (write_step(), decode_step()))
        g_call, ev_call = capture(decode_step)
        for _ in range(2):
            l2_flush(flush, args.l2_flush)
            g_step.replay()
            l2_flush(flush, args.l2_flush)
            g_call.replay()
        torch.cuda.synchronize()
        mode = ("CUDA graph replays: the step (cache write + decode call) as one graph, the decode "
                "call alone as another; events as graph nodes")
        run = lambda: timed_graphs(g_step, ev_step, g_call, ev_call, K)

    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    step_ms, decode_ms = run()
    clocks = sampler.stop() if sampler else None
    if pkv.device_error():
        raise RuntimeError("device error flags set during the timed steps")

    ms_per_step, value, seqs_per_s = job_throughput(step_ms, nbytes["step"], w.num_seqs, device)
    peak, peak_kind = measured_hbm_peak()
    dec_ms = statistics.mean(decode_ms)
    achieved = nbytes["decode"] / (dec_ms * 1e-3) / 1e9
    traffic = profile_traffic(nbytes["decode"])

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.DTYPE_NAMES[w.dtype], "data": "synthetic (seeded; workloads.py)",
        "config": workload_config(w, inp, world),
        "timing": {
            "l2": ("flushed before every timed step (256 MiB write, then a 256 MiB read of another buffer, "
                   "so no dirty lines remain)"
                   if args.l2_flush == "clean" else "flushed before every timed step (256 MiB write)")
                  + "; K/V read per step > L2",
            "execution": mode, "partition_size": part if part else "0 (default policy)",
        },
        "seqs_per_s": round(seqs_per_s, 1),
        "pct_of_nominal_8tbs": round(100 * value / NOMINAL_HBM_GBS, 2),
        "bytes_per_step": nbytes,
        "eager_ms_per_step": round(statistics.mean(eager_step_ms), 5),
        # timed region: K step graphs plus K decode-call graphs (eager: K steps)
        "gpu_launches": (launches_per_step + (0 if args.eager else decode_launches)) * K,
        "roofline": {
            "bound": "hbm", "kernel": "paged_attention_decode call (plan + decode + partition merge kernels)",
            "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
            "frac": round(achieved / peak, 4),
            "traffic": traffic,
            "decode_ms": round(dec_ms, 5),
        },
        "clocks": clocks,
    }

    out_step = b["out"].clone()   # the timed steps' output, for the parity check below
    if not args.no_contiguous:
        result["contiguous"] = contiguous_compare(args, inp, b, ws, flush, part, device)
    if not args.no_e2e:
        result["e2e"] = e2e_run(args, inp, b, ws, part, nbytes, device)
    if rank == 0 and not args.no_configs:
        try:  # the other workloads never cost the headline line
            result["configs"] = config_sweep(args, flush, device, peak)
        except Exception as e:
            result["configs"] = {"error": f"{type(e).__name__}: {e}"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(inp, nbytes, args.cpu_seconds, out_step)
        result["parity"] = result["cpu_baseline"].pop("parity", None)
    if rank == 0:
        result["kv_memory"] = kv_memory_report(w, inp.context_lens)
        print(json.dumps(result), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def workload_config(w: wl.Workload, inp: wl.DecodeInputs, world: int) -> dict:
    """The workload as both arms report it: what is computed, not how."""
    return {
        "workload": f"{w.name}: Llama-3-8B-shaped GQA decode step" if w.name == "gqa8b" else w.name,
        "num_seqs_per_gpu": w.num_seqs, "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
        "head_dim": w.head_dim, "block_size": w.block_size, "num_blocks": w.num_blocks,
        "context_tokens_per_gpu": int(inp.context_lens.sum()),
        "parallelism": f"dp{world} (sequences sharded, no collective)",
    }


def contiguous_compare(args, inp, b, ws, flush, part, device):
    """Paged vs contiguous decode, kernel level, same values and launch shape, each
    call timed as a CUDA graph with its events as graph nodes."""
    from paged_kv_cache_419_b200 import binding as pkv

    w = inp.w
    k, v = build_contiguous(inp, device)
    out_c = torch.empty_like(b["out"])
    K = max(args.steps, 5)

    def time_it(fn):
        if args.eager:
            for _ in range(3):
                l2_flush(flush, args.l2_flush)
                fn()
            evs = []
            for _ in range(K):
                l2_flush(flush, args.l2_flush)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                evs.append((e0, e1))
            torch.cuda.synchronize()
            return statistics.mean(a.elapsed_time(c) for a, c in evs)
        return graph_time_ms(fn, flush, args.l2_flush, K)

    t_paged = time_it(lambda: pkv.paged_attention_decode(
        b["out"], b["q"], b["k_cache"], b["v_cache"], b["tables"], b["lens"], w.scale,
        partition_size=part, workspace=ws))
    t_contig = time_it(lambda: pkv.contiguous_attention_decode(
        out_c, b["q"], k, v, b["lens"], w.scale, partition_size=part, workspace=ws))
    same = bool(torch.equal(out_c, b["out"]))
    del k, v
    torch.cuda.empty_cache()
    nb = algorithmic_bytes(w, inp.context_lens)["decode"]
    return {"paged_ms": round(t_paged, 5), "contiguous_ms": round(t_contig, 5),
            "paged_gbs": round(nb / (t_paged * 1e-3) / 1e9, 1),
            "contiguous_gbs": round(nb / (t_contig * 1e-3) / 1e9, 1),
            "overhead": round(t_paged / t_contig - 1.0, 4), "outputs_identical": same}


class WriteCombinedHost:
    """Pinned, write-combined host memory (cudaHostAlloc with
    cudaHostAllocWriteCombined) as a uint8 CPU tensor: the staging buffer for a
    step's inputs.  The host only writes it; its stores bypass the CPU caches, so
    the GPU's reads of it over the host link do not snoop freshly written lines
    (a cached pinned buffer that the host has just written reads at ~15 GB/s on
    these boxes, a write-combined one at ~50).  Freed with the object."""

    def __init__(self, nbytes: int):
        import ctypes
        from cuda.bindings import runtime as rt

        self._rt = rt
        err, ptr = rt.cudaHostAlloc(nbytes, rt.cudaHostAllocWriteCombined)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaHostAlloc: {err}")
        self.ptr = int(ptr)
        arr = np.ctypeslib.as_array((ctypes.c_uint8 * nbytes).from_address(self.ptr))
        self.tensor = torch.from_numpy(arr)

    def __del__(self):
        try:
            self.tensor = None
            self._rt.cudaFreeHost(self.ptr)
        except Exception:
            pass


def e2e_run(args, inp, b, ws, part, nbytes, device):
    """The same step through the public API from pinned host buffers: host->device
    copies of the step's inputs (q, the new token's K/V, its slots, the block tables
    and context lengths), the cache write and decode, and the device->host read of
    the step's output, every step.

    The inputs of a step cross the host link as one packed copy, from a pinned,
    write-combined staging buffer (the host writes it and never reads it).  Steps are
    pipelined the way a serving loop overlaps its transfers: inputs and
    outputs are double-buffered, the copies in run on one stream, the kernels on
    another and the copies out on a third, so step k+1's inputs and step k-1's
    output cross the host link while step k computes.  Each stage of each buffer
    is a CUDA graph of the public calls (eager calls with --eager); the stages are
    ordered by events.  The time is the device time from the first step's input
    copy to the last step's output copy, divided by the steps."""
    from paged_kv_cache_419_b200 import binding as pkv

    w = inp.w
    names = ("q", "new_k", "new_v", "slots", "tables", "lens")
    # The step's inputs are packed into one pinned buffer (each at a 256-byte
    # aligned offset) and cross the host link as one copy into a device buffer
    # of the same layout; the API calls take typed views of that buffer.
    offs, pos = {}, 0
    for n in names:
        offs[n] = pos
        pos += (b[n].numel() * b[n].element_size() + 255) // 256 * 256

    def views(buf):
        return {n: buf[offs[n]:offs[n] + b[n].numel() * b[n].element_size()].view(b[n].dtype).view(b[n].shape)
                for n in names}

    try:
        staging = [WriteCombinedHost(pos) for _ in range(2)]
        host_buf = [st.tensor for st in staging]
        host_kind = "pinned, write-combined (cudaHostAllocWriteCombined)"
    except Exception as e:  # no cuda-python: cached pinned memory
        staging = None
        host_buf = [torch.zeros(pos, dtype=torch.uint8).pin_memory() for _ in range(2)]
        host_kind = f"pinned (write-combined unavailable: {type(e).__name__})"
    for i in range(2):
        for n, t in views(host_buf[i]).items():
            t.copy_(b[n].cpu())
    dev_buf = [torch.empty(pos, dtype=torch.uint8, device=device) for _ in range(2)]
    dev = [views(dev_buf[i]) for i in range(2)]
    out_h = [torch.empty(b["out"].shape, dtype=b["out"].dtype).pin_memory() for _ in range(2)]
    h2d = pos
    d2h = out_h[0].numel() * out_h[0].element_size()
    out_d = [torch.empty_like(b["out"]) for _ in range(2)]
    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def copy_in(i):
        dev_buf[i].copy_(host_buf[i], non_blocking=True)

    def compute(i):
        d = dev[i]
        pkv.reshape_and_cache(d["new_k"], d["new_v"], b["k_cache"], b["v_cache"], d["slots"])
        pkv.paged_attention_decode(out_d[i], d["q"], b["k_cache"], b["v_cache"], d["tables"], d["lens"],
                                   w.scale, partition_size=part, workspace=ws)

    def copy_out(i):
        out_h[i].copy_(out_d[i], non_blocking=True)

    stages = {"in": copy_in, "comp": compute, "out": copy_out}
    streams = {"in": s_in, "comp": s_comp, "out": s_out}
    run = {(k, i): (lambda f=f, i=i: f(i)) for k, f in stages.items() for i in range(2)}
    for _ in range(2):  # warm-up (and first-call set-up) in stream order
        for i in range(2):
            for k in ("in", "comp", "out"):
                run[(k, i)]()
    torch.cuda.synchronize()
    mode = "eager public-API calls, pipelined over 3 streams"
    if not args.eager:
        graphs = {}
        for key in run:
            st = streams[key[0]]
            st.wait_stream(torch.cuda.current_stream())
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                run[key]()
            graphs[key] = g
        torch.cuda.synchronize()
        run = {key: g.replay for key, g in graphs.items()}
        mode = "CUDA graphs of the public-API calls, pipelined over 3 streams (copies in, kernels, copy out)"

    K = max(args.steps, 4)
    in_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for k in range(K):
        i = k % 2
        with torch.cuda.stream(s_in):
            if k == 0:
                t0.record()
            if k >= 2:
                s_in.wait_event(comp_done[i])   # step k-2 no longer reads these inputs
            run[("in", i)]()
            in_done[i].record()
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[i])
            if k >= 2:
                s_comp.wait_event(out_done[i])  # step k-2's output has been read out
            run[("comp", i)]()
            comp_done[i].record()
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[i])
            run[("out", i)]()
            out_done[i].record()
            if k == K - 1:
                t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / K
    ms_max, _, _ = aggregate(ms, 0.0, 0.0, device)
    return {"value": round(nbytes["step"] / (ms_max * 1e-3) / 1e9, 1), "unit": "GB/s",
            "ms_per_step": round(ms_max, 5), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "execution": mode, "input_staging": host_kind,
            "host_link": host_link(copy_in, copy_out, s_in, s_out, h2d, d2h)}


def host_link(copy_in, copy_out, s_in, s_out, h2d, d2h, reps=10):
    """The step's own copies timed alone on their streams: the packed input copy
    host->device, the output copy device->host, and both at once (the pipelined
    steady state can go no faster than the slower direction)."""
    def timed(fns):
        evs = {s: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _, s in fns}
        torch.cuda.synchronize()
        for f, s in fns:
            with torch.cuda.stream(s):
                evs[s][0].record()
                for r in range(reps):
                    f(r % 2)
                evs[s][1].record()
        torch.cuda.synchronize()
        return {s: evs[s][0].elapsed_time(evs[s][1]) / reps for _, s in fns}

    t_in = timed([(copy_in, s_in)])[s_in]
    t_out = timed([(copy_out, s_out)])[s_out]
    both = timed([(copy_in, s_in), (copy_out, s_out)])
    gbs = lambda nbytes, ms: round(nbytes / (ms * 1e-3) / 1e9, 1)
    return {"h2d_gbs": gbs(h2d, t_in), "d2h_gbs": gbs(d2h, t_out),
            "h2d_gbs_concurrent": gbs(h2d, both[s_in]), "d2h_gbs_concurrent": gbs(d2h, both[s_out]),
            "h2d_us": round(1e3 * t_in, 1), "d2h_us": round(1e3 * t_out, 1),
            "concurrent_us": round(1e3 * max(both.values()), 1)}


# ------------------------------------------------------------------ cache ops alone
def run_cache_ops(args, local):
    """reshape_and_cache and copy_blocks on their own at sizes where HBM bounds
    them (the decode step's own cache write moves only 1 MB and is launch-bound):
    a gqa8b-shaped pool of 16,384 frames (8 kv heads x 16 x 128 bf16, 1.07 GB for
    K and V), 32,768 new tokens written at distinct random slots, and 2,048 copy
    pairs between distinct random frames.  L2 flushed before every launch; CUDA
    events on the launching stream.  Algorithmic bytes: the cache write reads key
    and value and writes both (plus the int64 slots); the block copy reads and
    writes both frames of every pair.  One JSON line per kernel."""
    from paged_kv_cache_419_b200 import binding as pkv

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    N, Hkv, B, D, T, P = 16384, 8, 16, 128, 32768, 2048
    rng = np.random.default_rng(21)
    kc = torch.zeros((N, Hkv, B, D), dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    key = torch.randn((T, Hkv, D), dtype=torch.bfloat16, device=device)
    val = torch.randn_like(key)
    slots = torch.from_numpy(rng.choice(N * B, size=T, replace=False).astype(np.int64)).to(device)
    frames = rng.permutation(N)[: 2 * P].astype(np.int64)
    pairs = torch.from_numpy(np.stack([frames[:P], frames[P:]], axis=1).copy()).to(device)
    flush = torch.zeros(2 * L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    frame_bytes = Hkv * B * D * 2
    ops = {
        "reshape_and_cache": (lambda: pkv.reshape_and_cache(key, val, kc, vc, slots),
                              4 * T * Hkv * D * 2 + T * 8, f"{T} tokens, 8 kv heads x 128 bf16"),
        "copy_blocks": (lambda: pkv.copy_blocks(kc, vc, pairs),
                        2 * 2 * P * frame_bytes, f"{P} pairs of 32 KB frames, K and V"),
    }
    peak, peak_kind = measured_hbm_peak()
    for name, (fn, nbytes, what) in ops.items():
        for _ in range(max(args.warmup, 3)):
            l2_flush(flush, args.l2_flush)
            fn()
        torch.cuda.synchronize()
        times = []
        for _ in range(args.steps):
            l2_flush(flush, args.l2_flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        if pkv.device_error():
            raise RuntimeError(f"device error flags set by {name}")
        ms = statistics.mean(times)
        gbs = nbytes / (ms * 1e-3) / 1e9
        print(json.dumps({"op": name, "metric": f"{name} HBM GB/s", "value": round(gbs, 1), "unit": "GB/s",
                          "ms": round(ms, 5), "bytes": int(nbytes), "workload": what, "steps": args.steps,
                          "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak,
                                       "peak_kind": peak_kind, "frac": round(gbs / peak, 4)}}), flush=True)


# ------------------------------------------------------------------ KV memory
def kv_memory_report(w: wl.Workload, lens: np.ndarray) -> dict:
    """KV-cache memory use of this batch and of the parallel-sampling batch, from
    the native block allocator (host only; nothing here is timed).

    useful_kv_pct: context tokens / token capacity of the frames the batch holds
    (only each sequence's last block is partial); the pages report 96.3 % useful
    KV memory against 20-38 % for max-length reservation (dataarena note section 2).
    sharing_saving_pct: 1 - frames held / frames the same tables would need
    unshared, for 16 prompts of 1000 tokens x 4 samples that each decode 0-200
    tokens with copy-on-write (slides 13-14 report 6-66 % savings).
    beam_saving_pct: the same for 4 beams over a block tree (slide 14), 200 steps
    from one 1000-token prompt (kashii section 3: beam search memory cut by up to
    55 %).
    prefix_cache_*: 64 requests on 4 shared 1024-token system prompts through
    the prefix cache (dataarena note section 3.1): prompt tokens whose KV is
    reused instead of written, and frames held against the frames the same
    prompts take without the cache.
    """
    from paged_kv_cache_419_b200 import binding as pkv

    a = pkv.BlockAllocator(w.num_blocks, w.block_size)
    for s, L in enumerate(lens):
        a.add_seq(s, int(L))
    st = a.stats()
    a.close()
    capacity = st["used_blocks"] * w.block_size
    max_len = w.max_blocks_per_seq * w.block_size
    sh = wl.make_shared_inputs()
    ws = sh.w
    a = pkv.BlockAllocator(ws.num_blocks, ws.block_size, sh.frame_order)
    n = ws.samples_per_prompt
    for p in range(ws.num_prompts):
        a.add_seq(p * n, sh.prompt_len)
        for c in range(1, n):
            a.fork(p * n, p * n + c)
    copies = 0
    for step in range(int(sh.gen_lens.max())):
        ids = np.nonzero(sh.gen_lens > step)[0]
        _, pairs = a.append_batch(ids)
        copies += len(pairs)
    ss = a.stats()
    a.close()
    bm = wl.make_beam_inputs()
    wb = bm.w
    a = pkv.BlockAllocator(wb.num_blocks, wb.block_size, bm.frame_order)
    a.add_seq(0, bm.prompt_len)
    beams, nid, beam_copies = np.zeros(1, np.int32), 1, 0
    for step in range(bm.steps):
        beams, _, pairs, nid = a.beam_step(beams, bm.parents[step], nid)
        beam_copies += len(pairs)
    bs = a.stats()
    a.close()
    px = wl.make_prefix_inputs()
    wp = px.w
    a = pkv.BlockAllocator(wp.num_blocks, wp.block_size, px.frame_order)
    cached = sum(a.add_seq_cached(i, px.token_ids[i])[1] for i in range(wp.num_seqs))
    ps = a.stats()
    a.close()
    prompt_tokens = int(sum(len(t) for t in px.token_ids))
    return {
        "useful_kv_pct": round(100.0 * st["tokens"] / capacity, 2),
        "frames": int(st["used_blocks"]), "tokens": int(st["tokens"]), "block_size": w.block_size,
        "max_length_reservation_useful_pct": round(100.0 * st["tokens"] / (len(lens) * max_len), 2),
        "sharing_saving_pct": round(100.0 * (1 - ss["used_blocks"] / ss["logical_blocks"]), 2),
        "sharing_frames": int(ss["used_blocks"]), "sharing_unshared_frames": int(ss["logical_blocks"]),
        "sharing_cow_copies": int(copies),
        "beam_saving_pct": round(100.0 * (1 - bs["used_blocks"] / bs["logical_blocks"]), 2),
        "beam_frames": int(bs["used_blocks"]), "beam_unshared_frames": int(bs["logical_blocks"]),
        "beam_cow_copies": int(beam_copies),
        "prefix_cache_reused_tokens_pct": round(100.0 * cached / prompt_tokens, 2),
        "prefix_cache_frames": int(ps["used_blocks"]), "prefix_cache_uncached_frames": int(ps["logical_blocks"]),
    }


# ------------------------------------------------------------------ CPU oracle
def oracle_pool(inp: wl.DecodeInputs):
    """The batch's cache built on the host with the oracle's own allocator model
    and scatter (the oracle's inputs never come from the CUDA path).  Also
    returns the slots of the tokens the decode step appends (each sequence's last)."""
    import oracle
    from oracle.allocator_model import AllocatorModel

    w = inp.w
    m = AllocatorModel(w.num_blocks, w.block_size, inp.frame_order)
    slots = []
    for s in range(w.num_seqs):
        slots += m.add_seq(s, int(inp.context_lens[s]))
    shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
    kc = np.zeros(shape, np.uint16)
    vc = np.zeros(shape, np.uint16)
    slots = np.array(slots, np.int64)
    oracle.reshape_and_cache(kc, vc, inp.k_stream, inp.v_stream, slots, w.block_size)
    tables, lens = m.block_table(range(w.num_seqs), w.max_blocks_per_seq)
    return kc, vc, np.array(tables, np.int32), np.array(lens, np.int32), slots[inp.offsets[1:] - 1]


def parity_vs_oracle(gpu_out: torch.Tensor, ref: np.ndarray, dtype: int) -> dict:
    """Max-abs error of the GPU output against the fp64 oracle, and its distance in
    ulps from the oracle rounded to the output type (one round-to-nearest-even
    step from fp64)."""
    import oracle

    got_bits = gpu_out.detach().cpu().view(torch.int16).numpy().view(np.uint16).reshape(-1).astype(np.int64)
    got = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    want_bits = oracle.round_to_dtype(ref, dtype).reshape(-1).astype(np.int64)

    def line(b):  # sign-magnitude patterns onto one ordered integer line
        mag = b & 0x7FFF
        return np.where(b & 0x8000, -mag, mag)

    d = np.abs(line(got_bits) - line(want_bits))
    tol = 2e-3 if dtype == wl.F16 else 1e-2
    return {"max_abs_err": float(np.abs(got - ref).max()), "tolerance": tol,
            "elements": int(d.size), "identical_to_rounded_oracle": round(float(np.mean(d == 0)), 6),
            "within_1_ulp": round(float(np.mean(d <= 1)), 6), "max_ulp": int(d.max()),
            "checked": "every element of the timed steps' output against the oracle of the same step"}


def cpu_baseline(inp, nbytes, seconds, gpu_out=None):
    """The oracle (plain C, fp64, one thread) on this host over the same batch,
    repeated until `seconds` have passed; GB/s with the same byte count.  With
    `gpu_out`, also the parity of the GPU output with the oracle's result."""
    import oracle

    w = inp.w
    kc, vc, tables, lens, _ = oracle_pool(inp)
    runs, t0 = 0, time.perf_counter()
    while True:
        ref = oracle.paged_decode(inp.q, kc, vc, tables, lens, w.scale, w.num_kv_heads, w.block_size,
                                  w.dtype)
        runs += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per = el / runs
    res = {"value": round(nbytes["decode"] / per / 1e9, 4), "unit": "GB/s", "cores": 1,
           "kind": "oracle", "seqs_per_s": round(w.num_seqs / per, 2),
           "sample": f"the whole {w.num_seqs}-sequence batch (decode attention only), {runs} run(s), "
                     f"{el:.1f} s; host {os.cpu_count()} logical cores, oracle single-threaded"}
    if gpu_out is not None:
        res["parity"] = parity_vs_oracle(gpu_out, ref, w.dtype)
    try:  # the extra all-core figure never costs the bench line
        res["all_cores"] = oracle_all_cores(inp, kc, vc, tables, lens, nbytes, seconds)
    except Exception as e:
        res["all_cores"] = {"error": f"{type(e).__name__}: {e}"}
    return res


def sequence_ranges(lens: np.ndarray, parts: int):
    """Contiguous sequence ranges with about equal context tokens each."""
    work = np.cumsum(np.maximum(lens.astype(np.int64), 1))
    cuts = np.searchsorted(work, work[-1] * np.arange(1, parts) / parts, side="right")
    bounds = [0] + [int(c) for c in cuts] + [len(lens)]
    return [(a, b) for a, b in zip(bounds[:-1], bounds[1:]) if b > a]


def oracle_all_cores(inp, kc, vc, tables, lens, nbytes, seconds):
    """The same oracle, unchanged, on every host core: one thread per core, each
    calling it on a contiguous range of sequences (ranges balanced by context
    tokens).  The oracle is C behind ctypes, which drops the GIL during the call,
    so the threads run in parallel over shared arrays."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    w = inp.w
    ranges = sequence_ranges(lens, max(1, os.cpu_count() or 1))

    def part(r):
        oracle.paged_decode(inp.q, kc, vc, tables, lens, w.scale, w.num_kv_heads, w.block_size, w.dtype,
                            seqs=r)

    with ThreadPoolExecutor(max_workers=len(ranges)) as pool:
        runs, t0 = 0, time.perf_counter()
        while True:
            list(pool.map(part, ranges))
            runs += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
    per = el / runs
    return {"value": round(nbytes["decode"] / per / 1e9, 4), "unit": "GB/s", "cores": len(ranges),
            "kind": "oracle", "seqs_per_s": round(w.num_seqs / per, 2),
            "sample": f"the whole batch, {runs} run(s), {el:.1f} s; one thread per core over "
                      f"{len(ranges)} sequence ranges"}


def run_reference(args, world, rank, local):
    """The CPU oracle as the reference arm, on our arm's workload and step: per
    step, the oracle's cache write of each sequence's new token, then decode
    attention over the whole batch, on every host core (one thread per core over
    sequence ranges balanced by context tokens; the oracle is C behind ctypes,
    which drops the GIL).  Rank 0 only."""
    if rank != 0:
        return
    import oracle
    from concurrent.futures import ThreadPoolExecutor

    w = workload(args)
    inp = wl.make_decode_inputs(w)
    kc, vc, tables, lens, new_slots = oracle_pool(inp)
    last = inp.offsets[1:] - 1
    new_k, new_v = inp.k_stream[last], inp.v_stream[last]
    nbytes = algorithmic_bytes(w, inp.context_lens)
    ranges = sequence_ranges(lens, max(1, os.cpu_count() or 1))

    def part(r):
        oracle.paged_decode(inp.q, kc, vc, tables, lens, w.scale, w.num_kv_heads, w.block_size, w.dtype,
                            seqs=r)

    with ThreadPoolExecutor(max_workers=len(ranges)) as pool:
        def step():
            oracle.reshape_and_cache(kc, vc, new_k, new_v, new_slots, w.block_size)
            list(pool.map(part, ranges))

        for _ in range(max(args.warmup, 0)):
            step()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            step()
        el = time.perf_counter() - t0
    ms = el / max(args.steps, 1) * 1e3
    value = nbytes["step"] / (ms * 1e-3) / 1e9
    sample = (f"the whole {w.num_seqs}-sequence batch per step (cache write + decode), "
              f"{len(ranges)} threads over sequence ranges")
    res = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded; workloads.py)",
        "config": workload_config(w, inp, world),
        "seqs_per_s": round(w.num_seqs / (ms * 1e-3), 2),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": len(ranges), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def free_port() -> int:
    import socket

    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def rank_launch_command(argv, n: int, port: int):
    """The command that runs this script as n ranks on one node (one per GPU)."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    args = parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # no launcher around us: start one rank per GPU and report their line
        return subprocess.call(rank_launch_command(argv, args.gpus, free_port()))
    world, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, world, rank, local)
    elif args.op == "cache-ops":
        if rank == 0:
            run_cache_ops(args, local)
    elif args.op == "prefill":
        if rank == 0:
            torch.cuda.set_device(local)
            device = torch.device("cuda", local)
            flush = torch.zeros(2 * L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
            print(json.dumps({"op": "prefill", **time_prefill(args, flush, device)}), flush=True)
    elif args.op == "shared":
        if rank == 0:
            torch.cuda.set_device(local)
            device = torch.device("cuda", local)
            flush = torch.zeros(2 * L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
            peak, kind = measured_hbm_peak()
            res = time_shared_decode(args, flush, device, peak, args.partition)
            print(json.dumps({"op": "shared", "peak_gbs": peak, "peak_kind": kind, **res}), flush=True)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
