#!/usr/bin/env python
"""Benchmark: paged decode attention on B200 (one JSON line on rank 0).

A step is one pass of the whole hot path over one batch:
``kv_cache_append`` of every sequence's newest token (through its slot
mapping), then ``paged_attn_decode`` over all cached tokens. The decode
includes the split-context merge when a context exceeds one partition. The
default workload is the Llama-8B-shaped GQA batch:

  * 256 sequences, 32 query heads / 8 KV heads, head_dim 128, bf16
  * 16-token blocks, lognormal context lengths (median 512, capped at 4096)
  * shuffled physical blocks

Copy-on-write block copies happen only on forks; the shared-prefix workload
(``--workload shared_prefix``) includes them.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun each rank runs its own batch: weak scaling, no data collective.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "paged decode attention: effective KV GB/s (% of HBM peak), seq-steps/s"
HBM_SPEC_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DECODE_SOURCES = ("paged_kv_cache_387_b200/csrc/decode_tc.cu",
                  "paged_kv_cache_387_b200/csrc/pkv_device.cuh")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama8b_gqa_b256")
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="keep only the first sequences of the workload (small profiling cases)")
    ap.add_argument("--partition-size", type=int, default=None,
                    help="tokens per split-context partition (default: the workload's)")
    ap.add_argument("--soak-seconds", type=float, default=2.0,
                    help="back-to-back steps before the timed region (clock sampling, warm clocks)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--contiguous", action="store_true",
                    help="also time the same batch with identity block placement")
    ap.add_argument("--e2e-steps", type=int, default=200,
                    help="steps of the end-to-end loop (at least --steps): a serving loop runs "
                         "for many steps, and a short loop would charge each step a share of "
                         "the first upload and the last download, which nothing overlaps")
    ap.add_argument("--e2e-buffers", type=int, default=4,
                    help="device input/output buffers in the end-to-end loop (>= 2)")
    ap.add_argument("--e2e-steps-per-upload", type=int, default=4,
                    help="end-to-end loop: steps whose inputs go up in one copy and whose "
                         "results come back in one copy (>= 1); the calls of a group run "
                         "back to back on the compute stream")
    ap.add_argument("--e2e-compute-streams", type=int, default=1,
                    help="compute streams that take turns with the end-to-end loop's steps, "
                         "each with its own workspace (>= 1)")
    ap.add_argument("--e2e-result-in-host-memory", action="store_true",
                    help="end-to-end loop: the decode writes its result straight into pinned "
                         "host memory instead of a device buffer plus a device-to-host copy")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads' device-timed lines (OPT-13B, long split, "
                         "shared prefix, beam search, prefix cache, identity placement, "
                         "standalone append and copy)")
    ap.add_argument("--separate-append", action="store_true",
                    help="run kv_cache_append and paged_attn_decode as two calls instead of "
                         "the fused paged_attn_decode_append")
    ap.add_argument("--small-batch-only", action="store_true",
                    help="time only the small calls (the line's small_batch entry) on one GPU "
                         "and print them")
    ap.add_argument("--small-batch-shapes", default=None,
                    help="comma-separated subset of the small calls, e.g. 1x4096,256x16")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def decode_source_hash():
    """Hash of the decode kernel's code: its sources with comments and
    whitespace removed, so that an edited comment does not mark recorded
    counters as stale."""
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)  # block comments
        src = re.sub(r"//[^\n]*", " ", src)                # line comments
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per decode launch from a committed ncu summary, if it was
    taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", f"decode_tc_{workload}.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.strip().startswith(("source_sha256", "traffic_bytes_per_launch")):
                k, v = line.strip().split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    try:
        if vals.get("source_sha256") == decode_source_hash():
            return int(vals["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples (timestamps on the host clock)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.samples = []
        self.proc = None
        self.gpu_index = gpu_index
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1, window):
        sel = [p for (t, p) in self.samples if t0 <= t <= t1]
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": window}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in sel if num(p[1]) is not None]
        smax = [num(p[2]) for p in sel if num(p[2]) is not None]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for p in sel:
            for name, v in zip(names, p[5:9]):
                if v.strip().lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sel), "window": window,
                "power_w_max": max((num(p[3]) or 0.0) for p in sel)}


# ---------------------------------------------------------------------------
# multi-rank host logic (one process per GPU; no data collective)
# ---------------------------------------------------------------------------

def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank decodes its own batch (weak scaling): same workload, another seed."""
    return int(base_seed) + 1000 * int(rank)


def max_over_ranks(values, device):
    """Element-wise maximum of per-rank timings (the job is as slow as its slowest rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_gbs(bytes_per_rank: int, world: int, seconds: float) -> float:
    """Aggregate throughput: the bytes every rank moved / the slowest rank's time."""
    return bytes_per_rank * world / seconds / 1e9


# ---------------------------------------------------------------------------
# the reference arm: the CPU oracle, timed on the host cores
# ---------------------------------------------------------------------------

def oracle_sample_step(case_cpu, nseq):
    """One oracle step (append + decode) over the first ``nseq`` sequences."""
    import torch
    import oracle
    sl = slice(0, nseq)
    if case_cpu.slot_mapping is not None:
        oracle.cache_append(case_cpu.k_pool, case_cpu.v_pool, case_cpu.k_new[sl].contiguous(),
                            case_cpu.v_new[sl].contiguous(),
                            case_cpu.slot_mapping[sl].contiguous())
    oracle.paged_decode(case_cpu.q[sl].contiguous(), case_cpu.k_pool, case_cpu.v_pool,
                        case_cpu.block_tables[sl].contiguous(),
                        case_cpu.context_lens[sl].contiguous(), case_cpu.scale)


def size_oracle_sample(case_cpu, target_s):
    """Pick the number of leading sequences whose oracle step takes about target_s."""
    n = 1
    t = 0.0
    while True:
        t0 = time.perf_counter()
        oracle_sample_step(case_cpu, n)
        t = time.perf_counter() - t0
        if t >= 0.05 * target_s or n >= case_cpu.num_seqs:
            break
        n = min(case_cpu.num_seqs, n * 4)
    est = max(1, int(n * target_s / max(t, 1e-6)))
    return min(case_cpu.num_seqs, est)


def step_bytes(case, nseq=None):
    """Algorithmic bytes of one step (decode + the append that precedes it)."""
    from pkv_inputs import decode_algorithmic_bytes
    lens = case.context_lens.cpu().tolist()
    if nseq is not None:
        lens = lens[:nseq]
    es = case.q.element_size()
    b = decode_algorithmic_bytes(lens, case.num_heads, case.num_kv_heads, case.head_dim,
                                 case.block_size, es)
    app = 0
    if case.slot_mapping is not None:
        t = len(lens)
        # read new K and V + slot, write them into the pool
        app = t * (2 * 2 * case.num_kv_heads * case.head_dim * es + 8)
    return b, app


def case_unique_kv_bytes(case):
    """K/V bytes of the distinct physical blocks the step reads."""
    from pkv_inputs import unique_kv_bytes
    return unique_kv_bytes(case.block_tables.cpu().tolist(), case.context_lens.cpu().tolist(),
                           case.block_size, case.num_kv_heads, case.head_dim,
                           case.k_pool.element_size())


def measure_swap(case, dev, stream, pkv, nseq=32, reps=5):
    """Swap the blocks of the batch's first `nseq` sequences out to a swap
    space in pinned host memory and back in (kv_block_swap, both directions),
    as preemption does. Times each direction with CUDA events; the bound is
    the host link, so the measured pinned copy rates are reported beside."""
    import torch
    B = case.block_size
    lens = case.context_lens[:nseq].cpu().tolist()
    bt = case.block_tables[:nseq].cpu()
    blk_bytes = 2 * case.k_pool[0].numel() * case.k_pool.element_size()
    blocks, seen = [], set()
    for s, L in enumerate(lens):  # whole sequences, up to ~128 MB
        if blocks and len(blocks) * blk_bytes >= (128 << 20):
            nseq = s
            break
        for b in bt[s, :-(-L // B)].tolist():
            if b not in seen:
                seen.add(b)
                blocks.append(int(b))
    n = len(blocks)
    if n == 0:
        return None
    shape = (n,) + tuple(case.k_pool.shape[1:])
    hk = torch.empty(shape, dtype=case.k_pool.dtype, pin_memory=True)
    hv = torch.empty(shape, dtype=case.k_pool.dtype, pin_memory=True)
    out_pairs = torch.tensor([[b, i] for i, b in enumerate(blocks)], dtype=torch.int32,
                             device=dev)
    in_pairs = out_pairs.flip(1).contiguous()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    nbytes = 2 * n * case.k_pool[0].numel() * case.k_pool.element_size()

    def timed(dst_k, dst_v, src_k, src_v, pairs):
        ts = []
        for _ in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            pkv.kv_block_swap(dst_k, dst_v, src_k, src_v, pairs, err=err)
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts[1:])
    out_ms = timed(hk, hv, case.k_pool, case.v_pool, out_pairs)
    in_ms = timed(case.k_pool, case.v_pool, hk, hv, in_pairs)  # same data back in place
    if int(err.item()) != 0:
        raise RuntimeError("kv_block_swap reported a bad pair")
    return {"sequences": min(nseq, len(lens)), "blocks": n, "bytes": nbytes,
            "out_ms": out_ms, "out_gbs": nbytes / (out_ms * 1e-3) / 1e9,
            "in_ms": in_ms, "in_gbs": nbytes / (in_ms * 1e-3) / 1e9,
            "note": "device pool <-> swap space in pinned host memory, SM copies over the "
                    "host link (no copy engine)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    import torch
    import oracle
    from pkv_inputs import make_case
    oracle.build()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    case = make_case(args.workload, device=dev, with_append=True,
                     num_seqs=args.num_seqs).to("cpu")
    budget = 150.0  # seconds for warmup + steps
    per_step = min(2.0, budget / max(1, args.steps + args.warmup))
    nseq = size_oracle_sample(case, per_step)
    for _ in range(args.warmup):
        oracle_sample_step(case, nseq)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(case, nseq)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    dec, app = step_bytes(case, nseq)
    gbs = (dec + app) / dt / 1e9
    sample = (f"first {nseq} of {case.num_seqs} sequences "
              f"({int(case.context_lens[:nseq].sum())} tokens), append + decode, fp64 oracle")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config_block(case, args.workload, args.gpus),
                       call=call_description(case, args)),
        "seq_steps_per_s": nseq / dt,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def call_description(case, args):
    """The library call a step makes (the same text in both arms' config)."""
    fused = not args.separate_append and case.q.dtype != __import__("torch").float32
    return ("paged_attn_decode_append (append fused into the decode)" if fused else
            "kv_cache_append + paged_attn_decode")


def config_block(case, workload, n_gpus):
    from pkv_inputs.workloads import WORKLOADS
    desc = WORKLOADS.get(workload, {}).get(
        "desc", "shared prefix / parallel sampling: 16 prompts x 6 samples, 40 heads MHA, "
                "head_dim 128, fp16, block 16, prompt 1000 tokens shared through refcounted "
                "blocks, CoW copy of the partial block, then 64 divergent decode tokens "
                "(the timed step is the 64th)" if workload == "shared_prefix" else
        "beam search: 32 requests x 4 beams, 32 q heads / 8 kv heads, head_dim 128, bf16, "
        "block 16, prompt 512, seeded random parents each step; the timed step is the 128th "
        "(append + decode of the 128 beams)" if workload == "beam_search" else
        "automatic prefix caching: 64 requests, 1024-token system prompt shared by all, 8 "
        "groups sharing a 512-token prefix, unique 128-256-token suffixes; 32 q / 8 kv heads, "
        "head_dim 128, bf16, block 16; blocks keyed by a hash of the whole prefix"
        if workload == "prefix_cache" else workload)
    return {
        "workload": workload, "desc": desc, "num_seqs_per_gpu": case.num_seqs,
        "num_heads": case.num_heads, "num_kv_heads": case.num_kv_heads,
        "head_dim": case.head_dim, "block_size": case.block_size,
        "partition_size": case.partition_size,
        "context_tokens_per_gpu": int(case.context_lens.sum()),
        "max_context_len": case.max_context_len,
        "step": "append of each sequence's newest token + paged decode over its whole context",
        "accumulate": "fp32",
        "l2": "inputs larger than L2: the K/V pool read each step is "
              f"{case.k_pool.numel() * case.k_pool.element_size() * 2 / 1e9:.2f} GB per GPU",
        "parallelism": f"{n_gpus} independent batches, one per GPU (no data collective)",
    }


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_bench_case(args, dev, rank, workload=None):
    """The step's inputs, plus extra report fields for special workloads."""
    import torch
    from pkv_inputs import make_case
    from pkv_inputs.workloads import WORKLOADS, DecodeCase, make_shared_prefix_case
    workload = args.workload if workload is None else workload
    if workload == "beam_search":
        # 32 requests x 4 beams, Llama-8B-shaped heads: after 127 steps with seeded
        # random parents, the timed step is the 128th (copies applied, then the
        # fused append + decode of all 128 beams).
        from pkv_inputs import make_beam_search_case
        case = make_beam_search_case(device=dev, seed=rank_seed(393, rank))
        m = case.meta
        per_tok = 2 * case.num_kv_heads * case.head_dim * case.k_pool.element_size()
        extras = {"beam_search": {
            "requests": m["requests"], "width": m["width"],
            "blocks_in_use": m["blocks_in_use"], "blocks_unshared": m["blocks_unshared"],
            "memory_saving": 1.0 - m["blocks_in_use"] / m["blocks_unshared"],
            "logical_kv_bytes": int(case.context_lens.sum()) * per_tok,
            "unique_kv_bytes": case_unique_kv_bytes(case),
            "note": "value/roofline count logical bytes; unique_kv_bytes counts each "
                    "physical block the beams share once"}}
        case.meta = {k: v for k, v in m.items() if k not in ("allocator", "searches")}
        return case, extras
    if workload == "prefix_cache":
        # 64 requests: a 1024-token system prompt shared by all, 8 groups sharing a
        # 512-token prefix, unique 128-256-token suffixes; blocks from the prefix
        # cache; the timed step appends each request's last token and decodes.
        from pkv_inputs import make_prefix_cache_case
        case = make_prefix_cache_case(device=dev, seed=rank_seed(394, rank))
        m = case.meta
        per_tok = 2 * case.num_kv_heads * case.head_dim * case.k_pool.element_size()
        extras = {"prefix_cache": {
            "hits": m["hits"], "misses": m["misses"],
            "blocks_in_use": m["blocks_in_use"], "blocks_unshared": m["blocks_unshared"],
            "memory_saving": 1.0 - m["blocks_in_use"] / m["blocks_unshared"],
            "logical_kv_bytes": int(case.context_lens.sum()) * per_tok,
            "unique_kv_bytes": case_unique_kv_bytes(case),
            "note": "value/roofline count logical bytes; unique_kv_bytes counts each "
                    "cached block the requests share once"}}
        case.meta = {k: v for k, v in m.items() if k not in ("cache", "tokens")}
        return case, extras
    if workload != "shared_prefix":
        case = make_case(workload, device=dev, with_append=True,
                         num_seqs=args.num_seqs if workload == args.workload else None,
                         seed=rank_seed(WORKLOADS[workload]["seed"], rank))
        return case, {}
    # 16 prompts x 6 samples sharing refcounted prompt blocks: the copy-on-write
    # block copies run once, then the samples decode 64 divergent tokens. The
    # timed step is the last one (append + decode at context 1064).
    import paged_kv_cache_387_b200 as pkv
    sp = make_shared_prefix_case(device=dev, seed=rank_seed(391, rank))
    pairs = sp.cow_pairs
    pkv.kv_block_copy(sp.k_pool, sp.v_pool, pairs)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    reps = 20
    for _ in range(reps):  # idempotent: the same copies again
        pkv.kv_block_copy(sp.k_pool, sp.v_pool, pairs)
    b.record()
    torch.cuda.synchronize()
    copy_ms = a.elapsed_time(b) / reps
    blk = sp.num_kv_heads * sp.block_size * sp.head_dim * sp.k_pool.element_size()
    copy_bytes = 2 * 2 * blk * int(pairs.shape[0])  # read + write, K and V
    last = len(sp.steps) - 1
    for k in range(last):
        _, kn, vn = sp.step_tokens(k)
        pkv.kv_cache_append(sp.k_pool, sp.v_pool, kn, vn, sp.steps[k]["slot_mapping"])
    q, kn, vn = sp.step_tokens(last)
    st = sp.steps[last]
    case = DecodeCase(name="shared_prefix", q=q, k_pool=sp.k_pool, v_pool=sp.v_pool,
                      block_tables=st["block_tables"], context_lens=st["context_lens"],
                      num_heads=sp.num_heads, num_kv_heads=sp.num_kv_heads,
                      head_dim=sp.head_dim, block_size=sp.block_size, scale=sp.scale,
                      partition_size=sp.partition_size, k_new=kn, v_new=vn,
                      slot_mapping=st["slot_mapping"])
    # unique K/V bytes: the shared full prompt blocks once per prompt, plus every
    # sample's own blocks
    lens = st["context_lens"].cpu()
    per_tok = 2 * sp.num_kv_heads * sp.head_dim * sp.k_pool.element_size()
    extras = {"block_copy": {"pairs": int(pairs.shape[0]), "ms": copy_ms,
                             "us": copy_ms * 1e3,
                             "GB/s": copy_bytes / (copy_ms * 1e-3) / 1e9,
                             "bytes": copy_bytes},
              "shared_prefix": {"logical_kv_bytes": int(lens.sum()) * per_tok,
                                "unique_kv_bytes": case_unique_kv_bytes(case),
                                "prompts": sp.num_prompts, "samples": sp.samples,
                                "note": "value/roofline count logical bytes; unique_kv_bytes "
                                        "counts each block the samples of a prompt share "
                                        "once"}}
    return case, extras

EXTRA_WORKLOADS = ("opt13b_mha_b64", "long_split_b8", "shared_prefix", "beam_search",
                   "prefix_cache")


def time_fused_call(pkv, case, steps, warmup, stream):
    """Device milliseconds of one paged_attn_decode_append call on `case`, the
    mean over `steps` back-to-back calls after `warmup` (appending the same
    newest token again leaves the pools unchanged)."""
    import torch
    dev = case.q.device
    mcl = case.max_context_len
    out = torch.empty_like(case.q)
    wsb = pkv.decode_workspace_bytes(case.num_seqs, case.num_heads, case.head_dim, mcl,
                                     case.partition_size)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def call():
        pkv.paged_attn_decode_append(out, case.q, case.k_new, case.v_new, case.k_pool,
                                     case.v_pool, case.block_tables, case.context_lens,
                                     case.scale, mcl, partition_size=case.partition_size,
                                     workspace=ws, err=err)
    for _ in range(max(3, warmup)):
        call()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        call()
    b.record(stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word set: {pkv.device_error_message(int(err.item()))}")
    return a.elapsed_time(b) / steps


# Small calls: Llama-8B heads (32 query / 8 KV, d128), bf16, 16-token blocks,
# one step of the fused append + decode with PARTITION_AUTO.
SMALL_BATCHES = {"1x16": [16], "1x4096": [4096], "1x8192": [8192], "1x32768": [32768],
                 "1x131072": [131072], "4x16384": [16384] * 4, "32x1024": [1024] * 32,
                 "256x16": [16] * 256}


def small_batch_lines(pkv, dev, stream, shapes=None):
    """Device microseconds per small call, under the default kernel selection
    (these calls take the single-wave kernel) and with the persistent kernel
    forced:
      graph_us: 50 back-to-back calls replayed from a CUDA graph, per call
        (the K/V, 0.07-537 MB, stays in the 126 MB L2 when it fits);
      cold_us: one call after a 256 MB write has evicted L2, timed by events
        around it (median of 15), with its K/V GB/s."""
    import torch
    from pkv_inputs import make_random_case
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    res = {}
    try:
        for name, lens in SMALL_BATCHES.items():
            if shapes and name not in shapes:
                continue
            c = make_random_case("small_" + name, 32, 8, 128, 16, lens, torch.bfloat16, seed=1,
                                 device=dev, with_append=True)
            mcl = c.max_context_len
            out = torch.empty_like(c.q)
            wsb = pkv.decode_workspace_bytes(c.num_seqs, c.num_heads, c.head_dim, mcl,
                                             pkv.PARTITION_AUTO)
            ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=dev)
            kv_bytes = int(c.context_lens.sum()) * 8 * 128 * 2 * 2

            def call(st):
                pkv.paged_attn_decode_append(out, c.q, c.k_new, c.v_new, c.k_pool, c.v_pool,
                                             c.block_tables, c.context_lens, c.scale, mcl,
                                             partition_size=pkv.PARTITION_AUTO, workspace=ws,
                                             stream=st)
            entry = {"kv_bytes": kv_bytes}
            for mode, key in ((pkv.DISPATCH_AUTO, "single_wave"),
                              (pkv.DISPATCH_PERSISTENT, "persistent")):
                pkv.set_decode_dispatch(mode)
                for _ in range(5):
                    call(stream)
                torch.cuda.synchronize()
                cap = torch.cuda.Stream(device=dev)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap, capture_error_mode="relaxed"):
                    for _ in range(50):
                        call(cap)
                g.replay()
                torch.cuda.synchronize()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g.replay()
                b.record(stream)
                torch.cuda.synchronize()
                graph_us = a.elapsed_time(b) / 50 * 1e3
                del g
                cold = []
                for i in range(15):
                    flush.fill_(i & 0xff)
                    a.record(stream)
                    call(stream)
                    b.record(stream)
                    b.synchronize()
                    cold.append(a.elapsed_time(b) * 1e3)
                cold_us = statistics.median(cold)
                entry[key] = {"graph_us": graph_us, "cold_us": cold_us,
                              "cold_kv_GB/s": kv_bytes / (cold_us * 1e-6) / 1e9}
            res[name] = entry
            del c, out, ws
    finally:
        pkv.set_decode_dispatch(pkv.DISPATCH_AUTO)
    del flush
    torch.cuda.empty_cache()
    return {"shape": "32 query / 8 KV heads, d128, bf16, block 16, fused append, "
                     "PARTITION_AUTO", "calls": res}


def extra_lines(args, dev, rank, pkv, stream, peak):
    """The other workloads of the scope, each timed on the device like the
    headline (the fused append + decode call, `--steps` calls after
    `--warmup`): logical GB/s and, for the workloads that share blocks, the
    GB/s of the distinct blocks read, with their fractions of the copy peak."""
    import torch
    lines = {}
    for w in EXTRA_WORKLOADS:
        if w == args.workload:
            continue
        case, ex = build_bench_case(args, dev, rank, workload=w)
        ms = time_fused_call(pkv, case, args.steps, args.warmup, stream)
        dec, app = step_bytes(case)
        d = {"ms_per_step": ms, "GB/s": (dec + app) / (ms * 1e-3) / 1e9,
             "frac": (dec + app) / (ms * 1e-3) / 1e9 / peak,
             "seq_steps_per_s": case.num_seqs / (ms * 1e-3),
             "num_seqs": case.num_seqs, "context_tokens": int(case.context_lens.sum()),
             "partition_size": case.partition_size, "dtype": str(case.q.dtype)}
        for key in ("shared_prefix", "beam_search", "prefix_cache"):
            if key in ex:
                info = ex[key]
                # the unique step: each distinct block's K/V once, plus the q/o,
                # table and append bytes of every sequence
                ub = info["unique_kv_bytes"] + (dec + app - info["logical_kv_bytes"])
                d.update({k: v for k, v in info.items() if k != "note"})
                d["unique_bytes"] = ub
                d["unique_GB/s"] = ub / (ms * 1e-3) / 1e9
                d["unique_frac"] = d["unique_GB/s"] / peak
        if "block_copy" in ex:
            lines["block_copy"] = ex["block_copy"]
        lines[w] = d
        del case
        torch.cuda.empty_cache()
    lines["small_batch"] = small_batch_lines(pkv, dev, stream)
    return lines


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import paged_kv_cache_387_b200 as pkv
    from paged_kv_cache_387_b200 import build as pkv_build
    from pkv_inputs import make_case

    if rank == 0 or not os.path.exists(pkv.LIB_PATH):
        pkv_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    case, extras = build_bench_case(args, dev, rank)
    if args.partition_size is not None:
        case.partition_size = args.partition_size
    stream = torch.cuda.current_stream(dev)

    S, Hq, D = case.num_seqs, case.num_heads, case.head_dim
    mcl = case.max_context_len
    out = torch.empty_like(case.q)
    ws_bytes = pkv.decode_workspace_bytes(S, Hq, D, mcl, case.partition_size)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # 16-bit: plan + decode (append and merge fused in), or append + plan +
    # decode with --separate-append; fp32: append + decode (+ merge when split)
    if case.q.dtype == torch.float32:
        launches_per_step = 2 + (1 if mcl > case.partition_size > 0 else 0)
    else:
        launches_per_step = 3 if args.separate_append else 2

    def decode(c, o):
        pkv.paged_attn_decode(o, c.q, c.k_pool, c.v_pool, c.block_tables, c.context_lens,
                              c.scale, mcl, partition_size=c.partition_size, workspace=ws,
                              err=err)

    fused = not args.separate_append and case.q.dtype != torch.float32

    def step(ev_pair=None):
        if not fused:
            pkv.kv_cache_append(case.k_pool, case.v_pool, case.k_new, case.v_new,
                                case.slot_mapping, err=err)
        if ev_pair is not None:
            ev_pair[0].record(stream)
        if fused:
            pkv.paged_attn_decode_append(out, case.q, case.k_new, case.v_new, case.k_pool,
                                         case.v_pool, case.block_tables, case.context_lens,
                                         case.scale, mcl, partition_size=case.partition_size,
                                         workspace=ws, err=err)
        else:
            decode(case, out)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(dev)
    uuid = getattr(props, "uuid", None)
    sampler = ClockSampler(f"GPU-{uuid}" if uuid is not None else local_rank)
    if rank == 0:
        sampler.start()
    t_soak0 = time.time()
    # soak: back-to-back steps so clocks settle and samples exist next to the timed region
    while time.time() - t_soak0 < args.soak_seconds:
        for _ in range(20):
            step()
        torch.cuda.synchronize()

    # With the append fused in, a step is exactly one decode call, so the
    # region's time per step is the call's average duration. Only the separate
    # append + decode step brackets each decode call with its own events
    # (which cost a few microseconds of stream time per step).
    dec_events = None if fused else [
        (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
        for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_host0 = time.time()
    start.record(stream)
    for i in range(args.steps):
        step(dec_events[i] if dec_events else None)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t_host1 = time.time()
    time.sleep(0.25)
    sampler.stop()

    ms = start.elapsed_time(end) / args.steps
    dec_ms = (statistics.mean(a.elapsed_time(b) for a, b in dec_events) if dec_events
              else start.elapsed_time(end) / args.steps)
    ms, dec_ms = max_over_ranks([ms, dec_ms], dev)

    dec_bytes, app_bytes = step_bytes(case)
    value = whole_job_gbs(dec_bytes + app_bytes, world, ms * 1e-3)

    # ---- end to end: host buffers, copies inside the timed region ----
    # Every step's inputs go up from pinned host memory and every step's
    # result comes back to the host, as in a serving loop; the inputs of
    # `--e2e-steps-per-upload` steps travel in one copy. Uploads and
    # downloads run on two copy streams with `--e2e-buffers` device buffers,
    # so later groups' uploads and earlier groups' downloads overlap a
    # group's kernels.
    # With `--e2e-result-in-host-memory` the decode writes its result straight
    # into a pinned host buffer instead (the C ABI accepts page-locked host
    # memory for `out`), leaving the copy engines to the uploads. The host
    # link of a shared machine varies from run to run, so the measured pinned
    # copy rates are reported beside the number.
    names = ("q", "k_new", "v_new", "block_tables", "context_lens")
    if not fused:
        names = names + ("slot_mapping",)
    # The step's inputs live in one pinned staging buffer (256-byte aligned
    # segments) and go up in one copy, as a serving loop stages them.
    segs, off = {}, 0
    for k in names:
        t = getattr(case, k)
        nbytes = t.numel() * t.element_size()
        segs[k] = (off, nbytes, t.dtype, tuple(t.shape))
        off += (nbytes + 255) // 256 * 256
    h2d = off

    def views(buf):
        return {k: buf[o:o + n].view(dt).view(shp) for k, (o, n, dt, shp) in segs.items()}
    nb = max(2, args.e2e_buffers)
    d2h = out.numel() * out.element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ncs = max(1, args.e2e_compute_streams)
    comp = [stream] + [torch.cuda.Stream(dev) for _ in range(ncs - 1)]
    wss = [ws] + [torch.empty_like(ws) for _ in range(ncs - 1)]

    def run_step(inp, o, cs, wsi):
        if fused:
            pkv.paged_attn_decode_append(o, inp["q"], inp["k_new"], inp["v_new"], case.k_pool,
                                         case.v_pool, inp["block_tables"], inp["context_lens"],
                                         case.scale, mcl, partition_size=case.partition_size,
                                         workspace=wsi, err=err, stream=cs)
            return
        pkv.kv_cache_append(case.k_pool, case.v_pool, inp["k_new"], inp["v_new"],
                            inp["slot_mapping"], err=err, stream=cs)
        pkv.paged_attn_decode(o, inp["q"], case.k_pool, case.v_pool, inp["block_tables"],
                              inp["context_lens"], case.scale, mcl,
                              partition_size=case.partition_size, workspace=wsi, err=err,
                              stream=cs)

    def make_e2e(G):
        """The end-to-end loop with G steps per upload: one pinned staging
        buffer holds G steps' inputs (each step its own segment), goes up in
        one copy, and the G steps' results come back in one copy. Between the
        G calls of a group no stream operation intervenes, so their launches
        keep their programmatic overlap; every step's input and result bytes
        still cross the host link inside the timed region."""
        host_stage = torch.empty(G * h2d, dtype=torch.uint8, pin_memory=True)
        for g in range(G):
            for k, t in views(host_stage[g * h2d:(g + 1) * h2d]).items():
                t.copy_(getattr(case, k).cpu())
        dev_stage = [torch.empty(G * h2d, dtype=torch.uint8, device=dev) for _ in range(nb)]
        dev_sets = [[views(b[g * h2d:(g + 1) * h2d]) for g in range(G)] for b in dev_stage]
        outs = [torch.empty((G,) + tuple(out.shape), dtype=out.dtype, device=dev)
                for _ in range(nb)]
        host_outs = [torch.empty((G,) + tuple(out.shape), dtype=out.dtype, pin_memory=True)
                     for _ in range(nb)]
        # Per buffer b: in_ready (upload done), done (decodes done), out_free
        # (download done, which follows `done`). The upload into buffer b
        # waits for out_free of the group that used b before, so a compute
        # stream only waits for in_ready and records done, once per group.
        # Groups take turns on `--e2e-compute-streams` compute streams, each
        # with its own workspace.
        in_ready = [torch.cuda.Event() for _ in range(nb)]
        done = [torch.cuda.Event() for _ in range(nb)]
        out_free = [torch.cuda.Event() for _ in range(nb)]

        def steps(n, start_event=None):
            for j in range(n // G):
                b = j % nb
                with torch.cuda.stream(h2d_stream):
                    if j >= nb:
                        h2d_stream.wait_event(out_free[b])  # buffer b's previous group is over
                    elif start_event is not None:
                        h2d_stream.wait_event(start_event)
                    dev_stage[b].copy_(host_stage, non_blocking=True)
                    in_ready[b].record(h2d_stream)
                cs, wsi = comp[j % ncs], wss[j % ncs]
                cs.wait_event(in_ready[b])
                if args.e2e_result_in_host_memory:
                    # the decode writes its result straight into pinned host memory
                    for g in range(G):
                        run_step(dev_sets[b][g], host_outs[b][g], cs, wsi)
                    done[b].record(cs)
                    out_free[b] = done[b]
                    continue
                for g in range(G):
                    run_step(dev_sets[b][g], outs[b][g], cs, wsi)
                done[b].record(cs)
                with torch.cuda.stream(d2h_stream):
                    d2h_stream.wait_event(done[b])
                    host_outs[b].copy_(outs[b], non_blocking=True)
                    out_free[b].record(d2h_stream)
            for other in [d2h_stream] + comp[1:]:
                last = torch.cuda.Event()
                last.record(other)
                stream.wait_event(last)
        return steps

    def time_e2e(G):
        steps = make_e2e(G)
        steps(3 * G)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        n = max(args.steps, args.e2e_steps) // G * G
        e0.record(stream)
        t0 = time.perf_counter()
        steps(n, start_event=e0)
        submit_ms = (time.perf_counter() - t0) * 1e3 / n
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks([e0.elapsed_time(e1) / n], dev)[0], n, submit_ms

    G = max(1, args.e2e_steps_per_upload)
    # The device-only step again, right before the end-to-end loops: the
    # ratio of the two is taken at the same clocks (the power cap moves them
    # over a run).
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_adj = min(args.steps, 100)
    a0.record(stream)
    for _ in range(n_adj):
        step()
    a1.record(stream)
    torch.cuda.synchronize()
    adj_ms = max_over_ranks([a0.elapsed_time(a1) / n_adj], dev)[0]
    e2e_ms, n_e2e, host_submit_ms = time_e2e(G)
    # the same loop with one upload and one download per step (diagnostic)
    e2e_ms_1 = time_e2e(1)[0] if G > 1 else e2e_ms

    # the copy engines' own rates for this step's transfer sizes (diagnostic)
    def copy_gbs(dst, src, nbytes, reps=20):
        for _ in range(3):
            dst.copy_(src, non_blocking=True)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            dst.copy_(src, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        return nbytes * reps / (a.elapsed_time(b) * 1e-3) / 1e9
    flat_h = torch.empty(h2d, dtype=torch.uint8, pin_memory=True)
    flat_d = torch.empty(h2d, dtype=torch.uint8, device=dev)
    h2d_gbs = copy_gbs(flat_d, flat_h, h2d)
    d2h_gbs = copy_gbs(torch.empty(out.shape, dtype=out.dtype, pin_memory=True), out, d2h)
    del flat_h, flat_d
    e2e_value = whole_job_gbs(dec_bytes + app_bytes, world, e2e_ms * 1e-3)

    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word set: {pkv.device_error_message(int(err.item()))}")

    swap = measure_swap(case, dev, stream, pkv) if args.workload != "shared_prefix" else None

    # standalone kv_cache_append of the step's tokens (through the slot mapping)
    append_line = None
    if case.slot_mapping is not None and not args.no_extras:
        for _ in range(3):
            pkv.kv_cache_append(case.k_pool, case.v_pool, case.k_new, case.v_new,
                                case.slot_mapping, err=err)
        a_ev, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a_ev.record(stream)
        for _ in range(args.steps):
            pkv.kv_cache_append(case.k_pool, case.v_pool, case.k_new, case.v_new,
                                case.slot_mapping, err=err)
        b_ev.record(stream)
        torch.cuda.synchronize()
        app_ms = a_ev.elapsed_time(b_ev) / args.steps
        append_line = {"tokens": S, "us": app_ms * 1e3, "bytes": app_bytes,
                       "GB/s": app_bytes / (app_ms * 1e-3) / 1e9}

    contiguous = None
    if (args.contiguous or not args.no_extras) and args.workload != "shared_prefix":
        ccase = make_case(args.workload, device=dev, with_append=False, placement="identity",
                          num_seqs=args.num_seqs)
        cout = torch.empty_like(ccase.q)

        def decode_ms(c, o):
            for _ in range(3):
                decode(c, o)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(stream)
            for _ in range(args.steps):
                decode(c, o)
            b.record(stream)
            torch.cuda.synchronize()
            return a.elapsed_time(b) / args.steps
        # the same decode call (no append) on both placements
        sms = decode_ms(case, out)
        cms = decode_ms(ccase, cout)
        contiguous = {"decode_ms_identity_placement": cms, "decode_ms_shuffled": sms,
                      "paged_over_contiguous_time": sms / cms}
        del ccase, cout

    peak, peak_kind = measured_peaks()
    # every rank times the same extra workloads on its own GPU (no collective);
    # rank 0 reports its own
    extras_all = {} if args.no_extras else extra_lines(args, dev, rank, pkv, stream, peak)

    if rank != 0:
        return None

    # the fused call also reads the new K/V rows and writes them to the pool
    call_bytes = dec_bytes + (app_bytes if fused else 0)
    achieved = call_bytes / (dec_ms * 1e-3) / 1e9
    traffic = recorded_traffic(args.workload)
    clocks = sampler.summary(t_soak0, t_host1,
                             "soak + timed region" if t_host1 - t_host0 < 1.0 else "timed region")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": str(case.q.dtype).replace("torch.", "").replace("bfloat16", "bf16")
                 .replace("float16", "f16").replace("float32", "f32"),
        "data": "synthetic",
        "config": config_block(case, args.workload, world),
        "seq_steps_per_s": S * world / (ms * 1e-3),
        "pct_of_hbm_peak": {"of_spec_8000_gbs": value / (HBM_SPEC_GBS * world),
                            f"of_{peak_kind}_{peak:.0f}_gbs": value / (peak * world)},
        "roofline": {"kernel": "decode call (plan_kernel + decode_tc_kernel)",
                     "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "algorithmic_bytes": call_bytes,
                     "decode_ms": dec_ms,
                     "timing": ("timed region / steps (one call per step)" if fused
                                else "events around each decode call")},
        "e2e": {"value": e2e_value, "unit": "GB/s", "ms_per_step": e2e_ms, "steps": n_e2e,
                "device_ms_per_step_adjacent": adj_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps_per_upload": G,
                "ms_per_step_one_upload_per_step": e2e_ms_1,
                "pipelining": f"inputs of {G} step(s) staged in one pinned buffer, one upload "
                              "per group on a copy stream, overlapping the neighbouring groups' "
                              "kernels; each step's result comes back in one download per "
                              f"group; groups take turns on {ncs} compute stream(s), each with "
                              "its own workspace",
                "result_to_host": ("written by the decode kernels into pinned host memory"
                                   if args.e2e_result_in_host_memory else
                                   "device-to-host copy on a second copy stream"),
                "buffers": nb,
                "pinned_h2d_gbs": h2d_gbs, "pinned_d2h_gbs": d2h_gbs,
                "host_submit_ms_per_step": host_submit_ms,
                "transfer_bound_ms": max(h2d / h2d_gbs, d2h / d2h_gbs) * 1e-6},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if contiguous:
        line["paged_vs_contiguous"] = contiguous
    if append_line:
        line["kv_cache_append"] = append_line
    line.update(extras_all)
    if swap:
        swap["pinned_h2d_gbs"], swap["pinned_d2h_gbs"] = h2d_gbs, d2h_gbs
        line["swap"] = swap
    line["config"]["call"] = call_description(case, args)
    line.update(extras)
    for key in ("shared_prefix", "beam_search", "prefix_cache"):
        if key in extras:
            # the unique step: each distinct block's K/V once, plus the q/o,
            # table and append bytes of every sequence
            bx = extras[key]
            bx["unique_bytes"] = bx["unique_kv_bytes"] + (call_bytes - bx["logical_kv_bytes"])
            bx["unique_GB/s"] = bx["unique_bytes"] / (dec_ms * 1e-3) / 1e9
            bx["unique_frac"] = bx["unique_GB/s"] / peak
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, args.cpu_seconds)
    return line


def cpu_baseline(case, target_s):
    import oracle
    oracle.build()
    c = case.to("cpu")
    nseq = size_oracle_sample(c, target_s)
    t0 = time.perf_counter()
    oracle_sample_step(c, nseq)
    dt = time.perf_counter() - t0
    dec, app = step_bytes(c, nseq)
    return {"value": (dec + app) / dt / 1e9, "unit": "GB/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {nseq} of {c.num_seqs} sequences "
                      f"({int(c.context_lens[:nseq].sum())} tokens), one append + decode step, "
                      f"{dt:.1f} s"}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if args.small_batch_only:
        import torch
        import paged_kv_cache_387_b200 as pkv
        from paged_kv_cache_387_b200 import build as pkv_build
        pkv_build.build()
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        shapes = args.small_batch_shapes.split(",") if args.small_batch_shapes else None
        if rank == 0:
            print(json.dumps({"small_batch": small_batch_lines(
                pkv, dev, torch.cuda.current_stream(dev), shapes)}), flush=True)
        return
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
