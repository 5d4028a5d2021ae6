#!/usr/bin/env python
"""Decode-attention benchmark: µs per call and achieved HBM GB/s.

Default workload: decode GQA bf16, Llama-3-70B-like shape (batch 32, 64 query / 8 KV heads,
head_dim 128, cache lengths uniform in [1024, 32768], capacity 32768, planner splits). One step is
one fd_decode_attention call (device planner + split kernel + LSE combine) over resident inputs.
Workload 5 (mixed chunked-prefill step) times one fd_chunk_prefill_attention call instead.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl fd|reference] [--workload 1-5]
                    [--batch B] [--page-size P]

--page-size P reads a decode workload's cache through fd_decode_attention_paged, in pages of P
keys at shuffled physical positions.

Prints one JSON line on rank 0. `value` is the whole-job GB/s: the algorithmic bytes every rank
processed (K+V bytes of the valid keys plus the Q bytes) over the slowest rank's device time.
With N > 1 every rank runs an independent replica: the path has no exchange step. Under torchrun
--gpus must equal WORLD_SIZE; without it, --gpus N > 1 starts the N processes itself.
`--impl reference` times the float64 CPU oracle on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn µs/call and achieved HBM GB/s vs 8 TB/s peak (Llama-3-70B GQA)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["fd", "reference"], default="fd")
    ap.add_argument("--workload", type=int, default=3, choices=[1, 2, 3, 4, 5, 6])
    ap.add_argument("--batch", type=int, default=None,
                    help="batch of workload 4; for workloads 3 and 5, keep the first B requests")
    ap.add_argument("--page-size", type=int, default=0,
                    help="decode workloads: read the cache through fd_decode_attention_paged, in "
                         "pages of this many keys at shuffled physical positions (0: contiguous)")
    ap.add_argument("--kv-dtype", choices=["native", "e4m3"], default="native",
                    help="e4m3: the workload's cache quantized to FP8 E4M3 (one scale per tensor), "
                         "timed through fd_decode_attention_fp8 / fd_decode_attention_paged_fp8")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--profile-calls", type=int, default=200,
                    help="calls timed with per-kernel events after the timed region (0: skip)")
    ap.add_argument("--cpu-seconds", type=float, default=20.0,
                    help="host-time budget of the oracle CPU baseline samples (half with every "
                         "thread, half on one thread)")
    return ap.parse_args()


# ------------------------------------------------------------------------------ helpers -------

def log(*a):
    print(*a, file=sys.stderr, flush=True)


def is_chunk(inp) -> bool:
    return hasattr(inp, "q_chunk")


def key_lens(inp):
    """Valid keys per request: cache_lens, or prefix + chunk for a chunked-prefill step."""
    cap = inp.k_cache.shape[2]
    if is_chunk(inp):
        raw = [int(p) + int(c) for p, c in zip(inp.prefix_lens.tolist(), inp.chunk_lens.tolist())]
    else:
        raw = inp.cache_lens.tolist()
    return [max(0, min(int(x), cap)) for x in raw]


def queries(inp):
    return inp.q_chunk if is_chunk(inp) else inp.q


def algorithmic_bytes(inp) -> int:
    """K+V bytes of the valid keys (each read once) plus the Q bytes."""
    B, hkv, cap, d = inp.k_cache.shape
    es = inp.k_cache.element_size()
    q = queries(inp)
    return 2 * sum(key_lens(inp)) * hkv * d * es + q.numel() * q.element_size()


def chunk_tile_flops(inp) -> int:
    """Algorithmic FLOPs of the chunked-prefill tile rows (chunk_len > 1): per (row, query head),
    2 D for q.k and 2 D for p.v per visible key; row i of a request sees prefix + i + 1 keys."""
    cap = inp.k_cache.shape[2]
    hq, d = inp.q_chunk.shape[1], inp.q_chunk.shape[2]
    keys = 0
    for p, c in zip(inp.prefix_lens.tolist(), inp.chunk_lens.tolist()):
        if int(c) > 1:
            keys += sum(min(int(p) + i + 1, cap) for i in range(int(c)))
    return 4 * d * hq * keys


def measured_peak(key: str = "hbm_gbs"):
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j[key]), "measured"
    except Exception:
        return (FALLBACK_HBM_GBS if key == "hbm_gbs" else FALLBACK_BF16_TFLOPS), "fallback"


def kernel_source_sha(name: str) -> str:
    path = os.path.join(ROOT, "split_kv_decode_flashdecoding_b200", "csrc", name)
    h = hashlib.sha256()
    for f in sorted([path, os.path.join(os.path.dirname(path), "common.cuh")]):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            j = json.load(f)
        e = j[f"{workload}:{kernel_file}"]
        if e.get("source_sha") == kernel_source_sha(kernel_file):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="fd_clocks_", suffix=".csv")
        self.proc = None
        self.gpu = gpu_index

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.5)
        except Exception as e:  # no nvidia-smi: report that instead of clocks
            log(f"clock sampler unavailable: {e}")
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) < 10:
                    continue
                try:
                    sm.append(float(p[2]))
                    smax.append(float(p[3]))
                except ValueError:
                    continue
                for n, v in zip(names, p[6:10]):
                    if v.lower().startswith("active"):
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value: float, world: int, device) -> float:
    """The largest of the ranks' values (all_reduce MAX); the value itself on one rank. Every
    rank must call it, in the same order as every other collective."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank_step: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job GB/s of `world` replicas, each processing bytes_per_rank_step per step, over the
    slowest rank's time for `steps` steps."""
    return world * bytes_per_rank_step * steps / (ms_max * 1e-3) / 1e9


def emit(line: dict, rank: int) -> None:
    """Rank 0 prints the one JSON line; the other ranks stay silent."""
    if rank == 0:
        print(json.dumps(line), flush=True)


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [int(x.get("num_threads", 1)) for x in threadpool_info() if x.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


def cpu_model() -> str:
    """The host CPU's model name (first processor in /proc/cpuinfo) and its logical CPU count."""
    name = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    name = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return f"{name}, {os.cpu_count() or 1} logical CPUs"


def oracle_sample(inp, seconds: float, seed: int = 0, quant=None):
    """Time the oracle on whole (query row, KV head) groups of the workload, all G query heads
    each, in a seeded order, until `seconds` of host time are spent. `quant` = (k_scale, v_scale):
    the cache holds E4M3 codes.
    Returns (bytes/s, description, groups, elapsed)."""
    from oracle import attention as oracle
    from workloads import to_numpy_exact
    q = to_numpy_exact(queries(inp))
    k = to_numpy_exact(inp.k_cache)
    v = to_numpy_exact(inp.v_cache)
    R, hq, d = q.shape
    hkv = k.shape[1]
    g = hq // hkv
    es = inp.k_cache.element_size()
    vis = []
    if is_chunk(inp):
        prefix, chunk = inp.prefix_lens.tolist(), inp.chunk_lens.tolist()
        cap = k.shape[2]
        for p, c in zip(prefix, chunk):
            vis.extend(min(int(p) + i + 1, cap) for i in range(int(c)))

        def run(rows):
            oracle.chunk_prefill_attention(q, k, v, prefix, chunk, rows=rows)
    else:
        lens = inp.cache_lens.tolist()
        vis = key_lens(inp)

        def run(rows):
            if quant is not None:
                oracle.decode_attention_fp8(q, k, v, quant[0], quant[1], lens, rows=rows)
            else:
                oracle.decode_attention(q, k, v, lens, rows=rows)
    order = np.random.default_rng(seed).permutation(R * hkv)
    done, nbytes = 0, 0
    t0 = time.perf_counter()
    for idx in order:
        r, h = divmod(int(idx), hkv)
        run([(r, h * g + j) for j in range(g)])
        nbytes += 2 * vis[r] * d * es + g * d * queries(inp).element_size()
        done += 1
        if time.perf_counter() - t0 >= seconds:
            break
    el = time.perf_counter() - t0
    desc = (f"{done} of {R * hkv} (query row, KV head) groups of the workload, all {g} query "
            f"heads each, seeded order; float64 numpy")
    return nbytes / el, desc, done, el


def load_workload(args):
    """The workload's inputs and, with --kv-dtype e4m3, its E4M3 cache (the codes replace the
    bf16 cache tensors; the scales are returned beside them)."""
    from workloads import WORKLOADS, workload
    t0 = time.time()
    inp = workload(args.workload, batch=args.batch)
    f8 = None
    if args.kv_dtype == "e4m3":
        if is_chunk(inp) or inp.k_cache.dtype != torch.bfloat16:
            raise SystemExit("--kv-dtype e4m3 needs a bf16 decode workload (2, 3 or 4)")
        from workloads import make_fp8
        f8 = make_fp8(inp.k_cache, inp.v_cache)
        inp.k_cache, inp.v_cache = f8.k_codes, f8.v_codes
        inp.name = f"{inp.name}_e4m3"
    log(f"generated {inp.name} in {time.time() - t0:.1f}s")
    return inp, f8


# ------------------------------------------------------------------------------ arms ----------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    inp, f8 = load_workload(args)
    quant = (f8.k_scale, f8.v_scale) if f8 else None
    per_step = max(0.2, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(inp, per_step / 4, seed=1, quant=quant)
    rates = []
    t0 = time.perf_counter()
    total_bytes = 0
    for s in range(args.steps):
        r, desc, groups, el = oracle_sample(inp, per_step, seed=100 + s, quant=quant)
        rates.append(r)
        total_bytes += r * el
    el = time.perf_counter() - t0
    value = total_bytes / el / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * el / max(1, args.steps), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": inp.name},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cpu_threads(),
                         "kind": "oracle", "cpu": cpu_model(),
                         "sample": f"per step: whole (query row, KV head) groups of the workload in a "
                                   f"seeded order until {per_step:.2f}s of host time (or all groups)"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    emit(line, rank)
    return 0


def run_fd(args, rank, world, local_rank):
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    inp, f8 = load_workload(args)
    chunk = is_chunk(inp)
    paged = args.page_size > 0 and not chunk
    fp8 = f8 is not None
    if paged:
        from workloads import make_paged
        pgc = make_paged(inp.k_cache, inp.v_cache, inp.cache_lens.tolist(), args.page_size,
                         seed=7000 + args.workload, pad_fill=0.0)
        inp.name = f"{inp.name}_paged{args.page_size}"
    alg = algorithmic_bytes(inp)
    R, hq, d = queries(inp).shape
    B, hkv = inp.k_cache.shape[:2]
    g = hq // hkv
    q = queries(inp).to(dev)
    if paged:
        k = pgc.k_pages.to(dev)
        v = pgc.v_pages.to(dev)
        table = pgc.block_table.to(dev)
    else:
        k = inp.k_cache.to(dev)
        v = inp.v_cache.to(dev)
    if chunk:
        lens_h = [inp.prefix_lens, inp.chunk_lens]
    else:
        lens_h = [inp.cache_lens]
    lens = [t.to(dev) for t in lens_h]
    out = torch.empty_like(q)
    lse = torch.empty((R, hq), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ns = 0 if chunk else inp.num_splits
    input_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    l2_policy = ("inputs larger than L2 (valid K/V bytes per call exceed the 126 MB L2)"
                 if alg > 2 * L2_BYTES else "inputs smaller than L2: measured with warm L2")
    # the tensor-core split kernel: decode calls of bf16 groups of 2..16 (or any E4M3 group of
    # <= 8) with head_dim 128, and the decode rows of every chunked call with head_dim 128
    use_tc = (inp.k_cache.dtype == torch.bfloat16 and d == 128 and (chunk or 2 <= g <= 16)) or \
             (fp8 and d == 128 and g <= 8)
    if chunk:
        # planner, decode-row split kernel, chunk tile kernel, combine
        launches_per_step = 4

        def step():
            fd.fd_chunk_prefill_attention(q, k, v, lens[0], lens[1], out=out, lse=lse, stream=stream)
    else:
        # the tensor-core split kernel plans batches of up to 256 sequences itself and is
        # followed by the combine kernel; the CUDA-core split kernel follows the planner kernel
        # and merges its splits itself
        launches_per_step = ((0 if B <= 256 else 1) + 2) if use_tc else 2

        if fp8 and paged:
            def step():
                fd.fd_decode_attention_paged_fp8(q, k, v, f8.k_scale, f8.v_scale, table, lens[0],
                                                 ns, out=out, lse=lse, stream=stream)
        elif fp8:
            def step():
                fd.fd_decode_attention_fp8(q, k, v, f8.k_scale, f8.v_scale, lens[0], ns, out=out,
                                           lse=lse, stream=stream)
        elif paged:
            def step():
                fd.fd_decode_attention_paged(q, k, v, table, lens[0], ns, out=out, lse=lse,
                                             stream=stream)
        else:
            def step():
                fd.fd_decode_attention(q, k, v, lens[0], ns, out=out, lse=lse, stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    # ---- timed region: K calls, CUDA events on the launching stream ----
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    ms_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_per_step = ms_max / args.steps
    value = whole_job_gbs(alg, args.steps, world, ms_max)

    # ---- per-kernel durations (same calls, with events between the launches) ----
    nprof = min(args.steps, args.profile_calls)
    prof = [(float("nan"),) * 4]
    if nprof > 0:
        fd.fd_profile_begin(nprof)
        for _ in range(nprof):
            step()
        torch.cuda.synchronize()
        prof = fd.fd_profile_end(nprof)

    def _mean(i):
        x = statistics.mean(p[i] for p in prof)
        return None if x != x else x
    plan_ms, split_ms, tile_ms, comb_ms = _mean(0), _mean(1), _mean(2), _mean(3)
    peak, peak_kind = measured_peak("hbm_gbs")
    kfile = "decode_tc.cu" if use_tc else "decode_simt.cu"
    split_bytes = alg
    if chunk:
        # the decode-row split kernel streams the decode rows' K/V; the tile kernel the rest
        dec_keys = sum(n for n, c in zip(key_lens(inp), inp.chunk_lens.tolist()) if int(c) == 1)
        split_bytes = 2 * dec_keys * hkv * d * inp.k_cache.element_size()
    achieved = split_bytes / (split_ms * 1e-3) / 1e9 if split_ms else None
    roofline = {"bound": "hbm", "kernel": kfile.replace(".cu", "_kernel"),
                "achieved": round(achieved, 1) if achieved else None, "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4) if achieved else None,
                "peak_kind": f"{peak_kind} copy bandwidth",
                "algorithmic_bytes_per_launch": split_bytes,
                "traffic": traffic_from_profiles(kfile, inp.name),
                "kernel_ms": {k_: (round(x, 5) if x is not None else None) for k_, x in
                              (("planner", plan_ms), ("split", split_ms),
                               ("chunk_tiles", tile_ms), ("combine", comb_ms))}}
    roofline_tiles = None
    if chunk and tile_ms:
        flops = chunk_tile_flops(inp)
        tpeak, tkind = measured_peak("bf16_tflops")
        ach = flops / (tile_ms * 1e-3) / 1e12
        # the tile kernel's own K+V+Q bytes: requests of more than one row, keys read once per
        # KV head (head-packed tiles) or once per query head from L2 (per-head tiles)
        ck = inp.chunk_lens.tolist()
        es = inp.k_cache.element_size()
        tile_bytes = (2 * sum(n for n, c in zip(key_lens(inp), ck) if int(c) > 1) * hkv * d * es +
                      sum(int(c) for c in ck if int(c) > 1) * hq * d * inp.q_chunk.element_size())
        ridge = tpeak * 1e12 / (peak * 1e9)
        tensor_view = {"bound": "tensor", "kernel": "chunk_tc_kernel", "achieved": round(ach, 2),
                       "peak": tpeak, "unit": "TFLOP/s", "frac": round(ach / tpeak, 4),
                       "peak_kind": f"{tkind} dense bf16 (burst)",
                       "algorithmic_flops_per_launch": flops,
                       "traffic": traffic_from_profiles("chunk_tc.cu", inp.name),
                       "kernel_ms": roofline["kernel_ms"]}
        hb = tile_bytes / (tile_ms * 1e-3) / 1e9
        hbm_view = {"bound": "hbm", "kernel": "chunk_tc_kernel", "achieved": round(hb, 1),
                    "peak": peak, "unit": "GB/s", "frac": round(hb / peak, 4),
                    "peak_kind": f"{peak_kind} copy bandwidth",
                    "algorithmic_bytes_per_launch": tile_bytes,
                    "traffic": traffic_from_profiles("chunk_tc.cu", inp.name),
                    "kernel_ms": roofline["kernel_ms"]}
        # below the ridge point (flops per byte of the measured peaks) the tiles are memory-bound
        roofline_tiles = hbm_view if flops / max(1, tile_bytes) < ridge else tensor_view
        if tile_ms > split_ms:
            roofline, roofline_tiles = roofline_tiles, roofline

    # ---- end to end: host buffers, copies inside the timed region ----
    # The step's inputs are q, the lengths and the cache rows that hold keys: each (sequence, KV
    # head)'s first len rows of K and V (rows past the lengths are padding, not input), or the
    # whole page pool and block table of a paged cache. They are copied from pinned host memory,
    # one contiguous copy per (sequence, KV head) slab, and out / lse are read back every step.
    e2e = None
    if args.e2e_steps > 0:
        hq_ = queries(inp).pin_memory()
        hl = [t_.pin_memory() for t_ in lens_h]
        ho = torch.empty_like(queries(inp)).pin_memory()
        hlse = torch.empty((R, hq), dtype=torch.float32).pin_memory()
        copies = [(q, hq_)] + list(zip(lens, hl))
        if paged:
            copies += [(k, pgc.k_pages.pin_memory()), (v, pgc.v_pages.pin_memory()),
                       (table, pgc.block_table.pin_memory())]
            what = "q, lengths, the whole page pool (all pages but 3 spares hold keys) and the block table"
        else:
            hk = inp.k_cache.pin_memory()
            hv = inp.v_cache.pin_memory()
            for b_, n_ in enumerate(key_lens(inp)):
                if n_ > 0:
                    for h_ in range(hkv):
                        copies.append((k[b_, h_, :n_], hk[b_, h_, :n_]))
                        copies.append((v[b_, h_, :n_], hv[b_, h_, :n_]))
            what = ("q, lengths and the valid cache rows (the first len keys of every (sequence, KV "
                    "head), one copy per slab); padding rows past the lengths are not copied")
        h2d = sum(src.numel() * src.element_size() for _, src in copies)
        d2h = ho.numel() * ho.element_size() + hlse.numel() * 4

        def e2e_step():
            for dst, src in copies:
                dst.copy_(src, non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        a1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(a0.elapsed_time(a1), world, dev)
        e2e = {"value": round(whole_job_gbs(alg, args.e2e_steps, world, te), 3),
               "unit": "GB/s", "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps, "copies_per_step": len(copies) + 2,
               "note": f"host->device every step: {what}; out and lse read back"}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        # the oracle as it stands on the host's cores: once with every thread its numpy uses,
        # once limited to one thread, each on a bounded sample of the same workload
        from threadpoolctl import threadpool_limits
        quant = (f8.k_scale, f8.v_scale) if fp8 else None
        rate, desc, groups, el = oracle_sample(inp, args.cpu_seconds / 2, quant=quant)
        with threadpool_limits(limits=1):
            rate1, desc1, groups1, el1 = oracle_sample(inp, args.cpu_seconds / 2, quant=quant)
        cpu = {"value": round(rate / 1e9, 4), "unit": "GB/s", "cores": cpu_threads(),
               "kind": "oracle", "cpu": cpu_model(), "sample": f"{desc}; {el:.1f}s",
               "single_core": {"value": round(rate1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                               "sample": f"{desc1}; {el1:.1f}s"}}

    if rank == 0:
        config = {"workload": inp.name, "batch": R if not chunk else B, "q_heads": hq, "kv_heads": hkv,
                  "head_dim": d, "cache_capacity": int(inp.k_cache.shape[2]),
                  "sum_key_len": int(sum(key_lens(inp))),
                  "num_splits": "planner" if ns == 0 else ns,
                  "algorithmic_bytes_per_call": alg, "input_bytes_resident": input_bytes,
                  "l2": l2_policy, "parallelism": f"replicas x{world}"}
        if fp8:
            config["kv_cache"] = {"format": "E4M3", "k_scale": f8.k_scale, "v_scale": f8.v_scale}
        if paged:
            config["page_size"] = args.page_size
            config["pages_in_pool"] = int(k.shape[0])
        if chunk:
            config["chunk_rows"] = int(R)
            config["chunk_tile_flops_per_call"] = chunk_tile_flops(inp)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup),
            "ms_per_step": round(ms_per_step, 5), "us_per_call": round(ms_per_step * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if inp.k_cache.dtype == torch.bfloat16 else
                     ("bf16 (E4M3 cache expanded exactly to bf16)" if fp8 else "f32"),
            "data": "synthetic",
            "config": config,
            "roofline": roofline,
            "clocks": clocks,
            "e2e": e2e,
            "gpu_launches": launches_per_step * args.steps,
            "cpu_baseline": cpu,
        }
        if roofline_tiles is not None:
            line["roofline_secondary"] = roofline_tiles
        if chunk:
            line["note"] = ("the tile kernel and the decode-row split kernel run side by side (the "
                            "planner splits the multiprocessors between them); each kernel's "
                            "duration is measured while they share the device")
        emit(line, rank)
    return 0


def free_port() -> int:
    import socket
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def main():
    args = parse_args()
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # not under torchrun: start the N replicas (one process per GPU) here
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
               f"--nproc-per-node={args.gpus}", "--master-addr=127.0.0.1",
               f"--master-port={free_port()}", os.path.abspath(__file__), *sys.argv[1:]]
        return subprocess.call(cmd)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        log(f"bench.py: --gpus {args.gpus} but WORLD_SIZE is {world}; launch one process per GPU "
            f"(torchrun --nproc-per-node {args.gpus}) or pass --gpus {world}")
        return 2
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_fd(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
