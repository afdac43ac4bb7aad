"""Benchmark of one dynamic-sparse-attention prefill layer on B200.

One step = the whole hot path over one layer of synthetic input: build the
per-head sparse indices (dsa_build_indices) and run the sparse attention forward
(dsa_sparse_prefill).  The default workload is the FlashPrefill-style
block-threshold layer: 32 q / 8 KV heads, d = 128, N = 131072 tokens, bf16, K/V/Q
built from 512 latent topics per 128-token block, every head keeping the blocks
whose pooled score is within alpha = 0.5 (probability space) of the row maximum,
plus the sink and local block, block 128.  The attention kernel's tensor-peak
target is stated on this layer.  The other layers (VS 4K, Llama-3-8B-shaped mixed
32K, MoBA 64K, VS 1M) are behind --workload.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dsa|reference]

With torchrun (N > 1) every rank runs its own independent layer (heads and
layers shard with no data-path exchange: weak scaling); the only collectives are
the timing barrier and the max-over-ranks reduction.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "sparse prefill tokens/s per layer and % of B200 bf16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if "Active" in r[5 + k]
                          and "Not" not in r[5 + k]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def algorithmic_index_bytes(w, pats):
    """Bytes the index build must move: Q read once for pooled-Q heads, K read once
    per KV head that is pooled or scanned by a VS estimate, the last_q query rows,
    the VS score arrays written and read once, and the index lists written."""
    N, d, Bk, G = w["N"], w["d"], w["B"], w["Hq"] // w["Hkv"]
    nqb = (N + Bk - 1) // Bk
    byt = 0
    kv_read = set()
    for h, p in enumerate(pats):
        if p["kind"] in ("block_topk", "block_threshold", "moba", "unified"):
            byt += N * d * 2
            kv_read.add(h // G)
        elif p["kind"] in ("vs", "vs_windows"):
            byt += min(p["last_q"], N) * d * 2 + 2 * 2 * 4 * N
            kv_read.add(h // G)
    byt += len(kv_read) * N * d * 2
    return byt, nqb


def reduce_max_over_ranks(values, device="cpu"):
    """Max over all ranks of each value (timings: the slowest rank sets the pace).
    Identity when torch.distributed is not initialised."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


# the sources the attention kernel is compiled from (its .cu and the headers it includes)
ATTN_SOURCES = ("dsa_attn.cu", "dsa_common.cuh", "dsa_internal.h")


def kernel_source_hash(paths):
    """16 hex digits of the SHA-256 of CUDA sources (in the given order) with their
    // comments and blank lines removed: profiler counters stay tied to the code,
    not its prose."""
    import hashlib
    if isinstance(paths, str):
        paths = [paths]
    lines = []
    for path in paths:
        lines.append("@" + os.path.basename(path))
        for ln in open(path, encoding="utf-8").read().splitlines():
            code = ln.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def whole_job_tokens_per_s(N, world, ms_per_step):
    """Every rank processes its own N-token layer per step (weak scaling)."""
    return N * world / (ms_per_step * 1e-3)


def build_workload(w, device, seed_offset=0):
    w = dict(w)
    w["seed"] = w["seed"] + seed_offset
    Q, K, V, planted = synth.make_inputs(w, device=device)
    pats = synth.head_patterns(w)
    convs = synth.conv_weights(w, device=device)
    if convs is not None:
        G = w["Hq"] // w["Hkv"]
        pats = [dict(p, conv=convs[h // G]) if p["kind"] == "moba" else p for h, p in enumerate(pats)]
    return Q, K, V, pats


def key_tiles_per_item(bufs, N, B):
    """64-key tiles the attention kernel runs per 128-row item, from the index
    lists, the kernel's own tiling: per item the union of its two 64-row halves'
    64-key units (of listed blocks, or touched by the slash runs of the half's
    query block), each unit only up to the half's last row, plus the gathered
    column tiles (a half that shares its query block with the other adds none of
    its own); averaged over items."""
    nqb = (N + B - 1) // B
    tiles = items = 0
    for hl in bufs.host_lists():
        for r0 in range(0, N, 128):
            units = set()
            t = 0
            seen = set()
            for hh in (0, 1):
                rs = r0 + 64 * hh
                if rs >= N:
                    continue
                qb, r1h = rs // B, min(N - 1, rs + 63)
                if hl["kind"] == 6:
                    lst = hl["dist"]
                    n, nl = int(lst[0]), int(lst[1])
                    last = qb == nqb - 1
                    iv = lst[2 + (2 * n if last else 0): 2 + 2 * n + (2 * nl if last else 0)].reshape(-1, 2)
                    r1 = min(N - 1, qb * B + B - 1)
                    for a, b in iv:
                        hi, lo = r1 - int(a), max(0, r1 - int(b))
                        if hi >= lo:
                            units.update(range(lo // 64, min(hi, r1h) // 64 + 1))
                else:
                    if hl["kind"] == 1:
                        blocks = [qb - int(dd) for dd in hl["dist"] if dd <= qb]
                    else:
                        blocks = [int(x) for x in hl["blocks"][qb]]
                    for kb in blocks:
                        for u in range(kb * B // 64, (kb * B + B) // 64):
                            if u * 64 <= r1h:
                                units.add(u)
                if qb in seen:
                    continue
                seen.add(qb)
                t += (len(hl["cols"][qb]) + 63) // 64
            tiles += t + len(units)
            items += 1
    return tiles / max(1, items)


def kernel_launches_per_step(pats):
    kinds = [p["kind"] for p in pats]
    n = 4  # head info, A-shape counts, scan, block fill
    if any(k in ("block_topk", "block_threshold", "moba") for k in kinds):
        n += 2  # pool, block score/select
    if "vs" in kinds:
        n += 9  # VS pass 1, row stats, pass 2, slash combine, top-k, distances, column count, distance fill, column fill
    return n + 1  # attention


# --------------------------------------------------------------------------- oracle timing
ORACLE_SAMPLE_ROWS = 512


def oracle_sample(w, Q, K, V, pats, rows_per_kind=ORACLE_SAMPLE_ROWS):
    """Times the CPU oracle on one fixed, bounded sample of the layer and
    extrapolates to the whole layer.  The sample: the full index build of one
    head of each pattern kind present, and the attention of `rows_per_kind`
    evenly spaced rows of those heads (a row's cost grows with its allowed keys,
    so the rows are spread over the sequence).  Layer estimate = index time x
    heads of that kind + attention time per row x N x heads of that kind.  The
    CPU-baseline leg and the reference arm both use this same sample.
    Returns (estimated layer seconds, description, threads, seconds spent)."""
    from oracle import dsa_oracle as orc
    N, B, G = w["N"], w["B"], w["Hq"] // w["Hkv"]
    q = Q.to("cpu", torch.float64).numpy()
    k = K.to("cpu", torch.float64).numpy()
    v = V.to("cpu", torch.float64).numpy()
    by_kind = {}
    for h, p in enumerate(pats):
        by_kind.setdefault(p["kind"], []).append(h)
    rows = np.unique(np.linspace(0, N - 1, min(N, rows_per_kind)).astype(np.int64))
    est = spent = 0.0
    for kind, hs in by_kind.items():
        h = hs[0]
        conv = None
        p = dict(pats[h])
        if "conv" in p:
            cw, cb = p.pop("conv")
            conv = (cw.double().cpu().numpy(), cb.double().cpu().numpy())
        t0 = time.perf_counter()
        hi = orc.build_head_index(q[h], k[h // G], p, B, conv)
        t1 = time.perf_counter()
        orc.attention_rows(q[h], k[h // G], v[h // G], hi, rows)
        t2 = time.perf_counter()
        est += (t1 - t0) * len(hs) + (t2 - t1) / rows.size * N * len(hs)
        spent += t2 - t0
    desc = (f"full index build of one head per pattern kind ({', '.join(sorted(by_kind))}) and attention of "
            f"{rows.size} evenly spaced rows of each; extrapolated to {w['Hq']} heads x {N} rows")
    threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return est, desc, threads, spent


def oracle_baseline(w, Q, K, V, pats, min_seconds=10.0):
    """The sample of oracle_sample repeated until at least `min_seconds` of CPU
    work are spent; the mean layer estimate."""
    ests, spent = [], 0.0
    while spent < min_seconds or not ests:
        est, desc, threads, s = oracle_sample(w, Q, K, V, pats)
        ests.append(est)
        spent += s
    return statistics.mean(ests), desc + f" ({len(ests)} repetitions, {spent:.1f} s of CPU work)", threads


# --------------------------------------------------------------------------- main
# what each workload's heads do (synth.head_patterns)
PATTERN_TEXT = {
    "vs": "all heads Vertical-Slash (last_q 64, n_vert/n_slash per workload)",
    "mixed": "seeded per head: 20% A-shape 128/1024, 60% VS 64/1000/6096, 20% block top-100",
    "threshold": "all heads block threshold, alpha 0.5 in probability space, sink and local block kept",
    "moba": "all heads MoBA top-8 over earlier blocks plus the diagonal block",
}


def build_arg_parser():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="dsa", choices=["dsa", "reference"])
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--e2e-chunks", type=int, default=8, help="KV-group chunks of the overlapped host path")
    ap.add_argument("--N", type=int, default=0, help="override the token count (smaller profiling cases)")
    ap.add_argument("--B", type=int, default=0, help="override the block size (the MoBA workload's B sweep)")
    ap.add_argument("--conv", type=int, default=-1, help="override the MoBA key-conv width (0 = off)")
    ap.add_argument("--slash-cover", default="blocks", choices=["blocks", "windows"],
                    help="VS heads: cover the slashes by aligned key blocks or by their exact key runs")
    ap.add_argument("--shard-heads", action="store_true",
                    help="strong scaling: the ranks split ONE layer by KV groups (default: one layer per rank)")
    ap.add_argument("--gather", action="store_true",
                    help="with --shard-heads: all-gather every rank's O into the full layer output each step")
    return ap


def main():
    args = build_arg_parser().parse_args()
    rank, world, local = dist_env()
    over = {}
    if args.N:
        over["N"] = args.N
    if args.B:
        over["B"] = args.B
    if args.conv >= 0:
        over["conv_width"] = args.conv
    w = synth.workload(args.workload, **over)

    if args.impl == "reference":
        # the oracle, as it stands, on the host cores; rank 0 only
        if rank != 0:
            return
        torch.manual_seed(0)
        Q, K, V, pats = build_workload(w, "cuda" if torch.cuda.is_available() else "cpu")
        for _ in range(args.warmup):
            oracle_sample(w, Q, K, V, pats)
        times, spent = [], 0.0
        desc = threads = None
        for _ in range(args.steps):
            est, desc, threads, s = oracle_sample(w, Q, K, V, pats)
            times.append(est)
            spent += s
        t = statistics.mean(times)
        val = w["N"] / t
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
                "ms_per_step_kind": (f"extrapolated: each step times the oracle on one fixed sample "
                                     f"({spent / max(1, args.steps):.2f} s of CPU work) and scales it to the layer"),
                "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": w["name"], "Hq": w["Hq"], "Hkv": w["Hkv"], "N": w["N"], "d": w["d"],
                           "block": w["B"]},
                "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                 "sample": desc + f" (one sample per step, {args.steps} steps)"},
                "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import dynamic_sparse_attention_build_b200 as dsa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=dev)
    if args.slash_cover == "windows":
        w = dict(w, name=w["name"] + "_slash_runs")
    if args.shard_heads:
        # every rank builds the same layer and keeps its KV groups (heads are independent)
        from dynamic_sparse_attention_build_b200 import shard
        Qf, Kf, Vf, pf = build_workload(w, dev)
        Q, K, V, pats = shard.shard_inputs(Qf, Kf, Vf, pf, rank, world)
        del Qf, Kf, Vf
    else:
        Q, K, V, pats = build_workload(w, dev, seed_offset=rank)
    N, Hq, d = w["N"], Q.shape[0], w["d"]
    if args.slash_cover == "windows":
        pats = [dict(p, kind="vs_windows") if p["kind"] == "vs" else p for p in pats]
    gather = args.shard_heads and args.gather and world > 1
    pats_c = dsa.make_patterns(pats)
    bufs = dsa.build_indices(Q, K, pats_c, w["B"])
    O = torch.empty_like(Q)
    O, _ = dsa.sparse_prefill(Q, K, V, bufs, O=O)
    torch.cuda.synchronize()
    st, det = dsa.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det}")
    pairs = dsa.count_pairs(Q, K, bufs).sum().item()
    tiles_item = key_tiles_per_item(bufs, N, w["B"]) if N <= 65536 else None
    f_sel = 4.0 * d * pairs
    causal_pairs = Hq * N * (N + 1) / 2
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        dsa.build_indices(Q, K, pats_c, w["B"], bufs=bufs)
        if ev is not None:
            ev[1].record(stream)
        dsa.sparse_prefill(Q, K, V, bufs, O=O)
        if gather:
            shard.gather_heads(O, w["Hq"], w["Hkv"])
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    for i in range(args.steps):
        flush.zero_()  # L2 flush between timed steps, outside the step's events
        step(evs[i])
    torch.cuda.synchronize()
    clocks = sampler.stop()
    t_build = [e[0].elapsed_time(e[1]) for e in evs]
    t_attn = [e[1].elapsed_time(e[2]) for e in evs]
    t_step = [a + b for a, b in zip(t_build, t_attn)]
    tot = reduce_max_over_ranks([sum(t_step), sum(t_build), sum(t_attn)], device=dev)
    ms_step = tot[0] / args.steps
    ms_build = tot[1] / args.steps
    ms_attn = tot[2] / args.steps
    st, det = dsa.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} detail {det}")

    # end to end through the public API with pinned host buffers: HostPrefill
    # uploads, computes and downloads KV-group chunks on three streams
    Qh = Q.cpu().pin_memory()
    Kh = K.cpu().pin_memory()
    Vh = V.cpu().pin_memory()
    Oh = torch.empty_like(Qh).pin_memory()
    hp = dsa.HostPrefill(Hq, K.shape[0], N, d, pats, w["B"], chunks=args.e2e_chunks, device=dev)

    def e2e_step():
        hp.run(Qh, Kh, Vh, Oh)

    e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max_over_ranks([e0.elapsed_time(e1) / args.e2e_steps], device=dev)[0]

    pk, pk_src = peaks()
    tflops = f_sel / (ms_attn * 1e-3) / 1e12
    # one fixed denominator for the fraction: the measured dense bf16 burst peak;
    # the fraction of the sustained (power-capped) peak is reported beside it
    peak_tf = pk["bf16_tflops"]
    peak_kind = "bf16 burst (cuBLAS)"
    peak_sus = pk.get("bf16_tflops_sustained")
    idx_bytes, nqb = algorithmic_index_bytes(w, pats)
    idx_gbs = idx_bytes / (ms_build * 1e-3) / 1e9
    traffic = None
    tp = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if os.path.exists(tp):
        # DRAM bytes per launch from an ncu capture of a smaller case of the same
        # workload, scaled by the token count (the kernel's DRAM traffic is Q read,
        # O written and K/V first touches, each proportional to N); only valid
        # for the kernel source it was taken on
        csrc = os.path.join(ROOT, "dynamic_sparse_attention_build_b200", "csrc")
        sha = kernel_source_hash([os.path.join(csrc, f) for f in ATTN_SOURCES])
        for rec in json.load(open(tp)).get("records", []):
            if (rec.get("workload") == w["name"] and rec.get("kernel_source_sha256_16") == sha
                    and rec.get("block") == w["B"]):
                traffic = int(round(rec["dram_bytes_per_launch_at_capture"] * w["N"] / rec["captured_N"]))
                break

    line = {
        "metric": METRIC, "value": (N / (ms_step * 1e-3) if args.shard_heads else whole_job_tokens_per_s(N, world, ms_step)),
        "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.shard_heads else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w["name"], "Hq": Hq, "Hkv": w["Hkv"], "N": N, "d": d, "block": w["B"],
                   "slash_cover": args.slash_cover,
                   "key_conv_width": int(w.get("conv_width", 0) or 0),
                   "patterns": PATTERN_TEXT.get(w["mix"], w["mix"]),
                   "l2": "flushed by a 256 MiB write before every timed step (outside its events)",
                   "parallelism": (f"one layer, heads sharded by KV group x{world}"
                                   + (", O all-gathered each step" if gather else "")
                                   if args.shard_heads else f"independent layer per rank x{world}")},
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": tflops / peak_tf, "traffic": traffic,
                     "kernel": "sparse_attn_kernel<128>", "peak_source": f"{pk_src} {peak_kind}",
                     "work": f"F_sel = 4*d*|M| = {f_sel:.4e} FLOP per launch ({pairs} allowed pairs)"},
        "attention": {"ms": ms_attn, "tflops": tflops, "frac_peak": tflops / peak_tf,
                      "frac_sustained_peak": (tflops / peak_sus) if peak_sus else None,
                      "key_tiles_per_item": tiles_item,
                      "density_vs_causal": pairs / causal_pairs},
        "index_build": {"ms": ms_build, "algorithmic_bytes": idx_bytes, "gbs": idx_gbs,
                        "frac_hbm": idx_gbs / pk["hbm_gbs"], "hbm_peak_source": pk_src},
        "e2e": {"value": (N / (e2e_ms * 1e-3) if args.shard_heads else whole_job_tokens_per_s(N, world, e2e_ms)),
                "unit": "tokens/s",
                "h2d_bytes_per_step": (Q.numel() + K.numel() + V.numel()) * 2,
                "d2h_bytes_per_step": O.numel() * 2, "ms_per_step": e2e_ms},
        "gpu_launches": kernel_launches_per_step(pats) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        est, desc, threads = oracle_baseline(w, Q, K, V, pats)
        line["cpu_baseline"] = {"value": N / est, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
