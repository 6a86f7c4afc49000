#!/usr/bin/env python3
"""Throughput of the hashed n-gram (PLE / Engram) lookup on B200.

One step = the whole hot path over synthetic packed tokens: for each part
  forward  ple_lookup   (segment/EOS context, order hashes, head rows, row
                         gather; the rows are saved for the backward)
  backward ple_grad_scatter (deterministic table gradient of the gather)
Default step (--workload headline), the two largest single-GPU workloads:
  large_table      forward: 65536 tokens (14 packed sequences, 1k-8k),
                   Zipf(1.1) ids over 151936, EOS 0.5 %, ngram_size 4, 8
                   heads per order (24 heads), 24 primes >= 8.4e6 (201.6 M
                   rows), head_dim 128 bf16 table (51.6 GB);
  backward_stress  forward + backward: 131072 tokens, Zipf(1.3) with
                   repeated 64-token spans, 16 heads, 16 primes >= 1e6,
                   head_dim 128, bf16 grad_out N(0,1) into an 8.2 GB fp32
                   table gradient.
--workload NAME runs one workload (forward + backward, or --fwd-only).

Prints ONE JSON line on rank 0 (everything else goes to stderr).
Multi-GPU: the lookup has no exchange step on one node (one GPU holds the
whole table), so N GPUs run N independent replicas (weak scaling); ranks
only meet for a barrier and the max-over-ranks of the device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "PLE lookup tokens/s and achieved HBM GB/s (fwd gather, bwd scatter) vs 8 TB/s"
UNIT = "tokens/s"
NOMINAL_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 512 << 20   # > 4x the 126 MB L2: written, then a second buffer read (L2 left cold and clean)


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def workload(name: str, seed: int):
    import synth

    if name in synth.WORKLOADS:
        return synth.WORKLOADS[name](seed)
    if name.startswith("sweep:"):
        kw = dict(kv.split("=") for kv in name[len("sweep:"):].split(",") if kv)
        conv = {"tokens": int, "head_dim": int, "ngram_size": int, "heads_per_ngram": int, "table_gb": float,
                "ids": str, "table_dtype": lambda v: {"f32": 0, "bf16": 1, "e4m3": 2}[v]}
        return synth.sweep_point(seed=seed, **{k: conv[k](v) for k, v in kw.items()})
    raise SystemExit(f"unknown workload {name}")


DTYPE_NAMES = {0: "f32", 1: "bf16", 2: "e4m3"}
ELEM_BYTES = {0: 4, 1: 2, 2: 1}
HOST_DTYPE = {0: np.float32, 1: np.uint16, 2: np.uint8}  # the generator's host representation


def describe(w):
    return {"workload": w.name, "tokens": w.num_tokens, "sequences": int(len(w.cu_seqlens) - 1),
            "ngram_size": w.ngram_size, "heads_per_ngram": w.heads_per_ngram, "heads": w.num_heads,
            "head_dim": w.head_dim, "table_rows": w.num_rows,
            "table_dtype": DTYPE_NAMES[w.table_dtype],
            "table_gb": round(w.table_bytes / 1e9, 3), "grad_dtype": "bf16" if w.grad_dtype == 1 else "f32"}


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9 or not parts[0].isdigit() or int(parts[0]) != self.gpu:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def traffic_from_profiles(key: str, source_files):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (sha256 prefix recorded beside the number)."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    h = hashlib.sha256()
    for f in source_files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    sha = h.hexdigest()[:16]
    for line in open(p):
        parts = line.split()
        if len(parts) >= 3 and not line.startswith("#") and parts[0] == key and parts[2] == sha:
            return float(parts[1])
    return None


def backward_split(p, flush_l2, stream, peak: float, reps: int = 10) -> dict:
    """The backward of part p as its two halves, ple_grad_prepare (clear, key
    histogram, sort passes) and ple_grad_apply (fold, long-run finish), timed
    apart with CUDA events after the timed steps (L2 flushed before each
    prepare).  The apply moves all of the backward's algorithmic bytes (the
    sorted keys and hit ids in place of the row ids), so its GB/s is the
    fold's own roofline figure; the prepare is the sort's overhead."""
    import torch

    N = p.T_out * p.w.num_heads
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(reps)]
    for r in range(reps + 2):  # two untimed
        flush_l2()
        e = ev[r - 2] if r >= 2 else None
        if e is not None:
            e[0].record(stream)
        p.ple.ple_grad_prepare(p.plan, p.rows.view(-1), p.ws)
        if e is not None:
            e[1].record(stream)
        p.ple.ple_grad_apply(p.plan, N, p.grad, p.table_grad, p.ws)
        if e is not None:
            e[2].record(stream)
    torch.cuda.synchronize()
    status = p.ple.ple_status(p.table_grad.device)
    if status != p.ple.PLE_OK:
        raise SystemExit(f"libple async status {status}")
    prep = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    app = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    gbs = p.bwd_bytes() / (app * 1e-3) / 1e9
    return {"prepare_ms": prep, "apply_ms": app, "apply_gb_per_s": gbs, "apply_frac_of_measured": gbs / peak,
            "apply_frac_of_8tbs": gbs / NOMINAL_HBM_GBS,
            "what": "ple_grad_prepare (sort) and ple_grad_apply (fold) timed apart, CUDA events, L2 flushed "
                    "before each prepare, outside the timed steps"}


def size_matched_copy_gbs(nbytes: int, flush_l2, stream, device, reps: int = 10) -> float:
    """GB/s of a plain device-to-device copy moving the same bytes (nbytes/2
    read, nbytes/2 written): the practical ceiling for a kernel of this size,
    beside the large-buffer copy peak."""
    import torch

    half = max(16, (nbytes // 2) // 16 * 16)
    src = torch.ones(half, dtype=torch.uint8, device=device)
    dst = torch.empty_like(src)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    for k in range(reps + 3):
        flush_l2()
        e0.record(stream)
        dst.copy_(src)
        e1.record(stream)
        torch.cuda.synchronize()
        if k >= 3:
            times.append(e0.elapsed_time(e1))
    del src, dst
    return 2 * half / (statistics.mean(times) * 1e-3) / 1e9


def reduce_max(values, dist, device):
    """Element-wise max over ranks (replica timings are taken as the slowest
    rank's); a no-op without a process group."""
    import torch

    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def replica_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch."""
    return base + rank


# The default step: the forward on the large-table workload (65536 tokens,
# 24 heads, D=128, 51.6 GB bf16 table) and the forward + backward on the
# backward-stress workload (131072 tokens, 16 heads, D=128, Zipf(1.3) with
# repeated spans, bf16 grad_out into an 8.2 GB fp32 table gradient): the two
# largest single-GPU configurations, one for each direction.
HEADLINE = (("large_table", False), ("backward_stress", True))


def step_parts(args):
    """(workload name, with backward) for every part of one step."""
    if args.workload == "headline":
        return list(HEADLINE)
    return [(args.workload, not args.fwd_only)]


def compact_table(w, rows, table_rows):
    """A host table holding only the rows a pass touches, and the rows
    renumbered into it (the oracle's gather is a copy per hit, so a compact
    table gives it the same work without a table-sized host array)."""
    uniq, inv = np.unique(rows, return_inverse=True)
    return table_rows(uniq), inv.reshape(rows.shape).astype(np.int64)


def cpu_oracle_pass(w, tok, cu, table_c, rows_c, grad_host, threads):
    """The oracle, as it stands: rows, gather (from the compact table) and,
    with grad_host, the gradient sums.  Returns the seconds taken."""
    import oracle

    t0 = time.perf_counter()
    rows = oracle.rows(tok, cu, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes, w.offsets,
                       threads=threads)
    if w.table_dtype == 2:
        oracle.gather_e4m3(rows_c, table_c)
    else:
        oracle.gather(rows_c, table_c, threads=threads)
    if grad_host is not None:
        oracle.grad_sums(rows, grad_host, threads=threads)
    return time.perf_counter() - t0


def sample_prefix(w, tokens_limit):
    """The first tokens_limit tokens (whole sequences cut at that point)."""
    cu = w.cu_seqlens.astype(np.int64)
    if tokens_limit is None or tokens_limit >= w.num_tokens:
        return w.tokens, w.cu_seqlens.astype(np.int32)
    T = tokens_limit
    return w.tokens[:T], np.asarray(cu[cu < T].tolist() + [T], np.int32)


def oracle_inputs(w, tok, cu, with_grad, table_rows=None):
    """Host inputs of one oracle pass over (tok, cu): compact table, rows
    renumbered into it, and the grad_out rows (bookkeeping, untimed)."""
    import oracle
    import synth

    rows = oracle.rows(tok, cu, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes, w.offsets)
    table_c, rows_c = compact_table(w, rows, table_rows or w.table_rows)
    grad = None
    if with_grad:
        grad = synth.dense_values(w.grad_seed, rows.size * w.head_dim, w.grad_sigma,
                                  w.grad_dtype).reshape(rows.size, w.head_dim)
    return table_c, rows_c, grad


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on bounded samples of the workload
    (the first --ref-tokens tokens of every part of the step)."""
    if rank != 0:
        return 0
    threads = os.cpu_count() or 1
    parts = []
    for name, bwd in step_parts(args):
        w = workload(name, args.seed)
        tok, cu = sample_prefix(w, args.ref_tokens)
        parts.append((w, tok, cu) + oracle_inputs(w, tok, cu, bwd))

    def one_step():
        return sum(cpu_oracle_pass(w, tok, cu, tc, rc, g, threads) for w, tok, cu, tc, rc, g in parts)

    for _ in range(args.warmup):
        one_step()
    times = [one_step() for _ in range(args.steps)]
    T = sum(len(p[1]) for p in parts)
    ms = 1e3 * sum(times) / len(times)
    value = T / (ms / 1e3)
    what = "; ".join(f"{p[0].name}: first {len(p[1])} of {p[0].num_tokens} tokens (rows, gather"
                     f"{', grad sums' if p[5] is not None else ''})" for p in parts)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64+f32", "data": "synthetic",
            "config": config_of([p[0] for p in parts], step_parts(args)),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": what + " per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_of(ws, parts):
    if len(ws) == 1:
        return describe(ws[0])
    return {"workload": " + ".join(f"{w.name} ({'fwd+bwd' if bwd else 'fwd'})" for w, (_, bwd) in zip(ws, parts)),
            "parts": [dict(describe(w), timed="ple_lookup + ple_grad_scatter" if bwd else "ple_lookup")
                      for w, (_, bwd) in zip(ws, parts)]}


class Part:
    """Device state of one workload of the step: table, tokens, outputs and,
    with a backward, grad_out, table_grad and the gradient workspace."""

    def __init__(self, name, do_bwd, seed, dev, sl=None):
        import torch

        import hashed_gram_embedding_ple_b200 as ple
        from synth import gpu as sgpu

        self.ple = ple
        self.w = w = workload(name, seed)
        self.do_bwd = do_bwd
        self.sl = sl
        self.plan = ple.Plan.from_workload(w)
        T, H, D = w.num_tokens, w.num_heads, w.head_dim
        tdt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float8_e4m3fn}[w.table_dtype]
        self.table = torch.empty(w.num_rows, D, dtype=tdt, device=dev)
        sgpu.fill_(self.table, w.table_seed, w.table_sigma)
        self.tokens = torch.from_numpy(w.tokens).to(dev)
        self.cu = torch.from_numpy(w.cu_seqlens).to(dev)
        self.T_out = T if sl is None else (T // sl[0]) * (sl[2] - sl[1])  # tokens looked up per step
        self.out = torch.empty(self.T_out, H, D, dtype=self.plan.out_dtype, device=dev)
        self.rows = torch.empty(self.T_out, H, dtype=torch.int64, device=dev)
        self.grad = self.table_grad = self.ws = None
        if do_bwd:
            gdt = torch.bfloat16 if w.grad_dtype == 1 else torch.float32
            self.grad = torch.empty(self.T_out * H, D, dtype=gdt, device=dev)
            sgpu.fill_(self.grad, w.grad_seed, w.grad_sigma)
            self.table_grad = torch.zeros(w.num_rows, D, dtype=torch.float32, device=dev)
            self.ws = ple.alloc_workspace(self.plan, self.T_out * H, dev)
        self.U = None

    def lookup(self, tok=None, cu=None):
        tok = self.tokens if tok is None else tok
        cu = self.cu if cu is None else cu
        sl, T, H, D = self.sl, self.w.num_tokens, self.w.num_heads, self.w.head_dim
        if sl is None:
            self.ple.ple_lookup(self.plan, tok, cu, self.table, out=self.out, rows_out=self.rows)
        else:
            self.ple.ple_lookup_slice(self.plan, tok, cu, sl[0], sl[1], sl[2], self.table,
                                      out=self.out.view(T // sl[0], sl[2] - sl[1], H, D),
                                      rows_out=self.rows.view(T // sl[0], sl[2] - sl[1], H))

    def backward(self, grad=None):
        self.ple.ple_grad_scatter(self.plan, self.rows.view(-1), self.grad if grad is None else grad, self.table_grad,
                                  workspace=self.ws)

    def launches(self):
        """Kernels per step: the lookup; the backward's clear, key_hist, one
        sort pass per 8-bit digit of the row ids, the fold and the long-run
        finish."""
        passes = max(1, (int(self.w.num_rows).bit_length() + 7) // 8)
        return 1 + (4 + passes if self.do_bwd else 0)

    def fwd_bytes(self):
        w = self.w
        N_out = self.T_out * w.num_heads
        return 8 * w.num_tokens + N_out * w.head_dim * (ELEM_BYTES[w.table_dtype] + self.out.element_size()) + 8 * N_out

    def bwd_bytes(self):
        w = self.w
        N = self.T_out * w.num_heads
        e_g = 2 if w.grad_dtype == 1 else 4
        return 8 * N + N * w.head_dim * e_g + 2 * self.U * w.head_dim * 4


LOOKUP_SRC = ["hashed_gram_embedding_ple_b200/csrc/lookup.cu", "hashed_gram_embedding_ple_b200/csrc/common.cuh"]
GRAD_SRC = ["hashed_gram_embedding_ple_b200/csrc/grad.cu", "hashed_gram_embedding_ple_b200/csrc/sort.cuh",
            "hashed_gram_embedding_ple_b200/csrc/common.cuh"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="headline",
                    help="'headline' (large_table fwd + backward_stress fwd+bwd), a workload name, or "
                         "sweep:key=value,...")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--fwd-only", action="store_true", help="time the lookup alone (single workload)")
    ap.add_argument("--slice", default=None, metavar="ROW_LEN:START:END",
                    help="time the global-slice lookup of [START, END) of every ROW_LEN-token row (fwd only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=32768)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--conv", action="store_true",
                    help="time the PLE layer's short convolution (forward + backward) instead of the lookup")
    ap.add_argument("--conv-channels", type=int, default=8192, help="channels of the --conv workload")
    ap.add_argument("--host-table", action="store_true",
                    help="keep the table in pinned host memory: time ple_prefetch, the cached lookup and gradient, "
                         "and the two-stream pipeline (single_layer_bf16 unless --workload names another)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.host_table and args.workload == "headline":
        args.workload = "single_layer_bf16"  # the host-table mode's own default (a 2 GB table, pinned)
    if args.workload == "headline" and (args.fwd_only or args.slice):
        raise SystemExit("--fwd-only and --slice need a single --workload")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch

    import hashed_gram_embedding_ple_b200 as ple

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.conv:
        return run_conv(args, rank, world, dev, dist)
    if args.host_table:
        return run_host_table(args, rank, world, dev, dist)
    sl = None
    if args.slice:
        row_len, s0, s1 = (int(x) for x in args.slice.split(":"))
        sl = (row_len, s0, s1)
        args.fwd_only = True
    spec = step_parts(args)
    parts = []
    for name, bwd in spec:
        p = Part(name, bwd, replica_seed(args.seed, rank), dev, sl)
        if sl is not None and (sl[0] < 1 or p.w.num_tokens % sl[0] or not (0 <= sl[1] < sl[2] <= sl[0])):
            raise SystemExit("--slice needs ROW_LEN dividing the tokens and 0 <= START < END <= ROW_LEN")
        w = p.w
        log(f"[rank {rank}] {w.name}{' (fwd+bwd)' if bwd else ' (fwd)'}: T={w.num_tokens} H={w.num_heads} "
            f"D={w.head_dim} rows={w.num_rows} table {w.table_bytes / 1e9:.2f} GB")
        parts.append(p)
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    def step(evs=None):
        k = 0
        if evs is not None:
            evs[k].record(stream)
        for p in parts:
            p.lookup()
            k += 1
            if evs is not None:
                evs[k].record(stream)
            if p.do_bwd:
                p.backward()
                k += 1
                if evs is not None:
                    evs[k].record(stream)

    # unique rows for the backward's algorithmic bytes (bookkeeping, untimed)
    step()
    torch.cuda.synchronize()
    for p in parts:
        p.U = int(torch.unique(p.rows).numel())
    status = ple.ple_status(dev)
    if status != ple.PLE_OK:
        raise SystemExit(f"libple async status {status}")

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    n_ev = 1 + sum(1 + p.do_bwd for p in parts)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2()                         # L2 flush between steps, outside the events
        step(ev[k])
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    status = ple.ple_status(dev)
    if status != ple.PLE_OK:
        raise SystemExit(f"libple async status {status}")

    # per part: mean forward and backward times over the steps, max over ranks
    means, k = [], 0
    for p in parts:
        f = statistics.mean(ev[s][k].elapsed_time(ev[s][k + 1]) for s in range(args.steps))
        k += 1
        b = None
        if p.do_bwd:
            b = statistics.mean(ev[s][k].elapsed_time(ev[s][k + 1]) for s in range(args.steps))
            k += 1
        means += [f, b if b is not None else 0.0]
    ms_step = statistics.mean(ev[s][0].elapsed_time(ev[s][n_ev - 1]) for s in range(args.steps))
    red = reduce_max(means + [ms_step], dist, dev)
    ms_step = red[-1]
    for i, p in enumerate(parts):
        p.ms_fwd = red[2 * i]
        p.ms_bwd = red[2 * i + 1] if p.do_bwd else None

    peak, peak_kind = measured_peaks()
    fwd_part = parts[0]
    bwd_part = next((p for p in parts if p.do_bwd), None)

    def part_line(p):
        fb = p.fwd_bytes()
        d = {"workload": p.w.name, "fwd": {"ms": p.ms_fwd, "tokens_per_s": world * p.T_out / (p.ms_fwd * 1e-3),
                                           "gb_per_s": fb / (p.ms_fwd * 1e-3) / 1e9,
                                           "frac_of_8tbs": fb / (p.ms_fwd * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                                           "frac_of_measured": fb / (p.ms_fwd * 1e-3) / 1e9 / peak,
                                           "algorithmic_bytes": fb}}
        if p.do_bwd:
            bb = p.bwd_bytes()
            d["bwd"] = {"ms": p.ms_bwd, "tokens_per_s": world * p.T_out / (p.ms_bwd * 1e-3),
                        "gb_per_s": bb / (p.ms_bwd * 1e-3) / 1e9,
                        "frac_of_8tbs": bb / (p.ms_bwd * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
                        "frac_of_measured": bb / (p.ms_bwd * 1e-3) / 1e9 / peak,
                        "algorithmic_bytes": bb, "unique_rows": p.U}
        return d

    fwd_bytes = fwd_part.fwd_bytes()
    fwd_gbs = fwd_bytes / (fwd_part.ms_fwd * 1e-3) / 1e9
    copy_gbs = size_matched_copy_gbs(fwd_bytes, flush_l2, stream, dev)
    fwd_roof = {"bound": "hbm", "achieved": fwd_gbs, "peak": peak, "unit": "GB/s", "frac": fwd_gbs / peak,
                "size_matched_copy": {"gb_per_s": copy_gbs, "frac": fwd_gbs / copy_gbs,
                                      "what": "torch device copy of the lookup's algorithmic bytes (half read, "
                                              "half written), L2 flushed, CUDA events, outside the timed steps"},
                "frac_of_8tbs": fwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": fwd_bytes,
                "workload": fwd_part.w.name,
                "traffic": traffic_from_profiles(f"lookup_{fwd_part.w.name}", LOOKUP_SRC), "kernel": "lookup_kernel",
                "peak_source": f"{peak_kind} hbm_gbs"}
    roofline = fwd_roof
    bwd_roof = None
    if bwd_part is not None:
        bwd_bytes = bwd_part.bwd_bytes()
        bwd_gbs = bwd_bytes / (bwd_part.ms_bwd * 1e-3) / 1e9
        bwd_roof = {"bound": "hbm", "achieved": bwd_gbs, "peak": peak, "unit": "GB/s", "frac": bwd_gbs / peak,
                    "frac_of_8tbs": bwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": bwd_bytes,
                    "workload": bwd_part.w.name,
                    "traffic": traffic_from_profiles(f"grad_scatter_{bwd_part.w.name}", GRAD_SRC),
                    "kernel": "ple_grad_scatter (sort + fold kernels)", "unique_rows": bwd_part.U,
                    "peak_source": f"{peak_kind} hbm_gbs",
                    "split": backward_split(bwd_part, flush_l2, stream, peak)}
        if bwd_part.ms_bwd > fwd_part.ms_fwd:
            roofline = bwd_roof

    tokens_per_step = sum(p.T_out for p in parts)
    value = world * tokens_per_step / (ms_step * 1e-3)

    # end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        for p in parts:
            p.h_tok = torch.from_numpy(p.w.tokens).pin_memory()
            p.h_cu = torch.from_numpy(p.w.cu_seqlens).pin_memory()
            p.h_out = torch.empty_like(p.out, device="cpu").pin_memory()
            p.h_grad = p.grad.cpu().pin_memory() if p.do_bwd else None
            p.d_tok, p.d_cu = torch.empty_like(p.tokens), torch.empty_like(p.cu)
            p.d_grad = torch.empty_like(p.grad) if p.do_bwd else None
            p.ev_fwd, p.ev_up = torch.cuda.Event(), torch.cuda.Event()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # the link is full duplex: grad_out goes up on one copy stream from the
        # step's start, each lookup output comes down on another as soon as
        # its lookup is done, while the compute stream runs the next call
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_start, ev_down = torch.cuda.Event(), torch.cuda.Event()
        times = []
        for k in range(args.e2e_steps + 2):
            flush_l2()
            e0.record(stream)
            ev_start.record(stream)
            up.wait_event(ev_start)
            with torch.cuda.stream(up):
                for p in parts:
                    if p.do_bwd:
                        p.d_grad.copy_(p.h_grad, non_blocking=True)
                        p.ev_up.record(up)
            for p in parts:
                p.d_tok.copy_(p.h_tok, non_blocking=True)
                p.d_cu.copy_(p.h_cu, non_blocking=True)
                p.lookup(p.d_tok, p.d_cu)
                p.ev_fwd.record(stream)
                down.wait_event(p.ev_fwd)
                with torch.cuda.stream(down):
                    p.h_out.copy_(p.out, non_blocking=True)
                if p.do_bwd:
                    stream.wait_event(p.ev_up)
                    p.backward(p.d_grad)
            ev_down.record(down)
            stream.wait_event(ev_down)
            e1.record(stream)
            torch.cuda.synchronize()
            if k >= 2:
                times.append(e0.elapsed_time(e1))
        (t_e2e_ms,) = reduce_max([statistics.mean(times)], dist, dev)
        h2d = sum(8 * p.w.num_tokens + 4 * len(p.w.cu_seqlens) + (p.grad.numel() * p.grad.element_size()
                                                                     if p.do_bwd else 0) for p in parts)
        d2h = sum(p.out.numel() * p.out.element_size() for p in parts)
        e2e = {"value": world * tokens_per_step / (t_e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": t_e2e_ms,
               "what": "per part: pinned H2D tokens+cu_seqlens, ple_lookup, D2H of the lookup output on a second "
                       "copy stream; H2D of grad_out on a third stream from the step's start, then "
                       "ple_grad_scatter (full-duplex link); all inside the CUDA events"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and sl is None:
        threads = os.cpu_count() or 1
        inputs = []
        for p in parts:
            raw = p.table.view(torch.uint8) if p.w.table_dtype == 2 else p.table

            def from_device(uniq, raw=raw):  # the device table's rows (exactly the generator's values)
                idx = torch.from_numpy(uniq).to(dev)
                return torch_to_np(raw.index_select(0, idx))

            tc, rc, _ = oracle_inputs(p.w, p.w.tokens, p.w.cu_seqlens, False, from_device)
            g = torch_to_np(p.grad) if p.do_bwd else None
            inputs.append((p.w, p.w.tokens, p.w.cu_seqlens, tc, rc, g))
        tot_t, tot_s, reps = 0, 0.0, 0
        while tot_s < args.cpu_seconds and reps < 500:
            for w, tok, cu, tc, rc, g in inputs:
                tot_s += cpu_oracle_pass(w, tok, cu, tc, rc, g, threads)
                tot_t += len(tok)
            reps += 1
        cpu = {"value": tot_t / tot_s, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{reps} full passes of the step's workloads ({tokens_per_step} tokens each): rows, gather "
                         f"(from a host table of the touched rows), gradient sums for the backward part; "
                         f"std::thread over sequences / hits / rows, {tot_s:.1f} s"}
        del inputs

    if rank == 0:
        single = len(parts) == 1
        w0 = parts[0].w
        step_desc = " + ".join(("ple_lookup (rows saved) + ple_grad_scatter" if p.do_bwd else "ple_lookup")
                               + ("" if single else f" on {p.w.name}") for p in parts)
        if sl is not None:
            step_desc = f"ple_lookup_slice rows of {sl[0]}, positions [{sl[1]}, {sl[2]})"
        fl = part_line(fwd_part)["fwd"]
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None,
                "dtype": ("int64 hash, e4m3->bf16 widening copy, f32 grad" if w0.table_dtype == 2 else
                          f"int64 hash, {DTYPE_NAMES[w0.table_dtype]} copy, f32 grad"), "data": "synthetic",
                "config": dict(config_of([p.w for p in parts], spec), parallelism=f"replicas{world}",
                               l2="flushed between steps (512 MB written, then another 512 MB read); flush outside "
                                  "the step events",
                               step=step_desc),
                "fwd": dict(fl, workload=fwd_part.w.name),
                "bwd": None if bwd_part is None else dict(part_line(bwd_part)["bwd"], workload=bwd_part.w.name),
                "parts": [part_line(p) for p in parts],
                "roofline": roofline, "roofline_fwd": fwd_roof, "roofline_bwd": bwd_roof,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": sum(p.launches() for p in parts) * args.steps,
                "clocks": clocks, "wall_s_timed_region": wall}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_conv(args, rank, world, dev, dist):
    """--conv: the PLE layer's short convolution (segment-aware, causal,
    dilation = ngram_size, K = 4) over the single-layer packing with
    --conv-channels bf16 channels: one step = ple_conv_forward +
    ple_conv_backward (dx, dweight, dbias)."""
    import torch

    import hashed_gram_embedding_ple_b200 as ple
    import synth
    from synth import gpu as sgpu

    base = synth.single_layer_bf16(replica_seed(args.seed, rank))
    cu_np = base.cu_seqlens
    T, C, K, dil = int(cu_np[-1]), int(args.conv_channels), 4, base.ngram_size
    seed = 1000 + replica_seed(args.seed, rank)
    x = torch.empty(T, C, dtype=torch.bfloat16, device=dev)
    g = torch.empty(T, C, dtype=torch.bfloat16, device=dev)
    sgpu.fill_(x, seed, 1.0)
    sgpu.fill_(g, seed + 1, 1.0)
    gen = torch.Generator().manual_seed(seed)
    wt = (torch.randn(C, K, generator=gen) * 0.5).to(dev)
    bt = torch.randn(C, generator=gen).to(dev)
    cu = torch.from_numpy(cu_np).to(dev)
    y, dx = torch.empty_like(x), torch.empty_like(x)
    dw, db = torch.zeros(C, K, device=dev), torch.zeros(C, device=dev)
    ws = torch.empty(ple.conv_workspace_bytes(T, C, K), dtype=torch.uint8, device=dev)
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    def fwd(xin):
        ple.conv_forward(xin, cu, wt, dil, bt, out=y)

    def bwd(gin, xin):
        ple.conv_backward(gin, xin, cu, wt, dil, dx=dx, dweight=dw, dbias=db, workspace=ws)

    for _ in range(args.warmup):
        flush_l2()
        fwd(x)
        bwd(g, x)
    torch.cuda.synchronize()
    if ple.ple_status(dev) != ple.PLE_OK:
        raise SystemExit("libple async status after warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2()
        ev[k][0].record(stream)
        fwd(x)
        ev[k][1].record(stream)
        bwd(g, x)
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    if ple.ple_status(dev) != ple.PLE_OK:
        raise SystemExit("libple async status after the timed steps")
    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(args.steps)]
    bwd_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(args.steps)]
    ms_step, ms_fwd, ms_bwd = reduce_max([statistics.mean(a + b for a, b in zip(fwd_ms, bwd_ms)),
                                          statistics.mean(fwd_ms), statistics.mean(bwd_ms)], dist, dev)
    peak, peak_kind = measured_peaks()
    e = 2
    nchunks = max(1, -(-ws.numel() // (C * (K + 1) * 4)))
    fwd_bytes = 2 * T * C * e                                     # x read, y written
    bwd_bytes = 3 * T * C * e + 2 * nchunks * C * (K + 1) * 4    # dy and x read, dx written; partial sums
    fwd_gbs = fwd_bytes / (ms_fwd * 1e-3) / 1e9
    bwd_gbs = bwd_bytes / (ms_bwd * 1e-3) / 1e9
    src = ["hashed_gram_embedding_ple_b200/csrc/conv.cu", "hashed_gram_embedding_ple_b200/csrc/common.cuh"]
    roof_f = {"bound": "hbm", "achieved": fwd_gbs, "peak": peak, "unit": "GB/s", "frac": fwd_gbs / peak,
              "frac_of_8tbs": fwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": fwd_bytes,
              "traffic": traffic_from_profiles("conv_forward_conv_single_layer", src), "kernel": "conv_forward_kernel",
              "peak_source": f"{peak_kind} hbm_gbs"}
    roof_b = {"bound": "hbm", "achieved": bwd_gbs, "peak": peak, "unit": "GB/s", "frac": bwd_gbs / peak,
              "frac_of_8tbs": bwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": bwd_bytes,
              "traffic": traffic_from_profiles("conv_backward_conv_single_layer", src),
              "kernel": "conv_backward_kernel + conv_reduce_kernel", "peak_source": f"{peak_kind} hbm_gbs"}
    roofline = roof_b if ms_bwd > ms_fwd else roof_f

    e2e = None
    if args.e2e_steps > 0:
        hx, hg = x.cpu().pin_memory(), g.cpu().pin_memory()
        hy, hdx = torch.empty_like(hx).pin_memory(), torch.empty_like(hx).pin_memory()
        dxin, dgin = torch.empty_like(x), torch.empty_like(g)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # x goes up first; dy follows on a copy stream while the forward runs,
        # y comes down on another while dy goes up (full-duplex link), then dx
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_x, ev_y, ev_g, ev_dx, ev_down = (torch.cuda.Event() for _ in range(5))
        times = []
        for k in range(args.e2e_steps + 1):
            flush_l2()
            e0.record(stream)
            dxin.copy_(hx, non_blocking=True)
            ev_x.record(stream)
            up.wait_event(ev_x)
            with torch.cuda.stream(up):
                dgin.copy_(hg, non_blocking=True)
                ev_g.record(up)
            fwd(dxin)
            ev_y.record(stream)
            down.wait_event(ev_y)
            with torch.cuda.stream(down):
                hy.copy_(y, non_blocking=True)
            stream.wait_event(ev_g)
            bwd(dgin, dxin)
            ev_dx.record(stream)
            down.wait_event(ev_dx)
            with torch.cuda.stream(down):
                hdx.copy_(dx, non_blocking=True)
                ev_down.record(down)
            stream.wait_event(ev_down)
            e1.record(stream)
            torch.cuda.synchronize()
            if k >= 1:
                times.append(e0.elapsed_time(e1))
        (t_e2e,) = reduce_max([statistics.mean(times)], dist, dev)
        e2e = {"value": world * T / (t_e2e * 1e-3), "unit": UNIT, "h2d_bytes_per_step": 2 * T * C * e,
               "d2h_bytes_per_step": 2 * T * C * e, "ms_per_step": t_e2e,
               "what": "pinned H2D of x, ple_conv_forward, D2H of y; H2D of dy on a copy stream after x, "
                       "ple_conv_backward, D2H of dx; D2H on a third stream (full-duplex link); all inside the "
                       "CUDA events"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        sample = min(T, 1024)
        cu_s = np.asarray([c for c in cu_np if c < sample] + [sample], np.int32)
        xs = torch_to_np(x[:sample]).view(np.uint16)
        gs = torch_to_np(g[:sample]).view(np.uint16)
        xf = synth.bf16_bits_to_f32(xs).astype(np.float64)
        gf = synth.bf16_bits_to_f32(gs).astype(np.float64)
        wn, bn = wt.cpu().numpy().astype(np.float64), bt.cpu().numpy().astype(np.float64)
        tot_t, tot_s, reps = 0, 0.0, 0
        while tot_s < args.cpu_seconds and reps < 500:
            t0 = time.perf_counter()
            oracle.conv_forward(xf, cu_s, wn, dil, bn)
            oracle.conv_backward(gf, xf, cu_s, wn, dil)
            tot_s += time.perf_counter() - t0
            tot_t += sample
            reps += 1
        cpu = {"value": tot_t / tot_s, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{reps} passes over the first {sample} tokens x {C} channels (forward + backward, fp64 "
                         f"scalar loops, one thread), {tot_s:.1f} s"}

    if rank == 0:
        line = {"metric": "PLE short conv tokens/s and achieved HBM GB/s (fwd, bwd) vs 8 TB/s", "value":
                world * T / (ms_step * 1e-3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16 activations, f32 weights and accumulation", "data": "synthetic",
                "config": {"workload": "conv_single_layer", "tokens": T, "sequences": int(len(cu_np) - 1),
                           "channels": C, "kernel_size": K, "dilation": dil, "parallelism": f"replicas{world}",
                           "l2": "flushed between steps (512 MB written, then another 512 MB read); outside the events",
                           "step": "ple_conv_forward + ple_conv_backward (dx, dweight, dbias)"},
                "fwd": {"ms": ms_fwd, "gb_per_s": fwd_gbs, "frac_of_8tbs": fwd_gbs / NOMINAL_HBM_GBS,
                        "frac_of_measured": fwd_gbs / peak},
                "bwd": {"ms": ms_bwd, "gb_per_s": bwd_gbs, "frac_of_8tbs": bwd_gbs / NOMINAL_HBM_GBS,
                        "frac_of_measured": bwd_gbs / peak},
                "roofline": roofline, "roofline_fwd": roof_f, "roofline_bwd": roof_b, "cpu_baseline": cpu,
                "e2e": e2e, "gpu_launches": 3 * args.steps, "clocks": clocks, "wall_s_timed_region": wall}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_host_table(args, rank, world, dev, dist):
    """--host-table: the workload's table in pinned host memory.  Times, with
    CUDA events: ple_prefetch (the distinct rows over the host link), the
    cached lookup, the cached gradient, and a two-stream pipeline in which the
    prefetch of batch k+1 runs beside the lookup + gradient of batch k (two
    buffer sets, events between the streams).  The link's own peak is a
    pinned host-to-device copy of 256 MB measured in the same run."""
    import torch

    import hashed_gram_embedding_ple_b200 as ple
    from synth import gpu as sgpu

    w = workload(args.workload, replica_seed(args.seed, rank))
    plan = ple.Plan.from_workload(w)
    T, H, D, N = w.num_tokens, w.num_heads, w.head_dim, w.num_hits
    tdt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float8_e4m3fn}[w.table_dtype]
    dtab = torch.empty(w.num_rows, D, dtype=tdt, device=dev)
    sgpu.fill_(dtab, w.table_seed, w.table_sigma)
    table = torch.empty(w.num_rows, D, dtype=tdt, pin_memory=True)
    table.copy_(dtab)
    del dtab
    tokens = torch.from_numpy(w.tokens).to(dev)
    cu = torch.from_numpy(w.cu_seqlens).to(dev)
    grad = torch.empty(N, D, dtype=torch.bfloat16 if w.grad_dtype == 1 else torch.float32, device=dev)
    sgpu.fill_(grad, w.grad_seed, w.grad_sigma)
    bufs = [ple.Prefetched(plan, T, dev) for _ in range(2)]
    outs = [torch.empty(T, H, D, dtype=plan.out_dtype, device=dev) for _ in range(2)]
    cgrads = [torch.zeros(b.cache_rows, D, dtype=torch.float32, device=dev) for b in bufs]
    ws = ple.alloc_workspace(plan, N, dev)
    main = torch.cuda.current_stream(dev)
    side = torch.cuda.Stream(dev)
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    def compute(i):
        ple.ple_gather_cache(plan, bufs[i], out=outs[i])
        ple.ple_grad_scatter_cache(plan, bufs[i], grad, cache_grad=cgrads[i], workspace=ws)

    # link peak: pinned host -> device copy
    h = torch.empty(256 << 20, dtype=torch.uint8, pin_memory=True)
    d = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        d.copy_(h, non_blocking=True)
    e0.record(main)
    for _ in range(4):
        d.copy_(h, non_blocking=True)
    e1.record(main)
    torch.cuda.synchronize()
    link_gbs = 4 * h.numel() / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del h, d

    for _ in range(args.warmup):
        flush_l2()
        ple.ple_prefetch(plan, tokens, cu, table, bufs[0])
        compute(0)
    torch.cuda.synchronize()
    if ple.ple_status(dev) != ple.PLE_OK:
        raise SystemExit("libple async status after warm-up")
    U = int(bufs[0].num_unique.item())
    # each part alone
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for k in range(args.steps):
        flush_l2()
        ev[k][0].record(main)
        ple.ple_prefetch(plan, tokens, cu, table, bufs[0])
        ev[k][1].record(main)
        ple.ple_gather_cache(plan, bufs[0], out=outs[0])
        ev[k][2].record(main)
        ple.ple_grad_scatter_cache(plan, bufs[0], grad, cache_grad=cgrads[0], workspace=ws)
        ev[k][3].record(main)
    torch.cuda.synchronize()
    ms_pf = statistics.mean(ev[k][0].elapsed_time(ev[k][1]) for k in range(args.steps))
    ms_lk = statistics.mean(ev[k][1].elapsed_time(ev[k][2]) for k in range(args.steps))
    ms_bw = statistics.mean(ev[k][2].elapsed_time(ev[k][3]) for k in range(args.steps))
    # pipeline: prefetch of batch k+1 on the side stream beside batch k's compute
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    with torch.cuda.stream(side):
        ple.ple_prefetch(plan, tokens, cu, table, bufs[0])
        ready[0].record(side)
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else int(os.environ.get("LOCAL_RANK", "0")))
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    wall0 = time.perf_counter()
    p0.record(main)
    for k in range(args.steps):
        i, j = k % 2, (k + 1) % 2
        with torch.cuda.stream(side):  # the next batch (the same tokens, a new prefetch)
            if k > 0:
                side.wait_event(free[j])
            ple.ple_prefetch(plan, tokens, cu, table, bufs[j])
            ready[j].record(side)
        main.wait_event(ready[i])
        compute(i)
        free[i].record(main)
    p1.record(main)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    if ple.ple_status(dev) != ple.PLE_OK:
        raise SystemExit("libple async status after the pipeline")
    (ms_pipe,) = reduce_max([p0.elapsed_time(p1) / args.steps], dist, dev)
    ms_pf, ms_lk, ms_bw = reduce_max([ms_pf, ms_lk, ms_bw], dist, dev)
    pf_bytes = U * plan.table_dtype.itemsize * D  # the distinct rows over the link
    e_o = outs[0].element_size()
    lk_bytes = N * (8 + plan.table_dtype.itemsize * D + e_o * D)
    pf_gbs = pf_bytes / (ms_pf * 1e-3) / 1e9
    roof = {"bound": "pcie", "achieved": pf_gbs, "peak": link_gbs, "unit": "GB/s", "frac": pf_gbs / link_gbs,
            "algorithmic_bytes": pf_bytes, "traffic": None, "kernel": "ple_prefetch (finalize_kernel row copies)",
            "peak_source": "measured in this run: pinned host-to-device copy of 256 MB"}
    if rank == 0:
        line = {"metric": "PLE lookup tokens/s with the table in pinned host memory (prefetch pipelined)",
                "value": world * T / (ms_pipe * 1e-3), "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_pipe, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": f"int64 hash, {DTYPE_NAMES[w.table_dtype]} rows over the host link",
                "data": "synthetic",
                "config": dict(describe(w), parallelism=f"replicas{world}", table_location="pinned host memory",
                               unique_rows=U,
                               step="ple_prefetch of the next batch (side stream) beside ple_gather_cache + "
                                    "ple_grad_scatter_cache of the current one"),
                "parts_ms": {"prefetch": ms_pf, "gather_cache": ms_lk, "grad_scatter_cache": ms_bw},
                "prefetch_gb_per_s": pf_gbs, "link_peak_gb_per_s": link_gbs,
                "gather_cache_gb_per_s": lk_bytes / (ms_lk * 1e-3) / 1e9,
                "roofline": roof, "cpu_baseline": None, "e2e": None,
                "gpu_launches": None, "clocks": clocks, "wall_s_timed_region": wall}
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def torch_to_np(t):
    import torch

    c = t.detach().cpu()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16)
    return c.numpy()


if __name__ == "__main__":
    sys.exit(main())
