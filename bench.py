#!/usr/bin/env python3
"""Throughput of the hashed n-gram (PLE / Engram) lookup on B200.

One step = the whole hot path over one batch of synthetic packed tokens:
  forward  ple_lookup   (segment/EOS context, order hashes, head rows, row
                         gather; the rows are saved for the backward)
  backward ple_grad_scatter (deterministic table gradient of the gather)
Default workload: 8 packed sequences totalling 32768 tokens (lengths 1k-8k),
Zipf(1.1) ids over a 151936-id vocabulary, EOS 0.5 %, ngram_size 3, 8 heads
per order (16 heads), 16 consecutive primes >= 1e6 (16.0M rows), head_dim 64
bf16 table (2.05 GB); bf16 grad_out N(0,1) into an fp32 table gradient.

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


def cpu_oracle_step(w, table_host, grad_host, threads, tokens_limit=None):
    """The oracle, as it stands, on the first `tokens_limit` tokens (whole
    sequences cut at that point): rows, gather, gradient sums."""
    import oracle

    cu = w.cu_seqlens.astype(np.int64)
    if tokens_limit is not None and tokens_limit < w.num_tokens:
        T = tokens_limit
        cut = cu[cu < T].tolist() + [T]
        cu = np.asarray(cut, np.int64)
    else:
        T = w.num_tokens
    tok = w.tokens[:T]
    t0 = time.perf_counter()
    rows = oracle.rows(tok, cu.astype(np.int32), w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                       w.offsets, threads=threads)
    if w.table_dtype == 2:
        oracle.gather_e4m3(rows, table_host)
    else:
        oracle.gather(rows, table_host, threads=threads)
    oracle.grad_sums(rows, grad_host[: rows.size], threads=threads)
    return T, time.perf_counter() - t0


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle on bounded samples of the workload."""
    if rank != 0:
        return 0
    import synth

    w = workload(args.workload, args.seed)
    threads = os.cpu_count() or 1
    sample = min(w.num_tokens, args.ref_tokens)
    # host copies of the inputs the sample touches (table rows regenerated on the host)
    import oracle

    rows_s = oracle.rows(w.tokens[:sample], np.asarray([0] + [c for c in w.cu_seqlens[1:] if c < sample] + [sample],
                                                         np.int32), w.ngram_size, w.heads_per_ngram, w.eos_id,
                         w.mults, w.primes, w.offsets)
    # a full-size host table whose touched rows hold the generated values
    # (np.zeros pages stay unbacked until written, so untouched rows cost no RAM)
    table_host = np.zeros((w.num_rows, w.head_dim), HOST_DTYPE[w.table_dtype])
    uniq = np.unique(rows_s)
    table_host[uniq] = w.table_rows(uniq)
    grad_host = synth.dense_values(w.grad_seed, rows_s.size * w.head_dim, w.grad_sigma,
                                   w.grad_dtype).reshape(rows_s.size, w.head_dim)
    for _ in range(args.warmup):
        cpu_oracle_step(w, table_host, grad_host, threads, sample)
    times = []
    for _ in range(args.steps):
        T, dt = cpu_oracle_step(w, table_host, grad_host, threads, sample)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = T / (ms / 1e3)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int64+f32", "data": "synthetic",
            "config": describe(w),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"first {T} of {w.num_tokens} tokens per step (rows, gather, grad sums)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="single_layer_bf16")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--fwd-only", action="store_true", help="time the lookup alone (workloads marked fwd only)")
    ap.add_argument("--slice", default=None, metavar="ROW_LEN:START:END",
                    help="time the global-slice lookup of [START, END) of every ROW_LEN-token row (fwd only)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-tokens", type=int, default=8192)
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--conv", action="store_true",
                    help="time the PLE layer's short convolution (forward + backward) instead of the lookup")
    ap.add_argument("--conv-channels", type=int, default=8192, help="channels of the --conv workload")
    ap.add_argument("--host-table", action="store_true",
                    help="keep the table in pinned host memory: time ple_prefetch, the cached lookup and gradient, "
                         "and the two-stream pipeline")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch

    import hashed_gram_embedding_ple_b200 as ple
    import synth
    from synth import gpu as sgpu

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
    w = workload(args.workload, replica_seed(args.seed, rank))
    plan = ple.Plan.from_workload(w)
    T, H, D, N = w.num_tokens, w.num_heads, w.head_dim, w.num_hits
    sl = None
    if args.slice:
        row_len, s0, s1 = (int(x) for x in args.slice.split(":"))
        if row_len < 1 or T % row_len or not (0 <= s0 < s1 <= row_len):
            raise SystemExit("--slice needs ROW_LEN dividing the tokens and 0 <= START < END <= ROW_LEN")
        sl = (row_len, s0, s1)
        args.fwd_only = True
    tdt = {0: torch.float32, 1: torch.bfloat16, 2: torch.float8_e4m3fn}[w.table_dtype]
    odt = plan.out_dtype  # bf16 for an fp8 table
    gdt = torch.bfloat16 if w.grad_dtype == 1 else torch.float32
    log(f"[rank {rank}] workload {w.name}: T={T} H={H} D={D} rows={w.num_rows} table {w.table_bytes / 1e9:.2f} GB")

    table = torch.empty(w.num_rows, D, dtype=tdt, device=dev)
    sgpu.fill_(table, w.table_seed, w.table_sigma)
    tokens = torch.from_numpy(w.tokens).to(dev)
    cu = torch.from_numpy(w.cu_seqlens).to(dev)
    T_out = T if sl is None else (T // sl[0]) * (sl[2] - sl[1])  # tokens looked up per step
    out = torch.empty(T_out, H, D, dtype=odt, device=dev)
    rows = torch.empty(T_out, H, dtype=torch.int64, device=dev)

    def lookup(tok_in, cu_in):
        if sl is None:
            ple.ple_lookup(plan, tok_in, cu_in, table, out=out, rows_out=rows)
        else:
            ple.ple_lookup_slice(plan, tok_in, cu_in, sl[0], sl[1], sl[2], table,
                                 out=out.view(T // sl[0], sl[2] - sl[1], H, D),
                                 rows_out=rows.view(T // sl[0], sl[2] - sl[1], H))
    do_bwd = not args.fwd_only
    if do_bwd:
        grad = torch.empty(N, D, dtype=gdt, device=dev)
        sgpu.fill_(grad, w.grad_seed, w.grad_sigma)
        table_grad = torch.zeros(w.num_rows, D, dtype=torch.float32, device=dev)
        ws = ple.alloc_workspace(plan, N, dev)
    flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum()

    def step():
        lookup(tokens, cu)
        if do_bwd:
            ple.ple_grad_scatter(plan, rows.view(-1), grad, table_grad, workspace=ws)

    # unique rows for the backward's algorithmic bytes (bookkeeping, untimed)
    step()
    torch.cuda.synchronize()
    U = int(torch.unique(rows).numel())
    status = ple.ple_status(dev)
    if status != ple.PLE_OK:
        raise SystemExit(f"libple async status {status}")

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    sampler = ClockSampler(dev.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local_rank)
    sampler.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for k in range(args.steps):
        flush_l2()                         # L2 flush between steps, outside the events
        ev[k][0].record(stream)
        lookup(tokens, cu)
        ev[k][1].record(stream)
        if do_bwd:
            ple.ple_grad_scatter(plan, rows.view(-1), grad, table_grad, workspace=ws)
        ev[k][2].record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    status = ple.ple_status(dev)
    if status != ple.PLE_OK:
        raise SystemExit(f"libple async status {status}")

    fwd_ms = [ev[k][0].elapsed_time(ev[k][1]) for k in range(args.steps)]
    bwd_ms = [ev[k][1].elapsed_time(ev[k][2]) for k in range(args.steps)]
    step_ms = [a + b for a, b in zip(fwd_ms, bwd_ms)] if do_bwd else list(fwd_ms)
    ms_step, ms_fwd, ms_bwd = reduce_max([statistics.mean(step_ms), statistics.mean(fwd_ms),
                                          statistics.mean(bwd_ms)], dist, dev)

    peak, peak_kind = measured_peaks()
    e_t = ELEM_BYTES[w.table_dtype]
    e_o = out.element_size()
    e_g = 2 if w.grad_dtype == 1 else 4
    N_out = T_out * H
    fwd_bytes = 8 * T + N_out * D * (e_t + e_o) + 8 * N_out
    bwd_bytes = 8 * N + N * D * e_g + 2 * U * D * 4
    fwd_gbs = fwd_bytes / (ms_fwd * 1e-3) / 1e9
    bwd_gbs = bwd_bytes / (ms_bwd * 1e-3) / 1e9 if do_bwd else None

    # roofline of the dominant call of the step
    lookup_src = ["hashed_gram_embedding_ple_b200/csrc/lookup.cu", "hashed_gram_embedding_ple_b200/csrc/common.cuh"]
    grad_src = ["hashed_gram_embedding_ple_b200/csrc/grad.cu", "hashed_gram_embedding_ple_b200/csrc/sort.cuh",
                "hashed_gram_embedding_ple_b200/csrc/common.cuh"]
    copy_gbs = size_matched_copy_gbs(fwd_bytes, flush_l2, stream, dev)
    fwd_roof = {"bound": "hbm", "achieved": fwd_gbs, "peak": peak, "unit": "GB/s", "frac": fwd_gbs / peak,
                "size_matched_copy": {"gb_per_s": copy_gbs, "frac": fwd_gbs / copy_gbs,
                                      "what": "torch device copy of the lookup's algorithmic bytes (half read, "
                                              "half written), L2 flushed, CUDA events, outside the timed steps"},
                "frac_of_8tbs": fwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": fwd_bytes,
                "traffic": traffic_from_profiles(f"lookup_{w.name}", lookup_src), "kernel": "lookup_kernel",
                "peak_source": f"{peak_kind} hbm_gbs"}
    roofline = fwd_roof
    bwd_roof = None
    if do_bwd:
        bwd_roof = {"bound": "hbm", "achieved": bwd_gbs, "peak": peak, "unit": "GB/s", "frac": bwd_gbs / peak,
                    "frac_of_8tbs": bwd_gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": bwd_bytes,
                    "traffic": traffic_from_profiles(f"grad_scatter_{w.name}", grad_src),
                    "kernel": "ple_grad_scatter (sort + fold kernels)", "unique_rows": U,
                    "peak_source": f"{peak_kind} hbm_gbs"}
        if ms_bwd > ms_fwd:
            roofline = bwd_roof

    # lookup_kernel; the backward: clear, key_hist, one sort_pass per 8-bit digit of the row ids, the fold
    sort_passes = max(1, (int(w.num_rows).bit_length() + 7) // 8)
    launches_per_step = 1 + (3 + sort_passes if do_bwd else 0)
    value = world * T_out / (ms_step * 1e-3)

    # end to end through the public API with host buffers
    e2e = None
    if args.e2e_steps > 0:
        h_tok = torch.from_numpy(w.tokens).pin_memory()
        h_cu = torch.from_numpy(w.cu_seqlens).pin_memory()
        h_out = torch.empty(T_out, H, D, dtype=odt).pin_memory()
        h_grad = grad.cpu().pin_memory() if do_bwd else None
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        d_tok, d_cu = torch.empty_like(tokens), torch.empty_like(cu)
        d_grad = torch.empty_like(grad) if do_bwd else None
        # the link is full duplex: grad_out goes up on one copy stream from the
        # step's start, the lookup output comes down on another as soon as the
        # lookup is done, while the backward runs on the compute stream
        up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_start, ev_fwd, ev_up, ev_down = (torch.cuda.Event() for _ in range(4))
        times = []
        for k in range(args.e2e_steps + 2):
            flush_l2()
            e0.record(stream)
            ev_start.record(stream)
            if do_bwd:
                up.wait_event(ev_start)
                with torch.cuda.stream(up):
                    d_grad.copy_(h_grad, non_blocking=True)
                    ev_up.record(up)
            d_tok.copy_(h_tok, non_blocking=True)
            d_cu.copy_(h_cu, non_blocking=True)
            lookup(d_tok, d_cu)
            ev_fwd.record(stream)
            down.wait_event(ev_fwd)
            with torch.cuda.stream(down):
                h_out.copy_(out, non_blocking=True)
                ev_down.record(down)
            if do_bwd:
                stream.wait_event(ev_up)
                ple.ple_grad_scatter(plan, rows.view(-1), d_grad, table_grad, workspace=ws)
            stream.wait_event(ev_down)
            e1.record(stream)
            torch.cuda.synchronize()
            if k >= 2:
                times.append(e0.elapsed_time(e1))
        (t_e2e_ms,) = reduce_max([statistics.mean(times)], dist, dev)
        h2d = 8 * T + 4 * (len(w.cu_seqlens)) + (N * D * e_g if do_bwd else 0)
        e2e = {"value": world * T / (t_e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": N_out * D * e_o, "ms_per_step": t_e2e_ms,
               "what": "pinned H2D tokens+cu_seqlens, ple_lookup, D2H of the lookup output; H2D of grad_out on a "
                       "second copy stream from the step's start, then ple_grad_scatter; the D2H on a third stream "
                       "beside it (full-duplex link); all inside the CUDA events"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and sl is None:
        threads = os.cpu_count() or 1
        uniq_rows = torch.unique(rows)
        table_host = np.zeros((w.num_rows, D), HOST_DTYPE[w.table_dtype])
        raw = table.view(torch.uint8) if w.table_dtype == 2 else table
        table_host[uniq_rows.cpu().numpy()] = torch_to_np(raw.index_select(0, uniq_rows))
        grad_host = torch_to_np(grad) if do_bwd else np.zeros((N, D), np.float32)
        tot_t, tot_s, reps = 0, 0.0, 0
        while tot_s < args.cpu_seconds and reps < 500:
            tt, dt = cpu_oracle_step(w, table_host, grad_host, threads)
            tot_t += tt
            tot_s += dt
            reps += 1
        cpu = {"value": tot_t / tot_s, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": f"{reps} full passes of the workload ({T} tokens each): rows, gather, gradient sums; "
                         f"std::thread over sequences / hits / rows, {tot_s:.1f} s"}
        del table_host

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": ("int64 hash, e4m3->bf16 widening copy, f32 grad" if w.table_dtype == 2 else
                          f"int64 hash, {DTYPE_NAMES[w.table_dtype]} copy, f32 grad"), "data": "synthetic",
                "config": dict(describe(w), parallelism=f"replicas{world}",
                               l2="flushed between steps (512 MB written, then another 512 MB read); flush outside the step events",
                               step=("ple_lookup (rows saved) + ple_grad_scatter" if do_bwd else
                                     "ple_lookup" if sl is None else
                                     f"ple_lookup_slice rows of {sl[0]}, positions [{sl[1]}, {sl[2]})")),
                "fwd": {"ms": ms_fwd, "tokens_per_s": world * T_out / (ms_fwd * 1e-3), "gb_per_s": fwd_gbs,
                        "frac_of_8tbs": fwd_gbs / NOMINAL_HBM_GBS, "frac_of_measured": fwd_gbs / peak},
                "bwd": None if not do_bwd else {
                    "ms": ms_bwd, "tokens_per_s": world * T / (ms_bwd * 1e-3), "gb_per_s": bwd_gbs,
                    "frac_of_8tbs": bwd_gbs / NOMINAL_HBM_GBS, "frac_of_measured": bwd_gbs / peak},
                "roofline": roofline, "roofline_fwd": fwd_roof, "roofline_bwd": bwd_roof,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
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
