#!/usr/bin/env python
"""Benchmark of the paged-attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input: copy-on-write block
copies (when the workload has shared blocks), slot mapping, KV append, then paged attention over
the mixed batch (split-K decode kernel, tcgen05 prefill tiles when present, log-sum-exp merge).
The default workload is the largest single-GPU one: the 70B-shaped bf16 mixed batch (64/8 heads,
head_dim 128; 4 chunked-prefill requests of 512 rows at prior contexts 0/4k/16k/32k and 128 decode
rows with contexts U[256, 16384], one {request_id: num_tokens} step). --config c2 selects the
LLaMA-13B-shaped fp16 decode batch, and so on. Every workload's KV pool (>= 0.6 GB, 4.8 GB for the
default) is larger than the 126 MB L2; a second timed pass (--l2-flush, on by default) also
writes a 2 x L2-sized buffer between steps, outside the timed events, and reports that figure
beside the unflushed one.

Metric: KV bytes the step must read (every (request, KV head, context token) once as K and once as
V) divided by the step time, in GB/s; also decode sequence-tokens per second (sum of decode rows'
context lengths / time). Multi-GPU (torchrun): every rank runs its own replica with its own seed
(requests are independent: no data-path collective), and the whole-job value divides all ranks'
bytes by the slowest rank's time.

--impl reference times the CPU oracle (test infrastructure) on a bounded sample of the same
workload, on the host cores.
"""
from __future__ import annotations

import argparse
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

METRIC = "paged-attn KV-read GB/s (% of B200 HBM peak) and decode seqs·tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default="c5", choices=["c1", "c2", "c3", "c4", "c5", "c6"])
    ap.add_argument("--impl", default="pkv", choices=["pkv", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-l2-flush", action="store_true",
                    help="skip the second timed pass that flushes L2 between steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU work of the oracle sample")
    ap.add_argument("--split-blocks", type=int, default=0)
    ap.add_argument("--part", default="all", choices=["all", "prefill", "decode"],
                    help="time only the prefill or decode requests of the workload")
    ap.add_argument("--requests", type=int, default=0, help="keep only the first N requests (profiling subsets)")
    ap.add_argument("--heads-per-item", type=int, default=0, help="query heads per split-K work item")
    ap.add_argument("--rows-per-item", type=int, default=0, help="query rows of a request per split-K work item")
    ap.add_argument("--tc-min-rows", type=int, default=0, help="fewest rows a request needs for the tcgen05 tiles")
    ap.add_argument("--cuda-core-only", action="store_true", help="serve every row on CUDA cores")
    ap.add_argument("--decode-kernel", type=int, default=0, choices=[0, 1, 2],
                    help="kernel for split-K rows: 0 planner's choice, 1 FMA, 2 warp MMA")
    ap.add_argument("--decode-sms", type=int, default=0,
                    help="mixed batches: SMs of the split-K kernel running beside the tcgen05 tiles "
                         "(0 planner's choice, -1 the two kernels one after the other)")
    return ap.parse_args()


FALLBACK_BF16_TFLOPS = 1590.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense 16-bit tensor-core peak (TFLOP/s) for a kernel timed alone: the measured burst figure."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch recorded from an ncu capture (profiles/traffic.json), or None when there
    is no record for this workload or the kernel's source changed since the capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
        rec = data.get(f"{kernel}@{workload}") or data.get(kernel)
        if not rec or rec.get("workload") != workload:
            return None
        # the kernel's source files (one "source", or "sources" hashed in order as one byte string)
        h = hashlib.sha256()
        for src in rec.get("sources") or [rec["source"]]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != rec["source_sha256"]:
            return None
        return int(rec["dram_bytes_read"]) + int(rec["dram_bytes_write"])
    except (OSError, ValueError, KeyError):
        return None


def rank_seed(config: str, rank: int) -> int:
    """Each rank runs its own replica of the workload: same shapes, its own seeded data."""
    return 1000 + int(config[1]) + 100 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's time: every rank contributes its own device time, all receive the max."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: all ranks' bytes divided by the slowest rank's step time."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


def workload_desc(wl):
    ctx = np.asarray(wl.prior_lens, np.int64) + np.asarray(list(wl.batch.values()), np.int64)
    return ctx


def kv_bytes(wl) -> int:
    ctx = workload_desc(wl)
    eb = 4 if wl.dtype == "f32" else 2
    return int(ctx[np.asarray(list(wl.batch.values())) > 0].sum()) * wl.num_kv_heads * 2 * wl.head_dim * eb


def decode_seq_tokens(wl) -> int:
    ctx = workload_desc(wl)
    n = np.asarray(list(wl.batch.values()))
    return int(ctx[n == 1].sum())


def pool_waste(wl) -> dict:
    """Internal fragmentation of paging for the step's sequences (each holding its context after the
    step), from the library's host block manager (pkv_bm_*): blocks reserved, slots reserved but
    unfilled, and their fraction -- the quantity the pages put under 4 %. Sequences are counted
    independently (blocks shared between them would be counted once per sharer)."""
    from paged_kv_cache_446_b200 import pkv
    _, ctx = pkv.flatten_batch(wl.batch, wl.prior_lens)
    m = pkv.BlockManager(int(sum(-(-int(c) // 16) for c in ctx)) + 1)
    for r, c in enumerate(ctx):
        m.add(r, int(c))
    st = m.stats()
    return {"reserved_blocks": st["used_blocks"], "unfilled_slots": st["wasted_slots"],
            "frac": st["wasted_slots"] / max(1, 16 * st["used_blocks"])}


def kernel_work(plan, wl) -> dict:
    """Algorithmic work per launch from the plan: the split-K kernel reads K+V of its requests'
    contexts once per (request, KV head) plus its q rows and writes its output rows; the tcgen05
    tiles likewise for theirs, and compute 4*D flops per (row, head, attended key)."""
    eb = 4 if wl.dtype == "f32" else 2
    row_bytes = wl.num_q_heads * wl.head_dim * eb * 2
    core_rows = plan.num_q_tokens - plan.num_prefill_rows
    return {"decode": {"bytes": int(plan.core_kv_bytes) + core_rows * row_bytes},
            "prefill_tc": {"bytes": int(plan.tile_kv_bytes) + plan.num_prefill_rows * row_bytes,
                           "flops": int(plan.tile_flops)}}


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = bus_id
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(", ") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        if self.bus_id:
            mine = [r for r in rows if len(r) > 1 and r[1].strip().lower().endswith(self.bus_id.lower()[-12:])]
            rows = mine or rows
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[2]))
                mx.append(float(r[3]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[6:10]):
                if val.strip().lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def bus_id_of(dev) -> str | None:
    try:
        p = torch.cuda.get_device_properties(dev)
        return f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
    except Exception:
        return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_oracle_sample(wl, h, target_seconds: float, threads: int = 0, append: bool = True):
    """The oracle, as it stands, on a bounded sample of the step's query rows (all heads of each row):
    every k-th row of the flattened batch, so decode and prefill rows appear in their proportions,
    with the step's own KV append applied first (unless append=False: already applied to h). A
    sampled row counts its request's K/V bytes divided by the request's row count, so the whole
    batch counts each (request, KV head, context token) once, as the GPU metric does. The stride
    shrinks until the oracle has run for about target_seconds (the whole batch is repeated when it
    is faster than that). Returns dict(value_gbs, seconds, rows, of, cores, bytes, repeats).
    threads = 0: every host core."""
    import oracle
    cores = threads or os.cpu_count() or 1
    qsl, ctx = oracle.flatten_batch(wl.batch, wl.prior_lens)
    counts = np.asarray(list(wl.batch.values()), np.int64)
    if wl.write_batch and append:
        wcounts = np.asarray([wl.write_batch.get(r, 0) for r in wl.batch.keys()], np.int64)
        wqsl, wctx = oracle.flatten_batch(dict(zip(wl.batch.keys(), wcounts)), ctx.astype(np.int64) - wcounts)
        if len(wl.copy_pairs):
            oracle.copy_blocks([h["k_pool"]], [h["v_pool"]], wl.copy_pairs)
        slots = oracle.slot_mapping(wl.block_tables, wqsl, wctx)
        oracle.kv_cache_write(h["k_new"], h["v_new"], h["k_pool"], h["v_pool"], slots)
    eb = 4 if wl.dtype == "f32" else 2
    T = int(qsl[-1])
    req_of_row = np.repeat(np.arange(len(ctx)), counts)
    row_bytes = (ctx.astype(np.float64) * wl.num_kv_heads * 2 * wl.head_dim * eb / np.maximum(counts, 1))[req_of_row]

    def run(stride):
        rows = np.arange(stride // 2, T, stride, dtype=np.int32)
        t0 = time.perf_counter()
        oracle.paged_attention(h["q"], h["k_pool"], h["v_pool"], wl.block_tables, ctx, qsl, wl.scale, wl.dtype,
                               rows=rows, nthreads=cores)
        return time.perf_counter() - t0, float(row_bytes[rows].sum()), len(rows)

    stride = max(1, T // 8)
    dt, by, n = run(stride)
    while dt < target_seconds * 0.3 and stride > 1:
        stride = max(1, int(stride / min(8.0, max(1.5, 0.6 * target_seconds / max(dt, 1e-3)))))
        dt, by, n = run(stride)
    reps = 1
    if stride == 1 and dt < target_seconds * 0.5:
        # the whole batch is quick: repeat it to fill the measurement window
        reps = max(1, int(target_seconds / max(dt, 1e-3)))
        dt, by = 0.0, 0.0
        for _ in range(reps):
            t, b, n = run(1)
            dt += t
            by += b
    return {"value_gbs": by / dt / 1e9, "seconds": dt, "rows": n, "of": T, "stride": stride, "cores": cores,
            "bytes": int(by), "repeats": reps}


def storage(t):
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy().copy()
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def reference_arm(args, rank, world):
    if rank != 0:
        return
    from paged_kv_cache_446_b200 import workloads as W
    wl = W.make(args.config, device="cpu", part=args.part, max_requests=args.requests)
    h = {k: storage(getattr(wl, k)) for k in ("q", "k_pool", "v_pool", "k_new", "v_new")}
    per_step = max(1.0, 150.0 / max(1, args.steps + args.warmup))
    samples = []
    for i in range(args.warmup + args.steps):
        hh = {k: v.copy() for k, v in h.items()} if (wl.write_batch or len(wl.copy_pairs)) else h
        r = run_oracle_sample(wl, hh, per_step)
        if i >= args.warmup:
            samples.append(r)
    secs = sum(s["seconds"] for s in samples)
    by = sum(s["bytes"] for s in samples)
    value = by / secs / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(samples),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded N(0,1) q/k/v; seeded block placement)",
            "config": {"workload": wl.name, "rows_per_step_sample": samples[-1]["rows"],
                       "rows": samples[-1]["of"]},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": samples[-1]["cores"], "kind": "oracle",
                             "sample": f"every {samples[-1]['stride']}th of the {samples[-1]['of']} query rows of "
                                       f"{wl.name} per step (all heads, after the step's KV append)"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank, world)
        return
    import torch.distributed as dist
    from datetime import timedelta

    from paged_kv_cache_446_b200 import pkv
    from paged_kv_cache_446_b200 import workloads as W
    from paged_kv_cache_446_b200.step import PagedAttentionStep

    assert args.warmup >= 3, "at least 3 warm-up steps"
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wl = W.make(args.config, device=dev, seed=rank_seed(args.config, rank), part=args.part,
                max_requests=args.requests)
    dt = W.TORCH_DTYPES[wl.dtype]
    opts = {"split_blocks": args.split_blocks} if args.split_blocks else {}
    if args.heads_per_item:
        opts["heads_per_item"] = args.heads_per_item
    if args.rows_per_item:
        opts["rows_per_item"] = args.rows_per_item
    if args.tc_min_rows:
        opts["tc_min_rows"] = args.tc_min_rows
    if args.cuda_core_only:
        opts["cuda_core_only"] = True
    if args.decode_kernel:
        opts["decode_kernel"] = args.decode_kernel
    if args.decode_sms:
        opts["decode_sms"] = args.decode_sms
    step = PagedAttentionStep(wl.batch, wl.prior_lens, wl.block_tables, wl.num_blocks, wl.num_q_heads,
                              wl.num_kv_heads, wl.head_dim, dt, dev, write_batch=wl.write_batch or None,
                              copy_pairs=wl.copy_pairs, **opts)
    out = torch.empty_like(wl.q)
    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        h = {k: storage(getattr(wl, k)) for k in ("q", "k_pool", "v_pool", "k_new", "v_new")}
        r = run_oracle_sample(wl, h, args.cpu_seconds)
        cpu_baseline = {"value": r["value_gbs"], "unit": "GB/s", "cores": r["cores"], "kind": "oracle",
                        "sample": f"every {r['stride']}th of the {r['of']} query rows of {wl.name} ({r['rows']} rows, all "
                                  f"heads, after the step's KV append) x{r['repeats']}, {r['seconds']:.1f} s",
                        "cpu_model": cpu_model()}
        if args.config in ("c1", "c2"):
            r1 = run_oracle_sample(wl, h, args.cpu_seconds / 3, threads=1, append=False)
            cpu_baseline["single_thread"] = {
                "value": r1["value_gbs"], "unit": "GB/s", "cores": 1,
                "sample": f"every {r1['stride']}th of {r1['of']} rows x{r1['repeats']}, {r1['seconds']:.1f} s"}
        del h

    def run_step():
        step.run(wl.q, wl.k_pool, wl.v_pool, wl.scale, wl.k_new, wl.v_new, out=out)

    for _ in range(args.warmup):
        run_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(bus_id_of(dev)) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(args.steps):
        run_step()
    ev1.record()
    torch.cuda.synchronize()
    ms_total = ev0.elapsed_time(ev1)
    clocks = sampler.stop() if sampler else None
    # Per-kernel times: a second timed region of the same length with CUDA events around every
    # library launch, on the launch stream (the event pairs serialise back-to-back kernels, so the
    # step time above is taken without them).
    if world > 1:
        dist.barrier()
    pkv.profile_start(capacity=16 * args.steps + 16)
    for _ in range(args.steps):
        run_step()
    torch.cuda.synchronize()
    prof = pkv.profile_stop()
    ms_per_step = max_over_ranks(ms_total, dist, dev) / args.steps
    # When the step runs its split-K kernel beside the tcgen05 tiles, the intervals above are the
    # two kernels' overlapped spans; each kernel's own roofline comes from the same steps launched
    # one kernel after the other.
    prof_alone, run_alone = prof, run_step
    if step.plan.plan.decode_sms > 0:
        serial = PagedAttentionStep(wl.batch, wl.prior_lens, wl.block_tables, wl.num_blocks, wl.num_q_heads,
                                    wl.num_kv_heads, wl.head_dim, dt, dev, write_batch=wl.write_batch or None,
                                    copy_pairs=wl.copy_pairs, **dict(opts, decode_sms=-1))

        def run_alone():
            serial.run(wl.q, wl.k_pool, wl.v_pool, wl.scale, wl.k_new, wl.v_new, out=out)

        for _ in range(args.warmup):
            run_alone()
        torch.cuda.synchronize()
        pkv.profile_start(capacity=16 * args.steps + 16)
        for _ in range(args.steps):
            run_alone()
        torch.cuda.synchronize()
        prof_alone = pkv.profile_stop()
    code, detail = pkv.device_error()
    assert code == 0, f"device error {code} at {detail}"

    # ---- the same steps with L2 flushed between them ----
    # A write of twice the L2 size runs before every step, outside that step's event pair, so no
    # step finds its predecessor's K/V (or its own inputs) in L2. Step time = sum of the per-step
    # event intervals.
    flushed_ms, prof_flushed = None, None
    if not args.no_l2_flush:
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size or (126 << 20)
        flush_buf = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
        pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        if world > 1:
            dist.barrier()
        for a, b in pairs:
            flush_buf.fill_(1)
            a.record()
            run_step()
            b.record()
        torch.cuda.synchronize()
        flushed_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in pairs), dist, dev) / args.steps
        # once more with every library launch timed, for the kernels' flushed rooflines
        pkv.profile_start(capacity=16 * args.steps + 16)
        for _ in range(args.steps):
            flush_buf.fill_(1)
            run_alone()
        torch.cuda.synchronize()
        prof_flushed = pkv.profile_stop()
        del flush_buf

    # ---- end to end through the public API: pinned host inputs in, output back to the host ----
    e2e = None
    if not args.no_e2e:
        # End to end through the public API, as a serving loop runs it: every step copies its
        # inputs (q, new K/V, block tables) from pinned host memory, plans the batch on the host
        # (uploading the work lists), runs the step and reads the output back. Two sets of step
        # buffers alternate so that one step's host->device copies and the previous step's
        # device->host read run on two copy streams (PCIe is full duplex) while the compute stream
        # works; all of them fall inside the timed region.
        # The step's inputs travel as one packed pinned buffer (q, new K, new V, block tables at
        # 256-byte aligned offsets) in one copy; the device side is a matching buffer per set whose
        # typed views the step reads.
        host_parts = [wl.q, wl.k_new, wl.v_new, torch.from_numpy(wl.block_tables)]
        offs, total = [], 0
        for t in host_parts:
            offs.append(total)
            total += (t.numel() * t.element_size() + 255) // 256 * 256
        hbuf = torch.empty(total, dtype=torch.uint8).pin_memory()
        for t, o in zip(host_parts, offs):
            hbuf[o:o + t.numel() * t.element_size()].copy_(t.reshape(-1).view(torch.uint8).cpu())
        h2d_bytes = sum(t.numel() * t.element_size() for t in host_parts)
        comp = torch.cuda.current_stream()
        h2d_s, d2h_s = torch.cuda.Stream(), torch.cuda.Stream()
        steps2 = [step, PagedAttentionStep(wl.batch, wl.prior_lens, wl.block_tables, wl.num_blocks, wl.num_q_heads,
                                           wl.num_kv_heads, wl.head_dim, dt, dev, write_batch=wl.write_batch or None,
                                           copy_pairs=wl.copy_pairs, **opts)]
        dbuf = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]

        def dev_view(b, i):
            t = host_parts[i]
            n = t.numel() * t.element_size()
            return dbuf[b][offs[i]:offs[i] + n].view(t.dtype).view(t.shape)

        dq = [dev_view(b, 0) for b in range(2)]
        dkn = [dev_view(b, 1) for b in range(2)]
        dvn = [dev_view(b, 2) for b in range(2)]
        saved_tables = [st.block_tables for st in steps2]
        for b in range(2):
            steps2[b].block_tables = dev_view(b, 3)
        douts = [out, torch.empty_like(out)]
        houts = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        h2d_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        d2h_done = [torch.cuda.Event() for _ in range(2)]
        counter = [0]

        def e2e_step():
            i = counter[0]
            counter[0] += 1
            b = i & 1
            st = steps2[b]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(comp_done[b])   # step i-2 has finished with buffer set b
                dbuf[b].copy_(hbuf, non_blocking=True)
                # the work lists go up on the copy stream too, overlapping the previous step
                st.plan.replan(wl.batch, wl.prior_lens, stream=h2d_s)
                h2d_done[b].record(h2d_s)
            comp.wait_event(h2d_done[b])
            if i >= 2:
                comp.wait_event(d2h_done[b])          # step i-2's output has been read back
            st.run(dq[b], wl.k_pool, wl.v_pool, wl.scale, dkn[b], dvn[b], out=douts[b], stream=comp)
            comp_done[b].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[b])
                houts[b].copy_(douts[b], non_blocking=True)
                d2h_done[b].record(d2h_s)

        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        t_host = time.perf_counter()
        for _ in range(args.steps):
            e2e_step()
        host_ms = (time.perf_counter() - t_host) * 1e3 / args.steps   # host time to issue one step
        comp.wait_stream(d2h_s)         # the last output is back on the host
        e1.record(comp)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev) / args.steps
        for st, t in zip(steps2, saved_tables):
            st.block_tables = t
        h2d = h2d_bytes + int(step.plan.plan.meta_bytes) + 4 * (2 * len(wl.batch) + 1)
        d2h = houts[0].numel() * houts[0].element_size()
        e2e = {"value": whole_job_gbs(kv_bytes(wl), world, e2e_ms), "unit": "GB/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "pipelining": "2 buffer sets; one packed host->device copy of the inputs plus the work-list "
                             "upload on one copy stream, the output read on another",
               "host_issue_ms_per_step": host_ms}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    peak, peak_kind = peaks()
    value = whole_job_gbs(kv_bytes(wl), world, ms_per_step)
    # Rooflines of both attention kernels (each launch timed with CUDA events on its stream in the
    # profiling pass): the tcgen05 prefill tiles against the dense 16-bit tensor peak, the split-K
    # kernel against the HBM copy peak; `roofline` is the one that takes the most time per step.
    work = kernel_work(step.plan.plan, wl)
    tc_peak, tc_kind = tensor_peak()
    rooflines = {}
    for k, w in work.items():
        if not prof_alone[k][1]:
            continue
        avg_ms = prof_alone[k][0] / prof_alone[k][1]
        kname = "decode_mma_kernel" if (k == "decode" and step.plan.plan.decode_kernel == 2) else k + "_kernel"
        if k == "prefill_tc":
            achieved = w["flops"] / (avg_ms * 1e-3) / 1e12
            r = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                 "frac": achieved / tc_peak, "traffic": recorded_traffic(kname, wl.name),
                 "algorithmic_flops": w["flops"], "algorithmic_bytes": w["bytes"],
                 "peak_source": f"{tc_kind} bf16_tflops (burst cuBLAS)"}
        else:
            achieved = w["bytes"] / (avg_ms * 1e-3) / 1e9
            r = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                 "traffic": recorded_traffic(kname, wl.name), "algorithmic_bytes": w["bytes"],
                 "peak_source": f"{peak_kind} hbm_gbs (burst copy)"}
        r.update(kernel=kname, kernel_ms=avg_ms, launches_per_step=prof_alone[k][1] / max(1, args.steps),
                 timed="alone (kernels one after the other)" if prof_alone is not prof else "in the step")
        if prof_alone is not prof and prof[k][1]:
            r["kernel_ms_overlapped"] = prof[k][0] / prof[k][1]
        if prof_flushed and prof_flushed[k][1]:
            fms = prof_flushed[k][0] / prof_flushed[k][1]
            r["l2_flushed"] = {"kernel_ms": fms, "frac": r["frac"] * avg_ms / fms}
        rooflines[k] = r
    roof = None
    if rooflines:
        dom = max(rooflines, key=lambda k: prof_alone[k][0])
        roof = dict(rooflines[dom])
    # The step's own bound: every K/V byte once at the HBM peak, or every prefill flop at the tensor
    # peak, whichever is longer (the two can overlap in one step).
    t_bytes = kv_bytes(wl) / (peak * 1e9) * 1e3
    t_flops = work["prefill_tc"]["flops"] / (tc_peak * 1e12) * 1e3
    step_bound = {"ms": max(t_bytes, t_flops), "hbm_ms": t_bytes, "tensor_ms": t_flops,
                  "frac": max(t_bytes, t_flops) / ms_per_step}
    launches = sum(v[1] for k, v in prof.items() if k != "dropped")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded N(0,1) q/k/v drawn on the device; seeded random block placement)",
        "config": {"workload": wl.name, "requests": len(wl.batch), "num_q_heads": wl.num_q_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim, "block_size": 16,
                   "num_blocks": wl.num_blocks, "kv_bytes_per_step_per_gpu": kv_bytes(wl),
                   "l2": "inputs larger than L2 (KV pool read per step >> 126 MB); value taken without a "
                         "flush, l2_flushed taken with a 2 x L2 write between steps",
                   "parallelism": f"replicas x{world} (independent requests per GPU)",
                   "plan_options": opts, "decode_sms": int(step.plan.plan.decode_sms)},
        "frac_of_hbm_peak": value / world / peak,
        "frac_of_8tbs_spec": value / world / 8000.0,
        "kv_block_waste": pool_waste(wl),
        "decode_seq_tokens_per_s": world * decode_seq_tokens(wl) / (ms_per_step * 1e-3),
        "decode_steps_per_s": 1e3 / ms_per_step,
        "kernel_ms_per_step": {k: v[0] / max(1, args.steps) for k, v in prof.items() if k != "dropped"},
        "roofline": roof,
        "rooflines": rooflines,
        "step_bound": step_bound,
        "l2_flushed": None if flushed_ms is None else {
            "ms_per_step": flushed_ms, "value": whole_job_gbs(kv_bytes(wl), world, flushed_ms), "unit": "GB/s",
            "frac_of_hbm_peak": kv_bytes(wl) / (flushed_ms * 1e-3) / 1e9 / peak},
        "cpu_baseline": cpu_baseline,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
