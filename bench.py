#!/usr/bin/env python
"""Decode-attention benchmark on B200: one step = one cfr_paged_decode call over
every (sequence, query head) of the workload (schedule + decode + merge).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload alibi1m|cfr|tiny|gqa|tiered|mqa|gqa_d64|gqa_d64_i8p16|gqa_d64_mixed_p16|
                                gqa_i8p16|demote]
                    [--context N]
                    [--queries Q] [--sink S --window W]
    python bench.py --record-traffic NCU_CSV --workload W [--context N]

The default workload is the largest single-GPU one: 1,048,576 tokens of a
64-query / 8-kv-head bf16 cache with ALiBi (4 GiB of K/V).

Prints one JSON line (rank 0).  `value` is the effective KV-read bandwidth
(algorithmic K/V bytes of all ranks / step time, GB/s) with every input resident
in HBM; `ms_per_step` the device time of one step (CUDA events, max over ranks).
The decode kernel's own launches are bracketed by CUDA events inside the timed
steps for the roofline.  `e2e` repeats the measurement through the public call
with the step's inputs (q, seq_lens, page table) copied from pinned host memory
and (out, lse) read back, the KV cache staying resident.  `--impl reference`
times the fp64 CPU oracle on the host cores instead.  With N > 1 (torchrun) each
rank runs an independent replica of the workload (no collective on the path).

`--queries Q` makes the last Q positions of every sequence causal query rows
(cfr_paged_decode_multi); `--sink S --window W` restricts every softmax to the
first S and last W tokens (cfr_paged_decode_sink_window), the byte count then
covering only those tokens.  `--workload demote` measures page demotion instead: one step re-encodes the
cold pages of the tiered cache shape (768 bf16 pages of 8 kv heads x 256 tokens
x 128 dims) into int4 and int8 with cfr_demote_pages; `value` is HBM bytes
(read + written) per second.
"""
from __future__ import annotations

import argparse
import dataclasses
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_long_context_b200 import accounting, binding, demote_workload, synth  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
TRAFFIC_JSON = os.path.join(ROOT, "profiles", "traffic.json")
# the kernel sources whose code a traffic record is valid for
DECODE_SOURCES = ["cfr_decode_tc.cu", "cfr_decode_f32.cu", "cfr_decode_cc.cu", "cfr_common.cuh",
                  "cfr_tmap.cuh", "cfr_tmap.cu"]
DEMOTE_SOURCES = ["cfr_demote.cu", "cfr_common.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="alibi1m", choices=sorted(synth.WORKLOADS) + ["demote"])
    ap.add_argument("--context", type=int, default=None,
                    help="cut every sequence to CONTEXT tokens (the same shape, smaller)")
    ap.add_argument("--record-traffic", default=None, metavar="NCU_CSV",
                    help="store the DRAM traffic of the decode kernel from an ncu --csv "
                         "capture of this workload (at --context, scaled to the full size) "
                         "in profiles/traffic.json, then exit")
    ap.add_argument("--sink", type=int, default=0,
                    help="with --window: attend to the first SINK tokens of each sequence too")
    ap.add_argument("--window", type=int, default=0,
                    help="attend only to the last WINDOW tokens (and the sinks); 0 = every token")
    ap.add_argument("--queries", type=int, default=1,
                    help="query tokens per sequence (multi-query decode, causal over the last Q)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0,
                    help="seconds of oracle work for the CPU baseline")
    return ap.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing (replicas only)
# --------------------------------------------------------------------------

class Dist:
    """One process per GPU, each an independent replica of the workload; the
    process group only carries the barriers around the timed region and the
    max over ranks of the measured times (no collective on the data path).
    `backend` "gloo" runs the same logic on CPU processes."""

    def __init__(self, want: int, backend: str = "nccl"):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                self.device = f"cuda:{self.local}"
                dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                        device_id=torch.device("cuda", self.local))
            else:
                dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        elif torch.cuda.is_available():
            torch.cuda.set_device(0)

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


# --------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# --------------------------------------------------------------------------

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _reasons(self):
        f = getattr(self.nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            self.nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self._reasons()
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for bit, n in REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# --------------------------------------------------------------------------
# helpers
# --------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _code_only(text: str) -> str:
    """C++ source with its comments and blank lines removed (the kernel sources
    hold no string literal that contains a comment marker)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def kernel_source_digest(files=None) -> str:
    """Digest of kernel sources' code (comments do not change a capture's validity):
    the named files under csrc/, or all of them."""
    csrc = os.path.join(ROOT, "paged_long_context_b200", "csrc")
    paths = ([os.path.join(csrc, f) for f in files] if files else
             sorted(glob.glob(os.path.join(csrc, "*"))))
    h = hashlib.sha256()
    for f in paths:
        h.update(_code_only(open(f, encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def traffic_record(key: str):
    """The ncu DRAM figures of one kernel on one workload from profiles/traffic.json,
    only when the kernel's sources are unchanged since the capture (else None)."""
    if not os.path.exists(TRAFFIC_JSON):
        return None
    rec = json.load(open(TRAFFIC_JSON)).get(key)
    if not rec or rec.get("kernel_source_digest") != kernel_source_digest(rec["kernel_sources"]):
        return None
    return rec


_UNITS = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "tbyte": 1e12,
          "nsecond": 1e-3, "usecond": 1.0, "msecond": 1e3, "second": 1e6,
          "ns": 1e-3, "us": 1.0, "ms": 1e3, "s": 1e6, "%": 1.0, "": 1.0}


def ncu_csv_metrics(path: str, kernel_regex: str):
    """Per-launch metric values (bytes, microseconds, percent) of the launches whose
    kernel name matches, from `ncu --metrics ... --csv --log-file path`."""
    import csv
    launches = {}
    lines = [l for l in open(path) if l.startswith('"')]
    for row in csv.DictReader(lines):
        if not re.search(kernel_regex, row.get("Kernel Name", "")):
            continue
        unit = row.get("Metric Unit", "").strip().lower()
        val = float(row["Metric Value"].replace(",", "")) * _UNITS.get(unit, 1.0)
        launches.setdefault(row["ID"], {"kernel": row["Kernel Name"]})[row["Metric Name"]] = val
    return list(launches.values())


def record_traffic(args):
    """Writes the decode (or demotion) kernel's DRAM figures from an ncu CSV into
    profiles/traffic.json under this workload's key, scaled from the captured size
    to the full workload by the K/V bytes (DRAM traffic of these kernels grows in
    proportion to the tokens read)."""
    demote = args.workload == "demote"
    regex = r"demote_(staged_)?kernel" if demote else r"decode_kernel"
    rows = ncu_csv_metrics(args.record_traffic, regex)
    if not rows:
        raise SystemExit(f"no {regex} launch in {args.record_traffic}")
    r = rows[-1]
    rd, wr = r["dram__bytes_read.sum"], r["dram__bytes_write.sum"]
    scale = 1.0
    if demote:
        # a demotion step is two launches (int4 and int8 destinations): the
        # capture holds whole steps, and the record is per step
        steps = max(1, len(rows) // 2)
        rd = sum(x["dram__bytes_read.sum"] for x in rows) / steps
        wr = sum(x["dram__bytes_write.sum"] for x in rows) / steps
    elif args.context is not None:
        # K/V traffic grows with the tokens read; the workload's lengths come from
        # its shape alone (no cache is generated for this)
        spec = synth.WORKLOADS[args.workload][0]()
        if not spec.seq_lens:
            raise SystemExit("--context scaling needs a workload of fixed lengths")
        scale = sum(spec.seq_lens) / (args.context * spec.batch)
    rec = {
        "kernel": r["kernel"].split("(")[0],
        "workload": args.workload,
        "captured_context": args.context,
        "scale_to_workload": round(scale, 6),
        "dram_bytes_read_per_launch": int(round(rd * scale)),
        "dram_bytes_write_per_launch": int(round(wr * scale)),
        "dram_bytes_per_launch": int(round((rd + wr) * scale)),
        "dram_throughput_pct_of_peak_sustained_elapsed":
            r.get("dram__throughput.avg.pct_of_peak_sustained_elapsed"),
        "captured_gpu_time_us": r.get("gpu__time_duration.sum"),
        "kernel_sources": DEMOTE_SOURCES if demote else DECODE_SOURCES,
    }
    rec["kernel_source_digest"] = kernel_source_digest(rec["kernel_sources"])
    db = json.load(open(TRAFFIC_JSON)) if os.path.exists(TRAFFIC_JSON) else {}
    db[args.workload] = rec
    with open(TRAFFIC_JSON, "w") as f:
        json.dump(db, f, indent=1, sort_keys=True)
        f.write("\n")
    print(json.dumps(rec))


def dtype_name(case) -> str:
    fm = sorted({case.fmt_of_page(b, p) for b in range(case.batch)
                 for p in range(-(-int(case.seq_lens[b]) // case.page_tokens))})
    return "+".join(synth.FMT_NAMES[f] for f in fm)


def config_of(case, name, world, l2note):
    lens = [int(x) for x in case.seq_lens.cpu().tolist()]
    return {"workload": case.name, "short_name": name, "batch": case.batch,
            "q_heads": case.num_q_heads, "kv_heads": case.num_kv_heads,
            "head_dim": case.head_dim, "page_tokens": case.page_tokens,
            "context_tokens_total": sum(lens), "context_min": min(lens), "context_max": max(lens),
            "kv_formats": dtype_name(case), "alibi": case.alibi_slopes is not None,
            "l2": l2note, "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def _pair_bytes(case, b: int, sink: int, window: int) -> int:
    """K/V bytes one (sequence b, query head) pair's softmax reads (its subset's tokens)."""
    n_b = int(case.seq_lens[b])
    P = case.page_tokens
    kv = 0
    for p in range(-(-n_b // P)):
        f = case.fmt_of_page(b, p)
        kv += accounting._tokens_in_page(n_b, p, P, sink, window) * \
            accounting.kv_token_bytes(f, case.head_dim)
    return kv


def cpu_baseline(case, budget_s: float, host=None, sink: int = 0, window: int = 0):
    """Time the fp64 oracle (as it stands) on the host cores over a bounded sample."""
    import oracle
    oracle.build()
    hc = host if host is not None else case.to("cpu")
    pairs = [(b, h) for b in range(case.batch) for h in range(case.num_q_heads * case.num_queries)]
    sub = dict(sink_tokens=sink, window_tokens=window)
    # calibrate on one pair, then take as many pairs as fit the budget
    t0 = time.perf_counter()
    oracle.attend(hc, sel=[pairs[0]], nthreads=1, **sub)
    t1 = time.perf_counter() - t0
    threads = oracle.default_threads()
    n = max(1, min(len(pairs), int(budget_s * threads / max(t1, 1e-6))))
    # spread the sample over sequences and kv heads
    step = max(1, len(pairs) // n)
    sel = pairs[::step][:n]
    reps, t0 = 0, time.perf_counter()
    while True:                      # repeat a small sample until the timing is stable
        oracle.attend(hc, sel=sel, nthreads=threads, **sub)
        reps += 1
        if time.perf_counter() - t0 >= min(2.0, budget_s) or reps >= 1000:
            break
    dt = (time.perf_counter() - t0) / reps
    sample_bytes = sum(_pair_bytes(case, b, sink, window) for b, _ in sel)
    return {"value": sample_bytes / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{len(sel)} of {len(pairs)} (sequence, query head) pairs, "
                      f"{sample_bytes} K/V bytes, {dt:.3f} s per pass, {reps} passes",
            "seconds": dt}


# --------------------------------------------------------------------------
# our implementation
# --------------------------------------------------------------------------

def run_ours(args, dist):
    dev = torch.device("cuda", dist.local)
    case = synth.workload(args.workload, device=dev, num_queries=args.queries,
                          context=args.context)
    sw = (args.sink, args.window) if args.window > 0 else None
    acct = accounting.step_bytes(case, args.sink, args.window)
    kv_bytes = acct["kv"] + acct["scales"]
    bufs = binding.DecodeBuffers(case)
    path = binding.decode_path(case)
    stream = torch.cuda.current_stream(dev)
    st = binding.paged_decode_raw(case, bufs, stream, sink_window=sw)
    if st != 0:
        raise binding.CfrError(st, "cfr_paged_decode")
    torch.cuda.synchronize()
    if int(bufs.err.item()) != 0:
        raise RuntimeError(f"device error word {int(bufs.err.item()):#x}")

    flush = None
    if acct["total"] < 2 * L2_BYTES:
        flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
        l2note = "L2 flushed (512 MiB write) before every step, outside the timed events"
    else:
        l2note = f"inputs larger than L2 ({acct['total'] / 2**20:.0f} MiB > 126 MiB)"

    def full_step():
        binding.paged_decode_raw(case, bufs, stream, sink_window=sw)

    def phased_step(evs):
        binding.paged_decode_raw(case, bufs, stream, phases=binding.PHASE_SCHEDULE, sink_window=sw)
        evs[0].record(stream)
        binding.paged_decode_raw(case, bufs, stream, phases=binding.PHASE_DECODE, sink_window=sw)
        evs[1].record(stream)
        binding.paged_decode_raw(case, bufs, stream, phases=binding.PHASE_MERGE, sink_window=sw)

    for _ in range(args.warmup):
        if flush is not None:
            flush.fill_(1.0)
        full_step()
    torch.cuda.synchronize()
    # this library's kernels per step, counted from the device's own launch
    # record (outside the timed regions): the public call, and the phase-split
    # step of timed region 2
    n_full, names_full = count_launches(full_step)
    n_phased, names_phased = count_launches(
        lambda: phased_step([torch.cuda.Event(enable_timing=True) for _ in range(2)]))

    # timed region 1: K steps through the public call (schedule, decode, merge
    # launched back to back as a caller sees them)
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dist.local) as clk:
        for k in range(K):
            if flush is not None:
                flush.fill_(1.0)
            evs[k][0].record(stream)
            full_step()
            evs[k][1].record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        # timed region 2: the same K steps with the decode kernel's own launches
        # bracketed by events (the roofline's kernel time)
        kev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for k in range(K):
            if flush is not None:
                flush.fill_(1.0)
            phased_step(kev[k])
        torch.cuda.synchronize()
    dist.barrier()
    step_times = [a.elapsed_time(c) for a, c in evs]
    kern_times = [a.elapsed_time(c) for a, c in kev]
    step_ms = sum(step_times) / K
    kern_ms = sum(kern_times) / K
    l2_warm_ms = None
    if flush is not None:
        # the same steps back to back without the flush: the inputs stay in L2
        wev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for k in range(K):
            wev[k][0].record(stream)
            full_step()
            wev[k][1].record(stream)
        torch.cuda.synchronize()
        l2_warm_ms = dist.max(sum(a.elapsed_time(c) for a, c in wev) / K)
    step_ms_max = dist.max(step_ms)
    kern_ms_max = dist.max(kern_ms)
    err = int(bufs.err.item())

    # ---- end to end through the public call, host buffers ----
    # The step's inputs (q, seq_lens, page table, page formats) travel in one
    # pinned buffer and its results (out, lse) come back in one: one copy each
    # way per step.  The library is called on views into the packed device
    # buffers, exactly as a caller that packs its per-step tensors would.
    def layout(tensors):
        offs, o = [], 0
        for t in tensors:
            offs.append(o)
            o = (o + t.numel() * t.element_size() + 255) // 256 * 256
        return offs, o

    def views_of(buf, offs, tensors):
        return [buf[a:a + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
                for a, t in zip(offs, tensors)]

    ins = [case.q, case.seq_lens, case.page_table] + \
        ([case.page_fmt] if case.page_fmt is not None else [])
    in_offs, in_total = layout(ins)
    in_d = torch.empty((in_total,), dtype=torch.uint8, device=dev)
    in_h = torch.zeros((in_total,), dtype=torch.uint8).pin_memory()
    for v, t in zip(views_of(in_h, in_offs, ins), ins):
        v.copy_(t.cpu())
    in_v = views_of(in_d, in_offs, ins)
    e2e_case = dataclasses.replace(case, q=in_v[0], seq_lens=in_v[1], page_table=in_v[2],
                                   page_fmt=in_v[3] if case.page_fmt is not None else None)
    outs = [bufs.out, bufs.lse]
    out_offs, out_total = layout(outs)
    out_d = torch.empty((out_total,), dtype=torch.uint8, device=dev)
    e2e_bufs = binding.DecodeBuffers.__new__(binding.DecodeBuffers)
    e2e_bufs.out, e2e_bufs.lse = views_of(out_d, out_offs, outs)
    e2e_bufs.workspace, e2e_bufs.err = bufs.workspace, bufs.err
    out_h = torch.empty((out_total,), dtype=torch.uint8).pin_memory()
    h2d, d2h = in_total, out_total

    def e2e_step():
        in_d.copy_(in_h, non_blocking=True)
        binding.paged_decode_raw(e2e_case, e2e_bufs, stream, sink_window=sw)
        out_h.copy_(out_d, non_blocking=True)

    for _ in range(min(args.warmup, 10)):
        e2e_step()
    torch.cuda.synchronize()
    Ke = max(3, min(K, 500))
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
    dist.barrier()
    torch.cuda.synchronize()
    for k in range(Ke):
        if flush is not None:
            flush.fill_(1.0)
        ee[k][0].record(stream)
        e2e_step()
        ee[k][1].record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    e2e_ms = dist.max(sum(a.elapsed_time(b) for a, b in ee) / Ke)
    # the result read back through the packed buffer is the device-resident result
    assert torch.equal(views_of(out_h, out_offs, outs)[0], bufs.out.cpu())

    peak, peak_kind = measured_peaks()
    achieved = acct["total"] / (kern_ms_max * 1e-3) / 1e9
    # the committed capture is of the plain decode (no subset, one query per
    # sequence) at the workload's full size
    rec = (traffic_record(args.workload)
           if sw is None and args.queries == 1 and args.context is None else None)
    traffic = rec["dram_bytes_per_launch"] if rec else None
    world = dist.world
    value = world * kv_bytes / (step_ms_max * 1e-3) / 1e9
    res = {
        "metric": "decode-attn µs/step and KV-read GB/s as % of B200 HBM peak (1 GPU)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
        "us_per_step": round(step_ms_max * 1e3, 2),
        "us_per_step_median": round(statistics.median(step_times) * 1e3, 2),
        "us_per_step_min": round(min(step_times) * 1e3, 2),
        **({"us_per_step_l2_warm": round(l2_warm_ms * 1e3, 2)} if l2_warm_ms is not None else {}),
        "kv_read_gbs_per_gpu": round(kv_bytes / (step_ms_max * 1e-3) / 1e9, 2),
        "hbm_frac_of_measured": round(kv_bytes / (step_ms_max * 1e-3) / 1e9 / peak, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_name(case), "data": "synthetic (seeded N(0,1) K/V/q, page-shaped workload)",
        "config": dict(config_of(case, args.workload, world, l2note),
                       **({"sink_tokens": args.sink, "window_tokens": args.window} if sw else {}),
                       **({"queries_per_sequence": args.queries} if args.queries > 1 else {})),
        "kernel_path": {1: "cuda-core", 2: "tcgen05", 3: "cuda-core-f32-tma"}.get(path, "?"),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "peak_kind": peak_kind,
                     "ncu_dram_throughput_pct": (
                         rec["dram_throughput_pct_of_peak_sustained_elapsed"] if rec else None),
                     "traffic_source": ("profiles/traffic.json (ncu, kernel sources unchanged)"
                                        if rec else None),
                     "kernel_us": round(kern_ms_max * 1e3, 2),
                     "kernel_us_median": round(statistics.median(kern_times) * 1e3, 2),
                     "kernel_us_min": round(min(kern_times) * 1e3, 2),
                     "algorithmic_bytes_per_launch": acct["total"]},
        "e2e": {"value": round(world * kv_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": round(e2e_ms * 1e3, 2)},
        "gpu_launches": (n_full + n_phased) * K if n_full is not None else None,
        "gpu_launches_note": (
            f"{n_full} per step through the public call ({', '.join(names_full)}); the "
            f"kernel-time region repeats each step as separate schedule, decode and merge "
            f"calls ({n_phased}: {', '.join(names_phased)})" if n_full is not None else
            "the launch record could not be read"),
        "clocks": clk.summary(),
        "device_err_word": err,
    }
    return case, res


OUR_KERNELS = re.compile(r"(schedule|qimage|decode|merge|demote|demote_staged)_kernel")


def count_launches(step):
    """Kernels of this library that one call of `step` launches, read from the
    CUDA activity record (torch.profiler / CUPTI): (count, sorted kernel names),
    or (None, []) when the record is unavailable."""
    try:
        from torch.profiler import ProfilerActivity, profile
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            step()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events()
                 if e.device_type == torch.autograd.DeviceType.CUDA and OUR_KERNELS.search(e.name)]
    except Exception:  # noqa: BLE001 - the count is a report, not part of the measurement
        return None, []
    short = sorted({OUR_KERNELS.search(n).group(0) for n in names})
    return len(names), short


def run_reference(args, dist):
    """The fp64 CPU oracle, as it stands, timed on the host cores (rank 0 only)."""
    import oracle
    oracle.build()
    case = synth.workload(args.workload, device="cpu", num_queries=args.queries,
                          context=args.context)
    pairs = [(b, h) for b in range(case.batch) for h in range(case.num_q_heads * case.num_queries)]
    sub = dict(sink_tokens=args.sink, window_tokens=args.window)
    threads = oracle.default_threads()
    t0 = time.perf_counter()
    oracle.attend(case, sel=[pairs[0]], nthreads=1, **sub)
    t1 = time.perf_counter() - t0
    budget = 150.0 / max(1, args.steps + args.warmup)
    shortened = None
    if t1 > budget and max(int(x) for x in case.seq_lens.tolist()) > case.page_tokens:
        # even one (sequence, head) pair of the full length would overrun the run's
        # time budget (long contexts, many steps): the sample is the same shape cut
        # to a shorter context, whole pages, so the whole run still ends in minutes
        longest = max(int(x) for x in case.seq_lens.tolist())
        ctx = max(case.page_tokens, int(longest * budget / t1) // case.page_tokens * case.page_tokens)
        if ctx < longest:
            shortened = ctx
            case = synth.workload(args.workload, device="cpu", num_queries=args.queries, context=ctx)
            t0 = time.perf_counter()
            oracle.attend(case, sel=[pairs[0]], nthreads=1, **sub)
            t1 = time.perf_counter() - t0
    n = max(1, min(len(pairs), int(budget * threads / max(t1, 1e-6))))
    sel = pairs[::max(1, len(pairs) // n)][:n]
    sample_bytes = sum(_pair_bytes(case, b, args.sink, args.window) for b, _ in sel)
    # the run is bounded in time whatever K and W are: warm-up steps stop after
    # 20 s and timed steps after 120 s (at least one of each); the line reports
    # how many ran
    warm_done, t0 = 0, time.perf_counter()
    while warm_done < max(1, args.warmup) and (warm_done == 0 or time.perf_counter() - t0 < 20.0):
        oracle.attend(case, sel=sel, nthreads=threads, **sub)
        warm_done += 1
    steps_done, t0 = 0, time.perf_counter()
    while steps_done < max(1, args.steps) and (steps_done == 0 or time.perf_counter() - t0 < 120.0):
        oracle.attend(case, sel=sel, nthreads=threads, **sub)
        steps_done += 1
    dt = (time.perf_counter() - t0) / steps_done
    value = sample_bytes / dt / 1e9
    sample = (f"{len(sel)} of {len(pairs)} (sequence, query head) pairs per step, "
              f"{sample_bytes} K/V bytes"
              + (f", every sequence cut to {shortened} tokens (the full length would overrun "
                 f"the run's time budget)" if shortened else ""))
    cfg = config_of(case, args.workload, 1, "host memory")
    if args.window > 0:
        cfg.update(sink_tokens=args.sink, window_tokens=args.window)
    if args.queries > 1:
        cfg.update(queries_per_sequence=args.queries)
    return {
        "impl": "reference",
        "metric": "decode-attn µs/step and KV-read GB/s as % of B200 HBM peak (1 GPU)",
        "value": round(value, 4), "unit": "GB/s", "n_gpus": dist.world, "steps": steps_done,
        "warmup": warm_done, "steps_requested": args.steps, "warmup_requested": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) K/V/q, page-shaped workload)",
        "config": cfg,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# --------------------------------------------------------------------------
# page demotion (cfr_demote_pages)
# --------------------------------------------------------------------------

DEMOTE_METRIC = "page demotion bf16 -> int4/int8: HBM GB/s (read + write) (1 GPU)"


def demote_config(w, world):
    src = w.src
    return {"workload": demote_workload.NAME, "short_name": "demote", "pages": sum(j.n for j in w.jobs.values()),
            "pages_per_format": {synth.FMT_NAMES[f]: j.n for f, j in w.jobs.items()},
            "kv_heads": src.num_kv_heads, "head_dim": src.head_dim, "page_tokens": src.page_tokens,
            "source_format": "bf16", "l2": "inputs larger than L2",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def demote_cpu_baseline(w, budget_s: float, pages: int = 8):
    """The oracle's demotion, as it stands, on a bounded sample of pages (host)."""
    import oracle
    oracle.build()
    src = w.src
    Hkv, d, P = src.num_kv_heads, src.head_dim, src.page_tokens
    f = synth.I8
    j = w.jobs[f]
    idx = [int(x) for x in j.src_slots[:pages].cpu().tolist()]
    sk = src.k_pool[synth.BF16][idx].cpu().contiguous()
    sv = src.v_pool[synth.BF16][idx].cpu().contiguous()
    dk = torch.empty((pages, Hkv, P, synth.row_bytes(f, d)), dtype=torch.uint8)
    dv = torch.empty_like(dk)
    dsc = torch.empty((pages, Hkv, 2))
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.demote(Hkv, d, P, synth.BF16, sk, sv, None, f, dk, dv, dsc,
                      list(range(pages)), list(range(pages)))
        reps += 1
        if time.perf_counter() - t0 >= min(2.0, budget_s) or reps >= 1000:
            break
    dt = (time.perf_counter() - t0) / reps
    nbytes = pages * Hkv * P * 2 * (synth.row_bytes(synth.BF16, d) + synth.row_bytes(f, d))
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{pages} bf16 pages -> int8, {nbytes} bytes read + written, "
                      f"{dt:.3f} s per pass, {reps} passes (single-threaded oracle)",
            "seconds_per_pass": dt}


def run_demote(args, dist):
    dev = torch.device("cuda", dist.local)
    w = demote_workload.build(dev)
    acct = demote_workload.step_bytes(w)
    stream = torch.cuda.current_stream(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    demote_workload.run(w, err, stream)
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item()):#x}")
    jobs = list(w.jobs.values())
    for _ in range(args.warmup):
        demote_workload.run(w, err, stream)
    torch.cuda.synchronize()
    K = args.steps
    # each launch bracketed by events: [step][launch][start, end]
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in jobs] for _ in range(K)]
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dist.local) as clk:
        for k in range(K):
            for i, j in enumerate(jobs):
                evs[k][i][0].record(stream)
                st = binding.demote_pages(w.pool, synth.BF16, j.fmt, j.dst_k, j.dst_v,
                                          j.dst_scales, j.src_slots, j.dst_slots, None, err,
                                          stream)
                evs[k][i][1].record(stream)
                if st != 0:
                    raise binding.CfrError(st, "cfr_demote_pages")
        torch.cuda.synchronize()
    dist.barrier()
    step_ms = sum(evs[k][0][0].elapsed_time(evs[k][-1][1]) for k in range(K)) / K
    launch_ms = sum(e[0].elapsed_time(e[1]) for k in range(K) for e in evs[k]) / K
    step_ms_max, launch_ms_max = dist.max(step_ms), dist.max(launch_ms)

    # end to end: slot lists from pinned host memory, scales read back
    hs = [(j.src_slots.cpu().pin_memory(), j.dst_slots.cpu().pin_memory(),
           torch.empty_like(j.dst_scales, device="cpu").pin_memory()) for j in jobs]
    h2d = sum(a.numel() * 4 + b.numel() * 4 for a, b, _ in hs)
    d2h = sum(c.numel() * 4 for _, _, c in hs)

    def e2e_step():
        for j, (a, b, c) in zip(jobs, hs):
            j.src_slots.copy_(a, non_blocking=True)
            j.dst_slots.copy_(b, non_blocking=True)
        demote_workload.run(w, err, stream)
        for j, (a, b, c) in zip(jobs, hs):
            c.copy_(j.dst_scales, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    Ke = max(3, min(K, 200))
    ee = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(Ke)]
    for k in range(Ke):
        ee[k][0].record(stream)
        e2e_step()
        ee[k][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = dist.max(sum(a.elapsed_time(b) for a, b in ee) / Ke)

    peak, peak_kind = measured_peaks()
    achieved = acct["total"] / (launch_ms_max * 1e-3) / 1e9
    rec = traffic_record("demote")
    traffic = rec["dram_bytes_per_launch"] if rec else None   # per step (both launches)
    world = dist.world
    res = {
        "metric": DEMOTE_METRIC,
        "value": round(world * acct["total"] / (step_ms_max * 1e-3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(step_ms_max, 5), "us_per_step": round(step_ms_max * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->i4+i8", "data": "synthetic (seeded N(0,1) bf16 pages)",
        "config": demote_config(w, world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_kind": peak_kind, "kernel_us": round(launch_ms_max * 1e3, 2),
                     "algorithmic_bytes_per_step": acct["total"],
                     "launches_per_step": len(jobs)},
        "e2e": {"value": round(world * acct["total"] / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_step": round(e2e_ms * 1e3, 2)},
        "gpu_launches": len(jobs) * K,
        "gpu_launches_note": f"{len(jobs)} demote_staged_kernel launches per step (one per destination format)",
        "clocks": clk.summary(),
        "device_err_word": int(err.item()),
    }
    return w, res


def run_reference_demote(args):
    import oracle
    oracle.build()
    w = demote_workload.build("cpu")
    base = demote_cpu_baseline(w, 150.0 / max(1, args.steps + args.warmup))
    dt = base.pop("seconds_per_pass")
    return {
        "impl": "reference", "metric": DEMOTE_METRIC, "value": base["value"], "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32 decisions", "data": "synthetic (seeded N(0,1) bf16 pages)",
        "config": demote_config(w, 1),
        "cpu_baseline": base,
        "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    args = parse()
    if args.record_traffic:
        record_traffic(args)
        return 0
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        class _D:
            world = int(os.environ.get("WORLD_SIZE", "1"))
        res = run_reference_demote(args) if args.workload == "demote" else run_reference(args, _D())
        print(json.dumps(res), flush=True)
        return 0
    dist = Dist(args.gpus)
    try:
        if args.workload == "demote":
            w, res = run_demote(args, dist)
            if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
                base = demote_cpu_baseline(w, args.cpu_budget)
                base.pop("seconds_per_pass")
                res["cpu_baseline"] = base
        else:
            case, res = run_ours(args, dist)
            if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = {k: v for k, v in cpu_baseline(
                    case, args.cpu_budget, sink=args.sink, window=args.window).items()
                    if k != "seconds"}
        if dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
