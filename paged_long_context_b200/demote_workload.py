"""The page-demotion workload: the tiered cache's cold pages produced on the device.

Source: the tiered workload's shape (8 sequences of 32,768 tokens, 8 kv heads,
head_dim 128, 256-token pages) with every page in bf16.  Plan: logical pages
0-31 of each sequence are demoted to int4 and pages 32-95 to int8, so that the
demoted pools plus the untouched bf16 pages 96-127 form the tiered cache
(ARGUS page, "Visual Architecture": the compression cascade, oldest pages in
the lowest tier).  This module builds the inputs and the plan and calls the
library; it holds no arithmetic of the demotion itself.
"""
from __future__ import annotations

import dataclasses
from typing import Dict

import torch

from . import binding, synth

NAME = "demote_tiered_b8_32k_p256_bf16_to_i4i8"
TIERS = [(32, synth.I4), (96, synth.I8)]      # (end of logical page range, format), oldest first


def spec() -> synth.CaseSpec:
    return synth.CaseSpec(NAME, 8, 32, 8, 128, 256, seq_lens=[32768] * 8, fmt="bf16",
                          q_fmt="bf16")


@dataclasses.dataclass
class Job:
    fmt: int
    n: int
    src_slots: torch.Tensor
    dst_slots: torch.Tensor
    dst_k: torch.Tensor
    dst_v: torch.Tensor
    dst_scales: torch.Tensor


@dataclasses.dataclass
class Workload:
    src: synth.DecodeCase
    pool: binding.KvPool
    jobs: Dict[int, Job]


def build(device="cuda", seed: int = 4) -> Workload:
    src = synth.make_case(spec(), seed, device)
    P, Hkv, d = src.page_tokens, src.num_kv_heads, src.head_dim
    jobs = {}
    lo = 0
    for hi, f in TIERS:
        srcs = [int(src.page_table[b, p]) for b in range(src.batch) for p in range(lo, hi)]
        n = len(srcs)
        g = torch.Generator().manual_seed(seed * 31 + f)
        dst = torch.randperm(n, generator=g)
        rb = synth.row_bytes(f, d)
        jobs[f] = Job(f, n, torch.tensor(srcs, dtype=torch.int32, device=device),
                      dst.to(torch.int32).to(device),
                      torch.empty((n, Hkv, P, rb), dtype=torch.uint8, device=device),
                      torch.empty((n, Hkv, P, rb), dtype=torch.uint8, device=device),
                      torch.empty((n, Hkv, 2), dtype=torch.float32, device=device))
        lo = hi
    return Workload(src, binding.kv_pool_struct(src), jobs)


def run(w: Workload, err=None, stream=None) -> None:
    """One step: every planned page demoted (one library call per destination format)."""
    for f, j in w.jobs.items():
        st = binding.demote_pages(w.pool, synth.BF16, f, j.dst_k, j.dst_v, j.dst_scales,
                                  j.src_slots, j.dst_slots, None, err, stream)
        if st != binding.CFR_OK:
            raise binding.CfrError(st, "cfr_demote_pages")


def step_bytes(w: Workload) -> Dict[str, int]:
    """Algorithmic bytes of one step: every source page read once, every
    destination page and scale written once, the slot lists read."""
    src = w.src
    per_row_src = synth.row_bytes(synth.BF16, src.head_dim)
    rows = src.num_kv_heads * src.page_tokens * 2          # K and V rows of one page
    read = write = 0
    for f, j in w.jobs.items():
        read += j.n * rows * per_row_src + 8 * j.n
        write += j.n * rows * synth.row_bytes(f, src.head_dim) + j.n * src.num_kv_heads * 8
    return {"read": read, "write": write, "total": read + write,
            "pages": sum(j.n for j in w.jobs.values())}
