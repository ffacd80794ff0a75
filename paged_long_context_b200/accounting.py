"""Algorithmic byte and flop counts of one decode step (host logic for the roofline).

Bytes that any implementation must move at least once per step:
  K and V rows of every valid token of every (sequence, kv head), in their
  storage format; the int8/int4 scales of the pages read (8 bytes per page and
  kv head); the page-table entries (4 bytes per page of each sequence, plus 1
  byte of page format when a format array is used); q; out (fp32) and lse.
Flops: a q.k multiply-add and a p.v multiply-add per element per query head,
4 * Hq * d per token.
The per-head K+V byte count of an fp32 cache reproduces the CFR-Atlas page's
benchmark accounting (65,536 tokens x head_dim 64 -> 33,554,432 bytes).
With a sink + recent-window subset (window > 0) only the tokens j < sink and
j >= n - window count, and only the pages holding them.
"""
from __future__ import annotations

from . import synth


def kv_token_bytes(fmt: int, head_dim: int) -> int:
    """K+V bytes of one token of one kv head."""
    return 2 * synth.row_bytes(fmt, head_dim)


def _tokens_in_page(n: int, p: int, P: int, sink: int, window: int) -> int:
    lo, hi = p * P, min(n, (p + 1) * P)
    if window <= 0:
        return hi - lo
    keep = max(0, min(hi, sink) - lo)                      # sink tokens in [lo, hi)
    w0 = max(lo, n - window, min(hi, sink))                # window tokens not counted already
    return keep + max(0, hi - w0)


def step_bytes(case, sink: int = 0, window: int = 0) -> dict:
    lens = [int(x) for x in case.seq_lens.cpu().tolist()]
    P, d, Hkv = case.page_tokens, case.head_dim, case.num_kv_heads
    kv = 0
    scales = 0
    pages = 0
    tokens = 0
    for b, n in enumerate(lens):
        npg = -(-n // P)
        for p in range(npg):
            valid = _tokens_in_page(n, p, P, sink, window)
            if valid == 0:
                continue
            pages += 1
            tokens += valid
            f = case.fmt_of_page(b, p)
            kv += Hkv * valid * kv_token_bytes(f, d)
            if f in synth.QUANTISED:
                scales += Hkv * 8
    table = pages * (4 + (1 if case.page_fmt is not None else 0))
    rows = case.batch * case.num_q_heads * getattr(case, "num_queries", 1)   # query rows
    qb = rows * d * (4 if case.q_fmt == synth.F32 else 2)
    ob = rows * (d + 1) * 4
    total = kv + scales + table + qb + ob
    return {"kv": kv, "scales": scales, "page_table": table, "q": qb, "out": ob, "total": total,
            "tokens": tokens}


def step_flops(case) -> int:
    tokens = sum(int(x) for x in case.seq_lens.cpu().tolist())
    return 4 * case.num_q_heads * case.head_dim * tokens
