"""Seeded synthetic inputs for paged decode attention.

This module only *creates* inputs: query vectors, K/V page pools in their
storage formats, page tables, per-page formats, sequence lengths, ALiBi slopes
and head maps.  It holds none of the attention arithmetic (no dot products, no
softmax, no dequantisation, no merging).  Both the fp64 CPU oracle and the CUDA
library consume the bytes produced here; neither imports the other.

Storage layout (one pool per storage format, caller-owned):

    pool[f] : uint8 [pool_pages[f]][num_kv_heads][page_tokens][row_bytes(f)]

Each (physical page, kv head) sub-page is a contiguous row-major
[token][head_dim] block, the page content described on the CFR-Atlas page
(section "KvRegenerator": K and V written row-major [token][head_dim]).
row_bytes: F32 4*d, BF16 2*d, I8 d, I4 d/2, FP8 d.

Quantised pages (ARGUS page, "Visual Architecture": FP8, INT8, INT4 "2-way
bit-packed") carry one fp32 scale per (page, kv head, K-or-V):
scale = max|x| / 127 (int8), max|x| / 7 (int4) or max|x| / 448 (FP8 E4M3) over
the valid tokens of that block; integer codes = clamp(round_half_even(x /
scale)), FP8 codes = the E4M3 value nearest to x / scale.  int4 codes are 4-bit
two's complement; element 2i sits in the low nibble and element 2i+1 in the
high nibble of byte i of a row.  The quantiser is input generation: the
attention result depends only on the stored codes and scales.

Tokens past a sequence's length inside its last page are not part of the
input; float pools hold NaN there (and in unused pool slots) so that any stray
read shows up as a NaN in the output.

Every page is generated from its own seed (case seed, sequence, logical page),
so any page can be regenerated bit-identically into another physical slot; this
mirrors the deterministic page regeneration of the CFR-Atlas page
("KvRegenerator::regenerate_page(key, token_range, ...)").
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np
import torch

F32, BF16, I8, I4, FP8 = 0, 1, 2, 3, 4
FMT_COUNT = 5
FMT_NAMES = {F32: "f32", BF16: "bf16", I8: "i8", I4: "i4", FP8: "fp8"}
QUANTISED = (I8, I4, FP8)
FMT_BY_NAME = {v: k for k, v in FMT_NAMES.items()}

BF16_NAN_BITS = 0x7FC0
I8_FILL = 0x80  # code -128: never written by the quantiser
FP8_FILL = 0x7F  # E4M3 NaN: never written by the quantiser
FP8_MAX = 448.0  # largest finite E4M3 magnitude


def row_bytes(fmt: int, head_dim: int) -> int:
    """Bytes of one stored [head_dim] row in format ``fmt``."""
    if fmt == F32:
        return 4 * head_dim
    if fmt == BF16:
        return 2 * head_dim
    if fmt == I8:
        return head_dim
    if fmt == I4:
        return head_dim // 2
    if fmt == FP8:
        return head_dim
    raise ValueError(f"unknown page format {fmt}")


@dataclasses.dataclass
class DecodeCase:
    """One decode-attention problem: every buffer the library call takes."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_tokens: int
    max_pages: int
    seq_lens: torch.Tensor            # int32 [B]
    q_fmt: int                        # F32 or BF16
    q: torch.Tensor                   # f32 or bf16 bits [B][Q * Hq][d] = [B][Q][Hq][d]
    k_pool: Dict[int, torch.Tensor]   # fmt -> uint8 [pages][Hkv][P][row_bytes]
    v_pool: Dict[int, torch.Tensor]
    scales: Dict[int, torch.Tensor]   # I8/I4 -> f32 [pages][Hkv][2] (K scale, V scale)
    page_table: torch.Tensor          # int32 [B][max_pages]
    page_fmt: Optional[torch.Tensor]  # uint8 [B][max_pages] or None
    uniform_fmt: int
    head_map: Optional[torch.Tensor]  # int32 [Hq] or None
    alibi_slopes: Optional[torch.Tensor]  # f32 [Hq] or None
    softmax_scale: float              # 0.0 => 1/sqrt(head_dim)
    seed: int
    spec: dict
    num_queries: int = 1              # Q query tokens per sequence (the last Q positions)

    @property
    def device(self) -> torch.device:
        return self.page_table.device

    def pool_pages(self, fmt: int) -> int:
        t = self.k_pool.get(fmt)
        return 0 if t is None else int(t.shape[0])

    def to(self, device) -> "DecodeCase":
        """Copy of this case with every tensor on ``device``."""
        def mv(x):
            return None if x is None else x.to(device)
        return dataclasses.replace(
            self,
            seq_lens=mv(self.seq_lens), q=mv(self.q),
            k_pool={f: mv(t) for f, t in self.k_pool.items()},
            v_pool={f: mv(t) for f, t in self.v_pool.items()},
            scales={f: mv(t) for f, t in self.scales.items()},
            page_table=mv(self.page_table), page_fmt=mv(self.page_fmt),
            head_map=mv(self.head_map), alibi_slopes=mv(self.alibi_slopes))

    def fmt_of_page(self, b: int, p: int) -> int:
        if self.page_fmt is None:
            return self.uniform_fmt
        return int(self.page_fmt[b, p])


def _mix(*vals: int) -> int:
    """splitmix64-style combination of integers into one 63-bit seed."""
    x = 0x9E3779B97F4A7C15
    for v in vals:
        x = (x ^ (int(v) & 0xFFFFFFFFFFFFFFFF)) & 0xFFFFFFFFFFFFFFFF
        x = (x + 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & 0xFFFFFFFFFFFFFFFF
        x = z ^ (z >> 31)
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def alibi_slopes(num_q_heads: int) -> torch.Tensor:
    """Standard geometric ALiBi slopes 2^(-8(h+1)/Hq), h = 0..Hq-1, as fp32."""
    return torch.tensor([2.0 ** (-8.0 * (h + 1) / num_q_heads) for h in range(num_q_heads)],
                        dtype=torch.float32)


def _quant_int(x: torch.Tensor, valid: int, qmax: int):
    """Symmetric per-(kv head) quantisation of one page block x: f32 [Hkv][P][d].

    scale = max|x| / qmax over the first ``valid`` tokens; codes clamp to
    [-qmax, qmax].  Returns (int codes [Hkv][P][d] as int16, scale f32 [Hkv]).
    """
    xv = x[:, :valid, :]
    amax = xv.abs().amax(dim=(1, 2))                   # [Hkv]
    scale = amax / float(qmax)                         # fp32 division
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    codes = torch.round(x / safe[:, None, None]).clamp_(-qmax, qmax)
    codes = torch.where(scale[:, None, None] > 0, codes, torch.zeros_like(codes))
    return codes.to(torch.int16), scale


def _quant_fp8(x: torch.Tensor, valid: int):
    """E4M3 encoding of one page block x: f32 [Hkv][P][d] with scale max|x| / 448.

    Returns (uint8 codes [Hkv][P][d], scale f32 [Hkv]); an all-zero block gets
    scale 0 and zero codes.
    """
    xv = x[:, :valid, :]
    amax = xv.abs().amax(dim=(1, 2))
    scale = amax / FP8_MAX
    safe = torch.where(scale > 0, scale, torch.ones_like(scale))
    y = (x / safe[:, None, None]).clamp_(-FP8_MAX, FP8_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).clone()
    codes = torch.where(scale[:, None, None] > 0, codes, torch.zeros_like(codes))
    return codes, scale


def _pack_int4(codes: torch.Tensor) -> torch.Tensor:
    """codes int16 [..., d] in [-8, 7] -> uint8 [..., d/2]; even element in the low nibble."""
    nib = (codes & 0xF).to(torch.uint8)
    return nib[..., 0::2] | (nib[..., 1::2] << 4)


def _encode_page(x: torch.Tensor, fmt: int, valid: int):
    """Encode one page block x f32 [Hkv][P][d] into pool bytes uint8 [Hkv][P][row_bytes].

    Rows at or past ``valid`` are filled with NaN (float formats and FP8) or
    code -128 (int8) / nibble 8 (int4).  Returns (bytes, scale or None).
    """
    hkv, ptok, d = x.shape
    if fmt == F32:
        y = x.clone()
        y[:, valid:, :] = float("nan")
        return y.contiguous().view(torch.uint8).reshape(hkv, ptok, 4 * d), None
    if fmt == BF16:
        y = x.to(torch.bfloat16).view(torch.int16)
        y[:, valid:, :] = BF16_NAN_BITS
        return y.contiguous().view(torch.uint8).reshape(hkv, ptok, 2 * d), None
    if fmt == I8:
        codes, scale = _quant_int(x, valid, 127)
        b = codes.to(torch.int8).view(torch.uint8).clone()
        b[:, valid:, :] = I8_FILL
        return b, scale
    if fmt == I4:
        codes, scale = _quant_int(x, valid, 7)
        codes[:, valid:, :] = -8
        return _pack_int4(codes), scale
    if fmt == FP8:
        codes, scale = _quant_fp8(x, valid)
        codes[:, valid:, :] = FP8_FILL
        return codes, scale
    raise ValueError(fmt)


@dataclasses.dataclass
class CaseSpec:
    """Shape and structure of one synthetic decode problem."""

    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_tokens: int
    seq_lens: Sequence[int] = ()          # explicit lengths, or
    len_range: Optional[tuple] = None     # (lo, hi) inclusive, drawn uniformly from the seed
    fmt: str = "bf16"                     # uniform storage format, or "tiered"
    tiers: Optional[List[tuple]] = None   # [(fraction of oldest pages, fmt name), ...] oldest first
    q_fmt: str = "bf16"
    permute: bool = True                  # pages placed in the pool by a seeded permutation
    alibi: bool = False
    head_map: Optional[Sequence[int]] = None
    softmax_scale: float = 0.0
    spare_pages: int = 0                  # extra unused pool slots (NaN / fill bytes)
    use_page_fmt: Optional[bool] = None   # force passing a page_fmt array
    num_queries: int = 1                  # query tokens per sequence (speculative / chunked)


def tier_of_page(spec: CaseSpec, p: int, num_pages: int) -> int:
    """Storage format of logical page p of a sequence with num_pages pages.

    With ``tiers`` = [(frac_0, fmt_0), (frac_1, fmt_1), ...] listed oldest first,
    logical pages [0, round(frac_0*NP)) get fmt_0, the next round(frac_1*NP)
    get fmt_1, and the remainder the last format.
    """
    if spec.fmt != "tiered":
        return FMT_BY_NAME[spec.fmt]
    edge = 0
    for i, (frac, name) in enumerate(spec.tiers):
        if i == len(spec.tiers) - 1:
            return FMT_BY_NAME[name]
        edge += int(round(frac * num_pages))
        if p < edge:
            return FMT_BY_NAME[name]
    return FMT_BY_NAME[spec.tiers[-1][1]]


def make_case(spec: CaseSpec, seed: int, device="cpu") -> DecodeCase:
    """Build every input buffer of one decode problem, seeded, on ``device``."""
    device = torch.device(device)
    B, Hq, Hkv, d, P = spec.batch, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.page_tokens
    if spec.len_range is not None:
        lo, hi = spec.len_range
        g = _gen("cpu", _mix(seed, 0x5E9))
        lens = torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    else:
        lens = torch.tensor(list(spec.seq_lens), dtype=torch.int32)
        assert lens.numel() == B
    npages = [max(0, -(-int(n) // P)) for n in lens.tolist()]
    max_pages = max(1, max(npages))

    # formats of every (b, logical page) and the pool each one goes to
    fmts = [[tier_of_page(spec, p, npages[b]) for p in range(npages[b])] for b in range(B)]
    count = {f: 0 for f in range(FMT_COUNT)}
    for b in range(B):
        for f in fmts[b]:
            count[f] += 1
    used = [f for f in range(FMT_COUNT) if count[f] > 0]
    if not used:
        used = [FMT_BY_NAME[spec.fmt] if spec.fmt != "tiered" else BF16]
    total = {f: count[f] + spec.spare_pages for f in used}

    # seeded physical placement per format pool
    gperm = _gen("cpu", _mix(seed, 0x9E7))
    perm = {}
    for f in used:
        perm[f] = (torch.randperm(total[f], generator=gperm) if spec.permute
                   else torch.arange(total[f]))

    k_pool, v_pool, scales = {}, {}, {}
    for f in used:
        rb = row_bytes(f, d)
        shape = (total[f], Hkv, P, rb)
        if f == F32:
            k_pool[f] = torch.full((total[f], Hkv, P, d), float("nan"), device=device).view(torch.uint8).reshape(shape)
            v_pool[f] = torch.full((total[f], Hkv, P, d), float("nan"), device=device).view(torch.uint8).reshape(shape)
        elif f == BF16:
            k_pool[f] = torch.full((total[f], Hkv, P, d), BF16_NAN_BITS, dtype=torch.int16, device=device).view(torch.uint8).reshape(shape)
            v_pool[f] = torch.full((total[f], Hkv, P, d), BF16_NAN_BITS, dtype=torch.int16, device=device).view(torch.uint8).reshape(shape)
        else:
            fill = I8_FILL if f == I8 else FP8_FILL if f == FP8 else 0x88
            k_pool[f] = torch.full(shape, fill, dtype=torch.uint8, device=device)
            v_pool[f] = torch.full(shape, fill, dtype=torch.uint8, device=device)
            scales[f] = torch.zeros((total[f], Hkv, 2), dtype=torch.float32, device=device)

    page_table = torch.full((B, max_pages), -1, dtype=torch.int32)
    page_fmt = torch.full((B, max_pages), 255, dtype=torch.uint8)
    nxt = {f: 0 for f in used}
    for b in range(B):
        n = int(lens[b])
        for p in range(npages[b]):
            f = fmts[b][p]
            pid = int(perm[f][nxt[f]])
            nxt[f] += 1
            page_table[b, p] = pid
            page_fmt[b, p] = f
            valid = min(P, n - p * P)
            write_page(k_pool, v_pool, scales, f, pid, seed, b, p, Hkv, P, d, valid, device)

    uniform = fmts[0][0] if (B > 0 and npages[0] > 0) else used[0]
    mixed = len({f for row in fmts for f in row}) > 1
    use_pf = spec.use_page_fmt if spec.use_page_fmt is not None else mixed

    gq = _gen(device, _mix(seed, 0x0A11))
    Q = max(1, int(spec.num_queries))
    qf = torch.randn((B, Q * Hq, d), generator=gq, device=device, dtype=torch.float32)
    if spec.q_fmt == "f32":
        q, q_fmt = qf, F32
    else:
        q, q_fmt = qf.to(torch.bfloat16).view(torch.int16), BF16

    head_map = None if spec.head_map is None else torch.tensor(list(spec.head_map), dtype=torch.int32)
    slopes = alibi_slopes(Hq) if spec.alibi else None
    return DecodeCase(
        name=spec.name, batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=d, page_tokens=P,
        max_pages=max_pages, seq_lens=lens.to(device), q_fmt=q_fmt, q=q,
        k_pool=k_pool, v_pool=v_pool, scales=scales,
        page_table=page_table.to(device), page_fmt=page_fmt.to(device) if use_pf else None,
        uniform_fmt=uniform, head_map=None if head_map is None else head_map.to(device),
        alibi_slopes=None if slopes is None else slopes.to(device),
        softmax_scale=float(spec.softmax_scale), seed=seed, spec=dataclasses.asdict(spec), num_queries=Q)


def page_values(seed: int, b: int, p: int, hkv: int, P: int, d: int, device):
    """The fp32 N(0,1) K and V values of logical page p of sequence b: [Hkv][P][d] each."""
    gk = _gen(device, _mix(seed, b, p, 0xC0))
    gv = _gen(device, _mix(seed, b, p, 0xC1))
    k = torch.randn((hkv, P, d), generator=gk, device=device, dtype=torch.float32)
    v = torch.randn((hkv, P, d), generator=gv, device=device, dtype=torch.float32)
    return k, v


def write_page(k_pool, v_pool, scales, f, pid, seed, b, p, hkv, P, d, valid, device):
    """(Re)generate logical page p of sequence b into physical slot ``pid`` of pool ``f``."""
    k, v = page_values(seed, b, p, hkv, P, d, device)
    kb, ks = _encode_page(k, f, valid)
    vb, vs = _encode_page(v, f, valid)
    k_pool[f][pid].copy_(kb)
    v_pool[f][pid].copy_(vb)
    if ks is not None:
        scales[f][pid, :, 0] = ks
        scales[f][pid, :, 1] = vs


def regenerate_into(case: DecodeCase, b: int, p: int, new_pid: int) -> None:
    """Regenerate logical page p of sequence b into slot ``new_pid`` and repoint the page table."""
    f = case.fmt_of_page(b, p)
    valid = min(case.page_tokens, int(case.seq_lens[b]) - p * case.page_tokens)
    write_page(case.k_pool, case.v_pool, case.scales, f, new_pid, case.seed, b, p,
               case.num_kv_heads, case.page_tokens, case.head_dim, valid, case.device)
    case.page_table[b, p] = new_pid


def permute_pool(case: DecodeCase, seed: int) -> DecodeCase:
    """Same logical content with every format pool re-permuted (page table updated)."""
    g = _gen("cpu", _mix(seed, 0x7E7))
    new_k, new_v, new_s, perms = {}, {}, {}, {}
    for f in case.k_pool:
        n = case.k_pool[f].shape[0]
        perm = torch.randperm(n, generator=g)            # old slot i -> new slot perm[i]
        inv = torch.empty_like(perm)
        inv[perm] = torch.arange(n)
        idx = inv.to(case.device)
        new_k[f] = case.k_pool[f][idx].contiguous()
        new_v[f] = case.v_pool[f][idx].contiguous()
        if f in case.scales:
            new_s[f] = case.scales[f][idx].contiguous()
        perms[f] = perm
    pt = case.page_table.cpu().clone()
    lens = case.seq_lens.cpu()
    for b in range(case.batch):
        for p in range(-(-int(lens[b]) // case.page_tokens)):
            f = case.fmt_of_page(b, p)
            pt[b, p] = int(perms[f][int(pt[b, p])])
    return dataclasses.replace(case, k_pool=new_k, v_pool=new_v, scales=new_s,
                               page_table=pt.to(case.device))


# ---------------------------------------------------------------------------
# The five workloads of the pages (shapes only), plus the bounded samples used
# by tests.  Names describe the workload itself.
# ---------------------------------------------------------------------------

def spec_tiny_exact_fold() -> CaseSpec:
    """1 sequence, 1 head, d 64, 4096 tokens, 512-token pages (8), identity table, fp32."""
    return CaseSpec("tiny_exact_fold_4k_f32", 1, 1, 1, 64, 512, seq_lens=[4096], fmt="f32",
                    q_fmt="f32", permute=False, softmax_scale=1.0 / 8.0)


def spec_cfr_shaped() -> CaseSpec:
    """1 sequence, 32 MHA heads, d 64, 65,536 tokens, 512-token pages, fp32, permuted pool."""
    return CaseSpec("cfr_64k_mha32_d64_f32", 1, 32, 32, 64, 512, seq_lens=[65536], fmt="f32",
                    q_fmt="f32", permute=True)


def spec_gqa_ragged() -> CaseSpec:
    """16 sequences of 1K-32K tokens, 32 q / 8 kv heads, d 128, bf16, 16-token pages."""
    return CaseSpec("gqa_ragged_b16_1k32k_p16_bf16", 16, 32, 8, 128, 16, len_range=(1024, 32768),
                    fmt="bf16", q_fmt="bf16", permute=True)


def spec_tiered() -> CaseSpec:
    """8 x 32K tokens, 32 q / 8 kv heads, d 128, 256-token pages: int4 | int8 | bf16 tiers."""
    return CaseSpec("tiered_b8_32k_p256_i4i8bf16", 8, 32, 8, 128, 256, seq_lens=[32768] * 8,
                    fmt="tiered", tiers=[(0.25, "i4"), (0.50, "i8"), (0.25, "bf16")],
                    q_fmt="bf16", permute=True)


def spec_alibi_1m() -> CaseSpec:
    """1 x 1,048,576 tokens, 64 q / 8 kv heads, d 128, bf16, 512-token pages, ALiBi."""
    return CaseSpec("alibi_1m_gqa64x8_p512_bf16", 1, 64, 8, 128, 512, seq_lens=[1 << 20],
                    fmt="bf16", q_fmt="bf16", permute=True, alibi=True)


def spec_mqa() -> CaseSpec:
    """8 x 32,768 tokens, 32 q heads on 1 kv head (MQA), d 128, bf16, 256-token pages."""
    return CaseSpec("mqa_b8_32k_32q1kv_p256_bf16", 8, 32, 1, 128, 256, seq_lens=[32768] * 8,
                    fmt="bf16", q_fmt="bf16", permute=True)


def spec_gqa_d64() -> CaseSpec:
    """The ragged GQA batch at head_dim 64: 16 sequences of 1K-32K tokens, 32 q / 8 kv
    heads, bf16, 16-token pages (the tensor-core kernel, first half of its operands)."""
    return CaseSpec("gqa_ragged_b16_1k32k_p16_bf16_d64", 16, 32, 8, 64, 16,
                    len_range=(1024, 32768), fmt="bf16", q_fmt="bf16", permute=True)


def spec_gqa_d64_i8_p16() -> CaseSpec:
    """The same batch as int8 pages of 16 tokens, head_dim 64 (the tensor-core
    kernel: a tile holds 8 pages, each with its own scales)."""
    return CaseSpec("gqa_ragged_b16_1k32k_p16_i8_d64", 16, 32, 8, 64, 16,
                    len_range=(1024, 32768), fmt="i8", q_fmt="bf16", permute=True)


def spec_gqa_i8_p16() -> CaseSpec:
    """The ragged GQA batch as int8 pages of 16 tokens, head_dim 128 (the
    tensor-core kernel's int8 MMAs: a tile holds 8 pages, each with its scales)."""
    return CaseSpec("gqa_ragged_b16_1k32k_p16_i8", 16, 32, 8, 128, 16, len_range=(1024, 32768),
                    fmt="i8", q_fmt="bf16", permute=True)


def spec_gqa_d64_mixed_p16() -> CaseSpec:
    """The same batch with int8 and bf16 pages of 16 tokens mixed, head_dim 64: a
    shape only the general CUDA-core kernel takes (quantised pages under 128
    tokens among other formats)."""
    return CaseSpec("gqa_ragged_b16_1k32k_p16_i8bf16_d64", 16, 32, 8, 64, 16,
                    len_range=(1024, 32768), fmt="tiered", tiers=[(0.5, "i8"), (0.5, "bf16")],
                    q_fmt="bf16", permute=True)


WORKLOADS = {
    "tiny": (spec_tiny_exact_fold, 1),
    "cfr": (spec_cfr_shaped, 2),
    "gqa": (spec_gqa_ragged, 3),
    "tiered": (spec_tiered, 4),
    "alibi1m": (spec_alibi_1m, 5),
    "mqa": (spec_mqa, 6),
    "gqa_d64": (spec_gqa_d64, 7),
    "gqa_d64_i8p16": (spec_gqa_d64_i8_p16, 7),
    "gqa_d64_mixed_p16": (spec_gqa_d64_mixed_p16, 7),
    "gqa_i8p16": (spec_gqa_i8_p16, 3),
}


def workload(name: str, device="cpu", num_queries: int = 1,
             context: Optional[int] = None) -> DecodeCase:
    """One of the page-shaped workloads, with its fixed seed (optionally with
    several query tokens per sequence, or with every sequence cut to `context`
    tokens: the same shape at a smaller size, e.g. for a profiler capture)."""
    fn, seed = WORKLOADS[name]
    spec = fn()
    if num_queries > 1:
        spec = dataclasses.replace(spec, num_queries=num_queries,
                                   name=f"{spec.name}_q{num_queries}")
    if context is not None:
        spec = dataclasses.replace(spec, seq_lens=[int(context)] * spec.batch, len_range=None,
                                   name=f"{spec.name}_n{int(context)}")
    return make_case(spec, seed, device)


def merge_inputs(num_splits: Sequence[int], num_q_heads: int, head_dim: int, seed: int,
                 empty_frac: float = 0.0, device="cpu"):
    """Random split partials for the LSE merge: (part_acc, part_m, part_l, split_off).

    part_m are base-2 running maxima, part_l positive normalisers (0 for an
    empty split), part_acc arbitrary accumulators; split_off[b+1]-split_off[b]
    = num_splits[b].
    """
    g = _gen("cpu", _mix(seed, 0x3E6))
    S = int(sum(num_splits))
    off = torch.zeros(len(num_splits) + 1, dtype=torch.int32)
    off[1:] = torch.cumsum(torch.tensor(list(num_splits), dtype=torch.int64), 0).to(torch.int32)
    m = (torch.randn((S, num_q_heads), generator=g) * 8.0).float()
    l = (torch.rand((S, num_q_heads), generator=g) * 100.0 + 1.0).float()
    acc = (torch.randn((S, num_q_heads, head_dim), generator=g) * 10.0).float()
    if empty_frac > 0:
        e = torch.rand((S, num_q_heads), generator=g) < empty_frac
        l[e] = 0.0
        m[e] = float("-inf")
        acc[e] = 0.0
    return acc.to(device), m.to(device), l.to(device), off.to(device)
