"""GPU parity of page demotion and KV append against the oracle, through the C ABI.

Demotion codes and scales are integer / byte decisions taken in fp32 on both
sides, so the bar is bit-exact.  Append is a byte copy (with bf16 rounding),
also bit-exact.  A demoted or appended cache then decodes to the oracle's
attention result within the decode tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._gpu import check, run, small_case

pytestmark = pytest.mark.gpu

F32, BF16, I8, I4, FP8 = synth.F32, synth.BF16, synth.I8, synth.I4, synth.FP8
FMTS = [F32, BF16, I8, I4, FP8]
QUANTISED = synth.QUANTISED


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


def _src_case(fmt, d, P, lens, seed=5):
    return small_case(B=len(lens), Hq=4, Hkv=2, d=d, P=P, lens=lens, fmt=synth.FMT_NAMES[fmt],
                      q_fmt="bf16", seed=seed)


def _pages_of(case):
    """(slot, valid tokens) of every page of every sequence."""
    out = []
    P = case.page_tokens
    for b in range(case.batch):
        n = int(case.seq_lens[b])
        for p in range(-(-n // P)):
            out.append((int(case.page_table[b, p]), min(P, n - p * P)))
    return out


def _demote_both(case, src, dst, src_slots, dst_slots, valid, n_dst):
    """Demote on the GPU and in the oracle; returns both results on the host."""
    Hkv, d, P = case.num_kv_heads, case.head_dim, case.page_tokens
    rb = synth.row_bytes(dst, d)
    dk = torch.full((n_dst, Hkv, P, rb), 0xAB, dtype=torch.uint8, device="cuda")
    dv = torch.full_like(dk, 0xAB)
    dsc = torch.full((n_dst, Hkv, 2), -1.0, device="cuda") if dst in QUANTISED else None
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = binding.kv_pool_struct(case)
    st = binding.demote_pages(pool, src, dst, dk, dv, dsc,
                              torch.tensor(src_slots, dtype=torch.int32, device="cuda"),
                              torch.tensor(dst_slots, dtype=torch.int32, device="cuda"),
                              torch.tensor(valid, dtype=torch.int32, device="cuda"), err)
    assert st == 0
    torch.cuda.synchronize()
    hk, hv = dk.cpu(), dv.cpu()
    hsc = None if dsc is None else dsc.cpu()
    ok = torch.full((n_dst, Hkv, P, rb), 0xAB, dtype=torch.uint8)
    ov = ok.clone()
    osc = torch.full((n_dst, Hkv, 2), -1.0) if dst in QUANTISED else None
    sc = case.scales[src].cpu().contiguous() if src in QUANTISED else None
    oerr = oracle.demote(Hkv, d, P, src, case.k_pool[src].cpu().contiguous(),
                         case.v_pool[src].cpu().contiguous(), sc, dst, ok, ov, osc,
                         src_slots, dst_slots, valid)
    return (hk, hv, hsc, int(err.item())), (ok, ov, osc, oerr)


@pytest.mark.parametrize("src", FMTS, ids=lambda f: synth.FMT_NAMES[f])
@pytest.mark.parametrize("dst", FMTS, ids=lambda f: synth.FMT_NAMES[f])
@pytest.mark.parametrize("d,P", [(64, 16), (128, 256)])
def test_demote_bit_exact(src, dst, d, P):
    if src == dst:
        pytest.skip("same format")
    case = _src_case(src, d, P, lens=(5 * P + 3, P, 2 * P - 1))
    pages = _pages_of(case)
    n = len(pages)
    g = torch.Generator().manual_seed(n)
    dst_slots = torch.randperm(n + 3, generator=g)[:n].tolist()
    (hk, hv, hsc, err), (ok, ov, osc, oerr) = _demote_both(
        case, src, dst, [s for s, _ in pages], dst_slots, [v for _, v in pages], n + 3)
    assert err == 0 and oerr == 0
    assert torch.equal(hk, ok) and torch.equal(hv, ov)
    if hsc is not None:
        assert torch.equal(hsc, osc)


@pytest.mark.parametrize("dst", [I8, I4], ids=["int8", "int4"])
@pytest.mark.parametrize("d,P", [(64, 512), (128, 512), (128, 264)])
def test_demote_bf16_block_size_boundary(dst, d, P):
    # bf16 blocks of exactly 64 KiB (d 64, 512-token pages) take the shared-memory
    # kernel; larger ones (d 128 at 512 or 264 tokens) the general one: both
    # bit-exact, including a partial last page
    case = _src_case(BF16, d, P, lens=(2 * P - 5, P))
    pages = _pages_of(case)
    n = len(pages)
    (hk, hv, hsc, err), (ok, ov, osc, oerr) = _demote_both(
        case, BF16, dst, [s for s, _ in pages], list(range(n)), [v for _, v in pages], n)
    assert err == 0 and oerr == 0
    assert torch.equal(hk, ok) and torch.equal(hv, ov) and torch.equal(hsc, osc)


@pytest.mark.parametrize("src,dst", [(I8, I4), (I8, FP8), (FP8, I8), (FP8, I4)],
                         ids=["int8-int4", "int8-fp8", "fp8-int8", "fp8-int4"])
def test_demote_quantised_source_every_code(src, dst):
    # every one of the 256 source codes in each block, under K/V scales that
    # include zero, a subnormal, a negative, an infinite and a NaN scale; codes
    # and scales byte for byte against the oracle
    Hkv, P, d = 2, 16, 128
    scales = [1.0, 0.0123, 3.7e-3, 1e-39, 0.0, -0.5, float("inf"), float("nan")]
    nblk = len(scales)
    npages = -(-nblk // (2 * Hkv))
    case = _src_case(src, d, P, lens=(P * npages,), seed=17)
    pages = _pages_of(case)
    rng = np.random.default_rng(src * 7 + dst)
    k = case.k_pool[src]
    v = case.v_pool[src]
    sc = case.scales[src]
    for i, s_ in enumerate(scales):
        j, rest = divmod(i, 2 * Hkv)
        g, kv = divmod(rest, 2)
        codes = np.resize(np.arange(256, dtype=np.uint8), P * d)
        rng.shuffle(codes)
        (v if kv else k)[pages[j][0], g] = torch.from_numpy(codes.reshape(P, d)).to(k.device)
        sc[pages[j][0], g, kv] = s_
    n = len(pages)
    (hk, hv, hsc, err), (ok, ov, osc, oerr) = _demote_both(
        case, src, dst, [s for s, _ in pages], list(range(n)), [v_ for _, v_ in pages], n)
    assert err == 0 and oerr == 0
    assert torch.equal(hk, ok) and torch.equal(hv, ov)
    assert torch.equal(hsc.view(torch.int32), osc.view(torch.int32))


def test_demote_reports_and_skips_bad_pages():
    case = _src_case(BF16, 128, 16, lens=(64,))
    pages = _pages_of(case)
    src = [s for s, _ in pages] + [10_000, pages[0][0], pages[1][0]]
    dst = list(range(len(pages))) + [len(pages), 99, len(pages) + 1]
    valid = [v for _, v in pages] + [16, 16, 0]
    (hk, hv, hsc, err), (ok, ov, osc, oerr) = _demote_both(case, BF16, I8, src, dst, valid,
                                                           len(pages) + 2)
    assert err == binding.DEVERR_PAGE_ID | binding.DEVERR_SEQ_LEN
    assert oerr == oracle.DEV_PAGE_ID | oracle.DEV_SEQ_LEN
    assert torch.equal(hk, ok) and torch.equal(hsc, osc)
    assert int((hk[len(pages):] != 0xAB).sum()) == 0            # skipped pages untouched


# ---------------------------------------------------------------------------
# bf16 -> int8 / int4 over every bf16 input, and the blocks at the edges of the
# encoder (ties, NaN, infinities, zero and subnormal scales)
# ---------------------------------------------------------------------------

def _bf16_blocks_case(blocks, seed=11):
    """A bf16 cache (head_dim 128, 16-token pages, 2 kv heads) whose first
    len(blocks) (page, kv head, K-or-V) blocks hold the given bf16 bit patterns
    (2048 each, in the order the demotion numbers its blocks); the rest keep the
    generator's values."""
    Hkv, P, d = 2, 16, 128
    per_page = 2 * Hkv
    npages = -(-len(blocks) // per_page)
    case = _src_case(BF16, d, P, lens=(P * npages,), seed=seed)
    pages = _pages_of(case)
    k = case.k_pool[BF16].view(torch.int16)
    v = case.v_pool[BF16].view(torch.int16)
    for i, bits in enumerate(blocks):
        j, rest = divmod(i, per_page)
        g, kv = divmod(rest, 2)
        t = torch.from_numpy(np.asarray(bits, dtype=np.uint16).view(np.int16).reshape(P, d))
        (v if kv else k)[pages[j][0], g] = t.to(k.device)
    return case, pages


def _demote_blocks_exact(blocks, dst):
    case, pages = _bf16_blocks_case(blocks)
    n = len(pages)
    (hk, hv, hsc, err), (ok, ov, osc, oerr) = _demote_both(
        case, BF16, dst, [s for s, _ in pages], list(range(n)), [v for _, v in pages], n)
    assert err == 0 and oerr == 0
    assert torch.equal(hsc, osc)
    assert torch.equal(hk, ok) and torch.equal(hv, ov)
    return hsc


@pytest.mark.parametrize("dst", [I8, I4, FP8], ids=["int8", "int4", "fp8"])
@pytest.mark.parametrize("amax_bits", [0x3F80, 0x3F4A, 0x4040, 0x3FFE, 0x7F00, 0x0D80, 0x0400, 0x0300],
                         ids=lambda b: f"amax{b:04x}")
def test_demote_bf16_to_int_every_input(dst, amax_bits):
    # every bf16 value of magnitude up to max|x| (both signs, zeros and
    # subnormals included), shuffled over blocks that each also hold max|x|,
    # so every block has the same scale: each possible input of that scale is
    # encoded once and compared byte for byte with the oracle.  0x0400 gives
    # the smallest normal scales (2^-119 / Q); 0x0300 a subnormal scale.
    rng = np.random.default_rng(amax_bits)
    mags = np.arange(0, amax_bits + 1, dtype=np.uint32)
    vals = np.concatenate([mags, mags | 0x8000]).astype(np.uint16)
    rng.shuffle(vals)
    chunk = 2047
    blocks = []
    for c0 in range(0, len(vals), chunk):
        part = vals[c0:c0 + chunk]
        part = np.concatenate([part, np.full(chunk - len(part), amax_bits, np.uint16)])
        blk = np.concatenate([[amax_bits], part]).astype(np.uint16)
        rng.shuffle(blk)
        blocks.append(blk)
    sc = _demote_blocks_exact(blocks, dst)
    assert bool((sc.view(-1)[: len(blocks)] > 0).all())


@pytest.mark.parametrize("dst", [I8, I4, FP8], ids=["int8", "int4", "fp8"])
def test_demote_bf16_to_int_edge_blocks(dst):
    rng = np.random.default_rng(3)
    n = 2048

    def finite(lo_bits=0x3000, hi_bits=0x3F80):
        m = rng.integers(lo_bits, hi_bits, size=n, dtype=np.uint32)
        return (m | (rng.integers(0, 2, size=n, dtype=np.uint32) << 15)).astype(np.uint16)

    blocks = []
    if dst == FP8:
        # scale 1 (max|x| = 448): every midpoint between neighbouring E4M3 values,
        # both signs, each an exact tie of the E4M3 rounding
        vals = np.array([float(torch.tensor([c], dtype=torch.uint8).view(torch.float8_e4m3fn).float())
                         for c in range(0x7F)])
        mids = (vals[:-1] + vals[1:]) / 2
        mids = np.concatenate([mids, -mids])
        ties = np.resize(mids, n)
        rng.shuffle(ties)
        ties[0] = 448.0
        unit = 1.0
    else:
        # exact ties: scale = 2^-6 (int8) or 2^-2 (int4), values (k + 1/2) * scale
        q = 127 if dst == I8 else 7
        unit = 64 if dst == I8 else 4
        ks = rng.integers(-q, q, size=n)
        ties = (ks + 0.5) / unit
        ties[0] = q / unit
    blocks.append(torch.tensor(ties, dtype=torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    # NaNs (with payloads and signs) among finite values: max|x| ignores them, their codes are 0
    b = finite()
    b[rng.choice(n, 40, replace=False)] = np.array([0x7FC0, 0x7FC1, 0xFFC0, 0x7F81] * 10, np.uint16)
    blocks.append(b)
    # an infinity: scale is infinite and every code 0
    b = finite()
    b[5] = 0x7F80
    blocks.append(b)
    b = np.zeros(n, np.uint16)
    b[100] = 0xFF80
    blocks.append(b)
    # all zeros of both signs: scale 0
    blocks.append((rng.integers(0, 2, size=n, dtype=np.uint32) << 15).astype(np.uint16))
    # subnormals only (scale subnormal)
    blocks.append(finite(0x0001, 0x0080))
    # a subnormal maximum among zeros
    b = np.zeros(n, np.uint16)
    b[7] = 0x0001
    blocks.append(b)
    # large magnitudes next to the largest finite bf16
    blocks.append(finite(0x7E00, 0x7F80))
    # tiny values under a normal maximum (codes 0 and +-1)
    b = finite(0x0001, 0x0400)
    b[9] = 0x0C00
    blocks.append(b)
    sc = _demote_blocks_exact(blocks, dst)
    assert float(sc.view(-1)[0]) == 1.0 / unit


@pytest.mark.parametrize("P", [16, 256])
def test_demoted_cache_decodes(P):
    # a bf16 cache whose oldest pages are demoted on the GPU to int4 / int8 / FP8
    # (the compression cascade), then decoded: parity with the oracle on the
    # demoted cache
    case = small_case(B=3, Hq=8, Hkv=2, d=128, P=P, lens=(12 * P + 5, 6 * P, 3 * P + 1),
                      fmt="bf16", alibi=True, seed=21)
    Hkv, d = case.num_kv_heads, case.head_dim
    plan = {I4: [], I8: [], FP8: []}
    for b in range(case.batch):
        n = int(case.seq_lens[b])
        np_ = -(-n // P)
        for p in range(np_ - 1):                        # the last (hot) page stays bf16
            tier = I4 if p < np_ // 4 else I8 if p < np_ // 2 else FP8 if p < 3 * np_ // 4 else None
            if tier is not None:
                plan[tier].append((b, p, min(P, n - p * P)))
    pools_k, pools_v, scales = {BF16: case.k_pool[BF16]}, {BF16: case.v_pool[BF16]}, {}
    page_fmt = torch.full((case.batch, case.max_pages), BF16, dtype=torch.uint8)
    page_table = case.page_table.clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    src_pool = binding.kv_pool_struct(case)
    for f, items in plan.items():
        rb = synth.row_bytes(f, d)
        k = torch.zeros((len(items), Hkv, P, rb), dtype=torch.uint8, device="cuda")
        v = torch.zeros_like(k)
        s = torch.zeros((len(items), Hkv, 2), device="cuda")
        src_slots = torch.tensor([int(case.page_table[b, p]) for b, p, _ in items],
                                 dtype=torch.int32, device="cuda")
        valid = torch.tensor([n for _, _, n in items], dtype=torch.int32, device="cuda")
        dst_slots = torch.arange(len(items), dtype=torch.int32, device="cuda")
        assert binding.demote_pages(src_pool, BF16, f, k, v, s, src_slots, dst_slots, valid,
                                    err) == 0
        pools_k[f], pools_v[f], scales[f] = k, v, s
        for i, (b, p, _) in enumerate(items):
            page_table[b, p] = i
            page_fmt[b, p] = f
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    case.k_pool, case.v_pool, case.scales = pools_k, pools_v, scales
    case.page_table = page_table.to("cuda")
    case.page_fmt = page_fmt.to("cuda")
    out, lse, err2 = run(case)
    assert err2 == 0
    check(case, out, lse)


@pytest.mark.parametrize("page_fmt", [F32, BF16])
@pytest.mark.parametrize("new_fmt", [F32, BF16])
def test_append_bit_exact_and_decodes(page_fmt, new_fmt):
    P, d, Hkv = 16, 128, 2
    lens = (37, 16, 5)
    case = small_case(B=3, Hq=4, Hkv=Hkv, d=d, P=P, lens=lens, fmt=synth.FMT_NAMES[page_fmt],
                      q_fmt="bf16", spare_pages=2, seed=8)
    # sequence 1 fills its page exactly: give it the next page from the spare slots
    pt = case.page_table.clone()
    if pt.shape[1] < 3:
        pt = torch.cat([pt, torch.full((3, 3 - pt.shape[1]), -1, dtype=torch.int32,
                                       device=pt.device)], 1)
    used = set(int(x) for x in pt[pt >= 0].tolist())
    spare = [i for i in range(case.k_pool[page_fmt].shape[0]) if i not in used]
    pt[1, 1] = spare[0]
    case.page_table, case.max_pages = pt, pt.shape[1]
    g = torch.Generator().manual_seed(4)
    kn = torch.randn((3, Hkv, d), generator=g)
    vn = torch.randn((3, Hkv, d), generator=g)
    if new_fmt == BF16:
        kn, vn = kn.to(torch.bfloat16), vn.to(torch.bfloat16)
    positions = torch.tensor(lens, dtype=torch.int32)
    host_k = {page_fmt: case.k_pool[page_fmt].cpu().contiguous()}
    host_v = {page_fmt: case.v_pool[page_fmt].cpu().contiguous()}
    oerr = oracle.append(Hkv, d, P, host_k, host_v, pt.cpu(), None, page_fmt, positions, new_fmt,
                         kn, vn)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = binding.kv_pool_struct(case)
    st = binding.append_kv(pool, case.page_table, None, page_fmt, positions.cuda(), kn.cuda(),
                           vn.cuda(), err)
    assert st == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and oerr == 0
    assert torch.equal(case.k_pool[page_fmt].cpu(), host_k[page_fmt])
    assert torch.equal(case.v_pool[page_fmt].cpu(), host_v[page_fmt])
    # the extended sequences decode like the oracle says
    case.seq_lens = (positions + 1).cuda()
    out, lse, err2 = run(case)
    assert err2 == 0
    check(case, out, lse)


def test_append_faults_reported():
    case = small_case(B=2, Hq=4, Hkv=2, d=64, P=16, lens=(20, 20), fmt="tiered",
                      tiers=[(0.5, "i8"), (0.5, "bf16")])
    kn = torch.zeros((2, 2, 64), device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pool = binding.kv_pool_struct(case)
    before = case.k_pool[BF16].clone()
    # sequence 0 appends into its int8 page 0 (not a hot page); sequence 1 past the table
    pos = torch.tensor([3, 16 * case.max_pages], dtype=torch.int32, device="cuda")
    assert binding.append_kv(pool, case.page_table, case.page_fmt, BF16, pos, kn, kn, err) == 0
    torch.cuda.synchronize()
    assert int(err.item()) == binding.DEVERR_PAGE_FMT | binding.DEVERR_SEQ_LEN
    assert torch.equal(case.k_pool[BF16], before)


# ---------------------------------------------------------------------------
# full size, in the launch configuration the benchmark times
# ---------------------------------------------------------------------------

def test_demote_full_size_workload():
    from paged_long_context_b200 import demote_workload
    w = demote_workload.build("cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    demote_workload.run(w, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    src = w.src
    Hkv, d, P = src.num_kv_heads, src.head_dim, src.page_tokens
    for f, job in w.jobs.items():
        # every (page, kv head) block of random values is non-zero: its largest
        # code has magnitude Q (127, 7, or 448 = E4M3 0x7E)
        k = job.dst_k[: job.n]
        if f == I8:
            mag = k.view(torch.int8).to(torch.int32).abs()
            assert int(mag.amax(dim=(2, 3)).min()) == 127
        elif f == I4:
            lo = (k & 0xF).to(torch.int32)
            hi = (k >> 4).to(torch.int32)
            mag = torch.maximum(torch.where(lo >= 8, 16 - lo, lo), torch.where(hi >= 8, 16 - hi, hi))
            assert int(mag.amax(dim=(2, 3)).min()) == 7
        elif f == FP8:
            assert int((k & 0x7F).amax(dim=(2, 3)).min()) == 0x7E
        # sampled pages bit-exact against the oracle
        idx = list(range(0, job.n, max(1, job.n // 6)))[:6]
        s_slots = [int(job.src_slots[i]) for i in idx]
        dk = torch.full((len(idx), Hkv, P, synth.row_bytes(f, d)), 0xAB, dtype=torch.uint8)
        dv = dk.clone()
        dsc = torch.zeros((len(idx), Hkv, 2))
        src_k = src.k_pool[BF16][s_slots].cpu().contiguous()
        src_v = src.v_pool[BF16][s_slots].cpu().contiguous()
        assert oracle.demote(Hkv, d, P, BF16, src_k, src_v, None, f, dk, dv, dsc,
                             list(range(len(idx))), list(range(len(idx)))) == 0
        d_slots = [int(job.dst_slots[i]) for i in idx]
        assert torch.equal(job.dst_k[d_slots].cpu(), dk)
        assert torch.equal(job.dst_v[d_slots].cpu(), dv)
        assert torch.equal(job.dst_scales[d_slots].cpu(), dsc)
