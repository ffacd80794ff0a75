"""GPU parity of the decode path against the fp64 oracle, through the C ABI.

Tolerances (from the method's statement of the target): fp32 K/V max-abs error
1e-5; bf16 / int8 / int4 K/V max error 2e-3 * max|V| of the (sequence, kv
head); page-table and index resolution bit-exact.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._gpu import check, run, small_case
from tests._hostkv import decode_rows

pytestmark = pytest.mark.gpu

F32, BF16, I8, I4, FP8 = synth.F32, synth.BF16, synth.I8, synth.I4, synth.FP8


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


# ---------------------------------------------------------------------------
# parity matrix on small cases (several tiles, ragged tails)
# ---------------------------------------------------------------------------

HEADS = [(4, 4), (6, 3), (8, 2), (8, 1), (16, 1)]


@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "i4", "fp8"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("heads", HEADS, ids=lambda h: f"{h[0]}q{h[1]}kv")
def test_parity_formats_heads(fmt, d, heads):
    Hq, Hkv = heads
    q_fmt = "f32" if fmt == "f32" else "bf16"
    case = small_case(B=3, Hq=Hq, Hkv=Hkv, d=d, P=16, lens=(200, 17, 333), fmt=fmt, q_fmt=q_fmt)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("P", [8, 16, 32, 64, 128, 256, 512])
@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "fp8"])
def test_parity_page_sizes(P, fmt):
    lens = (1, P - 1 if P > 1 else 1, P, P + 1, 3 * P + 5, 1000)
    case = small_case(B=6, Hq=8, Hkv=2, d=128, P=P, lens=lens, fmt=fmt,
                      q_fmt="f32" if fmt == "f32" else "bf16", seed=P)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("P", [16, 64, 128, 256])
@pytest.mark.parametrize("d", [64, 128])
def test_parity_tiered_pages(P, d):
    case = small_case(B=3, Hq=8, Hkv=2, d=d, P=P, lens=(16 * P + 3, 9 * P, 2 * P + 1),
                      fmt="tiered", tiers=[(0.25, "i4"), (0.5, "i8"), (0.25, "bf16")])
    assert case.page_fmt is not None
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("P", [16, 128, 256])
def test_parity_tiered_with_fp8_pages(P):
    # the whole cascade: int4, int8, FP8, bf16 pages in one sequence
    case = small_case(B=3, Hq=8, Hkv=2, d=128, P=P, lens=(20 * P + 3, 9 * P, 2 * P + 1),
                      fmt="tiered", tiers=[(0.2, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.3, "bf16")])
    out, lse, err = run(case)
    assert err == 0
    assert binding.decode_path(case) == (binding.PATH_TENSOR_CORE if P >= 128
                                         else binding.PATH_CUDA_CORE)
    check(case, out, lse)


def test_parity_tiered_with_fp32_hot_pages():
    case = small_case(B=2, Hq=4, Hkv=2, d=64, P=32, lens=(700, 130), fmt="tiered",
                      tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "bf16"), (0.2, "f32")], q_fmt="f32")
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "i4", "fp8"])
def test_parity_alibi(fmt):
    case = small_case(B=2, Hq=8, Hkv=2, d=128, P=64, lens=(3000, 129), fmt=fmt,
                      q_fmt="f32" if fmt == "f32" else "bf16", alibi=True)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_parity_custom_head_map():
    case = small_case(B=2, Hq=6, Hkv=3, d=128, P=16, lens=(300, 45), fmt="bf16",
                      head_map=[2, 0, 1, 1, 0, 2], alibi=True)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_parity_uneven_groups():
    # kv head 0 serves 5 query heads, kv head 1 serves 1
    case = small_case(B=2, Hq=6, Hkv=2, d=64, P=16, lens=(250, 31), fmt="i8",
                      head_map=[0, 0, 1, 0, 0, 0])
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("q_fmt,fmt", [("f32", "bf16"), ("bf16", "f32"), ("f32", "i4")])
def test_parity_query_formats(q_fmt, fmt):
    case = small_case(B=2, Hq=8, Hkv=2, d=128, P=32, lens=(555, 64), fmt=fmt, q_fmt=q_fmt)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_parity_explicit_scale():
    case = small_case(B=2, Hq=4, Hkv=4, d=64, P=16, lens=(400, 77), fmt="f32", q_fmt="f32",
                      softmax_scale=0.37)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_parity_large_logits():
    # sigma large: exp of unshifted scores would overflow fp32
    case = small_case(B=1, Hq=4, Hkv=1, d=128, P=64, lens=(900,), fmt="bf16",
                      softmax_scale=4.0)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_parity_many_sequences_ragged():
    rng = np.random.default_rng(3)
    lens = [int(x) for x in rng.integers(1, 700, size=40)]
    case = small_case(B=40, Hq=8, Hkv=2, d=128, P=16, lens=lens, fmt="bf16")
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


# ---------------------------------------------------------------------------
# edge cases and device-side error reporting (host-made faults; nothing faults)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "i4", "fp8"])
def test_single_token_is_v0(fmt):
    case = small_case(B=2, Hq=4, Hkv=2, d=128, P=16, lens=(1, 1), fmt=fmt,
                      q_fmt="f32" if fmt == "f32" else "bf16")
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_full_page_table():
    case = small_case(B=2, Hq=4, Hkv=2, d=64, P=16, lens=(160, 160), fmt="f32", q_fmt="f32")
    assert case.max_pages * case.page_tokens == 160
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("path", ["cc", "tc", "f32"])
@pytest.mark.parametrize("bad_len", [0, -5, 10_000])
def test_bad_sequence_length(bad_len, path):
    # a sequence that gets no split: its rows are written as a merge of nothing
    # (0, lse -inf) by the decode that merges, on each kernel
    kw = {"cc": dict(d=64, fmt="tiered", tiers=[(0.5, "i8"), (0.5, "bf16")]),
          "tc": dict(d=128, fmt="bf16", q_fmt="bf16"),
          "f32": dict(d=64, fmt="f32", q_fmt="f32")}[path]
    case = small_case(B=3, Hq=4, Hkv=2, P=16, lens=(50, 33, 70), **kw)
    assert binding.decode_path(case) == {"cc": binding.PATH_CUDA_CORE, "tc": binding.PATH_TENSOR_CORE,
                                         "f32": binding.PATH_F32_TMA}[path]
    case.seq_lens[1] = bad_len
    out, lse, err = run(case)
    assert err & binding.DEVERR_SEQ_LEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    ok = dataclasses.replace(case, seq_lens=case.seq_lens.clone())
    check(ok, out, lse, sel=[(0, h) for h in range(4)] + [(2, h) for h in range(4)])


@pytest.mark.parametrize("how", ["id_too_big", "id_negative", "bad_fmt", "null_pool"])
def test_bad_page_is_skipped_and_reported(how):
    case = small_case(B=2, Hq=4, Hkv=2, d=64, P=16, lens=(100, 40), fmt="tiered",
                      tiers=[(0.5, "i8"), (0.5, "bf16")], q_fmt="bf16")
    expect = {"id_too_big": binding.DEVERR_PAGE_ID, "id_negative": binding.DEVERR_PAGE_ID,
              "bad_fmt": binding.DEVERR_PAGE_FMT, "null_pool": binding.DEVERR_POOL}[how]
    if how == "id_too_big":
        case.page_table[0, 2] = 1 << 20
    elif how == "id_negative":
        case.page_table[0, 2] = -3
    elif how == "bad_fmt":
        case.page_fmt[0, 2] = 9
    else:
        # the format of page 2 loses its pool (page 2 of sequence 0 is int8)
        assert int(case.page_fmt[0, 2]) == I8
        case = dataclasses.replace(case, k_pool={f: t for f, t in case.k_pool.items() if f != I8},
                                   v_pool={f: t for f, t in case.v_pool.items() if f != I8},
                                   scales={})
    out, lse, err = run(case)
    assert err & expect
    # the rest of the sequence equals attention without the skipped page(s)
    hc = case.to("cpu")
    ref_o, _ = oracle.attend(hc, mode=0, skip_invalid=True)
    ref_o = ref_o.reshape(2, 4, 64)
    vmax = pool_vmax(hc)
    np.testing.assert_allclose(out.double().numpy(), ref_o, atol=2e-3 * vmax, rtol=0)


def pool_vmax(case):
    """max |value| over every stored V element of every pool (NaN padding ignored)."""
    m = 0.0
    for f, t in case.v_pool.items():
        x = decode_rows(t.cpu().numpy(), f, case.head_dim)
        if f in synth.QUANTISED:
            x = x * case.scales[f].cpu().numpy()[:, :, None, 1:2].astype(np.float64)
        x = x[np.isfinite(x)]
        if x.size:
            m = max(m, float(np.abs(x).max()))
    return m


def test_workspace_checks():
    case = small_case(fmt="bf16")
    bufs = binding.DecodeBuffers(case)
    assert binding.paged_decode_raw(case, bufs, workspace_bytes=bufs.workspace.numel() - 256) == 7
    bad = binding.DecodeBuffers(case)
    bad.workspace = bufs.workspace[4:]
    assert binding.paged_decode_raw(case, bad) == 7
    bad.workspace = None
    assert binding.paged_decode_raw(case, bad, workspace_bytes=0) == 7


# ---------------------------------------------------------------------------
# determinism, placement independence, regeneration (bit-exact)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["f32", "bf16", "tiered"])
def test_bit_identical_runs_and_placements(fmt):
    kw = dict(tiers=[(0.25, "i4"), (0.5, "i8"), (0.25, "bf16")]) if fmt == "tiered" else {}
    case = small_case(B=3, Hq=8, Hkv=2, d=128, P=64, lens=(2000, 300, 65), fmt=fmt,
                      q_fmt="bf16", spare_pages=2, alibi=True, **kw)
    o1, l1, _ = run(case)
    o2, l2, _ = run(case)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    moved = synth.permute_pool(case, 5)
    o3, l3, _ = run(moved)
    assert torch.equal(o1, o3) and torch.equal(l1, l3)
    f = case.fmt_of_page(0, 3)
    used = set(case.page_table[case.page_fmt == f].tolist()) if case.page_fmt is not None \
        else set(case.page_table.flatten().tolist())
    spare = next(i for i in range(case.pool_pages(f)) if i not in used)
    synth.regenerate_into(case, 0, 3, spare)
    o4, l4, _ = run(case)
    assert torch.equal(o1, o4) and torch.equal(l1, l4)


def test_runs_on_a_side_stream():
    case = small_case(B=2, Hq=8, Hkv=2, d=128, P=16, lens=(500, 20), fmt="bf16")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        bufs = binding.paged_decode(case, stream=s)
    s.synchronize()
    check(case, bufs.out.cpu(), bufs.lse.cpu())


# ---------------------------------------------------------------------------
# the boundary's other entry points
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "i4", "fp8", "tiered"])
def test_gather_is_bit_exact(fmt):
    kw = dict(tiers=[(0.25, "i4"), (0.25, "i8"), (0.25, "fp8"), (0.25, "bf16")]) \
        if fmt == "tiered" else {}
    case = small_case(B=2, Hq=4, Hkv=2, d=128, P=16, lens=(150, 77), fmt=fmt, **kw)
    pitch = 512
    n = 150
    k_out = torch.full((n, pitch), 0xAB, dtype=torch.uint8, device="cuda")
    v_out = torch.full((n, pitch), 0xAB, dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = binding.gather_pages(case, 0, 1, n, k_out, v_out, pitch, err)
    assert st == 0
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # independent host gather with numpy indexing
    pt = case.page_table.cpu().numpy()
    kh, vh = k_out.cpu().numpy(), v_out.cpu().numpy()
    for j in range(n):
        p, t = divmod(j, 16)
        f = case.fmt_of_page(0, p)
        rb = synth.row_bytes(f, 128)
        krow = case.k_pool[f][int(pt[0, p]), 1, t].cpu().numpy()
        vrow = case.v_pool[f][int(pt[0, p]), 1, t].cpu().numpy()
        assert np.array_equal(kh[j, :rb], krow) and np.array_equal(vh[j, :rb], vrow), j
        assert np.all(kh[j, rb:] == 0xAB)


def test_schedule_properties():
    lens = torch.tensor([1, 16, 17, 1000, 0, 4096, 333], dtype=torch.int32, device="cuda")
    B, P, max_pages, target = 7, 16, 256, 9
    cap = target + B
    off = torch.full((B + 1,), -1, dtype=torch.int32, device="cuda")
    splits = torch.full((cap, 3), -1, dtype=torch.int32, device="cuda")
    ns = torch.zeros(2, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert binding.schedule_splits(lens, B, P, max_pages, target, off, splits, cap, ns, err) == 0
    torch.cuda.synchronize()
    off, splits, ns = off.cpu().tolist(), splits.cpu().tolist(), ns.cpu().tolist()
    nps = [(-(-int(n) // P)) if 0 < int(n) <= max_pages * P else 0 for n in lens.cpu().tolist()]
    chunk = max(1, -(-sum(nps) // target))
    assert ns[1] == chunk
    assert off[0] == 0 and off[B] == ns[0] <= target + B
    assert int(err.item()) & binding.DEVERR_SEQ_LEN       # the empty sequence
    for b in range(B):
        mine = splits[off[b]:off[b + 1]]
        assert len(mine) == -(-nps[b] // chunk)
        pos = 0
        for (bb, pb, pe) in mine:
            assert bb == b and pb == pos and pb < pe <= nps[b] and pe - pb <= chunk
            pos = pe
        assert pos == nps[b]


def test_merge_matches_oracle():
    num = [3, 1, 0, 7, 2]
    acc, m, l, off = synth.merge_inputs(num, 6, 128, seed=4, empty_frac=0.2, device="cuda")
    out = torch.empty((5, 6, 128), device="cuda")
    lse = torch.empty((5, 6), device="cuda")
    assert binding.merge_partials(acc, m, l, off, 5, 6, 128, out, lse) == 0
    torch.cuda.synchronize()
    ro, rl = oracle.merge(acc, m, l, off, 5, 6, 128)
    mag = np.abs(acc.cpu().numpy()).max()
    np.testing.assert_allclose(out.cpu().double().numpy(), ro, rtol=0, atol=1e-5 * mag)
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(lse.cpu().numpy()), fin)
    np.testing.assert_allclose(lse.cpu().double().numpy()[fin], rl[fin], rtol=1e-5, atol=1e-5)
    assert torch.all(out[2] == 0)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("P", [8, 16, 32, 64])
@pytest.mark.parametrize("fmt", ["i8", "i4", "fp8"])
def test_small_quantised_pages_on_the_tensor_core_kernel(fmt, P, d):
    # uniform int8 / int4 / FP8 caches with pages shorter than a 128-token tile:
    # a tile holds 128 / P pages, each with its own K and V scale
    lens = (1, P + 3, 3 * 128 + 5, 1000)
    case = small_case(B=len(lens), Hq=8, Hkv=2, d=d, P=P, lens=lens, fmt=fmt, q_fmt="bf16",
                      alibi=True, seed=P + d)
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


BAD_PAGE_SHAPES = {
    # uniform int8, one page per tile: the int8-MMA variant with six 32 KiB stages
    "i8_p128": dict(d=128, P=128, fmt="i8"),
    # uniform int8, eight pages per tile (one of them bad)
    "i8_p16": dict(d=128, P=16, fmt="i8"),
    # uniform int4, one page per tile: the int8-MMA variant with three stages
    "i4_p128": dict(d=128, P=128, fmt="i4"),
    # bf16, eight pages per tile
    "bf16_p16": dict(d=128, P=16, fmt="bf16"),
    # int8 at head_dim 64 (fp16 staging, six 32 KiB stages), two pages per tile
    "i8_d64_p64": dict(d=64, P=64, fmt="i8"),
}


@pytest.mark.parametrize("shape", list(BAD_PAGE_SHAPES))
@pytest.mark.parametrize("how", ["id_too_big", "id_negative"])
def test_bad_page_on_the_tensor_core_kernel(shape, how):
    # a tile whose only page (or one of whose pages) has a bad id: its tokens
    # are skipped and reported, the rest equals attention without them
    kw = BAD_PAGE_SHAPES[shape]
    P = kw["P"]
    case = small_case(B=2, Hq=8, Hkv=2, lens=(5 * P + 3, 2 * P + 1), q_fmt="bf16", alibi=True,
                      seed=P, **kw)
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    case.page_table[0, 1] = (1 << 20) if how == "id_too_big" else -3
    out, lse, err = run(case)
    assert err & binding.DEVERR_PAGE_ID
    hc = case.to("cpu")
    ref_o, _ = oracle.attend(hc, mode=0, skip_invalid=True)
    ref_o = ref_o.reshape(2, 8, kw["d"])
    np.testing.assert_allclose(out.double().numpy(), ref_o, atol=2e-3 * pool_vmax(hc), rtol=0)
