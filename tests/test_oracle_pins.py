"""Pins of the fp64 oracle against facts other than itself (CPU only).

Each test ties one part of the oracle to something fixed outside it: the
CFR-Atlas page's printed byte counts, byte patterns whose values the storage
formats define, closed forms of softmax attention, torch's scaled
dot-product attention evaluated in fp64 (the special case of an identity page
table), a 50-digit decimal brute force, and invariants the method guarantees
(fold and split exactness, regenerated pages, GQA replication).
"""
import dataclasses
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

from paged_long_context_b200 import synth
from tests._hostkv import host_kv, host_q, kv_head_of, sigma_of, decode_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32, BF16, I8, I4, FP8 = synth.F32, synth.BF16, synth.I8, synth.I4, synth.FP8
QUANTISED = synth.QUANTISED


def small(name="s", B=2, Hq=4, Hkv=2, d=16, P=8, lens=(37, 20), fmt="f32", q_fmt="f32",
          alibi=False, seed=11, **kw):
    spec = synth.CaseSpec(name, B, Hq, Hkv, d, P, seq_lens=list(lens), fmt=fmt, q_fmt=q_fmt,
                          alibi=alibi, **kw)
    return synth.make_case(spec, seed, "cpu")


def direct_numpy(case, b, h):
    """Textbook softmax attention over the host-decoded K/V (numpy, fp64)."""
    K, V = host_kv(case, b, kv_head_of(case, h))
    q = host_q(case)[b, h]
    n = K.shape[0]
    s = sigma_of(case) * (K @ q)
    if case.alibi_slopes is not None:
        s = s - float(case.alibi_slopes[h]) * (n - 1 - np.arange(n))
    w = np.exp(s - s.max())
    return (w @ V) / w.sum(), s.max() + np.log(w.sum())


# --------------------------------------------------------------------------
# 1. The CFR-Atlas page's printed byte accounting
# --------------------------------------------------------------------------

def _golden_kv(path):
    out = {}
    for line in open(path):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = v
    return out


def test_byte_accounting_matches_cfr_page(oracle_mod):
    g = _golden_kv(os.path.join(GOLDEN, "cfr_byte_accounting.txt"))
    ctx, d, P = int(g["context_tokens"]), int(g["head_dim"]), int(g["page_tokens"])
    base = oracle_mod.kv_bytes(F32, ctx, d)
    scratch = oracle_mod.kv_bytes(F32, P, d)
    assert base == int(g["baseline_kv_bytes"]) == 33554432
    assert scratch == int(g["cfr_scratch_bytes"]) == 262144
    assert f"{base / scratch:.2f}" == g["estimated_memory_reduction"]
    # the 32-head CFR-shaped workload holds 32 such baselines
    assert 32 * base == 1073741824


def test_byte_accounting_other_formats(oracle_mod):
    # bf16 halves, int8 quarters, int4 eighths of the fp32 bytes
    assert oracle_mod.kv_bytes(BF16, 65536, 64) == 33554432 // 2
    assert oracle_mod.kv_bytes(I8, 65536, 64) == 33554432 // 4
    assert oracle_mod.kv_bytes(I4, 65536, 64) == 33554432 // 8


# --------------------------------------------------------------------------
# 2. Stored bytes decode to the values the formats define (n = 1: o = V_0)
# --------------------------------------------------------------------------

def _patterns():
    rows = []
    for line in open(os.path.join(GOLDEN, "page_byte_patterns.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, hexb, vals = [x.strip() for x in line.split("|")]
        fmt, scale = head.split()
        rows.append((synth.FMT_BY_NAME[fmt], float(scale), bytes.fromhex(hexb),
                     [float(v) for v in vals.split()]))
    return rows


@pytest.mark.parametrize("pat", _patterns(), ids=lambda p: synth.FMT_NAMES[p[0]])
def test_byte_patterns_decode(oracle_mod, pat):
    fmt, scale, raw, expect = pat
    d = len(expect)
    case = small(B=1, Hq=1, Hkv=1, d=d, P=4, lens=(1,), fmt=synth.FMT_NAMES[fmt], q_fmt="f32")
    slot = int(case.page_table[0, 0])
    row = torch.tensor(list(raw), dtype=torch.uint8)
    case.v_pool[fmt][slot, 0, 0] = row
    if fmt in QUANTISED:
        case.scales[fmt][slot, 0, 1] = scale
    out, lse = oracle_mod.attend(case)
    # a single token has weight exactly 1: the output is its V row
    np.testing.assert_array_equal(out[0], np.array(expect, dtype=np.float64))
    # the independent numpy decoder agrees with the golden values too
    dec = decode_rows(row.numpy(), fmt, d) * (scale if fmt in QUANTISED else 1.0)
    np.testing.assert_array_equal(dec, np.array(expect))


def test_all_int8_and_int4_codes(oracle_mod):
    # every int8 byte and every int4 nibble, through the n = 1 closed form
    d = 256
    case = small(B=1, Hq=1, Hkv=1, d=d, P=4, lens=(1,), fmt="i8")
    slot = int(case.page_table[0, 0])
    case.v_pool[I8][slot, 0, 0] = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    case.scales[I8][slot, 0, 1] = 0.375
    out, _ = oracle_mod.attend(case)
    codes = np.array([c if c < 128 else c - 256 for c in range(256)], dtype=np.float64)
    np.testing.assert_array_equal(out[0], codes * 0.375)

    case = small(B=1, Hq=1, Hkv=1, d=32, P=4, lens=(1,), fmt="i4")
    slot = int(case.page_table[0, 0])
    raw = [lo | (hi << 4) for lo, hi in zip(range(16), reversed(range(16)))]
    case.v_pool[I4][slot, 0, 0] = torch.tensor(raw, dtype=torch.uint8)
    case.scales[I4][slot, 0, 1] = 1.0
    out, _ = oracle_mod.attend(case)
    two = lambda x: x - 16 if x >= 8 else x
    expect = []
    for lo, hi in zip(range(16), reversed(range(16))):
        expect += [two(lo), two(hi)]
    np.testing.assert_array_equal(out[0], np.array(expect, dtype=np.float64))


def test_all_fp8_codes(oracle_mod):
    # every E4M3 byte through the n = 1 closed form, against torch's float8 decoding
    d = 256
    case = small(B=1, Hq=1, Hkv=1, d=d, P=4, lens=(1,), fmt="fp8")
    slot = int(case.page_table[0, 0])
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    case.v_pool[FP8][slot, 0, 0] = codes
    case.scales[FP8][slot, 0, 1] = 0.5
    out, _ = oracle_mod.attend(case)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy() * 0.5
    np.testing.assert_array_equal(out[0], want)


# --------------------------------------------------------------------------
# 3. Closed forms of softmax attention
# --------------------------------------------------------------------------

FMTS = ["f32", "bf16", "i8", "i4", "fp8"]


@pytest.mark.parametrize("fmt", FMTS)
def test_single_token_is_v0(oracle_mod, fmt):
    case = small(lens=(1, 1), fmt=fmt, q_fmt="bf16")
    out, lse = oracle_mod.attend(case)
    for b in range(case.batch):
        for h in range(case.num_q_heads):
            K, V = host_kv(case, b, kv_head_of(case, h))
            np.testing.assert_array_equal(out[b * case.num_q_heads + h], V[0])
            s0 = sigma_of(case) * float(K[0] @ host_q(case)[b, h])
            assert lse[b * case.num_q_heads + h] == pytest.approx(s0, rel=1e-14, abs=1e-14)


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_query_gives_mean_of_v(oracle_mod, fmt):
    case = small(lens=(37, 20), fmt=fmt)
    case.q.zero_()
    out, lse = oracle_mod.attend(case)
    for b in range(case.batch):
        n = int(case.seq_lens[b])
        for h in range(case.num_q_heads):
            _, V = host_kv(case, b, kv_head_of(case, h))
            np.testing.assert_allclose(out[b * case.num_q_heads + h], V.mean(0), rtol=0,
                                       atol=1e-14 * max(1.0, np.abs(V).max()))
            assert lse[b * case.num_q_heads + h] == pytest.approx(math.log(n), rel=1e-14)


def test_equal_keys_give_mean_of_v(oracle_mod):
    case = small(lens=(37, 20), fmt="f32")
    pool = case.k_pool[F32]
    pool[:] = pool[int(case.page_table[0, 0]), :, 0:1, :].clone()  # every row equals one row
    out, _ = oracle_mod.attend(case)
    for b in range(case.batch):
        for h in range(case.num_q_heads):
            _, V = host_kv(case, b, kv_head_of(case, h))
            np.testing.assert_allclose(out[b * case.num_q_heads + h], V.mean(0), atol=1e-14)


def test_dominant_key_selects_its_row(oracle_mod):
    # one key whose score exceeds every other by far more than 745: exp() of the
    # gap underflows to 0 in fp64, so the output is exactly that row of V
    case = small(B=1, Hq=1, Hkv=1, d=16, P=8, lens=(29,), fmt="f32", softmax_scale=1.0)
    q = torch.zeros(16)
    q[3] = 1.0
    case.q[0, 0] = q
    K = case.k_pool[F32].view(torch.float32).view(-1, 1, 8, 16)
    j = 17
    p, t = j // 8, j % 8
    slot = int(case.page_table[0, p])
    for pp in range(4):
        sl = int(case.page_table[0, pp])
        K[sl, 0, :, 3] = torch.where(torch.isnan(K[sl, 0, :, 3]), K[sl, 0, :, 3],
                                     torch.zeros(8))
    K[slot, 0, t, 3] = 2000.0
    out, lse = oracle_mod.attend(case)
    _, V = host_kv(case, 0, 0)
    np.testing.assert_array_equal(out[0], V[j])
    assert lse[0] == 2000.0


@pytest.mark.parametrize("alibi", [False, True])
def test_two_tokens_logistic(oracle_mod, alibi):
    case = small(B=1, Hq=2, Hkv=1, d=16, P=8, lens=(2,), fmt="f32", alibi=alibi)
    out, _ = oracle_mod.attend(case)
    for h in range(2):
        K, V = host_kv(case, 0, 0)
        q = host_q(case)[0, h]
        s = sigma_of(case) * (K @ q)
        if alibi:
            s = s - float(case.alibi_slopes[h]) * np.array([1.0, 0.0])
        w0 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
        w1 = 1.0 / (1.0 + math.exp(s[0] - s[1]))
        np.testing.assert_allclose(out[h], w0 * V[0] + w1 * V[1], rtol=1e-14, atol=1e-15)


def test_zero_slope_alibi_is_no_bias(oracle_mod):
    a = small(lens=(37, 20), fmt="bf16", alibi=True)
    b = dataclasses.replace(a, alibi_slopes=torch.zeros_like(a.alibi_slopes))
    c = dataclasses.replace(a, alibi_slopes=None)
    ob, _ = oracle_mod.attend(b)
    oc, _ = oracle_mod.attend(c)
    np.testing.assert_array_equal(ob, oc)


def test_v_shift_moves_output(oracle_mod):
    # the softmax weights sum to one: adding c to every V value adds c to o
    case = small(lens=(37, 20), fmt="f32")
    V = case.v_pool[F32].view(torch.float32)
    V.copy_(torch.round(V * 4) / 4)          # quarter integers: the shift below is exact
    o1, _ = oracle_mod.attend(case)
    V.add_(0.5)
    o2, _ = oracle_mod.attend(case)
    np.testing.assert_allclose(o2, o1 + 0.5, atol=1e-13)


def test_token_order_does_not_matter_without_bias(oracle_mod):
    # with no positional bias, swapping two full pages in the page table permutes
    # the tokens and leaves the result unchanged up to rounding
    case = small(B=1, Hq=2, Hkv=1, lens=(40,), fmt="f32")
    o1, l1 = oracle_mod.attend(case)
    pt = case.page_table
    pt[0, 0], pt[0, 2] = pt[0, 2].clone(), pt[0, 0].clone()
    o2, l2 = oracle_mod.attend(case)
    np.testing.assert_allclose(o2, o1, atol=1e-14)
    np.testing.assert_allclose(l2, l1, rtol=1e-14)
    # with ALiBi the same swap changes the result
    case = small(B=1, Hq=2, Hkv=1, lens=(40,), fmt="f32", alibi=True)
    o1, _ = oracle_mod.attend(case)
    pt = case.page_table
    pt[0, 0], pt[0, 2] = pt[0, 2].clone(), pt[0, 0].clone()
    o2, _ = oracle_mod.attend(case)
    assert np.abs(o2 - o1).max() > 1e-6


# --------------------------------------------------------------------------
# 4. Library special case: identity page table == torch SDPA in fp64
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("alibi", [False, True])
def test_matches_torch_sdpa_fp64(oracle_mod, fmt, alibi):
    case = small(B=3, Hq=8, Hkv=2, d=32, P=16, lens=(53, 16, 100), fmt=fmt, q_fmt="bf16",
                 alibi=alibi, permute=False, seed=5)
    out, lse = oracle_mod.attend(case)
    q = torch.from_numpy(host_q(case))
    for b in range(case.batch):
        Ks, Vs = zip(*[host_kv(case, b, g) for g in range(case.num_kv_heads)])
        K = torch.from_numpy(np.stack(Ks))[None]       # [1, Hkv, n, d]
        V = torch.from_numpy(np.stack(Vs))[None]
        n = K.shape[2]
        mask = None
        if alibi:
            dist = (n - 1 - torch.arange(n, dtype=torch.float64))
            mask = (-case.alibi_slopes.double()[:, None] * dist[None, :])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b][None, :, None, :], K, V, attn_mask=mask, scale=sigma_of(case), enable_gqa=True)
        got = out[b * case.num_q_heads:(b + 1) * case.num_q_heads]
        np.testing.assert_allclose(got, ref[0, :, 0].numpy(), rtol=0,
                                   atol=1e-13 * max(1.0, float(V.abs().max())))


# --------------------------------------------------------------------------
# 5. Brute force at 50 decimal digits on tiny inputs with large logits
# --------------------------------------------------------------------------

def _decimal_attention(q, K, V, sigma, slope):
    getcontext().prec = 50
    n = K.shape[0]
    s = []
    for j in range(n):
        dot = sum(Decimal(float(q[i])) * Decimal(float(K[j, i])) for i in range(K.shape[1]))
        s.append(Decimal(sigma) * dot - Decimal(slope) * (n - 1 - j))
    m = max(s)
    w = [(x - m).exp() for x in s]
    L = sum(w)
    o = [sum(w[j] * Decimal(float(V[j, i])) for j in range(n)) / L for i in range(V.shape[1])]
    return np.array([float(x) for x in o]), float(m + L.ln())


@pytest.mark.parametrize("fmt,alibi,sigma", [("f32", False, 40.0), ("bf16", True, 25.0),
                                             ("i8", False, 0.9), ("i4", True, 3.0)])
def test_brute_force_decimal(oracle_mod, fmt, alibi, sigma):
    # sigma is large enough that exp() of an unshifted score overflows fp64
    case = small(B=1, Hq=2, Hkv=1, d=8, P=8, lens=(27,), fmt=fmt, q_fmt="f32", alibi=alibi,
                 softmax_scale=sigma)
    out, lse = oracle_mod.attend(case)
    K, V = host_kv(case, 0, 0)
    q = host_q(case)[0]
    for h in range(2):
        slope = float(case.alibi_slopes[h]) if alibi else 0.0
        ref, ref_lse = _decimal_attention(q[h], K, V, sigma, slope)
        scale = max(1.0, np.abs(V).max())
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-13 * scale)
        assert lse[h] == pytest.approx(ref_lse, rel=1e-13)


# --------------------------------------------------------------------------
# 6. Fold and split invariants (folded == direct, split + merge == direct)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", FMTS)
def test_fold_equals_direct_every_block_size(oracle_mod, fmt):
    case = small(B=2, Hq=4, Hkv=2, d=16, P=8, lens=(523, 64), fmt=fmt, alibi=True)
    o0, l0 = oracle_mod.attend(case)
    for blk in [1, 2, 3, 7, 16, 64, 512, 523]:
        o1, l1 = oracle_mod.attend(case, mode=1, arg=blk)
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l0, rtol=1e-12)


@pytest.mark.parametrize("fmt", FMTS)
def test_split_merge_equals_direct(oracle_mod, fmt):
    case = small(B=2, Hq=4, Hkv=2, d=16, P=8, lens=(523, 64), fmt=fmt)
    o0, l0 = oracle_mod.attend(case)
    for S in [1, 2, 5, 66]:
        o1, l1 = oracle_mod.attend(case, mode=2, arg=S)
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l0, rtol=1e-12)


# --------------------------------------------------------------------------
# 7. Regenerated pages and pool placement give bit-identical results
# --------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8", "tiered"])
def test_regenerated_copy_is_bit_identical(oracle_mod, fmt):
    kw = {}
    if fmt == "tiered":
        kw = dict(tiers=[(0.25, "i4"), (0.5, "i8"), (0.25, "bf16")])
    case = small(B=2, Hq=4, Hkv=2, d=16, P=8, lens=(61, 33), fmt=fmt, spare_pages=3, **kw)
    o0, l0 = oracle_mod.attend(case)
    f = case.fmt_of_page(0, 2)
    used = set(case.page_table[case.page_fmt == f].tolist()) if case.page_fmt is not None \
        else set(case.page_table.flatten().tolist())
    spare = next(i for i in range(case.pool_pages(f)) if i not in used)
    synth.regenerate_into(case, 0, 2, spare)
    o1, l1 = oracle_mod.attend(case)
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)
    moved = synth.permute_pool(case, 99)
    o2, l2 = oracle_mod.attend(moved)
    np.testing.assert_array_equal(o2, o0)
    np.testing.assert_array_equal(l2, l0)


# --------------------------------------------------------------------------
# 8. Head mapping: GQA equals MHA over replicated kv heads; custom head maps
# --------------------------------------------------------------------------

def _replicate_kv(case):
    """MHA case whose kv head h is a copy of kv head map(h) of ``case``."""
    Hq = case.num_q_heads
    idx = torch.tensor([kv_head_of(case, h) for h in range(Hq)])
    kp = {f: t[:, idx].contiguous() for f, t in case.k_pool.items()}
    vp = {f: t[:, idx].contiguous() for f, t in case.v_pool.items()}
    sc = {f: t[:, idx].contiguous() for f, t in case.scales.items()}
    return dataclasses.replace(case, num_kv_heads=Hq, k_pool=kp, v_pool=vp, scales=sc,
                               head_map=None)


@pytest.mark.parametrize("fmt", FMTS)
def test_gqa_equals_replicated_mha(oracle_mod, fmt):
    case = small(B=2, Hq=8, Hkv=2, d=16, lens=(45, 9), fmt=fmt, alibi=True)
    o0, l0 = oracle_mod.attend(case)
    o1, l1 = oracle_mod.attend(_replicate_kv(case))
    np.testing.assert_array_equal(o1, o0)
    np.testing.assert_array_equal(l1, l0)


def test_custom_head_map(oracle_mod):
    case = small(B=2, Hq=6, Hkv=3, d=16, lens=(45, 9), fmt="bf16", head_map=[2, 0, 1, 1, 0, 2])
    o0, _ = oracle_mod.attend(case)
    o1, _ = oracle_mod.attend(_replicate_kv(case))
    np.testing.assert_array_equal(o1, o0)
    for b in range(2):
        for h in range(6):
            ref, _ = direct_numpy(case, b, h)
            np.testing.assert_allclose(o0[b * 6 + h], ref, atol=1e-13)


# --------------------------------------------------------------------------
# 9. Invalid pages: skipping a page equals attending without its tokens
# --------------------------------------------------------------------------

def test_skip_invalid_page_equals_dropping_it(oracle_mod):
    case = small(B=1, Hq=2, Hkv=1, d=16, P=8, lens=(40,), fmt="f32")
    with pytest.raises(oracle_mod.OracleError):
        bad = dataclasses.replace(case, page_table=case.page_table.clone())
        bad.page_table[0, 1] = 10_000
        oracle_mod.attend(bad)
    o_skip, _ = oracle_mod.attend(bad, skip_invalid=True)
    # drop page 1: pages 0, 2, 3, 4 hold 32 tokens (all full)
    dropped = dataclasses.replace(case, page_table=case.page_table[:, [0, 2, 3, 4]].contiguous(),
                                  seq_lens=torch.tensor([32], dtype=torch.int32), max_pages=4)
    o_ref, _ = oracle_mod.attend(dropped)
    np.testing.assert_allclose(o_skip, o_ref, atol=1e-14)


def test_empty_sequence_gives_zero_and_minus_inf(oracle_mod):
    case = small(B=2, Hq=2, Hkv=1, lens=(5, 9), fmt="f32")
    case.seq_lens[1] = 0
    with pytest.raises(oracle_mod.OracleError) as e:
        oracle_mod.attend(case)
    assert e.value.code == oracle_mod.EMPTY
    out, lse = oracle_mod.attend(case, allow_empty=True)
    assert np.all(out[2:] == 0) and np.all(np.isneginf(lse[2:]))
    assert np.all(np.isfinite(lse[:2]))


# --------------------------------------------------------------------------
# 10. The log-sum-exp merge
# --------------------------------------------------------------------------

def test_merge_closed_forms(oracle_mod):
    d = 8
    acc = torch.randn(3, 1, d)
    m = torch.tensor([[2.0], [2.0], [-5.0]])
    l = torch.tensor([[3.0], [5.0], [0.0]])
    off = torch.tensor([0, 1, 3], dtype=torch.int32)
    out, lse = oracle_mod.merge(acc, m, l, off, 2, 1, d)
    # one split: a / l and (m + log2 l) ln 2
    np.testing.assert_allclose(out[0, 0], acc[0, 0].double().numpy() / 3.0, rtol=1e-15)
    assert lse[0, 0] == pytest.approx((2.0 + math.log2(3.0)) * math.log(2.0), rel=1e-15)
    # an empty split (l = 0) is skipped; the other one stands alone
    np.testing.assert_allclose(out[1, 0], acc[1, 0].double().numpy() / 5.0, rtol=1e-15)
    # equal maxima: (a1 + a2) / (l1 + l2)
    m2 = torch.tensor([[1.5], [1.5], [1.5]])
    l2 = torch.tensor([[2.0], [6.0], [0.0]])
    out, _ = oracle_mod.merge(acc, m2, l2, torch.tensor([0, 3, 3], dtype=torch.int32), 2, 1, d)
    np.testing.assert_allclose(out[0, 0], (acc[0, 0].double() + acc[1, 0].double()).numpy() / 8.0,
                               rtol=1e-14)
    assert np.all(out[1] == 0)


def test_merge_of_oracle_splits_equals_direct(oracle_mod):
    # partials of two halves of each sequence, rounded to fp32, then merged
    case = small(B=2, Hq=2, Hkv=1, d=16, P=8, lens=(64, 40), fmt="f32", alibi=True)
    o0, l0 = oracle_mod.attend(case)
    accs, ms, ls = [], [], []
    for b in range(2):
        K, V = host_kv(case, b, 0)
        n = K.shape[0]
        halves = [(0, n // 2), (n // 2, n)]
        for (j0, j1) in halves:
            row_a, row_m, row_l = [], [], []
            for h in range(2):
                s = sigma_of(case) * (K @ host_q(case)[b, h])
                s = s - float(case.alibi_slopes[h]) * (n - 1 - np.arange(n))
                ss = s[j0:j1]
                mm = ss.max()
                w = np.exp(ss - mm)
                row_a.append(w @ V[j0:j1])
                row_m.append(mm * math.log2(math.e))
                row_l.append(w.sum())
            accs.append(row_a); ms.append(row_m); ls.append(row_l)
    acc = torch.tensor(np.array(accs), dtype=torch.float32)
    m = torch.tensor(np.array(ms), dtype=torch.float32)
    l = torch.tensor(np.array(ls), dtype=torch.float32)
    out, lse = oracle_mod.merge(acc, m, l, torch.tensor([0, 2, 4], dtype=torch.int32), 2, 2, 16)
    np.testing.assert_allclose(out.reshape(4, 16), o0, atol=3e-6)
    np.testing.assert_allclose(lse.reshape(4), l0, atol=3e-6)
