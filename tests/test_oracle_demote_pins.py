"""Pins of the oracle's page demotion, KV append and FP8 tier (CPU only).

The demotion re-encodes pages down the compression cascade of the ARGUS page
("Visual Architecture": full precision, FP8, INT8, INT4); the append writes a
step's new K/V row into the hot tier.  Each test ties the oracle to something
fixed outside it: hand-derived byte patterns (``tests/golden``), the E4M3 and
bfloat16 format definitions as implemented by torch's float8 / bfloat16
conversions, reconstruction-error bounds, scaling invariances, and the decode
oracle's closed form for a single token.
"""
import math
import os

import numpy as np
import pytest
import torch

from paged_long_context_b200 import synth
from tests._hostkv import decode_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
F32, BF16, I8, I4, FP8 = synth.F32, synth.BF16, synth.I8, synth.I4, synth.FP8
QUANTISED = synth.QUANTISED
QMAX = {I8: 127, I4: 7, FP8: 448}


# --------------------------------------------------------------------------
# helpers: pools of P rows x d with Hkv heads, host tensors
# --------------------------------------------------------------------------

def pool(fmt, slots, hkv, P, d, fill=0):
    return torch.full((slots, hkv, P, synth.row_bytes(fmt, d)), fill, dtype=torch.uint8)


def encode_values(vals: np.ndarray, fmt: int) -> torch.Tensor:
    """float values [..., d] -> stored bytes of a float format (exact for the golden values)."""
    t = torch.from_numpy(np.asarray(vals, dtype=np.float32))
    if fmt == F32:
        return t.contiguous().view(torch.uint8)
    if fmt == BF16:
        return t.to(torch.bfloat16).contiguous().view(torch.uint8)
    raise ValueError(fmt)


def run_demote(oracle_mod, src_fmt, src_k, src_v, src_sc, dst_fmt, hkv, P, d, src_slots,
               dst_slots, valid=None, dst_slots_total=None):
    n_dst = dst_slots_total or (max(dst_slots) + 1 if len(dst_slots) else 1)
    dk, dv = pool(dst_fmt, n_dst, hkv, P, d, 0xAB), pool(dst_fmt, n_dst, hkv, P, d, 0xAB)
    dsc = torch.full((n_dst, hkv, 2), -1.0) if dst_fmt in QUANTISED else None
    err = oracle_mod.demote(hkv, d, P, src_fmt, src_k, src_v, src_sc, dst_fmt, dk, dv, dsc,
                            src_slots, dst_slots, valid)
    return dk, dv, dsc, err


# --------------------------------------------------------------------------
# 1. Hand-derived byte patterns
# --------------------------------------------------------------------------

def _demote_patterns():
    rows = []
    for line in open(os.path.join(GOLDEN, "demote_byte_patterns.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, src, dst, scale, out = [x.strip() for x in line.split("|")]
        sf, ss, valid = head.split()
        rows.append((synth.FMT_BY_NAME[sf], float(ss), int(valid),
                     [r.split() for r in src.split(";")], synth.FMT_BY_NAME[dst],
                     None if scale == "-" else float(scale),
                     [bytes.fromhex(r) for r in out.split(";")]))
    return rows


@pytest.mark.parametrize("pat", _demote_patterns(),
                         ids=lambda p: f"{synth.FMT_NAMES[p[0]]}-{synth.FMT_NAMES[p[4]]}")
def test_demote_byte_patterns(oracle_mod, pat):
    sf, ss, valid, src_rows, df, scale, expect = pat
    P, d = len(src_rows), len(src_rows[0])
    if sf in QUANTISED:
        blk = torch.tensor([[int(b, 16) for b in r] for r in src_rows], dtype=torch.uint8)
    else:
        blk = encode_values(np.array([[float(v) for v in r] for r in src_rows]), sf)
        blk = blk.reshape(P, synth.row_bytes(sf, d))
    sk = blk.reshape(1, 1, P, -1).clone()
    sv = blk.reshape(1, 1, P, -1).clone()
    ssc = torch.full((1, 1, 2), ss) if sf in QUANTISED else None
    dk, dv, dsc, err = run_demote(oracle_mod, sf, sk, sv, ssc, df, 1, P, d, [0], [0], [valid])
    assert err == 0
    for pool_ in (dk, dv):
        got = [bytes(pool_[0, 0, t].tolist()) for t in range(P)]
        assert got == expect
    if scale is not None:
        assert dsc[0, 0, 0].item() == scale and dsc[0, 0, 1].item() == scale


# --------------------------------------------------------------------------
# 2. Format definitions: E4M3 and bfloat16 against torch's conversions
# --------------------------------------------------------------------------

def test_e4m3_table_matches_torch_float8(oracle_mod):
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    ours = np.array([oracle_mod.e4m3_value(c) for c in range(256)])
    np.testing.assert_array_equal(ours, lib.numpy())
    assert math.isnan(ours[0x7F]) and math.isnan(ours[0xFF])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def _e4m3_probe_values():
    g = torch.Generator().manual_seed(7)
    vals = [torch.randn(4000, generator=g) * s for s in (1e-3, 1e-2, 0.3, 3.0, 60.0)]
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    fin = codes[torch.isfinite(codes)]
    srt = torch.sort(fin.unique()).values
    mids = (srt[1:] + srt[:-1]) / 2                     # every tie between neighbours
    vals += [fin, mids, mids.nextafter(torch.tensor(1e9)), mids.nextafter(torch.tensor(-1e9))]
    v = torch.cat(vals)
    return v[v.abs() < 448.0]


def test_e4m3_encoding_matches_torch_float8(oracle_mod):
    v = _e4m3_probe_values()
    lib = v.to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    ours = [oracle_mod.e4m3_code(x) for x in v.tolist()]
    assert ours == lib


def test_e4m3_saturates(oracle_mod):
    for x, c in [(448.0, 0x7E), (455.0, 0x7E), (470.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE),
                 (float("inf"), 0x7E), (-0.0, 0x80), (0.0, 0x00), (2.0 ** -11, 0x00)]:
        assert oracle_mod.e4m3_code(x) == c, x
    assert oracle_mod.e4m3_code(float("nan")) == 0x7F


def test_bf16_rounding_matches_torch(oracle_mod):
    g = torch.Generator().manual_seed(3)
    v = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-30, 1.0, 1e30)])
    base = torch.randn(500, generator=g).to(torch.bfloat16).float()
    ulp = (base.view(torch.int32) + (1 << 16)).view(torch.float32) - base
    v = torch.cat([v, base + ulp / 2, base - ulp / 2, torch.tensor([3.4028235e38, -3.4028235e38])])
    lib = v.to(torch.bfloat16).view(torch.int16).to(torch.int32).bitwise_and(0xFFFF).tolist()
    ours = [oracle_mod.bf16_bits(x) for x in v.tolist()]
    assert ours == lib


# --------------------------------------------------------------------------
# 3. Bounds and invariants of the quantiser on random pages
# --------------------------------------------------------------------------

def random_f32_pages(slots, hkv, P, d, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((slots, hkv, P, d), generator=g) * scale
    return x, x.contiguous().view(torch.uint8).reshape(slots, hkv, P, 4 * d)


def decoded(pool_, sc, fmt, d, kv):
    vals = decode_rows(pool_.numpy(), fmt, d)
    if fmt in QUANTISED:
        vals = vals * sc[..., kv].numpy().astype(np.float64)[:, :, None, None]
    return vals


@pytest.mark.parametrize("dst", [I8, I4, FP8])
def test_quantiser_error_bounds(oracle_mod, dst):
    hkv, P, d, slots = 3, 16, 32, 4
    x, raw = random_f32_pages(slots, hkv, P, d, seed=21)
    valid = [16, 5, 1, 16]
    dk, dv, dsc, err = run_demote(oracle_mod, F32, raw, raw.clone(), None, dst, hkv, P, d,
                                  list(range(slots)), list(range(slots)), valid)
    assert err == 0
    xs = x.double().numpy()
    for k in range(slots):
        n = valid[k]
        for g in range(hkv):
            blk = xs[k, g, :n]
            amax = np.float32(np.abs(blk).max())
            s = float(dsc[k, g, 0])
            assert s == float(np.float32(amax) / np.float32(QMAX[dst]))
            rec = decoded(dk, dsc, dst, d, 0)[k, g, :n]
            if dst == FP8:
                y = blk / s
                # E4M3: relative step 2^-3 for normals (half of it is the rounding bound),
                # absolute step 2^-9 below 2^-6
                bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
                assert np.all(np.abs(rec / s - y) <= bound)
            else:
                assert np.all(np.abs(rec / s - blk / s) <= 0.5 + 1e-5)
                codes = np.rint(rec / s)
                assert np.abs(codes).max() == QMAX[dst]      # the largest element maps to +-Q
            # rows past the valid count are zero bytes
            assert int(dk[k, g, n:].sum()) == 0


@pytest.mark.parametrize("dst", [I8, I4, FP8])
def test_power_of_two_scaling_keeps_codes(oracle_mod, dst):
    hkv, P, d = 2, 8, 16
    x, raw = random_f32_pages(1, hkv, P, d, seed=5)
    raw2 = (x * 8.0).contiguous().view(torch.uint8).reshape(1, hkv, P, 4 * d)
    a = run_demote(oracle_mod, F32, raw, raw.clone(), None, dst, hkv, P, d, [0], [0])
    b = run_demote(oracle_mod, F32, raw2, raw2.clone(), None, dst, hkv, P, d, [0], [0])
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert torch.equal(a[2] * 8.0, b[2])


def test_invalid_rows_do_not_matter(oracle_mod):
    hkv, P, d = 2, 8, 16
    x, raw = random_f32_pages(1, hkv, P, d, seed=9)
    raw2 = raw.clone()
    raw2[:, :, 3:] = 0xFF                                   # NaN bit patterns past valid
    for dst in (I8, I4, FP8, BF16):
        a = run_demote(oracle_mod, F32, raw, raw.clone(), None, dst, hkv, P, d, [0], [0], [3])
        b = run_demote(oracle_mod, F32, raw2, raw2.clone(), None, dst, hkv, P, d, [0], [0], [3])
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_float_destinations_are_conversions(oracle_mod):
    hkv, P, d = 2, 8, 16
    x, raw = random_f32_pages(2, hkv, P, d, seed=13)
    dk, dv, _, err = run_demote(oracle_mod, F32, raw, raw.clone(), None, BF16, hkv, P, d,
                                [1, 0], [0, 1])
    assert err == 0
    want = x.to(torch.bfloat16).contiguous().view(torch.uint8).reshape(2, hkv, P, 2 * d)
    assert torch.equal(dk[0], want[1]) and torch.equal(dk[1], want[0])
    # bf16 -> f32 widens exactly
    dk2, _, _, err = run_demote(oracle_mod, BF16, dk, dv, None, F32, hkv, P, d, [0], [0])
    assert torch.equal(dk2[0].view(torch.float32), x[1].to(torch.bfloat16).float())


def test_cascade_reencodes_decoded_values(oracle_mod):
    # i8 -> i4: the source values are code * scale rounded to fp32
    hkv, P, d = 1, 4, 8
    x, raw = random_f32_pages(1, hkv, P, d, seed=17)
    k8, v8, s8, _ = run_demote(oracle_mod, F32, raw, raw.clone(), None, I8, hkv, P, d, [0], [0])
    k4, v4, s4, _ = run_demote(oracle_mod, I8, k8, v8, s8, I4, hkv, P, d, [0], [0])
    vals = (torch.from_numpy(decode_rows(k8.numpy(), I8, d)).float() * s8[0, 0, 0]).float()
    rawv = vals.contiguous().view(torch.uint8).reshape(1, hkv, P, 4 * d)
    k4b, _, s4b, _ = run_demote(oracle_mod, F32, rawv, rawv.clone(), None, I4, hkv, P, d, [0], [0])
    assert torch.equal(k4, k4b) and s4[0, 0, 0] == s4b[0, 0, 0]


def test_demote_faults_are_skipped(oracle_mod):
    hkv, P, d = 1, 4, 8
    _, raw = random_f32_pages(2, hkv, P, d, seed=1)
    dk, dv, dsc, err = run_demote(oracle_mod, F32, raw, raw.clone(), None, I8, hkv, P, d,
                                  [0, 5, 1], [0, 1, 2], dst_slots_total=3)
    assert err == oracle_mod.DEV_PAGE_ID
    assert int((dk[1] != 0xAB).sum()) == 0                    # skipped page untouched
    dk, dv, dsc, err = run_demote(oracle_mod, F32, raw, raw.clone(), None, I8, hkv, P, d,
                                  [0, 1], [0, 1], [0, 5])
    assert err == oracle_mod.DEV_SEQ_LEN
    assert int((dk != 0xAB).sum()) == 0


# --------------------------------------------------------------------------
# 4. KV append
# --------------------------------------------------------------------------

def _append_case(fmt, P=8, d=16, hkv=2, B=2, max_pages=3):
    kp = {fmt: pool(fmt, 6, hkv, P, d, 0xFF)}
    vp = {fmt: pool(fmt, 6, hkv, P, d, 0xFF)}
    pt = torch.tensor([[4, 1, 0], [2, 5, 3]], dtype=torch.int32)[:B, :max_pages]
    return kp, vp, pt


@pytest.mark.parametrize("page_fmt", [F32, BF16])
@pytest.mark.parametrize("new_fmt", [F32, BF16])
def test_append_writes_the_row_the_decode_reads(oracle_mod, page_fmt, new_fmt):
    P, d, hkv = 8, 16, 2
    kp, vp, pt = _append_case(page_fmt)
    g = torch.Generator().manual_seed(2)
    kn = torch.randn((2, hkv, d), generator=g)
    vn = torch.randn((2, hkv, d), generator=g)
    if new_fmt == BF16:
        kn, vn = kn.to(torch.bfloat16), vn.to(torch.bfloat16)
    positions = [0, 13]                                   # page 0 row 0; page 1 row 5
    before_k = kp[page_fmt].clone()
    err = oracle_mod.append(hkv, d, P, kp, vp, pt, None, page_fmt, positions, new_fmt, kn, vn)
    assert err == 0
    conv = (lambda t: t.float()) if page_fmt == F32 else (lambda t: t.to(torch.bfloat16))
    for b, j in enumerate(positions):
        slot = int(pt[b, j // P])
        for gg in range(hkv):
            row = kp[page_fmt][slot, gg, j % P]
            assert torch.equal(row, conv(kn[b, gg]).contiguous().view(torch.uint8))
            row = vp[page_fmt][slot, gg, j % P]
            assert torch.equal(row, conv(vn[b, gg]).contiguous().view(torch.uint8))
    changed = (kp[page_fmt] != before_k).any(dim=-1)
    assert int(changed.sum()) <= len(positions) * hkv      # nothing else written

    # the decode oracle over the one appended token returns it (single-token closed form)
    spec = synth.CaseSpec("append", 1, hkv, hkv, d, P, seq_lens=[1], fmt=synth.FMT_NAMES[page_fmt],
                          q_fmt="f32")
    case = synth.make_case(spec, 1, "cpu")
    case.k_pool[page_fmt] = kp[page_fmt]
    case.v_pool[page_fmt] = vp[page_fmt]
    case.page_table = pt[:1].clone()
    case.max_pages = pt.shape[1]
    out, _ = oracle_mod.attend(case)
    for gg in range(hkv):
        np.testing.assert_array_equal(out[gg], conv(vn[0, gg]).double().numpy())


def test_append_faults(oracle_mod):
    P, d, hkv = 8, 16, 2
    kp, vp, pt = _append_case(BF16)
    kn = torch.zeros((2, hkv, d))
    before = kp[BF16].clone()
    # past max_pages * P
    assert oracle_mod.append(hkv, d, P, kp, vp, pt, None, BF16, [24, -1], F32, kn, kn) \
        == oracle_mod.DEV_SEQ_LEN
    # a quantised page is not a place for new tokens
    pf = torch.tensor([[BF16, I8, BF16], [BF16, BF16, BF16]], dtype=torch.uint8)
    assert oracle_mod.append(hkv, d, P, kp, vp, pt, pf, BF16, [9, -1], F32, kn, kn) \
        == oracle_mod.DEV_PAGE_FMT
    # a slot outside the pool
    pt2 = pt.clone()
    pt2[0, 0] = 99
    assert oracle_mod.append(hkv, d, P, kp, vp, pt2, None, BF16, [1, -1], F32, kn, kn) \
        == oracle_mod.DEV_PAGE_ID
    assert torch.equal(kp[BF16], before)
