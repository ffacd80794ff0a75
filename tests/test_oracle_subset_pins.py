"""Pins of the oracle's sink + recent-window token subsets (CPU only).

With window_tokens > 0 each softmax runs over the first sink_tokens tokens
(the attention sinks the ARGUS page keeps, "sink_tokens") and the last
window_tokens tokens (the recent window of the CFR-Atlas page's KeepRecent
policy) of its sequence, exactly, with ALiBi distances unchanged.  Pins: torch
scaled_dot_product_attention in fp64 with the subset as an additive -inf mask
(library special case), a 50-digit decimal brute force, closed forms, and the
fold / split invariants on the subset.
"""
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

from tests._hostkv import host_kv, host_q, sigma_of
from tests.test_oracle_pins import FMTS, small

SUBSETS = [(0, 1), (4, 16), (0, 40), (17, 5), (8, 200), (3, 8), (64, 64)]


def in_set(n, sink, window):
    j = np.arange(n)
    return (j < sink) | (j >= n - window)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("alibi", [False, True])
def test_subset_matches_torch_sdpa_fp64(oracle_mod, fmt, alibi):
    case = small(B=3, Hq=8, Hkv=2, d=32, P=16, lens=(153, 16, 100), fmt=fmt, q_fmt="bf16",
                 alibi=alibi, permute=False, seed=6)
    q = torch.from_numpy(host_q(case))
    for sink, window in SUBSETS:
        out, lse = oracle_mod.attend(case, sink_tokens=sink, window_tokens=window)
        for b in range(case.batch):
            Ks, Vs = zip(*[host_kv(case, b, g) for g in range(case.num_kv_heads)])
            K = torch.from_numpy(np.stack(Ks))[None]
            V = torch.from_numpy(np.stack(Vs))[None]
            n = K.shape[2]
            keep = torch.from_numpy(in_set(n, sink, window))
            mask = torch.where(keep, 0.0, -torch.inf).double()[None, None, None, :]
            if alibi:
                dist = (n - 1 - torch.arange(n, dtype=torch.float64))
                mask = mask + (-case.alibi_slopes.double()[:, None] * dist[None, :])[None, :, None, :]
            ref = torch.nn.functional.scaled_dot_product_attention(
                q[b][None, :, None, :], K, V, attn_mask=mask, scale=sigma_of(case), enable_gqa=True)
            got = out[b * case.num_q_heads:(b + 1) * case.num_q_heads]
            np.testing.assert_allclose(got, ref[0, :, 0].numpy(), rtol=0,
                                       atol=1e-13 * max(1.0, float(V.abs().max())))


def _decimal_subset(q, K, V, sigma, slope, keep):
    getcontext().prec = 50
    n = K.shape[0]
    s = {}
    for j in range(n):
        if keep[j]:
            dot = sum(Decimal(float(q[i])) * Decimal(float(K[j, i])) for i in range(K.shape[1]))
            s[j] = Decimal(sigma) * dot - Decimal(slope) * (n - 1 - j)
    m = max(s.values())
    w = {j: (x - m).exp() for j, x in s.items()}
    L = sum(w.values())
    o = [sum(w[j] * Decimal(float(V[j, i])) for j in w) / L for i in range(V.shape[1])]
    return np.array([float(x) for x in o]), float(m + L.ln())


@pytest.mark.parametrize("fmt,sink,window", [("f32", 3, 5), ("bf16", 0, 7), ("i8", 9, 2),
                                             ("fp8", 1, 1)])
def test_subset_brute_force_decimal(oracle_mod, fmt, sink, window):
    case = small(B=1, Hq=2, Hkv=1, d=8, P=8, lens=(27,), fmt=fmt, q_fmt="f32", alibi=True,
                 softmax_scale=20.0)
    out, lse = oracle_mod.attend(case, sink_tokens=sink, window_tokens=window)
    K, V = host_kv(case, 0, 0)
    q = host_q(case)[0]
    keep = in_set(27, sink, window)
    for h in range(2):
        ref, ref_lse = _decimal_subset(q[h], K, V, 20.0, float(case.alibi_slopes[h]), keep)
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-13 * max(1.0, np.abs(V).max()))
        assert lse[h] == pytest.approx(ref_lse, rel=1e-13)


@pytest.mark.parametrize("fmt", FMTS)
def test_subset_closed_forms(oracle_mod, fmt):
    case = small(B=2, Hq=4, Hkv=2, d=16, P=8, lens=(61, 9), fmt=fmt, alibi=True)
    full_o, full_l = oracle_mod.attend(case)
    # a window covering the whole sequence (with or without sinks) is full attention
    for sink, window in [(0, 61), (5, 100), (30, 31)]:
        o, l = oracle_mod.attend(case, sink_tokens=sink, window_tokens=window)
        np.testing.assert_array_equal(o[4:], full_o[4:])           # sequence 1 (n = 9)
        if sink + window >= 61:
            np.testing.assert_array_equal(o, full_o)
            np.testing.assert_array_equal(l, full_l)
    # a window of one token and no sink returns that token's V row
    o, _ = oracle_mod.attend(case, sink_tokens=0, window_tokens=1)
    for k, (b, h) in enumerate([(b, h) for b in range(2) for h in range(4)]):
        n = int(case.seq_lens[b])
        _, V = host_kv(case, b, h // 2)
        np.testing.assert_array_equal(o[k], V[n - 1])


@pytest.mark.parametrize("fmt", FMTS)
def test_subset_fold_and_split_equal_direct(oracle_mod, fmt):
    case = small(B=2, Hq=4, Hkv=2, d=16, P=8, lens=(523, 64), fmt=fmt, alibi=True)
    for sink, window in [(4, 100), (13, 9), (0, 64)]:
        o0, l0 = oracle_mod.attend(case, sink_tokens=sink, window_tokens=window)
        for blk in [1, 7, 64]:
            o1, l1 = oracle_mod.attend(case, mode=1, arg=blk, sink_tokens=sink,
                                       window_tokens=window)
            np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
        for S in [2, 5]:
            o2, _ = oracle_mod.attend(case, mode=2, arg=S, sink_tokens=sink, window_tokens=window)
            np.testing.assert_allclose(o2, o0, rtol=0, atol=1e-12)
