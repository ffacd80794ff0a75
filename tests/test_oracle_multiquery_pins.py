"""Pins of the oracle's multi-query decode (CPU only).

Q query tokens per sequence are its last Q positions; query i attends causally
to tokens j <= n - Q + i with ALiBi distance n - Q + i - j (the causal mask of
the RustAttention page's scaled dot-product definition, applied to the query
rows of a speculative / chunked step over the paged cache).  Pins: torch
scaled_dot_product_attention in fp64 with that causal mask (library special
case), a 50-digit decimal brute force, the reduction of each query row to the
single-query oracle over its prefix, and the fold / split invariants.
"""
import dataclasses
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle as oracle_pkg
from paged_long_context_b200 import synth
from tests._hostkv import host_kv, sigma_of
from tests.test_oracle_pins import FMTS


def mq_case(Q, B=2, Hq=4, Hkv=2, d=16, P=8, lens=(37, 20), fmt="f32", q_fmt="f32", alibi=False,
            seed=11, **kw):
    spec = synth.CaseSpec("mq", B, Hq, Hkv, d, P, seq_lens=list(lens), fmt=fmt, q_fmt=q_fmt,
                          alibi=alibi, num_queries=Q, **kw)
    return synth.make_case(spec, seed, "cpu")


def host_q_rows(case):
    """q as float64 [B][Q][Hq][d]."""
    q = case.q.cpu()
    if case.q_fmt == synth.F32:
        x = q.numpy().astype(np.float64)
    else:
        x = (q.numpy().view(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.reshape(case.batch, case.num_queries, case.num_q_heads, case.head_dim)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("alibi", [False, True])
@pytest.mark.parametrize("Q", [2, 4, 7])
def test_multiquery_matches_torch_sdpa_causal(oracle_mod, fmt, alibi, Q):
    case = mq_case(Q, B=3, Hq=8, Hkv=2, d=32, P=16, lens=(53, 16, 100), fmt=fmt, q_fmt="bf16",
                   alibi=alibi, permute=False, seed=5)
    out, lse = oracle_mod.attend(case)
    q = torch.from_numpy(host_q_rows(case))              # [B][Q][Hq][d]
    Hq = case.num_q_heads
    for b in range(case.batch):
        Ks, Vs = zip(*[host_kv(case, b, g) for g in range(case.num_kv_heads)])
        K = torch.from_numpy(np.stack(Ks))[None]        # [1, Hkv, n, d]
        V = torch.from_numpy(np.stack(Vs))[None]
        n = K.shape[2]
        pos = n - Q + torch.arange(Q, dtype=torch.float64)          # query positions
        j = torch.arange(n, dtype=torch.float64)
        mask = torch.where(j[None, :] <= pos[:, None], 0.0, -torch.inf).double()[None, None]
        if alibi:
            dist = pos[:, None] - j[None, :]
            mask = mask + (-case.alibi_slopes.double()[:, None, None] * dist[None])[None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b].permute(1, 0, 2)[None], K, V, attn_mask=mask, scale=sigma_of(case),
            enable_gqa=True)                                # [1, Hq, Q, d]
        got = out[b * Q * Hq:(b + 1) * Q * Hq].reshape(Q, Hq, -1)
        np.testing.assert_allclose(got, ref[0].permute(1, 0, 2).numpy(), rtol=0,
                                   atol=1e-13 * max(1.0, float(V.abs().max())))


@pytest.mark.parametrize("fmt", FMTS)
def test_each_query_row_is_a_single_query_decode(oracle_mod, fmt):
    Q, Hq = 3, 4
    case = mq_case(Q, fmt=fmt, alibi=True, lens=(45, 9))
    out, lse = oracle_mod.attend(case)
    qr = case.q.reshape(case.batch, Q, Hq, -1)
    for i in range(Q):
        one = dataclasses.replace(case, num_queries=1, q=qr[:, i].contiguous(),
                                  seq_lens=case.seq_lens - (Q - 1 - i))
        o1, l1 = oracle_mod.attend(one)
        for b in range(case.batch):
            rows = slice((b * Q + i) * Hq, (b * Q + i + 1) * Hq)
            np.testing.assert_array_equal(out[rows], o1[b * Hq:(b + 1) * Hq])
            np.testing.assert_array_equal(lse[rows], l1[b * Hq:(b + 1) * Hq])


def _decimal_causal(q, K, V, sigma, slope, pos):
    getcontext().prec = 50
    s = []
    for j in range(pos + 1):
        dot = sum(Decimal(float(q[i])) * Decimal(float(K[j, i])) for i in range(K.shape[1]))
        s.append(Decimal(sigma) * dot - Decimal(slope) * (pos - j))
    m = max(s)
    w = [(x - m).exp() for x in s]
    L = sum(w)
    o = [sum(w[j] * Decimal(float(V[j, i])) for j in range(pos + 1)) / L
         for i in range(V.shape[1])]
    return np.array([float(x) for x in o]), float(m + L.ln())


@pytest.mark.parametrize("fmt,Q", [("f32", 3), ("bf16", 5), ("fp8", 2), ("i4", 4)])
def test_multiquery_brute_force_decimal(oracle_mod, fmt, Q):
    case = mq_case(Q, B=1, Hq=2, Hkv=1, d=8, P=8, lens=(21,), fmt=fmt, alibi=True,
                   softmax_scale=15.0)
    out, lse = oracle_mod.attend(case)
    K, V = host_kv(case, 0, 0)
    q = host_q_rows(case)[0]
    for i in range(Q):
        for h in range(2):
            ref, ref_l = _decimal_causal(q[i, h], K, V, 15.0, float(case.alibi_slopes[h]),
                                         21 - Q + i)
            k = i * 2 + h
            np.testing.assert_allclose(out[k], ref, rtol=0, atol=1e-13 * max(1.0, np.abs(V).max()))
            assert lse[k] == pytest.approx(ref_l, rel=1e-13)


@pytest.mark.parametrize("fmt", FMTS)
def test_multiquery_fold_and_split_equal_direct(oracle_mod, fmt):
    case = mq_case(4, B=2, Hq=4, Hkv=2, d=16, P=8, lens=(523, 64), fmt=fmt, alibi=True)
    o0, l0 = oracle_mod.attend(case)
    for blk in [1, 7, 64]:
        o1, l1 = oracle_mod.attend(case, mode=1, arg=blk)
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-12)
        np.testing.assert_allclose(l1, l0, rtol=1e-12)
    for S in [2, 5]:
        o2, _ = oracle_mod.attend(case, mode=2, arg=S)
        np.testing.assert_allclose(o2, o0, rtol=0, atol=1e-12)


def test_query_rows_without_tokens_are_empty(oracle_mod):
    # n = 2 with Q = 4: queries 0 and 1 sit before the first cached token
    case = mq_case(4, B=1, Hq=2, Hkv=1, lens=(2,))
    with pytest.raises(oracle_pkg.OracleError):
        oracle_mod.attend(case)
    out, lse = oracle_mod.attend(case, allow_empty=True)
    assert np.all(out[:4] == 0) and np.all(np.isneginf(lse[:4]))
    assert np.all(np.isfinite(lse[4:]))
