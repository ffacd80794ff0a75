"""Shared helpers of the GPU parity tests: run the library, compare with the oracle."""
import numpy as np
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._hostkv import host_kv, kv_head_of

TOL_F32_ABS = 1e-5      # fp32 K/V: absolute max error
TOL_LOWP_REL = 2e-3     # bf16 / int8 / int4 K/V: max error relative to max|V|


def all_f32(case) -> bool:
    if case.page_fmt is None:
        return case.uniform_fmt == synth.F32
    return set(case.k_pool.keys()) == {synth.F32}


def run(case, stream=None):
    """Decode on the GPU; returns (out, lse, err) on the host."""
    bufs = binding.paged_decode(case, stream=stream)
    torch.cuda.synchronize()
    return bufs.out.cpu(), bufs.lse.cpu(), int(bufs.err.item())


def vmax_table(case, host_case):
    """max|V| over the valid tokens of each (b, kv head), from the independent host decode."""
    t = {}
    for b in range(case.batch):
        if int(case.seq_lens[b]) <= 0:
            continue
        for g in range(case.num_kv_heads):
            _, V = host_kv(host_case, b, g)
            t[(b, g)] = float(np.abs(V).max()) if V.size else 0.0
    return t


def check(case, out, lse, sel=None, host_case=None, lse_tol=1e-4, nthreads=None):
    """Compare GPU (out, lse) with the oracle on the (b, h) pairs in sel (default all).

    fp32 caches: |o_gpu - o_ref| <= 1e-5.  Other caches: <= 2e-3 * max|V| of that
    (b, kv head).  lse: |lse_gpu - lse_ref| <= lse_tol * max(1, |lse_ref|).
    Returns the worst normalised error (error / tolerance).
    """
    hc = host_case if host_case is not None else case.to("cpu")
    pairs = sel if sel is not None else [(b, h) for b in range(case.batch)
                                         for h in range(case.num_q_heads)]
    ref_o, ref_l = oracle.attend(hc, sel=pairs, nthreads=nthreads)
    f32 = all_f32(case)
    vmax = None if f32 else vmax_table_sel(hc, pairs)
    worst = 0.0
    for k, (b, h) in enumerate(pairs):
        g = out[b, h].double().numpy()
        err = np.abs(g - ref_o[k]).max()
        tol = TOL_F32_ABS if f32 else TOL_LOWP_REL * vmax[(b, kv_head_of(hc, h))]
        assert np.all(np.isfinite(g)), f"non-finite output at b={b} h={h}"
        assert err <= tol, f"b={b} h={h}: max err {err:.3e} > tol {tol:.3e}"
        worst = max(worst, err / tol)
        lg = float(lse[b, h])
        assert abs(lg - ref_l[k]) <= lse_tol * max(1.0, abs(ref_l[k])), \
            f"b={b} h={h}: lse {lg} vs {ref_l[k]}"
    return worst


def vmax_table_sel(hc, pairs):
    t = {}
    for (b, h) in pairs:
        g = kv_head_of(hc, h)
        if (b, g) not in t:
            _, V = host_kv(hc, b, g)
            t[(b, g)] = float(np.abs(V).max())
    return t


def small_case(B=2, Hq=4, Hkv=2, d=64, P=16, lens=(100, 37), fmt="bf16", q_fmt="bf16",
               alibi=False, seed=7, **kw):
    spec = synth.CaseSpec("t", B, Hq, Hkv, d, P, seq_lens=list(lens), fmt=fmt, q_fmt=q_fmt,
                          alibi=alibi, **kw)
    return synth.make_case(spec, seed, "cuda")
