"""Seeded random sweep of decode configurations against the oracle, through the
C ABI: batch, head counts and maps, head_dim, page size, storage-format mixes,
lengths (ragged tails, single tokens, exact page multiples), ALiBi, query
counts and sink + window subsets are drawn per case, so that combinations the
fixed parity matrix does not name are exercised on whichever kernel the
library selects for them."""
import random

import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._gpu import TOL_F32_ABS, TOL_LOWP_REL, all_f32, vmax_table_sel
from tests._hostkv import kv_head_of

pytestmark = pytest.mark.gpu

N_CASES = 160


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


def draw(i):
    rng = random.Random(1000 + i)
    d = rng.choice([64, 128])
    Hkv = rng.choice([1, 2, 3, 4, 8])
    G = rng.choice([1, 2, 3, 4, 5, 8])
    Q = rng.choice([1, 1, 1, 2, 3])
    while G * Q > 16:
        Q -= 1
    Hq = Hkv * G
    P = rng.choice([8, 16, 32, 64, 128, 256])
    B = rng.randint(1, 9)
    lens = []
    for _ in range(B):
        kind = rng.random()
        if kind < 0.15:
            lens.append(max(Q, 1))
        elif kind < 0.3:
            lens.append(P * rng.randint(1, 6))
        elif kind < 0.4:                              # long: many splits to merge
            lens.append(rng.randint(24 * P, 48 * P + 5))
        else:
            lens.append(rng.randint(max(Q, 1), 12 * P + 7))
    fmts = ["f32", "bf16", "i8", "i4", "fp8"]
    if rng.random() < 0.4:
        pick = rng.sample(fmts, rng.randint(2, 4))
        tiers = [(1.0 / len(pick), f) for f in pick]
        fmt = "tiered"
    else:
        fmt, tiers = rng.choice(fmts), None
    q_fmt = "f32" if (fmt == "f32" or rng.random() < 0.3) else "bf16"
    head_map = None
    if rng.random() < 0.25 and Q == 1:
        head_map = [rng.randrange(Hkv) for _ in range(Hq)]
        for g in range(Hkv):                      # every kv head keeps at least one row
            head_map[g % Hq] = g
        counts = [head_map.count(g) for g in range(Hkv)]
        if max(counts) > 16:
            head_map = None
    alibi = rng.random() < 0.5
    sw = None
    if Q == 1 and rng.random() < 0.3:
        sw = (rng.choice([0, 1, 4, P + 3]), rng.choice([1, 5, P, 3 * P + 1]))
    return dict(B=B, Hq=Hq, Hkv=Hkv, d=d, P=P, lens=lens, fmt=fmt, tiers=tiers, q_fmt=q_fmt,
                head_map=head_map, alibi=alibi, Q=Q, sw=sw, seed=2000 + i)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_case(i):
    c = draw(i)
    kw = dict(tiers=c["tiers"]) if c["tiers"] else {}
    if c["head_map"] is not None:
        kw["head_map"] = c["head_map"]
    spec = synth.CaseSpec("sweep", c["B"], c["Hq"], c["Hkv"], c["d"], c["P"],
                          seq_lens=c["lens"], fmt=c["fmt"], q_fmt=c["q_fmt"], alibi=c["alibi"],
                          num_queries=c["Q"], **kw)
    case = synth.make_case(spec, c["seed"], "cuda")
    bufs = binding.paged_decode(case, sink_window=c["sw"])
    torch.cuda.synchronize()
    assert int(bufs.err.item()) == 0, c
    out, lse = bufs.out.cpu(), bufs.lse.cpu()
    hc = case.to("cpu")
    rows = c["Hq"] * c["Q"]
    pairs = [(b, r) for b in range(c["B"]) for r in range(rows)]
    sub = dict(sink_tokens=c["sw"][0], window_tokens=c["sw"][1]) if c["sw"] else {}
    ref_o, ref_l = oracle.attend(hc, sel=pairs, **sub)
    f32 = all_f32(case)
    Hq = c["Hq"]
    vmax = None if f32 else vmax_table_sel(hc, [(b, r % Hq) for b, r in pairs])
    for k, (b, r) in enumerate(pairs):
        g = out[b, r].double().numpy()
        tol = TOL_F32_ABS if f32 else TOL_LOWP_REL * vmax[(b, kv_head_of(hc, r % Hq))]
        err = np.abs(g - ref_o[k]).max()
        assert np.all(np.isfinite(g)), f"{c}: non-finite output at b={b} row={r}"
        assert err <= tol, f"{c}: b={b} row={r} err {err:.3e} > {tol:.3e}"
        assert abs(float(lse[b, r]) - ref_l[k]) <= 1e-4 * max(1.0, abs(ref_l[k])), (c, b, r)
