"""GPU parity of multi-query decode (cfr_paged_decode_multi) against the oracle:
the last Q positions of every sequence as causal query rows, on every decode
kernel, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._gpu import TOL_F32_ABS, TOL_LOWP_REL, all_f32, vmax_table_sel
from tests._hostkv import host_kv, kv_head_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


def mq_case(Q, B=3, Hq=8, Hkv=2, d=128, P=64, lens=(700, 77, 300), fmt="bf16", q_fmt="bf16",
            alibi=True, seed=41, **kw):
    spec = synth.CaseSpec("mq", B, Hq, Hkv, d, P, seq_lens=list(lens), fmt=fmt, q_fmt=q_fmt,
                          alibi=alibi, num_queries=Q, **kw)
    return synth.make_case(spec, seed, "cuda")


def check_mq(case, out, lse, sel=None, allow_empty=False):
    hc = case.to("cpu")
    rows = case.num_q_heads * case.num_queries
    pairs = sel or [(b, r) for b in range(case.batch) for r in range(rows)]
    ref_o, ref_l = oracle.attend(hc, sel=pairs, allow_empty=allow_empty)
    f32 = all_f32(case)
    vmax = {}
    for b, r in pairs:
        g = kv_head_of(hc, r % case.num_q_heads)
        if (b, g) not in vmax:
            _, V = host_kv(hc, b, g)
            vmax[(b, g)] = float(np.abs(V).max())
    for k, (b, r) in enumerate(pairs):
        got = out[b, r].double().numpy()
        g = kv_head_of(hc, r % case.num_q_heads)
        tol = TOL_F32_ABS if f32 else TOL_LOWP_REL * vmax[(b, g)]
        err = np.abs(got - ref_o[k]).max()
        assert err <= tol, f"b={b} row={r}: {err:.3e} > {tol:.3e}"
        if np.isneginf(ref_l[k]):
            assert np.isneginf(float(lse[b, r]))
        else:
            assert abs(float(lse[b, r]) - ref_l[k]) <= 1e-4 * max(1.0, abs(ref_l[k]))


def run_mq(case):
    bufs = binding.paged_decode(case)
    torch.cuda.synchronize()
    return bufs.out.cpu(), bufs.lse.cpu(), int(bufs.err.item())


CONFIGS = {
    # (kernel it takes, case keywords)
    "tcgen05-8rows": dict(Q=2, Hq=8, Hkv=2),
    "tcgen05-16rows": dict(Q=4, Hq=8, Hkv=2),
    "tcgen05-mha-16": dict(Q=16, Hq=4, Hkv=4),
    "tcgen05-int-fp8": dict(Q=3, Hq=8, Hkv=2, P=128, fmt="tiered",
                            tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
    "cuda-core-d64": dict(Q=4, Hq=8, Hkv=2, d=64, P=16, fmt="tiered",
                          tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
    "tcgen05-d64": dict(Q=2, Hq=8, Hkv=2, d=64, P=32),
    "tcgen05-d64-int": dict(Q=3, Hq=8, Hkv=2, d=64, P=128, fmt="tiered",
                            tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
    "f32-tma": dict(Q=2, Hq=4, Hkv=4, d=64, fmt="f32", q_fmt="f32"),
    "cuda-core-f32": dict(Q=4, Hq=8, Hkv=4, d=64, fmt="f32", q_fmt="f32"),
}


@pytest.mark.parametrize("name", list(CONFIGS))
def test_multiquery_parity(name):
    case = mq_case(**CONFIGS[name])
    out, lse, err = run_mq(case)
    assert err == 0
    check_mq(case, out, lse)


def test_one_query_equals_decode():
    case = mq_case(1, Hq=8, Hkv=2)
    bufs = binding.DecodeBuffers(case)
    pool = binding.kv_pool_struct(case)
    st = binding.lib().cfr_paged_decode_multi(
        binding._p(case.q), case.q_fmt, __import__("ctypes").byref(pool), binding._p(case.page_table),
        case.max_pages, binding._p(case.seq_lens), case.batch, binding._p(case.page_fmt),
        case.uniform_fmt, case.num_q_heads, 1, None, binding._p(case.alibi_slopes), 0.0,
        binding._p(bufs.out), binding._p(bufs.lse), binding._p(bufs.workspace),
        bufs.workspace.numel(), binding._p(bufs.err), binding._stream(None), binding.PHASE_ALL)
    assert st == 0
    ref = binding.paged_decode(case)
    torch.cuda.synchronize()
    assert torch.equal(bufs.out, ref.out) and torch.equal(bufs.lse, ref.lse)


def test_sequence_shorter_than_queries():
    case = mq_case(4, lens=(300, 3, 100))
    out, lse, err = run_mq(case)
    assert err == binding.DEVERR_SEQ_LEN
    assert torch.all(out[1] == 0) and torch.all(torch.isneginf(lse[1]))
    rows = case.num_q_heads * case.num_queries
    check_mq(case, out, lse, sel=[(b, r) for b in (0, 2) for r in range(rows)])


@pytest.mark.parametrize("fmt", ["bf16", "i8", "f32"])
def test_more_than_16_rows_per_kv_head(fmt):
    # 8 heads x 4 queries = 32 rows per kv head: decoded as two groups of 16
    case = mq_case(4, Hq=16, Hkv=2, fmt=fmt, q_fmt="f32" if fmt == "f32" else "bf16",
                   P=128 if fmt == "i8" else 64)
    out, lse, err = run_mq(case)
    assert err == 0
    check_mq(case, out, lse)


@pytest.mark.parametrize("name,Q", [("gqa", 4), ("alibi1m", 2)])
def test_multiquery_full_size(name, Q):
    case = synth.workload(name, "cuda", num_queries=Q)
    out, lse, err = run_mq(case)
    assert err == 0
    rows = case.num_q_heads * Q
    G = case.num_q_heads // case.num_kv_heads
    if name == "alibi1m":
        sel = [(0, r) for r in (0, 1, case.num_q_heads + 7 * G, rows - 1)]
    else:
        sel = [(b, (b * 7 + k * G) % rows) for b in range(case.batch) for k in range(2)]
    check_mq(case, out, lse, sel=sel)
