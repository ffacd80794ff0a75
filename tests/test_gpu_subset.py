"""GPU parity of sink + recent-window decode (cfr_paged_decode_sink_window)
against the oracle on the same token subsets, on every decode kernel, plus the
guarantee that pages outside the subset are never read."""
import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import binding, synth
from tests._gpu import TOL_F32_ABS, TOL_LOWP_REL, all_f32, small_case, vmax_table_sel
from tests._hostkv import kv_head_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


def run_subset(case, sink, window):
    bufs = binding.paged_decode(case, sink_window=(sink, window))
    torch.cuda.synchronize()
    return bufs.out.cpu(), bufs.lse.cpu(), int(bufs.err.item())


def check_subset(case, out, lse, sink, window, sel=None):
    hc = case.to("cpu")
    pairs = sel or [(b, h) for b in range(case.batch) for h in range(case.num_q_heads)]
    ref_o, ref_l = oracle.attend(hc, sel=pairs, sink_tokens=sink, window_tokens=window)
    f32 = all_f32(case)
    vmax = None if f32 else vmax_table_sel(hc, pairs)
    for k, (b, h) in enumerate(pairs):
        g = out[b, h].double().numpy()
        tol = TOL_F32_ABS if f32 else TOL_LOWP_REL * vmax[(b, kv_head_of(hc, h))]
        err = np.abs(g - ref_o[k]).max()
        assert err <= tol, f"b={b} h={h} sink={sink} window={window}: {err:.3e} > {tol:.3e}"
        assert abs(float(lse[b, h]) - ref_l[k]) <= 1e-4 * max(1.0, abs(ref_l[k]))


SUBSETS = [(0, 1), (4, 16), (17, 5), (8, 200), (64, 64), (0, 700), (3, 129), (130, 1)]

PATHS = {
    "f32-tma": dict(d=64, P=64, fmt="f32", q_fmt="f32", Hq=4, Hkv=2),
    "tcgen05-bf16": dict(d=128, P=64, fmt="bf16", q_fmt="bf16", Hq=8, Hkv=2),
    "tcgen05-int": dict(d=128, P=128, fmt="tiered", q_fmt="bf16", Hq=8, Hkv=2,
                        tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
    "cuda-core": dict(d=64, P=16, fmt="tiered", q_fmt="bf16", Hq=8, Hkv=2,
                      tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
    "tcgen05-d64": dict(d=64, P=32, fmt="bf16", q_fmt="bf16", Hq=8, Hkv=2),
}
WANT = {"f32-tma": binding.PATH_F32_TMA, "tcgen05-bf16": binding.PATH_TENSOR_CORE,
        "tcgen05-int": binding.PATH_TENSOR_CORE, "cuda-core": binding.PATH_CUDA_CORE,
        "tcgen05-d64": binding.PATH_TENSOR_CORE}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("alibi", [False, True])
def test_subset_parity(path, alibi):
    kw = dict(PATHS[path])
    case = small_case(B=3, lens=(1500, 77, 600), alibi=alibi, seed=33, **kw)
    assert binding.decode_path(case) == WANT[path]
    for sink, window in SUBSETS:
        out, lse, err = run_subset(case, sink, window)
        assert err == 0
        check_subset(case, out, lse, sink, window)


def test_full_window_equals_full_decode():
    case = small_case(B=2, Hq=8, Hkv=2, d=128, P=64, lens=(900, 130), fmt="bf16", alibi=True)
    full = binding.paged_decode(case)
    out, lse, err = run_subset(case, 10, 900)
    torch.cuda.synchronize()
    assert err == 0
    assert torch.equal(out, full.out.cpu()) and torch.equal(lse, full.lse.cpu())


def test_pages_outside_the_subset_are_never_read():
    # the gap pages point at a slot far outside the pool: a read would set
    # CFR_DEVERR_PAGE_ID; none must happen
    P = 64
    case = small_case(B=2, Hq=8, Hkv=2, d=128, P=P, lens=(40 * P + 3, 20 * P), fmt="bf16")
    sink, window = 2 * P, 5 * P + 7
    pt = case.page_table.clone()
    for b in range(2):
        n = int(case.seq_lens[b])
        for p in range(-(-n // P)):
            if p * P < sink or (p + 1) * P > n - window:      # holds a token of the subset
                continue
            pt[b, p] = 1 << 30
    good = case.page_table
    case.page_table = pt
    out, lse, err = run_subset(case, sink, window)
    assert err == 0
    # the oracle resolves every page: compare on the original table (the gap
    # pages cannot change the result)
    case.page_table = good
    check_subset(case, out, lse, sink, window)


def test_subset_rejects():
    case = small_case(fmt="bf16")
    bufs = binding.DecodeBuffers(case)
    assert binding.paged_decode_raw(case, bufs, sink_window=(-1, 4)) == 1
    assert binding.paged_decode_raw(case, bufs, sink_window=(4, 0)) == 1


def test_subset_full_size_alibi_1m():
    # the 1M-token ALiBi workload with 4 attention sinks and a 32K recent window
    case = synth.workload("alibi1m", device="cuda")
    out, lse, err = run_subset(case, 4, 32768)
    assert err == 0
    G = case.num_q_heads // case.num_kv_heads
    check_subset(case, out, lse, 4, 32768, sel=[(0, h) for h in (0, 1, 3 * G, 8 * G - 1)])
