"""Decode split into its phases through cfr_paged_decode_phases: the schedule,
the decode and the merge as separate calls on one workspace, then the decode
and merge repeated on the same schedule.  The repeated calls rely on the decode
kernel leaving its work-item counter at zero (no schedule launch re-zeroes it),
so every repeat must give the same bits as the first result; all of them are
checked against the oracle."""
import pytest
import torch

from paged_long_context_b200 import binding
from tests._gpu import check, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    import oracle
    build.build()
    oracle.build()


CASES = {
    # bf16, d 128: tcgen05 path, items claimed at run time
    "bf16_claimed": dict(B=5, Hq=16, Hkv=4, d=128, P=16, lens=(3000, 17, 1500, 128, 2049),
                         fmt="bf16", q_fmt="bf16", alibi=True),
    # int4 / int8 / bf16 tiers: tcgen05 path, fixed share of items
    "tiered_fixed": dict(B=3, Hq=8, Hkv=2, d=128, P=128, lens=(2000, 700, 4096), fmt="tiered",
                         tiers=[(0.3, "i4"), (0.4, "i8"), (0.3, "bf16")], q_fmt="bf16"),
    # fp32, d 64: the fp32 kernel
    "f32": dict(B=2, Hq=4, Hkv=4, d=64, P=64, lens=(1000, 4000), fmt="f32", q_fmt="f32"),
    # int8 and bf16 pages of 32 tokens, d 64: the CUDA-core kernel
    "cc": dict(B=3, Hq=8, Hkv=2, d=64, P=32, lens=(2500, 31, 900), fmt="tiered",
               tiers=[(0.5, "i8"), (0.5, "bf16")], q_fmt="bf16"),
    # uniform int4 pages of 32 tokens: the tcgen05 path, per-page scales in a tile
    "i4_small_pages": dict(B=3, Hq=8, Hkv=2, d=128, P=32, lens=(2500, 31, 900), fmt="i4",
                           q_fmt="bf16", alibi=True),
    # bf16, d 64: the tcgen05 path reading the first half of its operands
    "bf16_d64": dict(B=3, Hq=8, Hkv=2, d=64, P=32, lens=(2500, 31, 900), fmt="bf16", q_fmt="bf16"),
    # uniform int8, 4 rows per kv head: tcgen05 int8-MMA variant, items claimed
    "i8_claimed": dict(B=3, Hq=8, Hkv=2, d=128, P=128, lens=(3000, 129, 5000), fmt="i8",
                       q_fmt="bf16", alibi=True),
    # 32 query heads on one kv head: two row groups per sequence, merged separately
    "mqa": dict(B=2, Hq=32, Hkv=1, d=128, P=64, lens=(4000, 700), fmt="bf16", q_fmt="bf16"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_phases_and_repeated_decode(name):
    case = small_case(seed=11, **CASES[name])
    bufs = binding.DecodeBuffers(case)
    for ph in (binding.PHASE_SCHEDULE, binding.PHASE_DECODE, binding.PHASE_MERGE):
        assert binding.paged_decode_raw(case, bufs, phases=ph) == binding.CFR_OK
    torch.cuda.synchronize()
    assert int(bufs.err.item()) == 0
    out0, lse0 = bufs.out.clone(), bufs.lse.clone()
    check(case, out0.cpu(), lse0.cpu())
    for _ in range(3):
        bufs.out.fill_(float("nan"))
        bufs.lse.fill_(float("nan"))
        assert binding.paged_decode_raw(
            case, bufs, phases=binding.PHASE_DECODE | binding.PHASE_MERGE) == binding.CFR_OK
        torch.cuda.synchronize()
        assert int(bufs.err.item()) == 0
        assert torch.equal(bufs.out, out0)
        assert torch.equal(bufs.lse, lse0)


FOREIGN = {
    # tcgen05 path, bf16 pages, claimed items
    "bf16": dict(d=128, fmt="bf16", q_fmt="bf16"),
    # tcgen05 path, quantised tiers, fixed share
    "tiered": dict(d=128, fmt="tiered", tiers=[(0.5, "i8"), (0.5, "bf16")], q_fmt="bf16", P=128),
    # fp32 TMA kernel
    "f32": dict(d=64, fmt="f32", q_fmt="f32", Hq=4, Hkv=4),
    # general CUDA-core kernel (int8 and bf16 pages of 16 tokens, head_dim 64)
    "cc": dict(d=64, fmt="tiered", tiers=[(0.5, "i8"), (0.5, "bf16")], q_fmt="bf16"),
}


@pytest.mark.parametrize("name", list(FOREIGN))
def test_decode_only_call_on_a_foreign_schedule_stays_in_its_workspace(name):
    """A decode-only call (no schedule launch) on a workspace that a call with
    other arguments scheduled breaks the documented rule of split-phase calls.
    The kernels must then cap the split count and skip foreign splits, report
    CFR_DEVERR_SCHEDULE, and write nothing past the bytes this call was given."""
    kw = dict(Hq=16, Hkv=4, P=16)
    kw.update(FOREIGN[name])
    P = kw.pop("P")
    big = small_case(seed=21, B=8, P=P, lens=(8192,) * 8, **kw)
    small = small_case(seed=22, B=1, P=P, lens=(4 * P,), **kw)
    assert small.max_pages == 4
    bb, sb = binding.DecodeBuffers(big), binding.DecodeBuffers(small)
    ws_big, ws_small = bb.workspace.numel(), sb.workspace.numel()
    assert ws_small < ws_big
    arena = torch.zeros(ws_big + (1 << 20), dtype=torch.uint8, device="cuda")
    bb.workspace = arena[:ws_big]
    sb.workspace = arena[:ws_small]
    assert binding.decode_path(small) == binding.decode_path(big)

    assert binding.paged_decode_raw(big, bb) == binding.CFR_OK
    torch.cuda.synchronize()
    assert int(bb.err.item()) == 0
    guard = arena[ws_small:].clone()

    assert binding.paged_decode_raw(
        small, sb, phases=binding.PHASE_DECODE | binding.PHASE_MERGE) == binding.CFR_OK
    torch.cuda.synchronize()
    assert int(sb.err.item()) & binding.DEVERR_SCHEDULE
    assert torch.equal(arena[ws_small:], guard)

    # the same call with its own schedule is clean and correct again
    sb.err.zero_()
    assert binding.paged_decode_raw(small, sb) == binding.CFR_OK
    torch.cuda.synchronize()
    assert int(sb.err.item()) == 0
    check(small, sb.out.cpu(), sb.lse.cpu())
