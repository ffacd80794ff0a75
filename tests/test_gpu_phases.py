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
