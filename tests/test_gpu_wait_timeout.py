"""The bounded on-chip wait of the decode kernels gives up instead of hanging.

cfr_wait_probe runs the kernels' own mbarrier wait with a short cycle limit on
a barrier that nothing arrives on: the wait must end, report
CFR_DEVERR_TIMEOUT through the error word, and leave the context usable (a
decode right after it is correct).  The same wait on a barrier that was arrived
on completes without an error bit."""
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


def _probe(limit, arrive):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    assert binding.wait_probe(limit, arrive, err, res) == binding.CFR_OK
    torch.cuda.synchronize()
    return int(err.item()), int(res.item())


def test_wait_that_nothing_completes_gives_up_with_timeout_bit():
    for limit in (1000, 100_000, 2_000_000):
        err, res = _probe(limit, arrive=False)
        assert err == binding.DEVERR_TIMEOUT
        assert res == 0


def test_wait_on_a_completed_phase_returns_clean():
    err, res = _probe(100_000, arrive=True)
    assert err == 0 and res == 1


def test_context_usable_after_a_timeout():
    _probe(100_000, arrive=False)
    case = small_case(seed=5, B=2, Hq=8, Hkv=2, d=128, P=16, lens=(300, 41), fmt="bf16",
                      q_fmt="bf16")
    bufs = binding.paged_decode(case)
    torch.cuda.synchronize()
    assert int(bufs.err.item()) == 0
    check(case, bufs.out.cpu(), bufs.lse.cpu())

