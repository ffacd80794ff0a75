"""Parity at the five page-shaped workloads' full sizes, in the launch
configuration bench.py times: the library call on the whole workload, then the
oracle on sampled (sequence, query head) outputs (every output where the oracle
finishes in seconds)."""
import numpy as np
import pytest
import torch

import oracle
from paged_long_context_b200 import accounting, binding, synth
from tests._gpu import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()
    oracle.build()


def _sample(case, name):
    B, Hq, G = case.batch, case.num_q_heads, case.num_q_heads // case.num_kv_heads
    if name in ("tiny", "cfr"):
        return None                                    # every output
    if name == "alibi1m":
        # two kv groups, four query heads each (one materialisation per group)
        return [(0, h) for h in (0, 1, 6, 7)] + [(0, h) for h in (5 * G, 5 * G + 3, 6 * G - 2, 6 * G - 1)]
    # every sequence, query heads rotating over the kv groups
    return [(b, (b * 5 + k * G) % Hq) for b in range(B) for k in range(2)]


@pytest.mark.parametrize("name", ["tiny", "cfr", "gqa", "tiered", "alibi1m"])
def test_full_size_workload(name):
    case = synth.workload(name, device="cuda")
    bufs = binding.paged_decode(case)
    torch.cuda.synchronize()
    assert int(bufs.err.item()) == 0
    out, lse = bufs.out.cpu(), bufs.lse.cpu()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    host = case.to("cpu")
    worst = check(case, out, lse, sel=_sample(case, name), host_case=host)
    print(f"{name}: worst error / tolerance = {worst:.3f}, path {binding.decode_path(case)}")
    # byte accounting of the CFR-shaped workload: 32 heads x the page's 33,554,432 bytes
    if name == "cfr":
        assert accounting.step_bytes(case)["kv"] == 32 * 33554432
