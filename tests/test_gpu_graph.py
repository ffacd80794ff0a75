"""The decode entry points enqueue only stream-ordered work (no allocation, no
host synchronisation), so a call can be captured in a CUDA graph and replayed.
Each replay must give exactly the eager call's result."""
import pytest
import torch

from paged_long_context_b200 import binding, synth
from tests._gpu import small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()


CASES = {
    "f32": dict(d=64, P=64, fmt="f32", q_fmt="f32", Hq=4, Hkv=2),
    "bf16-gqa": dict(d=128, P=16, fmt="bf16", Hq=8, Hkv=2),
    "tiered-fp8": dict(d=128, P=128, fmt="tiered", Hq=8, Hkv=2,
                       tiers=[(0.3, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.2, "bf16")]),
}


def _capture(call):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):                 # warm-up outside the capture
        assert call(s) == 0
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        st = call(s)
    assert st == 0
    return g


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("entry", ["decode", "sink_window", "multi"])
def test_graph_replay_equals_eager(name, entry):
    kw = dict(CASES[name])
    if entry == "multi":
        kw["num_queries"] = 2
    case = small_case(B=3, lens=(700, 77, 300), alibi=True, seed=51, **kw)
    sw = (4, 100) if entry == "sink_window" else None
    eager = binding.DecodeBuffers(case)
    assert binding.paged_decode_raw(case, eager, sink_window=sw) == 0
    torch.cuda.synchronize()
    bufs = binding.DecodeBuffers(case)
    g = _capture(lambda s: binding.paged_decode_raw(case, bufs, stream=s, sink_window=sw))
    for _ in range(2):
        bufs.out.fill_(float("nan"))
        bufs.lse.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(bufs.out, eager.out) and torch.equal(bufs.lse, eager.lse)
        assert int(bufs.err.item()) == 0
    # a replay sees new query values written into the same buffers
    case.q.copy_(torch.flip(case.q, dims=[1]))
    assert binding.paged_decode_raw(case, eager, sink_window=sw) == 0
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(bufs.out, eager.out)
