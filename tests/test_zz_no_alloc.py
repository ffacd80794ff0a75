"""cfr_paged_decode_static_workspace: decode for callers that cannot allocate
device memory.  Some callers only hand a kernel its inputs and outputs (plugin
and operator interfaces without a workspace argument, code running where
another component owns every device allocation); this entry point takes its
scratch from an array built into the library.  Checked through the C ABI: its
results are bit-identical to the workspace-taking entry point's on two calls in
a row (the same kernels run in the same order), one of them is compared with
the oracle, and free device memory does not move across the two calls (nothing
is allocated, by the library or anyone else).  This file is collected last so
that a run stopping at the first failure has already run every other test."""
import pytest
import torch

from paged_long_context_b200 import binding, synth
from tests._gpu import check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    import oracle
    build.build()
    oracle.build()


def _case(fmt, q_fmt, seed):
    kw = dict(tiers=[(0.25, "i4"), (0.5, "i8"), (0.25, "bf16")]) if fmt == "tiered" else {}
    spec = synth.CaseSpec("noalloc", 3, 8, 2, 128, 64, seq_lens=[1500, 64, 777], fmt=fmt,
                          q_fmt=q_fmt, alibi=True, **kw)
    return synth.make_case(spec, seed, "cuda")


@pytest.mark.parametrize("fmt,q_fmt", [("f32", "f32"), ("bf16", "bf16"), ("tiered", "bf16")])
def test_static_workspace_matches_workspace_entry(fmt, q_fmt):
    case = _case(fmt, q_fmt, 31)
    ref = binding.paged_decode(case)          # the entry point with caller-owned scratch
    torch.cuda.synchronize()
    assert int(ref.err.item()) == 0
    # every buffer of the calls below exists before free memory is read
    outs = [torch.full_like(ref.out, float("nan")) for _ in range(3)]
    lses = [torch.full_like(ref.lse, float("nan")) for _ in range(3)]
    errs = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(3)]
    # a first call loads the kernels and looks up the array's address
    assert binding.paged_decode_static_workspace(case, outs[0], lses[0], errs[0]) == binding.CFR_OK
    torch.cuda.synchronize()
    free_before, _ = torch.cuda.mem_get_info()
    for call in (1, 2):                       # two calls in a row share the array
        st = binding.paged_decode_static_workspace(case, outs[call], lses[call], errs[call])
        assert st == binding.CFR_OK, binding.STATUS.get(st, st)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert free_after == free_before, "device memory was allocated during the calls"
    for call in range(3):
        assert int(errs[call].item()) == 0
        assert torch.equal(outs[call], ref.out), call
        assert torch.equal(lses[call], ref.lse), call
    check(case, outs[2].cpu(), lses[2].cpu())


def test_static_workspace_rejects_oversized_problems():
    # 2048 one-page sequences x 64 query heads need far more than the built-in array
    spec = synth.CaseSpec("noalloc_big", 2048, 64, 8, 128, 16, seq_lens=[1] * 2048, fmt="bf16",
                          q_fmt="bf16", permute=False)
    case = synth.make_case(spec, 5, "cuda")
    need = binding.workspace_size(case.batch, case.num_q_heads, case.num_kv_heads, case.head_dim,
                                  case.max_pages, case.page_tokens)
    assert need > binding.STATIC_WORKSPACE_BYTES
    out = torch.zeros((2048, 64, 128), device="cuda")
    st = binding.paged_decode_static_workspace(case, out)
    assert st == binding.STATUS_CODES["CFR_ERR_WORKSPACE"]
    torch.cuda.synchronize()
    assert torch.all(out == 0)               # nothing was launched
