"""cfr_paged_decode_static_workspace: decode for callers that cannot allocate
device memory (they pass only inputs and outputs; the scratch comes from an
array built into the library).  Checked through the C ABI against the
workspace-taking entry point, on two calls in a row.  This file is collected
last so that a run stopping at the first failure has already run every other
test."""
import numpy as np
import pytest
import torch

from paged_long_context_b200 import binding, synth
from tests._gpu import TOL_F32_ABS, TOL_LOWP_REL, all_f32, vmax_table_sel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    build.build()


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
    hc = case.to("cpu")
    pairs = [(b, h) for b in range(case.batch) for h in range(case.num_q_heads)]
    if all_f32(case):
        tol = {p: TOL_F32_ABS for p in pairs}
    else:
        vmax = vmax_table_sel(hc, pairs)           # max|V| per (sequence, kv head)
        tol = {(b, h): TOL_LOWP_REL * vmax[(b, h // 4)] for (b, h) in pairs}
    for call in range(2):                     # two calls in a row share the array
        out = torch.full_like(ref.out, float("nan"))
        lse = torch.full_like(ref.lse, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = binding.paged_decode_static_workspace(case, out, lse, err)
        assert st == binding.CFR_OK, binding.STATUS.get(st, st)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        o, r = out.cpu().double().numpy(), ref.out.cpu().double().numpy()
        for (b, h) in pairs:
            assert np.abs(o[b, h] - r[b, h]).max() <= tol[(b, h)], (call, b, h)
        np.testing.assert_allclose(lse.cpu().numpy(), ref.lse.cpu().numpy(), rtol=1e-6, atol=1e-6)


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
    assert st == 7  # CFR_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 0)               # nothing was launched
