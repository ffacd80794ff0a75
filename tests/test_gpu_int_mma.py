"""Quantised pages on the tensor-core path, both ways it runs them.

With at most 4 query rows per kv head, int8 and int4 tiles run int8 MMAs: the
stored codes are the operand (int4 widened to one byte per code), the query and
the probabilities enter as columns of 8-bit digits, and the int32 products are
recombined in fp32.  With 5 to 16 rows per kv head the codes are expanded to
fp16 in shared memory instead.  FP8 tiles always take the fp16 expansion, bf16
tiles the bf16 MMAs, inside the same launch.  Every case is compared with the
oracle at the stated tolerance (2e-3 * max|V| of the (sequence, kv head))."""
import pytest
import torch

from paged_long_context_b200 import binding
from tests._gpu import check, run, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from paged_long_context_b200 import build
    import oracle
    build.build()
    oracle.build()


TIERS = {
    "i8": None,
    "i4": None,
    "i4_i8_bf16": [(0.25, "i4"), (0.5, "i8"), (0.25, "bf16")],
    "i4_i8_fp8_bf16": [(0.2, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.3, "bf16")],
}
# (query heads, kv heads): 1-4 rows per kv head run the int8 MMAs, 5-16 the fp16 expansion
HEADS = [(4, 4), (8, 4), (12, 4), (8, 2), (10, 2), (16, 2), (16, 1)]


def _case(fmt, heads, P, seed, q_fmt="bf16", alibi=False, lens=None, **kw):
    Hq, Hkv = heads
    tiers = TIERS[fmt]
    lens = lens or (9 * P + 3, 1, P, 2 * P + 77)
    return small_case(B=len(lens), Hq=Hq, Hkv=Hkv, d=128, P=P, lens=lens,
                      fmt="tiered" if tiers else fmt, tiers=tiers, q_fmt=q_fmt, alibi=alibi,
                      seed=seed, **kw)


@pytest.mark.parametrize("fmt", list(TIERS))
@pytest.mark.parametrize("heads", HEADS, ids=lambda h: f"{h[0]}q{h[1]}kv")
@pytest.mark.parametrize("P", [128, 256])
def test_int_pages_tensor_core(fmt, heads, P):
    case = _case(fmt, heads, P, seed=P + heads[0])
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("fmt", ["i8", "i4", "i4_i8_bf16"])
@pytest.mark.parametrize("q_fmt", ["f32", "bf16"])
def test_int_pages_alibi_and_query_formats(fmt, q_fmt):
    case = _case(fmt, (8, 2), 128, seed=5, q_fmt=q_fmt, alibi=True,
                 lens=(3000, 129, 128, 4097))
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("fmt", ["i8", "i4"])
def test_int_pages_large_logits(fmt):
    # sigma = 4: scores span hundreds of units, a few tokens carry the softmax
    case = _case(fmt, (4, 1), 128, seed=9, softmax_scale=4.0, lens=(900, 300))
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_int_pages_head_map():
    # an arbitrary query-head -> kv-head map with 1 to 4 rows per kv head
    case = _case("i4_i8_bf16", (8, 3), 128, seed=13, head_map=[2, 0, 0, 1, 2, 2, 0, 2])
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_int_pages_long_sequence():
    # 65,536 tokens of int8 codes in one sequence: the probability digits are
    # summed over every token of a split
    case = _case("i8", (8, 2), 256, seed=17, lens=(65536, 40000))
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse, sel=[(b, h) for b in range(2) for h in (0, 3, 5, 7)])


def test_int_pages_bit_identical_runs():
    case = _case("i4_i8_bf16", (8, 2), 128, seed=21, lens=(5000, 777))
    out0, lse0, _ = run(case)
    for _ in range(3):
        out, lse, err = run(case)
        assert err == 0
        assert torch.equal(out, out0) and torch.equal(lse, lse0)
