"""head_dim 64 on the tensor-core kernel.

The kernel's operand layout is built for 128 dims in two 64-dim halves; a
cache of head_dim 64 fills the first half of K and V, the QK products stop at
dim 64 and the P.V rows of dims 64..127 are never read or written.  Every
format the kernel takes (bf16 pages of any size that divides or is a multiple
of 128 tokens; int8, int4 and FP8 pages of 128 tokens or more, expanded to
fp16 by the staging warps) must match the oracle at the stated tolerance, with
ALiBi, GQA groups of 1 to 16 rows, more than 16 rows per kv head, several query
tokens per sequence and sink + window subsets."""
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


@pytest.mark.parametrize("fmt,P", [("bf16", 8), ("bf16", 16), ("bf16", 128), ("bf16", 512),
                                   ("i8", 128), ("i4", 256), ("fp8", 128)])
@pytest.mark.parametrize("heads", [(8, 8), (8, 2), (16, 1), (32, 4)], ids=lambda h: f"{h[0]}q{h[1]}kv")
def test_head_dim_64_parity(fmt, P, heads):
    Hq, Hkv = heads
    lens = (1, P - 1 if P > 1 else 1, 3 * P + 5, 1000, 2 * P)
    case = small_case(B=len(lens), Hq=Hq, Hkv=Hkv, d=64, P=P, lens=lens, fmt=fmt, q_fmt="bf16",
                      alibi=True, seed=P + Hq)
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_head_dim_64_tiered_and_f32_queries():
    case = small_case(B=3, Hq=8, Hkv=2, d=64, P=128, lens=(2000, 129, 4096), fmt="tiered",
                      tiers=[(0.2, "i4"), (0.3, "i8"), (0.2, "fp8"), (0.3, "bf16")], q_fmt="f32",
                      alibi=True, seed=5)
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_head_dim_64_large_logits():
    # sigma = 4 x the default scale: the running maximum moves a lot
    case = small_case(B=2, Hq=8, Hkv=2, d=64, P=64, lens=(3000, 77), fmt="bf16", q_fmt="bf16",
                      seed=9, softmax_scale=0.5)
    assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)
