"""MQA and wide GQA: more than 16 query rows per kv head.

The query rows of a kv head are decoded in groups of at most 16 (each group
reads the kv head's pages); every path -- the tensor-core kernel for bf16,
FP8, int8 and int4 pages (head_dim 128, and 64 for bf16), the CUDA-core kernels
for fp32 pages and small int8 pages -- must match the oracle at the stated tolerance, with contiguous and
arbitrary head maps, ALiBi, and several query tokens per sequence."""
import numpy as np
import pytest
import torch

from paged_long_context_b200 import binding, synth
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


@pytest.mark.parametrize("fmt", ["bf16", "i8", "i4", "fp8", "f32"])
@pytest.mark.parametrize("heads", [(32, 1), (64, 1), (24, 1), (64, 2)],
                         ids=lambda h: f"{h[0]}q{h[1]}kv")
def test_wide_groups_tensor_core_shapes(fmt, heads):
    Hq, Hkv = heads
    case = small_case(B=2, Hq=Hq, Hkv=Hkv, d=128, P=128, lens=(1300, 129), fmt=fmt,
                      q_fmt="f32" if fmt == "f32" else "bf16", alibi=True, seed=Hq + Hkv)
    if fmt != "f32":
        assert binding.decode_path(case) == binding.PATH_TENSOR_CORE
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


@pytest.mark.parametrize("fmt", ["bf16", "i8"])
def test_wide_groups_head_dim_64(fmt):
    # head_dim 64: the tensor-core kernel (bf16) or the CUDA-core kernel (int8
    # pages of 16 tokens)
    case = small_case(B=2, Hq=32, Hkv=1, d=64, P=16, lens=(700, 33), fmt=fmt, seed=3)
    assert binding.decode_path(case) == (binding.PATH_TENSOR_CORE if fmt == "bf16"
                                         else binding.PATH_CUDA_CORE)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_wide_groups_uneven_head_map():
    # 20 query heads on kv head 0, 3 on kv head 1, 1 on kv head 2, none on kv head 3
    hm = [0] * 20 + [1] * 3 + [2]
    rng = np.random.default_rng(5)
    hm = [int(x) for x in rng.permutation(hm)]
    case = small_case(B=2, Hq=24, Hkv=4, d=128, P=64, lens=(900, 64), fmt="bf16", head_map=hm,
                      seed=6)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_wide_groups_tiered_pages():
    case = small_case(B=2, Hq=32, Hkv=1, d=128, P=256, lens=(4000, 300), fmt="tiered",
                      tiers=[(0.25, "i4"), (0.25, "i8"), (0.25, "fp8"), (0.25, "bf16")], seed=8)
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse)


def test_wide_groups_multi_query():
    # 8 query heads per kv head x 4 query tokens = 32 rows per kv head
    from tests.test_gpu_multiquery import check_mq, mq_case, run_mq
    case = mq_case(4, B=2, Hq=16, Hkv=2, lens=(900, 40), seed=9)
    out, lse, err = run_mq(case)
    assert err == 0
    check_mq(case, out, lse)


def test_mqa_32k_full_size_sampled():
    # 8 sequences x 32,768 tokens, 32 query heads on 1 kv head, bf16, 256-token pages
    spec = synth.CaseSpec("mqa_32k", 8, 32, 1, 128, 256, seq_lens=[32768] * 8, fmt="bf16")
    case = synth.make_case(spec, 10, "cuda")
    out, lse, err = run(case)
    assert err == 0
    check(case, out, lse, sel=[(b, h) for b in (0, 5) for h in (0, 15, 16, 31)])
