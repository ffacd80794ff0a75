"""The C ABI without a GPU: the library loads, exports every declared symbol, and
rejects invalid arguments on the host before anything is launched."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from paged_long_context_b200 import binding, synth
from paged_long_context_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cfr_paged.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return binding.lib()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return sorted(set(re.findall(r"\b(cfr_\w+)\s*\(", src)))


def test_header_declares_the_entry_points():
    assert declared_functions() == sorted(binding.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (cfr_\w+)", out))
    assert set(declared_functions()) <= exported


def test_status_strings(lib):
    for code in range(8):
        assert binding.status_str(code) not in ("", "unknown status")
    assert binding.status_str(99) == "unknown status"


def _case(**kw):
    spec = dict(name="abi", batch=2, num_q_heads=4, num_kv_heads=2, head_dim=64, page_tokens=16,
                seq_lens=[40, 17], fmt="bf16", q_fmt="bf16")
    spec.update(kw)
    return synth.make_case(synth.CaseSpec(**spec), 3, "cpu")


class FakeBufs:
    """Host tensors standing in for device buffers: the calls below are all
    rejected on the host before any pointer is dereferenced or any kernel runs."""

    def __init__(self, case):
        self.out = torch.empty((case.batch, case.num_q_heads, case.head_dim))
        self.lse = torch.empty((case.batch, case.num_q_heads))
        self.workspace = torch.empty((1 << 16,), dtype=torch.uint8)
        self.err = torch.zeros((1,), dtype=torch.int32)


def _decode(case, **over):
    bufs = FakeBufs(case)
    pool = binding.kv_pool_struct(case)
    for k, v in over.pop("pool", {}).items():
        if k in ("k_pool", "v_pool", "scales", "pool_pages"):
            for f, val in v.items():
                getattr(pool, k)[f] = val
        else:
            setattr(pool, k, v)
    args = dict(q=binding._p(case.q), q_fmt=case.q_fmt, page_table=binding._p(case.page_table),
                max_pages=case.max_pages, seq_lens=binding._p(case.seq_lens), batch=case.batch,
                page_fmt=binding._p(case.page_fmt), uniform_fmt=case.uniform_fmt,
                num_q_heads=case.num_q_heads, head_map=None, slopes=None, scale=0.0,
                out=binding._p(bufs.out), lse=binding._p(bufs.lse),
                ws=binding._p(bufs.workspace), ws_bytes=bufs.workspace.numel(),
                err=binding._p(bufs.err))
    args.update(over)
    return binding.lib().cfr_paged_decode(
        args["q"], args["q_fmt"], ctypes.byref(pool), args["page_table"], args["max_pages"],
        args["seq_lens"], args["batch"], args["page_fmt"], args["uniform_fmt"],
        args["num_q_heads"], args["head_map"], args["slopes"], args["scale"], args["out"],
        args["lse"], args["ws"], args["ws_bytes"], args["err"], None)


E = binding.STATUS
INVALID, UNSUP, OVERFLOW = 1, 2, 3


def _hm(vals):
    t = torch.tensor(vals, dtype=torch.int32)
    _hm.keep.append(t)
    return ctypes.c_void_p(t.data_ptr())


_hm.keep = []


@pytest.mark.parametrize("what,over,code", [
    ("null q", dict(q=None), INVALID),
    ("null page table", dict(page_table=None), INVALID),
    ("null seq_lens", dict(seq_lens=None), INVALID),
    ("null out", dict(out=None), INVALID),
    ("batch 0", dict(batch=0), INVALID),
    ("q format i8", dict(q_fmt=2), INVALID),
    ("max_pages 0", dict(max_pages=0), INVALID),
    ("uniform format out of range", dict(uniform_fmt=7), INVALID),
    ("uniform format without pool", dict(uniform_fmt=0), INVALID),
    ("negative scale", dict(scale=-1.0), INVALID),
    ("nan scale", dict(scale=float("nan")), INVALID),
    ("head_dim 96", dict(pool={"head_dim": 96}), UNSUP),
    ("page_tokens 4", dict(pool={"page_tokens": 4}), UNSUP),
    ("kv heads 0", dict(pool={"num_kv_heads": 0}), INVALID),
    ("Hq not multiple of Hkv", dict(num_q_heads=3), INVALID),
    ("Hq above 256", dict(num_q_heads=258, pool={"num_kv_heads": 258}), UNSUP),
    ("head map out of range", dict(head_map=_hm([0, 1, 2, 0])), INVALID),
    ("negative head map", dict(head_map=_hm([0, -1, 1, 0])), INVALID),
    ("k pool without v pool", dict(pool={"k_pool": {1: None}}), INVALID),
    ("negative pool pages", dict(pool={"pool_pages": {1: -5}}), INVALID),
    ("pages x tokens overflow", dict(max_pages=1 << 28), OVERFLOW),
    ("batch x pages overflow", dict(batch=1 << 20, max_pages=1 << 12), OVERFLOW),
])
def test_host_rejects(lib, what, over, code):
    case = _case()
    assert _decode(case, **over) == code, what


def test_misaligned_pointers_rejected(lib):
    case = _case()
    k = case.k_pool[synth.BF16]
    assert _decode(case, pool={"k_pool": {synth.BF16: k.data_ptr() + 4}}) == INVALID
    qp = ctypes.c_void_p(case.q.data_ptr() + 2)
    assert _decode(case, q=qp) == INVALID


def test_quantised_pool_needs_scales(lib):
    case = _case(fmt="i8")
    assert _decode(case, pool={"scales": {synth.I8: None}}) == INVALID


def test_pool_byte_size_overflow(lib):
    case = _case()
    assert _decode(case, pool={"pool_pages": {synth.BF16: 1 << 60}}) == OVERFLOW


def test_merge_and_schedule_and_gather_rejects(lib):
    L = binding.lib()
    t = torch.zeros(64)
    p = ctypes.c_void_p(t.data_ptr())
    assert L.cfr_merge_partials(p, p, p, p, 1, 1, 96, p, None, None) == UNSUP
    assert L.cfr_merge_partials(None, p, p, p, 1, 1, 64, p, None, None) == INVALID
    assert L.cfr_merge_partials(p, p, p, p, 0, 1, 64, p, None, None) == INVALID
    assert L.cfr_schedule_splits(p, 1, 16, 4, 0, p, p, 8, p, None, None) == INVALID
    assert L.cfr_schedule_splits(None, 1, 16, 4, 4, p, p, 8, p, None, None) == INVALID
    case = _case()
    pool = binding.kv_pool_struct(case)
    args = (ctypes.byref(pool), binding._p(case.page_table), None, case.uniform_fmt,
            case.batch, case.max_pages)
    assert L.cfr_gather_pages(*args, 0, 0, 16, p, p, 24, None, None) == INVALID   # pitch % 16
    assert L.cfr_gather_pages(*args, 0, 0, 16, p, p, 64, None, None) == INVALID   # < row bytes
    assert L.cfr_gather_pages(*args, 0, 5, 16, p, p, 128, None, None) == INVALID  # kv head
    assert L.cfr_gather_pages(*args, 0, 0, 10_000, p, p, 128, None, None) == INVALID
    assert L.cfr_gather_pages(*args, 2, 0, 16, p, p, 128, None, None) == INVALID    # b >= batch


def test_workspace_size_rejects_bad_sizes(lib):
    assert binding.workspace_size(0, 4, 2, 64, 4, 16) == 0
    assert binding.workspace_size(1, 0, 2, 64, 4, 16) == 0
    assert binding.workspace_size(1, 4, 2, 64, -1, 16) == 0


def test_path_selection_is_host_only(lib):
    # fp32 caches with at most two query heads per kv head take the fp32 TMA kernel
    assert binding.decode_path(_case(fmt="f32", q_fmt="f32")) == binding.PATH_F32_TMA
    assert binding.decode_path(_case(fmt="f32", q_fmt="f32", head_dim=128)) == binding.PATH_F32_TMA
    assert binding.decode_path(_case(fmt="f32", q_fmt="bf16", num_q_heads=4, num_kv_heads=4)) == \
        binding.PATH_F32_TMA
    # wider groups, odd page sizes and format mixes with fp32 take the general kernel
    assert binding.decode_path(_case(fmt="f32", num_q_heads=8, num_kv_heads=2)) == binding.PATH_CUDA_CORE
    assert binding.decode_path(_case(fmt="f32", page_tokens=24)) == binding.PATH_CUDA_CORE
    assert binding.decode_path(_case(fmt="tiered", tiers=[(0.5, "i8"), (0.5, "f32")])) == \
        binding.PATH_CUDA_CORE
    # bf16 caches of head_dim 64 take the tensor-core kernel (the first half of
    # its 128-dim operands), and so do uniform int8 caches of any page size up to
    # 8 rows per group; quantised pages under 128 tokens in a cache of mixed
    # formats, or with wider groups, take the general kernel
    assert binding.decode_path(_case()) == binding.PATH_TENSOR_CORE
    assert binding.decode_path(_case(fmt="i8")) == binding.PATH_TENSOR_CORE
    assert binding.decode_path(_case(fmt="i8", page_tokens=128)) == binding.PATH_TENSOR_CORE
    assert binding.decode_path(_case(fmt="i8", num_q_heads=32, num_kv_heads=2)) == \
        binding.PATH_CUDA_CORE
    assert binding.decode_path(_case(fmt="tiered", tiers=[(0.5, "i8"), (0.5, "bf16")])) == \
        binding.PATH_CUDA_CORE
    # rejected configurations report 0
    assert binding.decode_path(_case(num_q_heads=3, num_kv_heads=2)) == 0


def test_path_selection_fp8(lib):
    # FP8 pages: head_dim 128 with 128-token pages take the tensor-core kernel
    assert binding.decode_path(_case(fmt="fp8", head_dim=128, page_tokens=128)) == \
        binding.PATH_TENSOR_CORE
    # and so do uniform FP8 caches with smaller pages; FP8 pages under 128
    # tokens among other formats take the general kernel
    assert binding.decode_path(_case(fmt="fp8")) == binding.PATH_TENSOR_CORE
    assert binding.decode_path(_case(fmt="fp8", head_dim=128, page_tokens=64)) == \
        binding.PATH_TENSOR_CORE
    assert binding.decode_path(_case(fmt="tiered", tiers=[(0.5, "fp8"), (0.5, "bf16")])) == \
        binding.PATH_CUDA_CORE


def test_fp8_pool_needs_scales(lib):
    case = _case(fmt="fp8")
    assert _decode(case, pool={"scales": {synth.FP8: None}}) == INVALID


def _demote(pool, src, dst, dk, dv, dsc, n=1, dst_pages=None, slots=True):
    t = torch.zeros(8, dtype=torch.int32)
    sp = ctypes.c_void_p(t.data_ptr()) if slots else None
    return binding.lib().cfr_demote_pages(
        ctypes.byref(pool), src, dst, dk, dv, dsc,
        dst_pages if dst_pages is not None else 4, sp, sp, None, n, None, None)


def test_demote_rejects(lib):
    case = _case()                          # bf16 pool, d 64, P 16
    pool = binding.kv_pool_struct(case)
    buf = torch.zeros(1 << 16, dtype=torch.uint8)
    sc = torch.zeros(64)
    p = ctypes.c_void_p(buf.data_ptr())
    ps = ctypes.c_void_p(sc.data_ptr())
    BF, I8, F32 = synth.BF16, synth.I8, synth.F32
    assert _demote(pool, BF, BF, p, p, ps) == INVALID                  # same format
    assert _demote(pool, BF, 9, p, p, ps) == INVALID                   # unknown format
    assert _demote(pool, F32, I8, p, p, ps) == INVALID                 # no source pool
    assert _demote(pool, BF, I8, None, p, ps) == INVALID               # no destination
    assert _demote(pool, BF, I8, p, p, None) == INVALID                # quantised without scales
    assert _demote(pool, BF, I8, ctypes.c_void_p(buf.data_ptr() + 8), p, ps) == INVALID
    assert _demote(pool, BF, I8, p, p, ps, n=-1) == INVALID
    assert _demote(pool, BF, I8, p, p, ps, slots=False) == INVALID     # slots missing
    assert _demote(pool, BF, I8, p, p, ps, dst_pages=-1) == OVERFLOW
    assert _demote(pool, BF, I8, p, p, ps, n=0) == 0                   # nothing to do
    pool.head_dim = 96
    assert _demote(pool, BF, I8, p, p, ps) == UNSUP
    case8 = _case(fmt="i8")
    pool8 = binding.kv_pool_struct(case8)
    pool8.scales[I8] = None
    assert _demote(pool8, I8, synth.I4, p, p, ps) == INVALID           # quantised source, no scales


def test_append_rejects(lib):
    case = _case()
    pool = binding.kv_pool_struct(case)
    t = torch.zeros(4096)
    p = ctypes.c_void_p(t.data_ptr())
    L = binding.lib()
    pt = binding._p(case.page_table)
    BF = synth.BF16
    args = lambda **o: (ctypes.byref(o.get("pool", pool)), o.get("pt", pt), o.get("mp", case.max_pages),
                        None, o.get("uf", BF), o.get("pos", p), o.get("b", case.batch),
                        o.get("kn", p), p, o.get("nf", synth.F32), None, None)
    assert L.cfr_append_kv(*args(pt=None)) == INVALID
    assert L.cfr_append_kv(*args(pos=None)) == INVALID
    assert L.cfr_append_kv(*args(kn=None)) == INVALID
    assert L.cfr_append_kv(*args(b=0)) == INVALID
    assert L.cfr_append_kv(*args(nf=synth.I8)) == INVALID
    assert L.cfr_append_kv(*args(uf=synth.I8)) == INVALID             # new tokens go to F32/BF16
    assert L.cfr_append_kv(*args(mp=1 << 28)) == OVERFLOW
    case8 = _case(fmt="i8")
    assert L.cfr_append_kv(*args(pool=binding.kv_pool_struct(case8))) == INVALID  # no hot pool


def test_sink_window_rejects(lib):
    case = _case()
    bufs = FakeBufs(case)
    pool = binding.kv_pool_struct(case)
    args = (binding._p(case.q), case.q_fmt, ctypes.byref(pool), binding._p(case.page_table),
            case.max_pages, binding._p(case.seq_lens), case.batch, binding._p(case.page_fmt),
            case.uniform_fmt, case.num_q_heads, None, None, 0.0, binding._p(bufs.out),
            binding._p(bufs.lse), binding._p(bufs.workspace), bufs.workspace.numel(),
            binding._p(bufs.err), None)
    L = binding.lib()
    assert L.cfr_paged_decode_sink_window(*args, -1, 16, binding.PHASE_ALL) == INVALID
    assert L.cfr_paged_decode_sink_window(*args, 4, 0, binding.PHASE_ALL) == INVALID
    assert L.cfr_paged_decode_sink_window(*args, 4, 16, 0) == INVALID
    assert L.cfr_paged_decode_sink_window(*args, 4, 16, 0x10) == INVALID


def test_multi_query_rejects(lib):
    case = _case()
    bufs = FakeBufs(case)
    pool = binding.kv_pool_struct(case)
    L = binding.lib()

    def call(nq, hq=case.num_q_heads, hkv=None, phases=binding.PHASE_ALL):
        p = binding.kv_pool_struct(case)
        if hkv is not None:
            p.num_kv_heads = hkv
        return L.cfr_paged_decode_multi(
            binding._p(case.q), case.q_fmt, ctypes.byref(p), binding._p(case.page_table),
            case.max_pages, binding._p(case.seq_lens), case.batch, binding._p(case.page_fmt),
            case.uniform_fmt, hq, nq, None, None, 0.0, binding._p(bufs.out), binding._p(bufs.lse),
            binding._p(bufs.workspace), bufs.workspace.numel(), binding._p(bufs.err), None, phases)
    assert call(0) == INVALID                     # at least one query per sequence
    assert call(17) == UNSUP                      # at most 16
    assert call(2, hq=130, hkv=130) == UNSUP      # 260 query rows per sequence
    assert call(2, phases=0) == INVALID


def test_wait_probe_rejects_limits_out_of_range(lib):
    # rejected on the host, before any launch
    assert binding.wait_probe(0, False) == 1
    assert binding.wait_probe(-5, True) == 1
    assert binding.wait_probe(4_000_000_001, False) == 1


def test_wide_groups_are_accepted(lib):
    # MQA and wide GQA: more than 16 query rows per kv head are split into groups
    # of at most 16 rows (host-only path query, nothing launched)
    for hq, hkv in [(17, 1), (32, 1), (64, 1), (64, 2), (48, 3)]:
        case = _case(num_q_heads=hq, num_kv_heads=hkv, head_dim=128, page_tokens=128,
                     seq_lens=[300, 17])
        assert binding.decode_path(case) != 0, (hq, hkv)
