"""Thin Python binding of the C ABI in include/cfr_paged.h (ctypes).

Argument marshalling only: every step of the attention computation runs in the
CUDA kernels of libcfr_paged.so.  There is no fallback: if the library is not
built, or a call is rejected, the binding raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

from . import synth

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcfr_paged.so")

CFR_OK = 0
STATUS = {0: "CFR_OK", 1: "CFR_ERR_INVALID_ARG", 2: "CFR_ERR_UNSUPPORTED", 3: "CFR_ERR_OVERFLOW",
          4: "CFR_ERR_PAGE_INDEX", 5: "CFR_ERR_CUDA", 6: "CFR_ERR_TIMEOUT", 7: "CFR_ERR_WORKSPACE"}
DEVERR_PAGE_ID, DEVERR_PAGE_FMT, DEVERR_SEQ_LEN, DEVERR_POOL, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
DEVERR_SCHEDULE = 0x20
STATUS_CODES = {v: k for k, v in STATUS.items()}
PATH_CUDA_CORE, PATH_TENSOR_CORE, PATH_F32_TMA = 1, 2, 3

# every exported symbol the header declares
EXPORTS = ["cfr_paged_decode_workspace_size", "cfr_paged_decode", "cfr_paged_decode_phases",
           "cfr_merge_partials",
           "cfr_schedule_splits", "cfr_gather_pages", "cfr_paged_decode_path", "cfr_status_str",
           "cfr_paged_decode_static_workspace", "cfr_demote_pages", "cfr_append_kv",
           "cfr_paged_decode_sink_window", "cfr_paged_decode_multi", "cfr_wait_probe"]
FMT_COUNT = 5


def _header_static_workspace_bytes() -> int:
    """CFR_STATIC_WORKSPACE_BYTES as the header defines it (one source of truth)."""
    import re
    hdr = os.path.join(os.path.dirname(_PKG), "include", "cfr_paged.h")
    m = re.search(r"#define\s+CFR_STATIC_WORKSPACE_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)",
                  open(hdr).read())
    if not m:
        raise RuntimeError("CFR_STATIC_WORKSPACE_BYTES not found in include/cfr_paged.h")
    return int(m.group(1)) << int(m.group(2))


STATIC_WORKSPACE_BYTES = _header_static_workspace_bytes()


class CfrError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class KvPool(ctypes.Structure):
    """Mirror of cfr_kv_pool."""
    _fields_ = [
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("page_tokens", ctypes.c_int32),
        ("k_pool", ctypes.c_void_p * FMT_COUNT), ("v_pool", ctypes.c_void_p * FMT_COUNT),
        ("scales", ctypes.c_void_p * FMT_COUNT), ("pool_pages", ctypes.c_int64 * FMT_COUNT),
    ]


_lib = None
_VP, _I32, _I64, _SZ, _F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float


def lib():
    """The loaded CUDA library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m paged_long_context_b200.build` (no CPU fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        L.cfr_paged_decode_workspace_size.restype = _SZ
        L.cfr_paged_decode_workspace_size.argtypes = [_I32] * 6
        L.cfr_paged_decode.restype = ctypes.c_int
        L.cfr_paged_decode.argtypes = [_VP, _I32, ctypes.POINTER(KvPool), _VP, _I32, _VP, _I32, _VP,
                                       _I32, _I32, _VP, _VP, _F32, _VP, _VP, _VP, _SZ, _VP, _VP]
        L.cfr_paged_decode_phases.restype = ctypes.c_int
        L.cfr_paged_decode_phases.argtypes = L.cfr_paged_decode.argtypes + [ctypes.c_uint32]
        L.cfr_merge_partials.restype = ctypes.c_int
        L.cfr_merge_partials.argtypes = [_VP, _VP, _VP, _VP, _I32, _I32, _I32, _VP, _VP, _VP]
        L.cfr_schedule_splits.restype = ctypes.c_int
        L.cfr_schedule_splits.argtypes = [_VP, _I32, _I32, _I32, _I32, _VP, _VP, _I32, _VP, _VP, _VP]
        L.cfr_gather_pages.restype = ctypes.c_int
        L.cfr_gather_pages.argtypes = [ctypes.POINTER(KvPool), _VP, _VP, _I32, _I32, _I32, _I32,
                                       _I32, _I32, _VP, _VP, _I64, _VP, _VP]
        L.cfr_paged_decode_path.restype = _I32
        L.cfr_paged_decode_path.argtypes = [_I32, ctypes.POINTER(KvPool), _I32, _VP, _I32, _I32, _VP]
        L.cfr_paged_decode_static_workspace.restype = ctypes.c_int
        L.cfr_paged_decode_static_workspace.argtypes = [_VP, _I32, ctypes.POINTER(KvPool), _VP, _I32,
                                                        _VP, _I32, _VP, _I32, _I32, _VP, _VP, _F32,
                                                        _VP, _VP, _VP, _VP]
        L.cfr_paged_decode_sink_window.restype = ctypes.c_int
        L.cfr_paged_decode_sink_window.argtypes = L.cfr_paged_decode.argtypes + [_I32, _I32,
                                                                                  ctypes.c_uint32]
        L.cfr_paged_decode_multi.restype = ctypes.c_int
        L.cfr_paged_decode_multi.argtypes = [_VP, _I32, ctypes.POINTER(KvPool), _VP, _I32, _VP, _I32,
                                             _VP, _I32, _I32, _I32, _VP, _VP, _F32, _VP, _VP, _VP,
                                             _SZ, _VP, _VP, ctypes.c_uint32]
        L.cfr_demote_pages.restype = ctypes.c_int
        L.cfr_demote_pages.argtypes = [ctypes.POINTER(KvPool), _I32, _I32, _VP, _VP, _VP, _I64,
                                       _VP, _VP, _VP, _I32, _VP, _VP]
        L.cfr_append_kv.restype = ctypes.c_int
        L.cfr_append_kv.argtypes = [ctypes.POINTER(KvPool), _VP, _I32, _VP, _I32, _VP, _I32,
                                    _VP, _VP, _I32, _VP, _VP]
        L.cfr_wait_probe.restype = ctypes.c_int
        L.cfr_wait_probe.argtypes = [_I64, _I32, _VP, _VP, _VP]
        L.cfr_status_str.restype = ctypes.c_char_p
        L.cfr_status_str.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> Optional[ctypes.c_void_p]:
    if stream is None:
        if torch.cuda.is_available():
            return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        return None
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def status_str(status: int) -> str:
    return lib().cfr_status_str(status).decode()


def pool_struct(num_kv_heads: int, head_dim: int, page_tokens: int, k_pool: dict, v_pool: dict,
                scales: Optional[dict] = None) -> KvPool:
    """cfr_kv_pool from dicts format -> device tensor."""
    s = KvPool()
    s.num_kv_heads, s.head_dim, s.page_tokens = num_kv_heads, head_dim, page_tokens
    scales = scales or {}
    for f in range(FMT_COUNT):
        s.k_pool[f] = k_pool[f].data_ptr() if f in k_pool else None
        s.v_pool[f] = v_pool[f].data_ptr() if f in v_pool else None
        s.scales[f] = scales[f].data_ptr() if f in scales else None
        s.pool_pages[f] = int(k_pool[f].shape[0]) if f in k_pool else 0
    return s


def kv_pool_struct(case: "synth.DecodeCase") -> KvPool:
    return pool_struct(case.num_kv_heads, case.head_dim, case.page_tokens, case.k_pool,
                       case.v_pool, case.scales)


def workspace_size(batch, num_q_heads, num_kv_heads, head_dim, max_pages, page_tokens) -> int:
    return int(lib().cfr_paged_decode_workspace_size(batch, num_q_heads, num_kv_heads, head_dim,
                                                     max_pages, page_tokens))


def _head_map_host(case):
    if case.head_map is None:
        return None, None
    hm = case.head_map.detach().to("cpu", torch.int32).contiguous()
    return hm, ctypes.c_void_p(hm.data_ptr())


def decode_path(case) -> int:
    """1 = general CUDA-core kernel, 2 = tcgen05 kernel, 3 = fp32 TMA kernel,
    0 = the call would be rejected."""
    pool = kv_pool_struct(case)
    hm, hmp = _head_map_host(case)
    return int(lib().cfr_paged_decode_path(case.q_fmt, ctypes.byref(pool), case.max_pages,
                                           _p(case.page_fmt), case.uniform_fmt, case.num_q_heads,
                                           hmp))


class DecodeBuffers:
    """Caller-owned output and scratch buffers of one decode call (device)."""

    def __init__(self, case, device=None, with_lse=True):
        dev = device or case.device
        rows = case.num_q_heads * getattr(case, "num_queries", 1)   # [Q][Hq] query rows
        self.out = torch.empty((case.batch, rows, case.head_dim), dtype=torch.float32, device=dev)
        self.lse = torch.empty((case.batch, rows), dtype=torch.float32,
                               device=dev) if with_lse else None
        n = workspace_size(case.batch, rows, case.num_kv_heads, case.head_dim,
                           case.max_pages, case.page_tokens)
        if n == 0:
            raise CfrError(1, "cfr_paged_decode_workspace_size")
        self.workspace = torch.empty((n,), dtype=torch.uint8, device=dev)
        self.err = torch.zeros((1,), dtype=torch.int32, device=dev)


PHASE_SCHEDULE, PHASE_DECODE, PHASE_MERGE, PHASE_ALL = 0x1, 0x2, 0x4, 0x7


def paged_decode_raw(case, bufs: DecodeBuffers, stream=None, workspace_bytes=None,
                     phases: Optional[int] = None, sink_window: Optional[tuple] = None) -> int:
    """Call cfr_paged_decode (cfr_paged_decode_phases when ``phases`` is given,
    cfr_paged_decode_sink_window when ``sink_window`` = (sink_tokens, window_tokens)
    is given, cfr_paged_decode_multi when the case has several queries per
    sequence) on a case whose tensors live on the GPU; returns the status."""
    pool = kv_pool_struct(case)
    hm, hmp = _head_map_host(case)
    nbytes = bufs.workspace.numel() if workspace_bytes is None else workspace_bytes
    args = (_p(case.q), case.q_fmt, ctypes.byref(pool), _p(case.page_table), case.max_pages,
            _p(case.seq_lens), case.batch, _p(case.page_fmt), case.uniform_fmt, case.num_q_heads,
            hmp, _p(case.alibi_slopes), float(case.softmax_scale), _p(bufs.out), _p(bufs.lse),
            _p(bufs.workspace), nbytes, _p(bufs.err), _stream(stream))
    if getattr(case, "num_queries", 1) > 1:
        if sink_window is not None:
            raise ValueError("sink/window subsets take one query per sequence")
        return int(lib().cfr_paged_decode_multi(
            _p(case.q), case.q_fmt, ctypes.byref(pool), _p(case.page_table), case.max_pages,
            _p(case.seq_lens), case.batch, _p(case.page_fmt), case.uniform_fmt, case.num_q_heads,
            case.num_queries, hmp, _p(case.alibi_slopes), float(case.softmax_scale), _p(bufs.out),
            _p(bufs.lse), _p(bufs.workspace), nbytes, _p(bufs.err), _stream(stream),
            PHASE_ALL if phases is None else phases))
    if sink_window is not None:
        return int(lib().cfr_paged_decode_sink_window(*args, int(sink_window[0]),
                                                      int(sink_window[1]),
                                                      PHASE_ALL if phases is None else phases))
    if phases is None:
        return int(lib().cfr_paged_decode(*args))
    return int(lib().cfr_paged_decode_phases(*args, phases))


def paged_decode(case, bufs: Optional[DecodeBuffers] = None, stream=None,
                 sink_window: Optional[tuple] = None) -> DecodeBuffers:
    """Decode attention for every (sequence, query head), over all tokens or a
    (sink_tokens, window_tokens) subset; raises on a rejected call."""
    bufs = bufs or DecodeBuffers(case)
    st = paged_decode_raw(case, bufs, stream, sink_window=sink_window)
    if st != CFR_OK:
        raise CfrError(st, "cfr_paged_decode")
    return bufs


def merge_partials(part_acc, part_m, part_l, split_off, batch, num_q_heads, head_dim, out,
                   lse=None, stream=None) -> int:
    return int(lib().cfr_merge_partials(_p(part_acc), _p(part_m), _p(part_l), _p(split_off),
                                        batch, num_q_heads, head_dim, _p(out), _p(lse),
                                        _stream(stream)))


def schedule_splits(seq_lens, batch, page_tokens, max_pages, target_splits, split_off, splits,
                    max_splits, num_splits, err=None, stream=None) -> int:
    return int(lib().cfr_schedule_splits(_p(seq_lens), batch, page_tokens, max_pages,
                                         target_splits, _p(split_off), _p(splits), max_splits,
                                         _p(num_splits), _p(err), _stream(stream)))


def gather_pages(case, b, kv_head, n_tokens, k_out, v_out, pitch, err=None, stream=None) -> int:
    pool = kv_pool_struct(case)
    return int(lib().cfr_gather_pages(ctypes.byref(pool), _p(case.page_table), _p(case.page_fmt),
                                      case.uniform_fmt, case.batch, case.max_pages, b, kv_head,
                                      n_tokens,
                                      _p(k_out), _p(v_out), pitch, _p(err), _stream(stream)))


def paged_decode_static_workspace(case, out, lse=None, err=None, stream=None) -> int:
    """cfr_paged_decode_static_workspace: decode with the library's built-in scratch array
    (for callers that cannot allocate device memory); returns the status."""
    pool = kv_pool_struct(case)
    hm, hmp = _head_map_host(case)
    return int(lib().cfr_paged_decode_static_workspace(
        _p(case.q), case.q_fmt, ctypes.byref(pool), _p(case.page_table), case.max_pages,
        _p(case.seq_lens), case.batch, _p(case.page_fmt), case.uniform_fmt, case.num_q_heads, hmp,
        _p(case.alibi_slopes), float(case.softmax_scale), _p(out), _p(lse), _p(err),
        _stream(stream)))


def wait_probe(limit_cycles: int, arrive: bool, err=None, result=None, stream=None) -> int:
    """cfr_wait_probe: the decode kernels' bounded on-chip wait, run once with a
    short cycle limit on a barrier that is (arrive) or is not arrived on."""
    return int(lib().cfr_wait_probe(int(limit_cycles), 1 if arrive else 0, _p(err), _p(result),
                                    _stream(stream)))


def demote_pages(pool: KvPool, src_fmt: int, dst_fmt: int, dst_k, dst_v, dst_scales,
                 src_slots, dst_slots, valid_tokens=None, err=None, stream=None) -> int:
    """cfr_demote_pages: re-encode pages of the src_fmt pool described by ``pool`` into
    the destination pool tensors (device uint8 [slots][Hkv][P][row_bytes]); returns the status."""
    n = int(src_slots.numel())
    return int(lib().cfr_demote_pages(ctypes.byref(pool), src_fmt, dst_fmt, _p(dst_k), _p(dst_v),
                                      _p(dst_scales), int(dst_k.shape[0]), _p(src_slots),
                                      _p(dst_slots), _p(valid_tokens), n, _p(err),
                                      _stream(stream)))


def append_kv(pool: KvPool, page_table, page_fmt, uniform_fmt: int, positions, k_new, v_new,
              err=None, stream=None) -> int:
    """cfr_append_kv: write one token per sequence into its F32/BF16 page; returns the status."""
    new_fmt = synth.F32 if k_new.dtype == torch.float32 else synth.BF16
    return int(lib().cfr_append_kv(ctypes.byref(pool), _p(page_table), int(page_table.shape[1]),
                                   _p(page_fmt), uniform_fmt, _p(positions),
                                   int(positions.numel()), _p(k_new), _p(v_new), new_fmt, _p(err),
                                   _stream(stream)))
