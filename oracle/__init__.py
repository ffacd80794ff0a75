"""fp64 CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and
shares no code with it; ``cfr_oracle.c`` decodes stored bytes, resolves page
indices and evaluates softmax(q K^T sigma + bias) V directly in double
precision.

Parity status of each oracle function (what pins it is listed in the tests):
  attend(mode=0)  pinned: closed forms, library SDPA special case, page-byte
                  decoding patterns, brute force on tiny inputs, invariants.
  attend(mode=1)  pinned against mode 0 (fold invariant, every block size).
  attend(mode=2)  pinned against mode 0 (split + merge invariant).
  merge           pinned: closed forms and against attend(mode=2).
  kv_bytes        pinned: the CFR-Atlas page's printed byte counts.
  demote          pinned: hand-derived byte patterns (rounding, clamping,
                  nibble order), the E4M3 table of the format definition and
                  the library's float8 conversion, reconstruction-error bounds,
                  scaling invariances, the all-zero block.
  attend(num_queries > 1)  pinned: one query row equals the single-query
                  definition over its prefix, torch SDPA in fp64 with the causal
                  mask of the last Q positions, decimal brute force.
  attend(sink, window)  pinned: full window equals full attention, a window of
                  one token returns its V row, without ALiBi equals attention
                  over a sequence holding only the chosen tokens, decimal brute
                  force with ALiBi.
  append          pinned: byte layout (a token appended to an empty page is
                  what a decode over one token returns), the library's bf16
                  rounding, fault cases.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cfr_oracle.c")
_LIB = os.path.join(_HERE, "libcfr_oracle.so")

OK, BAD_ARG, BAD_PAGE, NO_MEMORY, EMPTY = 0, 1, 2, 3, 4
NFMT = 5  # F32, BF16, I8, I4, FP8 (E4M3)
# bits the oracle reports for skipped pages or tokens
DEV_PAGE_ID, DEV_PAGE_FMT, DEV_SEQ_LEN = 0x1, 0x2, 0x4


def build(force: bool = False) -> str:
    """Compile cfr_oracle.c with gcc (-O2, no fast-math, OpenMP) into libcfr_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("page_tokens", ctypes.c_int32), ("max_pages", ctypes.c_int32),
        ("q_fmt", ctypes.c_int32), ("uniform_fmt", ctypes.c_int32),
        ("q", ctypes.c_void_p),
        ("k_pool", ctypes.c_void_p * 5), ("v_pool", ctypes.c_void_p * 5),
        ("scales", ctypes.c_void_p * 5), ("pool_pages", ctypes.c_int64 * 5),
        ("page_table", ctypes.c_void_p), ("page_fmt", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p), ("head_map", ctypes.c_void_p),
        ("alibi_slopes", ctypes.c_void_p), ("softmax_scale", ctypes.c_double),
        ("sink_tokens", ctypes.c_int32), ("window_tokens", ctypes.c_int32),
        ("num_queries", ctypes.c_int32),
    ]


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.cfr_oracle_attend.restype = ctypes.c_int
        lib.cfr_oracle_attend.argtypes = [
            ctypes.POINTER(_Problem), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_int, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_void_p]
        lib.cfr_oracle_merge.restype = ctypes.c_int
        lib.cfr_oracle_merge.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p]
        lib.cfr_oracle_kv_bytes.restype = ctypes.c_int64
        lib.cfr_oracle_kv_bytes.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int32]
        vp = ctypes.c_void_p
        lib.cfr_oracle_demote.restype = ctypes.c_int
        lib.cfr_oracle_demote.argtypes = [
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, vp, vp, vp, ctypes.c_int64,
            ctypes.c_int32, vp, vp, vp, ctypes.c_int64,
            vp, vp, vp, ctypes.c_int32, vp]
        lib.cfr_oracle_append.restype = ctypes.c_int
        lib.cfr_oracle_append.argtypes = [
            ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, vp, vp, vp,
            vp, ctypes.c_int32, vp, ctypes.c_int32, vp, ctypes.c_int32,
            ctypes.c_int32, vp, vp, vp]
        lib.cfr_oracle_e4m3_code.restype = ctypes.c_int32
        lib.cfr_oracle_e4m3_code.argtypes = [ctypes.c_float]
        lib.cfr_oracle_e4m3_value.restype = ctypes.c_double
        lib.cfr_oracle_e4m3_value.argtypes = [ctypes.c_int32]
        lib.cfr_oracle_bf16_bits.restype = ctypes.c_int32
        lib.cfr_oracle_bf16_bits.argtypes = [ctypes.c_float]
        _lib = lib
    return _lib


def _host(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return t.detach().to("cpu").contiguous()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned status {code}")
        self.code = code


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def attend(case, sel: Optional[Sequence[tuple]] = None, mode: int = 0, arg: int = 0,
           skip_invalid: bool = False, nthreads: Optional[int] = None,
           mem_limit: int = 16 << 30, allow_empty: bool = False, host_pools=None,
           sink_tokens: int = 0, window_tokens: int = 0):
    """Oracle output for a ``synth.DecodeCase``.

    sel: list of (b, h) pairs (default: every pair, b-major).  With Q =
    case.num_queries > 1, h is a query row qi * Hq + head: query qi of the last Q
    positions, attending causally.
    window_tokens > 0 restricts every softmax to the first ``sink_tokens`` and the
    last ``window_tokens`` tokens of its sequence.
    mode 0 direct definition, 1 fold with block ``arg`` tokens, 2 ``arg`` splits + merge.
    Returns (out float64 [n_sel][d], lse float64 [n_sel]).  ``host_pools`` may
    pass pre-copied host tensors (dict with keys k_pool, v_pool, scales) so a
    large case is copied to the host once.
    """
    lib = _load()
    keep = []

    def h(t):
        x = _host(t)
        if x is not None:
            keep.append(x)
        return x

    if host_pools is None:
        kp = {f: h(t) for f, t in case.k_pool.items()}
        vp = {f: h(t) for f, t in case.v_pool.items()}
        sc = {f: h(t) for f, t in case.scales.items()}
    else:
        kp, vp, sc = host_pools["k_pool"], host_pools["v_pool"], host_pools["scales"]
    pr = _Problem()
    pr.batch, pr.num_q_heads, pr.num_kv_heads = case.batch, case.num_q_heads, case.num_kv_heads
    pr.head_dim, pr.page_tokens, pr.max_pages = case.head_dim, case.page_tokens, case.max_pages
    pr.q_fmt, pr.uniform_fmt = case.q_fmt, case.uniform_fmt
    q = h(case.q)
    pr.q = q.data_ptr()
    for f in range(NFMT):
        pr.k_pool[f] = kp[f].data_ptr() if f in kp else None
        pr.v_pool[f] = vp[f].data_ptr() if f in vp else None
        pr.scales[f] = sc[f].data_ptr() if f in sc else None
        pr.pool_pages[f] = int(kp[f].shape[0]) if f in kp else 0
    pt = h(case.page_table.to(torch.int32))
    pr.page_table = pt.data_ptr()
    pf = h(case.page_fmt)
    pr.page_fmt = pf.data_ptr() if pf is not None else None
    sl = h(case.seq_lens.to(torch.int32))
    pr.seq_lens = sl.data_ptr()
    hm = h(case.head_map)
    pr.head_map = hm.data_ptr() if hm is not None else None
    al = h(case.alibi_slopes)
    pr.alibi_slopes = al.data_ptr() if al is not None else None
    pr.softmax_scale = float(case.softmax_scale)
    pr.sink_tokens, pr.window_tokens = int(sink_tokens), int(window_tokens)
    pr.num_queries = int(getattr(case, "num_queries", 1))

    if sel is None:
        n_sel = case.batch * case.num_q_heads * int(getattr(case, "num_queries", 1))
        sb = sh = None
    else:
        n_sel = len(sel)
        sb = torch.tensor([s[0] for s in sel], dtype=torch.int32)
        sh = torch.tensor([s[1] for s in sel], dtype=torch.int32)
    out = np.zeros((n_sel, case.head_dim), dtype=np.float64)
    lse = np.zeros((n_sel,), dtype=np.float64)
    nt = default_threads() if nthreads is None else nthreads
    rc = lib.cfr_oracle_attend(ctypes.byref(pr), _ptr(sb), _ptr(sh), n_sel, mode, arg,
                               int(skip_invalid), nt, mem_limit,
                               out.ctypes.data_as(ctypes.c_void_p),
                               lse.ctypes.data_as(ctypes.c_void_p))
    if rc != OK and not (rc == EMPTY and allow_empty):
        raise OracleError(rc)
    return out, lse


def merge(part_acc, part_m, part_l, split_off, batch: int, num_q_heads: int, head_dim: int):
    """Oracle log-sum-exp merge of split partials (base-2 maxima). Returns (out, lse) fp64."""
    lib = _load()
    a = _host(part_acc).float()
    m = _host(part_m).float()
    l = _host(part_l).float()
    off = _host(split_off).to(torch.int32)
    out = np.zeros((batch, num_q_heads, head_dim), dtype=np.float64)
    lse = np.zeros((batch, num_q_heads), dtype=np.float64)
    rc = lib.cfr_oracle_merge(_ptr(a), _ptr(m), _ptr(l), _ptr(off), batch, num_q_heads, head_dim,
                              out.ctypes.data_as(ctypes.c_void_p),
                              lse.ctypes.data_as(ctypes.c_void_p))
    if rc != OK:
        raise OracleError(rc)
    return out, lse


def kv_bytes(fmt: int, tokens: int, head_dim: int) -> int:
    """K+V bytes of `tokens` tokens of one head stored in format ``fmt``."""
    return int(_load().cfr_oracle_kv_bytes(fmt, tokens, head_dim))


def demote(num_kv_heads: int, head_dim: int, page_tokens: int, src_fmt: int, src_k, src_v,
           src_scales, dst_fmt: int, dst_k, dst_v, dst_scales, src_slots, dst_slots,
           valid_tokens=None) -> int:
    """Oracle page demotion on host tensors; writes dst_k/dst_v/dst_scales in place.

    Pools are contiguous uint8 CPU tensors [slots][Hkv][P][row_bytes], scales
    float32 [slots][Hkv][2] (None for float formats).  Returns the OR of the
    DEV_* bits of skipped pages.
    """
    lib = _load()
    for t in (src_k, src_v, dst_k, dst_v, src_scales, dst_scales):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError("oracle.demote needs contiguous CPU tensors")
    ss = _host(torch.as_tensor(src_slots, dtype=torch.int32))
    ds = _host(torch.as_tensor(dst_slots, dtype=torch.int32))
    vt = None if valid_tokens is None else _host(torch.as_tensor(valid_tokens, dtype=torch.int32))
    err = ctypes.c_uint32(0)
    rc = lib.cfr_oracle_demote(num_kv_heads, head_dim, page_tokens,
                               src_fmt, _ptr(src_k), _ptr(src_v), _ptr(src_scales),
                               int(src_k.shape[0]),
                               dst_fmt, _ptr(dst_k), _ptr(dst_v), _ptr(dst_scales),
                               int(dst_k.shape[0]),
                               _ptr(ss), _ptr(ds), _ptr(vt), int(ss.numel()), ctypes.byref(err))
    if rc != OK:
        raise OracleError(rc)
    return int(err.value)


def append(num_kv_heads: int, head_dim: int, page_tokens: int, k_pool: dict, v_pool: dict,
           page_table, page_fmt, uniform_fmt: int, positions, new_fmt: int, k_new, v_new) -> int:
    """Oracle KV append on host tensors (pools dict fmt -> uint8 CPU tensor, written in place).

    Returns the OR of the DEV_* bits of skipped sequences.
    """
    lib = _load()
    kp = (ctypes.c_void_p * NFMT)(*[k_pool[f].data_ptr() if f in k_pool else None
                                     for f in range(NFMT)])
    vpp = (ctypes.c_void_p * NFMT)(*[v_pool[f].data_ptr() if f in v_pool else None
                                      for f in range(NFMT)])
    pages = (ctypes.c_int64 * NFMT)(*[int(k_pool[f].shape[0]) if f in k_pool else 0
                                       for f in range(NFMT)])
    pt = _host(page_table.to(torch.int32))
    pf = _host(page_fmt)
    pos = _host(torch.as_tensor(positions, dtype=torch.int32))
    kn, vn = _host(k_new), _host(v_new)
    err = ctypes.c_uint32(0)
    rc = lib.cfr_oracle_append(num_kv_heads, head_dim, page_tokens, kp, vpp, pages,
                               _ptr(pt), int(pt.shape[1]), _ptr(pf), uniform_fmt,
                               _ptr(pos), int(pos.numel()), new_fmt, _ptr(kn), _ptr(vn),
                               ctypes.byref(err))
    if rc != OK:
        raise OracleError(rc)
    return int(err.value)


def e4m3_code(x: float) -> int:
    """The oracle's E4M3 code for fp32 x (nearest, ties to even, saturating)."""
    return int(_load().cfr_oracle_e4m3_code(float(x)))


def e4m3_value(code: int) -> float:
    """The value of E4M3 code ``code`` by the format definition."""
    return float(_load().cfr_oracle_e4m3_value(int(code)))


def bf16_bits(x: float) -> int:
    """The oracle's bfloat16 bits for fp32 x (nearest, ties to even)."""
    return int(_load().cfr_oracle_bf16_bits(float(x))) & 0xFFFF
