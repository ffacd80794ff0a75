"""Independent host-side (numpy) decoding of pool bytes, for test pins only.

Written separately from the C oracle: it gathers whole pages with numpy
indexing and decodes formats with numpy views, so a mistake in the oracle's
byte decoding or index arithmetic shows up as a disagreement.
"""
import numpy as np
import torch

F32, BF16, I8, I4, FP8 = 0, 1, 2, 3, 4
QUANTISED = (I8, I4, FP8)


def decode_rows(raw: np.ndarray, fmt: int, d: int) -> np.ndarray:
    """raw uint8 [..., row_bytes] -> float64 [..., d] codes/values (no scale)."""
    if fmt == F32:
        return raw.copy().view(np.float32).astype(np.float64)
    if fmt == BF16:
        u = raw.copy().view(np.uint16).astype(np.uint32) << 16
        return u.view(np.float32).astype(np.float64)
    if fmt == I8:
        return raw.view(np.int8).astype(np.float64)
    if fmt == I4:
        lo = (raw & 0x0F).astype(np.int16)
        hi = (raw >> 4).astype(np.int16)
        lo = np.where(lo >= 8, lo - 16, lo)
        hi = np.where(hi >= 8, hi - 16, hi)
        out = np.empty(raw.shape[:-1] + (2 * raw.shape[-1],), dtype=np.float64)
        out[..., 0::2] = lo
        out[..., 1::2] = hi
        return out
    if fmt == FP8:
        # E4M3 through torch's float8 dtype (a library decoder, not the oracle's)
        t = torch.from_numpy(np.ascontiguousarray(raw)).view(torch.float8_e4m3fn)
        return t.to(torch.float64).numpy()
    raise ValueError(fmt)


def host_kv(case, b: int, g: int):
    """Full K, V (float64 [n][d]) of sequence b, kv head g, gathered page by page."""
    n = int(case.seq_lens[b])
    P, d = case.page_tokens, case.head_dim
    pt = case.page_table.cpu().numpy()
    pf = None if case.page_fmt is None else case.page_fmt.cpu().numpy()
    Ks, Vs = [], []
    for p in range(-(-n // P)):
        f = case.uniform_fmt if pf is None else int(pf[b, p])
        slot = int(pt[b, p])
        kb = case.k_pool[f][slot, g].cpu().numpy()
        vb = case.v_pool[f][slot, g].cpu().numpy()
        k = decode_rows(kb, f, d)
        v = decode_rows(vb, f, d)
        if f in QUANTISED:
            s = case.scales[f][slot, g].cpu().numpy().astype(np.float64)
            k = k * s[0]
            v = v * s[1]
        Ks.append(k)
        Vs.append(v)
    K = np.concatenate(Ks, 0)[:n]
    V = np.concatenate(Vs, 0)[:n]
    return K, V


def host_q(case) -> np.ndarray:
    q = case.q.cpu()
    if case.q_fmt == F32:
        return q.numpy().astype(np.float64)
    u = q.numpy().view(np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def kv_head_of(case, h: int) -> int:
    if case.head_map is not None:
        return int(case.head_map[h])
    return h // (case.num_q_heads // case.num_kv_heads)


def sigma_of(case) -> float:
    return case.softmax_scale if case.softmax_scale != 0 else 1.0 / np.sqrt(case.head_dim)
