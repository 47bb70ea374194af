"""Decode the workspace regions documented in include/sage.h into plain arrays.

Tiles hold 128 tokens; within a tile, 128-byte rows store logical 16-byte
chunk c at chunk c ^ (row % 8), 64-byte rows store chunk c at c ^ ((row/2) % 4).
This is a layout decoder for tests, it holds none of the method's arithmetic.
"""
import numpy as np


def swz_index(rows: int, row_bytes: int) -> np.ndarray:
    r = np.arange(rows)[:, None]
    c = np.arange(row_bytes)[None, :]
    if row_bytes == 128:
        return r * 128 + (((c >> 4) ^ (r & 7)) << 4) + (c & 15)
    return r * 64 + (((c >> 4) ^ ((r >> 1) & 3)) << 4) + (c & 15)


def region(ws_bytes: np.ndarray, off: int, nbytes: int) -> np.ndarray:
    return ws_bytes[off:off + nbytes]


def codes_int8(ws_bytes, L, key, H, tiles, D):
    """[H, tiles, 128, D] int8 from q_codes / k_codes."""
    raw = region(ws_bytes, L[key], H * tiles * 128 * D).reshape(H, tiles, 128 * D)
    return raw[:, :, swz_index(128, D)].view(np.int8)


def scales(ws_bytes, L, key, H, tiles, ng_max):
    return region(ws_bytes, L[key], H * tiles * ng_max * 4).view(np.float32).reshape(H, tiles, ng_max)


def v_fp8(ws_bytes, L, H, tiles, D):
    """[H, tiles, 128 keys, D] E4M3 codes (transposed back)."""
    raw = region(ws_bytes, L["v_codes"], H * tiles * D * 128).reshape(H, tiles, D * 128)
    t = raw[:, :, swz_index(D, 128)]            # [H, tiles, D, 128 keys]
    return t.transpose(0, 1, 3, 2)


def v_16(ws_bytes, L, H, tiles, D):
    """[H, tiles, 128 keys, D] uint16 (transposed back from two 64-key halves)."""
    raw = region(ws_bytes, L["v_codes"], H * tiles * D * 256).reshape(H, tiles, 2, D * 128)
    idx = swz_index(D, 128)                     # bytes of [D rows][64 keys * 2 B]
    t = raw[:, :, :, idx].reshape(H, tiles, 2, D, 64, 2)
    u16 = t[..., 0].astype(np.uint16) | (t[..., 1].astype(np.uint16) << 8)   # [H, tiles, 2, D, 64]
    return u16.transpose(0, 1, 2, 4, 3).reshape(H, tiles, 128, D)


def f32(ws_bytes, L, key, n):
    return region(ws_bytes, L[key], n * 4).view(np.float32)
