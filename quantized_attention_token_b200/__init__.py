"""Python binding of libsage, the B200 (sm_100a) quantized-attention library.

Argument marshalling only: every step of the forward pass runs in the CUDA
kernels behind include/sage.h.  There is no CPU or PyTorch fallback -- if the
shared library is missing, importing the entry points raises.

Low-level functions carry the C names (sage_attn_fwd, sage_quant_qk, ...) and
take raw device pointers; ``sageattn`` / ``sageattn_varlen`` are the tensor
API of the pages (sageattn(q, k, v, tensor_layout="HND", is_causal=False),
from the install/tuning guide's quick-start and tuning sections; the varlen +
GQA entry point from the repository summary's feature list).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

__all__ = [
    "sageattn", "sageattn_varlen", "quant_qk", "quant_qkv", "quant_v", "attn_quantized", "workspace_layout",
    "get_device_error", "debug_qk_tile", "debug_set_max_ctas", "debug_withhold_k_tile",
    "debug_set_prepass_one_pass", "debug_last_prepass_path", "debug_set_out_map", "debug_last_out_path",
    "Workspace", "SageError",
    "lib", "LIB_PATH",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsage.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(6)
LAYOUT = {"HND": 0, "NHD": 1}
GRAN = {"per_block": 0, "per_warp": 1, "per_thread": 2, "per_token": 3}
PV = {"fp8": 0, "fp16": 1, "fp8_smooth_v": 2}   # fp8_smooth_v: FP8 with V smoothed by its channel mean
# fp32_lazy: one-level, conditional rescaling; fp32+fp16: two-level with a binary16 inner level (FP8 P~V)
ACC = {"fp32": 0, "fp32+fp32": 1, "fp32fp32": 1, "fp32_lazy": 2, "fp32+fp16": 3, "fp32fp16": 3}


class SageError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "err", "tile_off_q", "tile_off_k", "k_stat", "v_sum", "v_stat", "k_mean", "v_scale", "v_mean",
        "q_codes", "q_scale", "k_codes", "k_scale", "v_codes", "q_mean", "q_bias", "total")] + [
        ("tiles_q", ctypes.c_int), ("tiles_k", ctypes.c_int)]


_lib = None


def lib():
    """Load libsage.so (built in-tree by build.py); raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m quantized_attention_token_b200.build`"
                          " (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    sigs = {
        "sage_workspace_bytes": (Z, [I, I, I, I, I, I, I]),
        "sage_varlen_workspace_bytes": (Z, [I, I, I, I, I, I, I, I]),
        "sage_workspace_layout": (I, [I, I, I, I, I, I, I, I, I, I, ctypes.POINTER(WsLayout)]),
        "sage_quant_qk": (I, [P, P, I, I, I, I, I, I, I, I, I, I, P, Z, P]),
        "sage_quant_v": (I, [P, I, I, I, I, I, I, I, P, Z, P]),
        "sage_quant_qkv": (I, [P, P, P, I, I, I, I, I, I, I, I, I, I, I, P, Z, P]),
        "sage_attn_fwd": (I, [P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, I, I, I, P, Z, P]),
        "sage_attn_quantized": (I, [P, I, I, I, I, I, I, I, I, F, I, I, I, I, P, Z, P]),
        "sage_attn_varlen_fwd": (I, [P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, F, I, I, I, I, P, Z, P]),
        "sage_get_device_error": (I, [P, P, ctypes.POINTER(ctypes.c_uint32)]),
        "sage_debug_qk_tile": (I, [P, I, I, I, I, I, I, I, I, I, I, I, P, P]),
        "sage_status_string": (ctypes.c_char_p, [I]),
        "sage_last_cuda_error": (I, []),
        "sage_last_cuda_error_name": (ctypes.c_char_p, []),
        "sage_debug_set_max_ctas": (I, [I]),
        "sage_debug_withhold_k_tile": (I, [I]),
        "sage_debug_set_prepass_one_pass": (I, [I]),
        "sage_debug_last_prepass_path": (I, []),
        "sage_debug_set_out_map": (I, [I]),
        "sage_debug_last_out_path": (I, []),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(L, name)
        fn.restype, fn.argtypes = res, args
    _lib = L
    return L


def _check(fn: str, status: int):
    if status != OK:
        msg = lib().sage_status_string(status).decode()
        if status in (ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE):
            raise ValueError(f"{fn}: {msg} (status {status})")
        if status == ERR_CUDA:
            msg += f" ({lib().sage_last_cuda_error_name().decode()})"
        raise SageError(fn, status, msg)


# ----------------------------------------------------------------------------- C names
def sage_workspace_bytes(B, Hq, Hkv, S, D, pv=0, smooth_q=0) -> int:
    return int(lib().sage_workspace_bytes(B, Hq, Hkv, S, D, pv, smooth_q))


def sage_varlen_workspace_bytes(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv=0) -> int:
    return int(lib().sage_varlen_workspace_bytes(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv))


def workspace_layout(n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv=0, smooth_q=0, varlen=0) -> dict:
    L = WsLayout()
    _check("sage_workspace_layout", lib().sage_workspace_layout(
        n_seqs, total_q, total_k, max_seqlen, Hq, Hkv, D, pv, smooth_q, varlen, ctypes.byref(L)))
    return {n: getattr(L, n) for n, _ in WsLayout._fields_}


# ----------------------------------------------------------------------------- torch API
def _torch():
    import torch
    return torch


def _stream(device) -> int:
    torch = _torch()
    return torch.cuda.current_stream(device).cuda_stream


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float16:
        return 0
    if t.dtype == torch.bfloat16:
        return 1
    raise ValueError(f"sageattn: dtype {t.dtype} not supported (fp16 or bf16)")


class Workspace:
    """A growable device workspace per device (a torch uint8 buffer)."""

    _cache: dict = {}

    @classmethod
    def get(cls, nbytes: int, device):
        torch = _torch()
        key = torch.device(device).index or 0
        buf = cls._cache.get(key)
        if buf is None or buf.numel() < nbytes:
            # zeroed: the device error word at its start must begin at 0
            buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            cls._cache[key] = buf
        return buf


def _contig(t, name):
    if not t.is_cuda:
        raise ValueError(f"sageattn: {name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"sageattn: {name} must be contiguous")
    return t


def _pv_mode(pv_dtype: str, smooth_v: bool) -> str:
    if smooth_v and pv_dtype not in ("fp8", "fp8_smooth_v"):
        raise ValueError("smooth_v applies to FP8 P~V only")
    return "fp8_smooth_v" if smooth_v else pv_dtype


def sageattn(q, k, v, tensor_layout: str = "HND", is_causal: bool = False, sm_scale: Optional[float] = None,
             qk_quant_gran: str = "per_block", pv_dtype: str = "fp8", pv_accum_dtype: str = "fp32+fp32",
             smooth_k: bool = True, smooth_q: bool = False, smooth_v: bool = False, out=None,
             workspace=None):
    """Quantized attention forward; returns a tensor shaped like q.

    q: [B, Hq, S, D] (HND) or [B, S, Hq, D] (NHD); k, v likewise with Hkv
    heads; fp16 or bf16; D in {64, 128}.  smooth_v (FP8 P~V only) is the
    pv_dtype "fp8_smooth_v".
    """
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _contig(t, n)
    if tensor_layout not in LAYOUT:
        raise ValueError("sageattn: tensor_layout must be 'HND' or 'NHD'")
    if q.dim() != 4 or k.shape != v.shape or q.dtype != k.dtype or k.dtype != v.dtype:
        raise ValueError("sageattn: q, k, v must be 4-D with matching dtype and k.shape == v.shape")
    if tensor_layout == "HND":
        B, Hq, S, D = q.shape
        Hkv, Sk = k.shape[1], k.shape[2]
    else:
        B, S, Hq, D = q.shape
        Sk, Hkv = k.shape[1], k.shape[2]
    if Sk != S or k.shape[0] != B or k.shape[3] != D:
        raise ValueError("sageattn: q and k/v must share batch, sequence length and head dim")
    pv, acc, gran = PV[_pv_mode(pv_dtype, smooth_v)], ACC[pv_accum_dtype], GRAN[qk_quant_gran]
    nbytes = sage_workspace_bytes(B, Hq, Hkv, S, D, pv, int(smooth_q))
    if nbytes == 0:
        raise ValueError("sageattn: unsupported sizes")
    ws = workspace if workspace is not None else Workspace.get(nbytes, q.device)
    if out is None:
        out = torch.empty_like(q)
    st = lib().sage_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q), B, Hq,
                             Hkv, S, D, LAYOUT[tensor_layout], int(is_causal), float(sm_scale or 0.0), gran, pv,
                             acc, int(smooth_k), int(smooth_q), ws.data_ptr(), ws.numel(), _stream(q.device))
    _check("sage_attn_fwd", st)
    return out


def sageattn_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen: int, is_causal: bool = False,
                    sm_scale: Optional[float] = None, qk_quant_gran: str = "per_block", pv_dtype: str = "fp8",
                    pv_accum_dtype: str = "fp32+fp32", smooth_k: bool = True, smooth_v: bool = False, out=None,
                    workspace=None):
    """Packed variable-length attention with GQA: q [Tq, Hq, D], k/v [Tk, Hkv, D],
    cu_seqlens_* int32 CUDA tensors [n+1]."""
    torch = _torch()
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (cu_seqlens_q, "cu_seqlens_q"), (cu_seqlens_k, "cu_seqlens_k")):
        _contig(t, n)
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("sageattn_varlen: cu_seqlens must be int32")
    n = cu_seqlens_q.numel() - 1
    if n < 1 or cu_seqlens_k.numel() != n + 1:
        raise ValueError("sageattn_varlen: cu_seqlens_q/k must have the same n+1 >= 2 entries")
    Tq, Hq, D = q.shape
    Tk, Hkv = k.shape[0], k.shape[1]
    pv, acc, gran = PV[_pv_mode(pv_dtype, smooth_v)], ACC[pv_accum_dtype], GRAN[qk_quant_gran]
    nbytes = sage_varlen_workspace_bytes(n, Tq, Tk, max_seqlen, Hq, Hkv, D, pv)
    if nbytes == 0:
        raise ValueError("sageattn_varlen: unsupported sizes")
    ws = workspace if workspace is not None else Workspace.get(nbytes, q.device)
    if out is None:
        out = torch.empty_like(q)
    st = lib().sage_attn_varlen_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _dtype_code(q),
                                    cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), n, Tq, Tk, int(max_seqlen),
                                    Hq, Hkv, D, int(is_causal), float(sm_scale or 0.0), gran, pv, acc,
                                    int(smooth_k), ws.data_ptr(), ws.numel(), _stream(q.device))
    _check("sage_attn_varlen_fwd", st)
    return out


def quant_qk(q, k, ws, tensor_layout="HND", qk_quant_gran="per_block", smooth_k=True, smooth_q=False):
    """The smooth + quantize pre-pass for Q and K into workspace `ws`."""
    if tensor_layout == "HND":
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
    else:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
    st = lib().sage_quant_qk(q.data_ptr(), k.data_ptr(), _dtype_code(q), LAYOUT[tensor_layout], B, Hq, Hkv, S, D,
                             GRAN[qk_quant_gran], int(smooth_k), int(smooth_q), ws.data_ptr(), ws.numel(),
                             _stream(q.device))
    _check("sage_quant_qk", st)


def quant_qkv(q, k, v, ws, tensor_layout="HND", qk_quant_gran="per_block", pv_dtype="fp8", smooth_k=True,
              smooth_q=False):
    """The whole smooth + quantize pre-pass (Q, K and V) in one launch."""
    if tensor_layout == "HND":
        B, Hq, S, D = q.shape
        Hkv = k.shape[1]
    else:
        B, S, Hq, D = q.shape
        Hkv = k.shape[2]
    st = lib().sage_quant_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), LAYOUT[tensor_layout], B,
                              Hq, Hkv, S, D, GRAN[qk_quant_gran], PV[pv_dtype], int(smooth_k), int(smooth_q),
                              ws.data_ptr(), ws.numel(), _stream(q.device))
    _check("sage_quant_qkv", st)


def quant_v(v, ws, tensor_layout="HND", pv_dtype="fp8"):
    if tensor_layout == "HND":
        B, H, S, D = v.shape
    else:
        B, S, H, D = v.shape
    st = lib().sage_quant_v(v.data_ptr(), _dtype_code(v), LAYOUT[tensor_layout], B, H, S, D, PV[pv_dtype],
                            ws.data_ptr(), ws.numel(), _stream(v.device))
    _check("sage_quant_v", st)


def attn_quantized(out, ws, B, Hq, Hkv, S, D, tensor_layout="HND", is_causal=False, sm_scale=None,
                   qk_quant_gran="per_block", pv_dtype="fp8", pv_accum_dtype="fp32+fp32", smooth_q=False):
    """The attention kernel alone on a workspace filled by quant_qk + quant_v
    (smooth_q as given to quant_qk)."""
    st = lib().sage_attn_quantized(out.data_ptr(), _dtype_code(out), B, Hq, Hkv, S, D, LAYOUT[tensor_layout],
                                   int(is_causal), float(sm_scale or 0.0), GRAN[qk_quant_gran], PV[pv_dtype],
                                   ACC[pv_accum_dtype], int(smooth_q), ws.data_ptr(), ws.numel(),
                                   _stream(out.device))
    _check("sage_attn_quantized", st)


def get_device_error(ws) -> tuple:
    """(status, raw bits) of the workspace's device error word; synchronizes."""
    bits = ctypes.c_uint32(0)
    st = lib().sage_get_device_error(ws.data_ptr(), _stream(ws.device), ctypes.byref(bits))
    return st, bits.value


def debug_qk_tile(ws, B, Hq, Hkv, S, D, b, h, q_tile, k_tile, pv_dtype="fp8"):
    """int32 [128, 128] scores of one tile, from the tensor-core MMA path."""
    torch = _torch()
    out = torch.empty(128, 128, dtype=torch.int32, device=ws.device)
    st = lib().sage_debug_qk_tile(ws.data_ptr(), B, Hq, Hkv, S, D, PV[pv_dtype], 0, b, h, q_tile, k_tile,
                                  out.data_ptr(), _stream(ws.device))
    _check("sage_debug_qk_tile", st)
    return out


def debug_set_max_ctas(n: int):
    """Cap the attention kernel's persistent grid at n CTAs (0: one per SM).
    Process-wide; results do not depend on it."""
    _check("sage_debug_set_max_ctas", lib().sage_debug_set_max_ctas(int(n)))


def debug_withhold_k_tile(ring_index: int):
    """Make CTA 0 of the following attention launches skip one K tile copy, so
    that its bounded wait runs out (-1: off).  Tests the timeout path."""
    _check("sage_debug_withhold_k_tile", lib().sage_debug_withhold_k_tile(int(ring_index)))


PREPASS_PATH = {0: None, 1: "one_pass", 2: "two_launch"}


def debug_set_prepass_one_pass(on: bool):
    """Send K / V of the following pre-passes through the one-pass cluster
    path wherever a head fits it (default: the two-launch path).
    Process-wide; both paths write identical bytes."""
    _check("sage_debug_set_prepass_one_pass", lib().sage_debug_set_prepass_one_pass(int(bool(on))))


def debug_last_prepass_path():
    """"one_pass", "two_launch" or None: the K / V path of this thread's last
    pre-pass."""
    return PREPASS_PATH[lib().sage_debug_last_prepass_path()]


OUT_PATH = {0: None, 1: "tensor_map", 2: "warp_stores"}


def debug_set_out_map(on: bool):
    """Let dense one-level attention store its output through a tensor map
    (the default) or make every launch use per-warp stores.  Process-wide;
    both paths write identical bytes."""
    _check("sage_debug_set_out_map", lib().sage_debug_set_out_map(int(bool(on))))


def debug_last_out_path():
    """"tensor_map", "warp_stores" (stores from the threads: per-warp rows in
    one-level modes, each thread's row in two-level modes) or None: the output
    store path of this thread's last attention launch."""
    return OUT_PATH[lib().sage_debug_last_out_path()]
