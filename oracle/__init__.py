"""CPU oracle for SageAttention-style quantized attention -- TEST INFRASTRUCTURE.

Only tests/, the smoke check of the package entry file and the benchmark's
CPU-baseline / reference leg may import this module.  It is a plain, slow,
independent statement of the method (sage_oracle.c, compiled with gcc) used to
check the CUDA library; the product path never calls it.

This file does argument marshalling only: it turns fp16/bf16 CPU tensors in
the HND / NHD / packed-varlen layouts of the pages' API into one [L, D] fp64
array per (sequence, head) and calls the C routines, which hold all of the
method's arithmetic.  Conversions fp16/bf16 -> fp64 are exact.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch

from . import build as _build

GRAN = {"per_block": 0, "per_warp": 1, "per_thread": 2, "per_token": 3}
PV = {"fp8": 0, "fp16": 1, "identity": 2}
ACC = {"fp32": 0, "fp32+fp32": 0, "fp32_lazy": 0, "fp32+fp16": 1}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        sig = {
            "orc_e4m3_to_float": (f32, [ctypes.c_uint8]),
            "orc_e4m3_from_float": (ctypes.c_uint8, [f32]),
            "orc_e4m3_from_float_array": (None, [P, P, i64]),
            "orc_e4m3_to_float_array": (None, [P, P, i64]),
            "orc_round_f16": (f64, [f64]),
            "orc_e4m3_alt_step": (f64, [f64, f64]),
            "orc_h16_alt_step": (f64, [f64, i32, f64]),
            "orc_p_band": (f64, [f64, f64, i32, i32, f64]),
            "orc_round_bf16": (f64, [f64]),
            "orc_q_groups_per_block": (i32, [i32]),
            "orc_k_groups_per_block": (i32, [i32]),
            "orc_q_group": (i32, [i32, i32]),
            "orc_k_group": (i32, [i32, i32]),
            "orc_channel_mean": (None, [P, i64, i32, i32, P]),
            "orc_subtract_channel": (None, [P, i64, i32, P, P]),
            "orc_smooth_q_blocks": (None, [P, i64, i32, P, P]),
            "orc_quant_int8": (None, [P, i64, i32, i32, i32, P, P]),
            "orc_row_scales": (None, [P, i64, i32, i32, P]),
            "orc_quant_v_fp8": (None, [P, i64, i32, P, P]),
            "orc_scores_int32": (None, [P, P, i64, i64, i32, P]),
            "orc_smooth_q_bias": (None, [P, i64, P, P, i64, i32, P]),
            "orc_attn_quant_head": (None, [P, P, P, P, P, P, P, P, P, i32, i32, i32, P, i64, i64, i32,
                                           i32, f32, i64, i64, P, P, i32]),
            "orc_attn_exact_head": (None, [P, P, P, i64, i64, i32, i32, f64, i64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------- codecs
def e4m3_encode(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint8)
    lib().orc_e4m3_from_float_array(_p(x), _p(out), x.size)
    return out


def e4m3_decode(c: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float32)
    lib().orc_e4m3_to_float_array(_p(c), _p(out), c.size)
    return out


def q_group(gran: str, r: int) -> int:
    return lib().orc_q_group(GRAN[gran], r)


def k_group(gran: str, r: int) -> int:
    return lib().orc_k_group(GRAN[gran], r)


def q_groups_per_block(gran: str) -> int:
    return lib().orc_q_groups_per_block(GRAN[gran])


def k_groups_per_block(gran: str) -> int:
    return lib().orc_k_groups_per_block(GRAN[gran])


# --------------------------------------------------------------------------- layouts
def _f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def seq_heads(x: torch.Tensor, layout: str, cu_seqlens: Optional[np.ndarray]) -> List[List[np.ndarray]]:
    """Split an input tensor into [sequence][head] -> contiguous [L, D] fp64."""
    x64 = _f64(x)
    out: List[List[np.ndarray]] = []
    if cu_seqlens is not None:                       # packed [T, H, D]
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        for b in range(len(cu) - 1):
            out.append([np.ascontiguousarray(x64[cu[b]:cu[b + 1], h]) for h in range(x64.shape[1])])
    elif layout == "HND":                            # [B, H, S, D]
        for b in range(x64.shape[0]):
            out.append([np.ascontiguousarray(x64[b, h]) for h in range(x64.shape[1])])
    else:                                            # NHD [B, S, H, D]
        for b in range(x64.shape[0]):
            out.append([np.ascontiguousarray(x64[b, :, h]) for h in range(x64.shape[2])])
    return out


def assemble(per: List[List[np.ndarray]], like: torch.Tensor, layout: str,
             cu_seqlens: Optional[np.ndarray]) -> np.ndarray:
    """Inverse of seq_heads for outputs (fp64, same shape as `like`)."""
    out = np.zeros(tuple(like.shape), dtype=np.float64)
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        for b, hs in enumerate(per):
            for h, a in enumerate(hs):
                out[cu[b]:cu[b + 1], h] = a
    elif layout == "HND":
        for b, hs in enumerate(per):
            for h, a in enumerate(hs):
                out[b, h] = a
    else:
        for b, hs in enumerate(per):
            for h, a in enumerate(hs):
                out[b, :, h] = a
    return out


# --------------------------------------------------------------------------- steps
@dataclass
class QuantK:
    mu: Optional[np.ndarray]      # [D] float32 (None when smooth_k is off)
    codes: np.ndarray             # [L, D] int8
    scales: np.ndarray            # [nblk, groups] float32
    row_scales: np.ndarray        # [L] float32


@dataclass
class QuantQ:
    mu_blk: Optional[np.ndarray]  # [nblk, D] float32 (smooth_q only)
    codes: np.ndarray
    scales: np.ndarray
    row_scales: np.ndarray


@dataclass
class QuantV:
    codes: np.ndarray             # [L, D] uint8 E4M3
    scales: np.ndarray            # [D] float32
    mu: Optional[np.ndarray] = None   # [D] float32 channel mean (smooth V only)


def quant_k(k: np.ndarray, gran: str, smooth_k: bool, is_fp16: bool) -> QuantK:
    L, D = k.shape
    mu = None
    xs = np.empty((L, D), dtype=np.float32)
    if smooth_k:
        mu = np.empty(D, dtype=np.float32)
        lib().orc_channel_mean(_p(k), L, D, int(is_fp16), _p(mu))
    lib().orc_subtract_channel(_p(k), L, D, _p(mu), _p(xs))
    return _quant_int8(xs, False, gran, mu)


def quant_q(q: np.ndarray, gran: str, smooth_q: bool) -> QuantQ:
    L, D = q.shape
    xs = np.empty((L, D), dtype=np.float32)
    mu_blk = None
    if smooth_q:
        mu_blk = np.empty(((L + 127) // 128, D), dtype=np.float32)
        lib().orc_smooth_q_blocks(_p(q), L, D, _p(mu_blk), _p(xs))
    else:
        lib().orc_subtract_channel(_p(q), L, D, None, _p(xs))
    r = _quant_int8(xs, True, gran, None)
    return QuantQ(mu_blk, r.codes, r.scales, r.row_scales)


def _quant_int8(xs: np.ndarray, is_q: bool, gran: str, mu) -> QuantK:
    L, D = xs.shape
    ng = (q_groups_per_block if is_q else k_groups_per_block)(gran)
    codes = np.empty((L, D), dtype=np.int8)
    scales = np.empty(((L + 127) // 128, ng), dtype=np.float32)
    lib().orc_quant_int8(_p(xs), L, D, int(is_q), GRAN[gran], _p(codes), _p(scales))
    rs = np.empty(L, dtype=np.float32)
    lib().orc_row_scales(_p(scales), L, int(is_q), GRAN[gran], _p(rs))
    return QuantK(mu, codes, scales, rs)


def quant_v(v: np.ndarray, smooth: bool = False, is_fp16: bool = True) -> QuantV:
    """Per-channel E4M3 V [SA2, FP8 quantization of P~V].  smooth: the
    optional smooth-V step the same page names next to the FP32 buffer (no
    formula given; reading): V is first reduced by its channel mean over the
    sequence's tokens (exact sum, as for K) with one float32 subtraction, and
    attention adds the mean back to its output (rows of softmax sum to 1)."""
    L, D = v.shape
    codes = np.empty((L, D), dtype=np.uint8)
    dv = np.empty(D, dtype=np.float32)
    mu = None
    if smooth:
        mu = np.empty(D, dtype=np.float32)
        lib().orc_channel_mean(_p(v), L, D, int(is_fp16), _p(mu))
        xs = np.empty((L, D), dtype=np.float32)
        lib().orc_subtract_channel(_p(v), L, D, _p(mu), _p(xs))
        v = xs.astype(np.float64)
    lib().orc_quant_v_fp8(_p(v), L, D, _p(codes), _p(dv))
    return QuantV(codes, dv, mu)


def scores_int32(qc: np.ndarray, kc: np.ndarray) -> np.ndarray:
    qc = np.ascontiguousarray(qc, dtype=np.int8)
    kc = np.ascontiguousarray(kc, dtype=np.int8)
    out = np.empty((qc.shape[0], kc.shape[0]), dtype=np.int32)
    lib().orc_scores_int32(_p(qc), _p(kc), qc.shape[0], kc.shape[0], qc.shape[1], _p(out))
    return out


def smooth_q_bias(qq: QuantQ, kq: QuantK) -> np.ndarray:
    nb, D = qq.mu_blk.shape
    Lk = kq.codes.shape[0]
    out = np.empty((nb, Lk), dtype=np.float64)
    lib().orc_smooth_q_bias(_p(qq.mu_blk), nb, _p(kq.codes), _p(kq.row_scales), Lk, D, _p(out))
    return out


def attn_head(qq: QuantQ, kq: QuantK, vq: Optional[QuantV], v16: Optional[np.ndarray],
              pv: str, v_is_bf16: bool, causal: bool, sm_scale: float,
              rows: Optional[Tuple[int, int]] = None, bias: Optional[np.ndarray] = None,
              allow: Optional[np.ndarray] = None, lazy_tau: int = 0, acc: str = "fp32") -> np.ndarray:
    """pv "fp8" / "fp16"; acc "fp32+fp16" selects the binary16 inner
    accumulation of each tile's P~V (FP8 only; see sage_oracle.c)."""
    Lq, D = qq.codes.shape
    Lk = kq.codes.shape[0]
    r0, r1 = rows if rows is not None else (0, Lq)
    if ACC[acc] == 1 and (pv != "fp8" or lazy_tau):
        raise ValueError("fp32+fp16 accumulation is defined for FP8 P~V with the plain online softmax")
    out = np.zeros((Lq, D), dtype=np.float64)
    lib().orc_attn_quant_head(
        _p(qq.codes), _p(qq.row_scales), _p(kq.codes), _p(kq.row_scales),
        _p(vq.codes) if vq is not None else None, _p(vq.scales) if vq is not None else None,
        _p(v16), None, None, PV[pv], ACC[acc], int(v_is_bf16), _p(bias), Lq, Lk, D, int(causal),
        ctypes.c_float(sm_scale), r0, r1, _p(out), _p(allow), int(lazy_tau))
    if vq is not None and vq.mu is not None and Lk > 0:
        out[r0:r1] += vq.mu.astype(np.float64)      # smooth V: the mean comes back (no keys: rows stay 0)
    return out


def attn_exact_head(q, k, v, causal, sm_scale, row_offset: int = 0) -> np.ndarray:
    q = np.ascontiguousarray(q)
    out = np.zeros(q.shape, dtype=np.float64)
    lib().orc_attn_exact_head(_p(q), _p(k), _p(v), q.shape[0], k.shape[0], q.shape[1],
                              int(causal), float(sm_scale), int(row_offset), _p(out))
    return out


def attn_tiled_fp64_head(q, k, v, causal, sm_scale, lazy_tau: int = 0) -> np.ndarray:
    """The quantized routine with its identity-quantizer switch: the same
    tiled online-softmax loop on unquantized fp64 q, k, P~ and v."""
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    Lq, D = q.shape
    out = np.zeros(q.shape, dtype=np.float64)
    lib().orc_attn_quant_head(None, None, None, None, None, None, _p(v), _p(q), _p(k), PV["identity"], 0, 0, None,
                              Lq, k.shape[0], D, int(causal), ctypes.c_float(sm_scale), 0, Lq, _p(out), None,
                              int(lazy_tau))
    return out


# --------------------------------------------------------------------------- full problems
@dataclass
class Problem:
    """Inputs of one sageattn call, split per (sequence, head)."""
    q: List[List[np.ndarray]]
    k: List[List[np.ndarray]]
    v: List[List[np.ndarray]]
    Hq: int
    Hkv: int
    D: int
    is_fp16: bool


def problem(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: str = "HND",
            cu_seqlens: Optional[np.ndarray] = None, cu_seqlens_k: Optional[np.ndarray] = None) -> Problem:
    """cu_seqlens splits packed q (and k, v unless cu_seqlens_k is given:
    then sequence b attends with its queries cu_seqlens[b]..[b+1] to the keys
    cu_seqlens_k[b]..[b+1])."""
    cu_k = cu_seqlens if cu_seqlens_k is None else cu_seqlens_k
    qs = seq_heads(q, layout, cu_seqlens)
    ks, vs = (seq_heads(t, layout, cu_k) for t in (k, v))
    return Problem(qs, ks, vs, len(qs[0]), len(ks[0]), q.shape[-1], q.dtype == torch.float16)


def default_scale(D: int, sm_scale: Optional[float]) -> float:
    return float(np.float32(1.0 / math.sqrt(D))) if not sm_scale or sm_scale <= 0 else float(sm_scale)


def quantize(pb: Problem, gran: str = "per_block", smooth_k: bool = True, smooth_q: bool = False,
             pv: str = "fp8") -> Dict[str, list]:
    """Pre-pass: per-sequence lists of per-head QuantQ / QuantK / QuantV."""
    res = {"q": [], "k": [], "v": []}
    for b in range(len(pb.q)):
        res["q"].append([quant_q(x, gran, smooth_q) for x in pb.q[b]])
        res["k"].append([quant_k(x, gran, smooth_k, pb.is_fp16) for x in pb.k[b]])
        res["v"].append([quant_v(x) if pv == "fp8" else None for x in pb.v[b]])
    return res


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: str = "HND",
              causal: bool = False, sm_scale: Optional[float] = None, gran: str = "per_block",
              pv: str = "fp8", smooth_k: bool = True, smooth_q: bool = False,
              cu_seqlens: Optional[np.ndarray] = None, smooth_v: bool = False, lazy_tau: int = 0,
              q_rows: Optional[Dict[Tuple[int, int], Tuple[int, int]]] = None,
              heads: Optional[List[Tuple[int, int]]] = None, with_allowance: bool = False,
              cu_seqlens_k: Optional[np.ndarray] = None, acc: str = "fp32"):
    """The quantized forward pass; returns fp64 output shaped like q.

    q_rows optionally restricts (seq, head) -> [row0, row1); heads restricts
    which (seq, head) pairs are computed (others stay zero).  with_allowance:
    return (out, allow), allow being the per-output bound on what ambiguous
    roundings of P~ (and, with acc "fp32+fp16", the binary16 roundings of the
    partial sums) can change (see sage_oracle.c).  acc: "fp32" / "fp32+fp32"
    / "fp32_lazy" (the same exact per-tile sums; lazy_tau selects the lazy
    bookkeeping) or "fp32+fp16".  cu_seqlens_k: packed
    keys with their own sequence boundaries (causal masks key j > query i,
    both counted from their sequence's start; a row with no visible key is 0).
    """
    pb = problem(q, k, v, layout, cu_seqlens, cu_seqlens_k)
    scale = default_scale(pb.D, sm_scale)
    group = pb.Hq // pb.Hkv
    outs, allows = [], []
    for b in range(len(pb.q)):
        needed_kv = {h // group for h in range(pb.Hq) if heads is None or (b, h) in heads}
        kq = {hk: quant_k(pb.k[b][hk], gran, smooth_k, pb.is_fp16) for hk in needed_kv}
        vq = {hk: (quant_v(pb.v[b][hk], smooth_v, pb.is_fp16) if pv == "fp8" else None) for hk in needed_kv}
        row, arow = [], []
        for h in range(pb.Hq):
            al = np.zeros_like(pb.q[b][h])
            arow.append(al)
            if heads is not None and (b, h) not in heads:
                row.append(np.zeros_like(pb.q[b][h]))
                continue
            hk = h // group
            qq = quant_q(pb.q[b][h], gran, smooth_q)
            bias = smooth_q_bias(qq, kq[hk]) if smooth_q else None
            rows = q_rows.get((b, h)) if q_rows else None
            row.append(attn_head(qq, kq[hk], vq[hk], pb.v[b][hk] if pv != "fp8" else None, pv,
                                 not pb.is_fp16, causal, scale, rows, bias,
                                 al if with_allowance else None, lazy_tau, acc))
        outs.append(row)
        allows.append(arow)
    out = assemble(outs, q, layout, cu_seqlens)
    if with_allowance:
        return out, assemble(allows, q, layout, cu_seqlens)
    return out


def attention_exact(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, layout: str = "HND",
                    causal: bool = False, sm_scale: Optional[float] = None,
                    cu_seqlens: Optional[np.ndarray] = None, tiled: bool = False,
                    cu_seqlens_k: Optional[np.ndarray] = None) -> np.ndarray:
    """fp64 softmax attention of the unquantized inputs (tiled=True: the
    128-key online-softmax loop with quantization switched off)."""
    pb = problem(q, k, v, layout, cu_seqlens, cu_seqlens_k)
    scale = default_scale(pb.D, sm_scale)
    group = pb.Hq // pb.Hkv
    fn = attn_tiled_fp64_head if tiled else attn_exact_head
    outs = [[fn(pb.q[b][h], pb.k[b][h // group], pb.v[b][h // group], causal, scale)
             for h in range(pb.Hq)] for b in range(len(pb.q))]
    return assemble(outs, q, layout, cu_seqlens)
