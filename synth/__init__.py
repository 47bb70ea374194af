"""Seeded synthetic inputs for the quantized attention forward pass.

This module holds no arithmetic of the method: it only draws random numbers
and arranges them in the tensor layouts the pages use.  It is the one module
that both the CPU oracle's tests and the CUDA path's tests/bench import, so
that both sides see the very same input bits.

Generator: numpy's Philox4x32-10 counter-based bit generator (Salmon et al.,
"Parallel random numbers: as easy as 1, 2, 3", SC'11), keyed by
(seed, tensor id); normals come from numpy's standard_normal.  Values are
drawn in float32 and rounded once (round-to-nearest-even) to fp16 or bf16.

Workload shapes follow the pages' own examples:
  * the quick-start call of the SageAttention install/tuning guide
    ("SageAttention量化加速框架完整指南", section 五分钟跑通): B=2, H=32,
    S=4096, D=128, fp16, HND;
  * the 1K-32K sequence axis and head_dim 64/128 of that guide's benchmark
    figures (section 性能调优实战);
  * video-DiT attention (Kairos page, section 四; dim 2560 = 20 heads x 128),
    where K carries per-channel outliers and Q carries a per-64-token block
    offset -- synthetic stand-ins, no model or dataset item is used;
  * packed variable-length batches with grouped-query attention (SageAttention
    repo summary, "Tính năng chính": sageattn_varlen + native GQA).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import numpy as np
import torch

__all__ = ["Spec", "CONFIGS", "make", "normal"]

_TENSOR_IDS = {"q": 1, "k": 2, "v": 3, "k_bias": 4, "q_offset": 5}


def normal(seed: int, tensor: str, shape: Sequence[int], std: float = 1.0) -> np.ndarray:
    """float32 N(0, std^2) samples from Philox keyed by (seed, tensor)."""
    key = (int(seed) << 8) | _TENSOR_IDS[tensor]
    rng = np.random.Generator(np.random.Philox(key=key))
    x = rng.standard_normal(size=tuple(int(s) for s in shape), dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


@dataclass
class Spec:
    """One synthetic workload.

    Dense problems use (B, S); variable-length problems use ``seqlens`` (then
    B == len(seqlens) and the tensors are packed [total_tokens, H, D]).
    """
    name: str
    Hq: int
    Hkv: int
    D: int
    B: int = 1
    S: int = 0
    seqlens: Optional[List[int]] = None
    dtype: str = "fp16"          # "fp16" | "bf16"
    layout: str = "HND"          # "HND" | "NHD" (dense only)
    causal: bool = False
    k_bias_std: float = 0.0      # per-(head, channel) K offset shared by all tokens
    q_block_offset_std: float = 0.0   # per-(head, 64-token block, channel) Q offset
    seed: int = 0x5A6E
    gran: str = "per_block"
    pv: str = "fp8"
    pv_accum: str = "fp32+fp32"
    extra: dict = field(default_factory=dict)

    @property
    def varlen(self) -> bool:
        return self.seqlens is not None

    @property
    def total_tokens(self) -> int:
        return int(sum(self.seqlens)) if self.varlen else self.B * self.S

    def cu_seqlens(self) -> np.ndarray:
        lens = self.seqlens if self.varlen else [self.S] * self.B
        return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)

    def attention_ops(self) -> float:
        """4*H*L^2*D per sequence (halved for causal): the pages' TOPS numerator."""
        lens = self.seqlens if self.varlen else [self.S] * self.B
        ops = sum(4.0 * self.Hq * float(L) * float(L) * self.D for L in lens)
        return ops / 2.0 if self.causal else ops


def _to_dtype(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to(torch.float16 if dtype == "fp16" else torch.bfloat16)


def make(spec: Spec):
    """Return (q, k, v) as CPU torch tensors in the spec's layout.

    Dense HND: [B, H, S, D]; dense NHD: [B, S, H, D]; varlen: [total, H, D].
    """
    T = spec.total_tokens
    # Draw everything token-major [T, H, D] (one stream per tensor), then lay out.
    q = normal(spec.seed, "q", (T, spec.Hq, spec.D))
    k = normal(spec.seed, "k", (T, spec.Hkv, spec.D))
    v = normal(spec.seed, "v", (T, spec.Hkv, spec.D))
    if spec.k_bias_std:
        k += normal(spec.seed, "k_bias", (1, spec.Hkv, spec.D), spec.k_bias_std)
    if spec.q_block_offset_std:
        lens = spec.seqlens if spec.varlen else [spec.S] * spec.B
        nblk = max((L + 63) // 64 for L in lens)
        off = normal(spec.seed, "q_offset", (nblk, spec.Hq, spec.D), spec.q_block_offset_std)
        start = 0
        for L in lens:
            tok = np.arange(L)
            q[start:start + L] += off[tok // 64]
            start += L
    q, k, v = (_to_dtype(t, spec.dtype) for t in (q, k, v))
    if spec.varlen:
        return q, k, v
    B, S = spec.B, spec.S

    def lay(t, H):
        t = t.reshape(B, S, H, spec.D)
        return t.permute(0, 2, 1, 3).contiguous() if spec.layout == "HND" else t.contiguous()

    return lay(q, spec.Hq), lay(k, spec.Hkv), lay(v, spec.Hkv)


def _sweep() -> List[Spec]:
    out = []
    for D in (64, 128):
        for S in (1024, 2048, 4096, 8192, 16384, 32768):
            for causal in (False, True):
                out.append(Spec(f"sweep_S{S}_D{D}{'_causal' if causal else ''}", Hq=32, Hkv=32,
                                D=D, B=32768 // S, S=S, causal=causal, seed=0x5A6E + 3))
    return out


CONFIGS = {
    # Small correctness case: outlier channels in K (per-channel bias N(0, 3^2)).
    "tiny": Spec("tiny", Hq=2, Hkv=2, D=64, B=1, S=256, k_bias_std=3.0, seed=0x5A6E + 1),
    # The pages' quick-start shape; the headline throughput workload.
    "b2_h32_s4096_d128": Spec("b2_h32_s4096_d128", Hq=32, Hkv=32, D=128, B=2, S=4096,
                              seed=0x5A6E + 2),
    # Video-DiT attention: 20 heads x 128 = model dim 2560, 32K tokens, bf16, NHD.
    "video_dit": Spec("video_dit", Hq=20, Hkv=20, D=128, B=1, S=32768, dtype="bf16",
                      layout="NHD", k_bias_std=4.0, q_block_offset_std=1.0, seed=0x5A6E + 4),
    # Packed varlen batch with GQA 32/8, causal.
    "varlen_gqa": Spec("varlen_gqa", Hq=32, Hkv=8, D=128, seqlens=[1024, 3072, 7168, 16384],
                       causal=True, seed=0x5A6E + 5),
}
for _s in _sweep():
    CONFIGS[_s.name] = _s
