"""The allocation-free entry point, sage_attn_fwd_noalloc, against the
ordinary one.

It exists for callers that cannot allocate device memory where they run
attention (an engine that reserved all device memory for its own pool, a
fixed memory budget, no tolerance for cudaMalloc's implicit synchronization).
It keeps its workspace in a static device array inside the library, so two
calls in a row reuse the same memory: both must still match sage_attn_fwd.
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import synth
import quantized_attention_token_b200 as sage

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    L = sage.lib()
    fn = L.sage_attn_fwd_noalloc
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    fn.restype = I
    fn.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, I, I, P]
    return fn


def _call(fn, q, k, v, causal, pv, acc):
    B, Hq, S, D = q.shape
    out = torch.empty_like(q)
    st = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), 0, B, Hq, k.shape[1], S, D, 0, int(causal),
            0.0, 0, sage.PV[pv], sage.ACC[acc], 1, torch.cuda.current_stream().cuda_stream)
    assert st == 0, sage.lib().sage_status_string(st)
    return out


def test_noalloc_matches_sage_attn_fwd_twice():
    fn = _noalloc_fn()
    cases = [
        (synth.Spec("a", Hq=4, Hkv=2, D=128, B=2, S=700, causal=True, seed=91), "fp8", "fp32+fp32"),
        (synth.Spec("b", Hq=8, Hkv=8, D=64, B=1, S=1500, causal=False, k_bias_std=3.0, seed=92), "fp16", "fp32"),
    ]
    for spec, pv, acc in cases:
        q, k, v = (t.cuda() for t in synth.make(spec))
        got = _call(fn, q, k, v, spec.causal, pv, acc)
        ref = sage.sageattn(q, k, v, "HND", spec.causal, pv_dtype=pv, pv_accum_dtype=acc)
        torch.cuda.synchronize()
        # the same deterministic kernels on the same inputs: identical bits
        assert torch.equal(got, ref), (spec.name, float((got.float() - ref.float()).abs().max()))


def test_noalloc_rejects_problems_beyond_its_array():
    fn = _noalloc_fn()
    B, H, S, D = 1, 32, 8192, 128            # workspace well above the 32 MiB array
    assert sage.sage_workspace_bytes(B, H, H, S, D, 0, 0) > (32 << 20)
    q = torch.empty(B, H, S, D, dtype=torch.float16, device="cuda")
    out = torch.empty_like(q)
    st = fn(q.data_ptr(), q.data_ptr(), q.data_ptr(), out.data_ptr(), 0, B, H, H, S, D, 0, 0, 0.0, 0, 0, 1, 1,
            torch.cuda.current_stream().cuda_stream)
    assert st == sage.ERR_WORKSPACE
