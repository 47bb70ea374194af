"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer / byte work (INT8 codes, E4M3 codes, int32 scores) must match bit for
bit; outputs within max-abs 2e-3 of the oracle (plus half an ulp of the
output's 16-bit type, which the rounded output carries on top, plus the
oracle's per-output allowance for P~ values whose rounding is ambiguous within
the derived exp2 error band); accuracy against exact fp64 attention: cosine >=
0.999 and relative L1 <= 0.02 with 16-bit P~V.  With FP8 P~V the method itself
(the oracle, computed exactly) lands at 0.034-0.038 relative L1 on zero-mean
iid inputs -- E4M3 keeps three fraction bits -- so the GPU output is held to
the oracle's own relative L1 + 0.002 there.
"""
import contextlib
import math

import numpy as np
import pytest
import torch

import oracle
import synth
import quantized_attention_token_b200 as sage
from tests import wsdecode

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _dev(t):
    return t.cuda()


def _tol(ref: np.ndarray, dtype: str, allow=None) -> np.ndarray:
    """2e-3, plus half an ulp of the output's 16-bit type, plus the oracle's
    allowance for P~ values whose rounding is ambiguous (within the exp2
    error band of a rounding midpoint, both neighbours are correct)."""
    ulp_bits = 10 if dtype == "fp16" else 7
    t = TOL + 0.5 * np.abs(ref) * 2.0 ** -ulp_bits + 2.0 ** -24
    return t if allow is None else t + allow


def _assert_close(out: torch.Tensor, ref, dtype: str, what=""):
    ref, allow = ref if isinstance(ref, tuple) else (ref, None)
    o = out.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - ref)
    bad = ~(err <= _tol(ref, dtype, allow))          # a NaN anywhere counts as outside
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {np.nanmax(err):.3e}"


def _accuracy(o: np.ndarray, ex: np.ndarray):
    o, ex = np.asarray(o, np.float64).ravel(), np.asarray(ex, np.float64).ravel()
    cos = float(o @ ex / (np.linalg.norm(o) * np.linalg.norm(ex)))
    rl1 = float(np.abs(o - ex).sum() / np.abs(ex).sum())
    return cos, rl1


def _check_accuracy(out, ex: np.ndarray, ref: np.ndarray, pv: str, what=""):
    """cosine >= 0.999 against exact fp64 attention, and relative L1 <= 0.02
    (16-bit P~V) or <= the oracle's own relative L1 + 0.002 (FP8 P~V)."""
    o = out.double().cpu().numpy() if isinstance(out, torch.Tensor) else out
    cos, rl1 = _accuracy(o, ex)
    assert cos >= 0.999, (what, cos)
    bound = 0.02 if pv == "fp16" else _accuracy(ref, ex)[1] + 0.002
    assert rl1 <= bound, (what, rl1, bound)
    return cos, rl1


@contextlib.contextmanager
def max_ctas(n):
    """Cap the attention kernel's persistent grid for the duration."""
    sage.debug_set_max_ctas(int(n or 0))
    try:
        yield
    finally:
        sage.debug_set_max_ctas(0)


@contextlib.contextmanager
def prepass_path(path):
    """Run the block with K / V of the pre-pass on `path`: "two_launch" (the
    default) or "one_pass" (the cluster path, wherever a head fits it)."""
    sage.debug_set_prepass_one_pass(path == "one_pass")
    try:
        yield
    finally:
        sage.debug_set_prepass_one_pass(False)


def _ws_bytes(ws: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    return ws.cpu().numpy()


# ----------------------------------------------------------------------------- pre-pass
@pytest.mark.parametrize("D,S,gran,dtype,layout", [
    (128, 256, "per_block", "fp16", "HND"),
    (128, 300, "per_warp", "bf16", "NHD"),
    (64, 1000, "per_thread", "fp16", "HND"),
    (64, 129, "per_block", "bf16", "HND"),
    (128, 700, "per_thread", "bf16", "NHD"),
    (128, 333, "per_token", "fp16", "HND"),
    (64, 200, "per_token", "bf16", "NHD"),
])
@pytest.mark.parametrize("smooth_k", [True, False])
@pytest.mark.parametrize("path", ["two_launch", "one_pass"])
def test_prepass_codes_bit_exact(D, S, gran, dtype, layout, smooth_k, path):
    """Codes and scales of Q, K and V against the oracle, bit for bit, on both
    K / V paths of the pre-pass."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=D, B=2, S=S, dtype=dtype, layout=layout, k_bias_std=3.0, seed=31)
    q, k, v = synth.make(sp)
    nb = sage.sage_workspace_bytes(2, 4, 2, S, D, 0, 0)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    expect = path
    with prepass_path(path):
        sage.quant_qk(_dev(q), _dev(k), ws, layout, gran, smooth_k=smooth_k)
        assert sage.debug_last_prepass_path() == expect
        sage.quant_v(_dev(v), ws, layout, "fp8")
        assert sage.debug_last_prepass_path() == expect
    assert sage.get_device_error(ws) == (0, 0)
    L = sage.workspace_layout(2, 2 * S, 2 * S, S, 4, 2, D)
    W = _ws_bytes(ws)
    tps = (S + 127) // 128
    qc = wsdecode.codes_int8(W, L, "q_codes", 4, L["tiles_q"], D)
    kc = wsdecode.codes_int8(W, L, "k_codes", 2, L["tiles_k"], D)
    qs = wsdecode.scales(W, L, "q_scale", 4, L["tiles_q"], 128)
    ks = wsdecode.scales(W, L, "k_scale", 2, L["tiles_k"], 16)
    v8 = wsdecode.v_fp8(W, L, 2, L["tiles_k"], D)
    vs = wsdecode.f32(W, L, "v_scale", 2 * 2 * D).reshape(2, 2, D)
    km = wsdecode.f32(W, L, "k_mean", 2 * 2 * D).reshape(2, 2, D)
    pb = oracle.problem(q, k, v, layout)
    for b in range(2):
        for h in range(4):
            r = oracle.quant_q(pb.q[b][h], gran, False)
            g = qc[h, b * tps:(b + 1) * tps].reshape(-1, D)
            assert np.array_equal(g[:S], r.codes), (b, h)
            assert np.all(g[S:] == 0)
            ng = oracle.q_groups_per_block(gran)
            assert np.array_equal(qs[h, b * tps:(b + 1) * tps, :ng], r.scales)
        for h in range(2):
            r = oracle.quant_k(pb.k[b][h], gran, smooth_k, dtype == "fp16")
            g = kc[h, b * tps:(b + 1) * tps].reshape(-1, D)
            assert np.array_equal(g[:S], r.codes), (b, h)
            assert np.all(g[S:] == 0)
            ng = oracle.k_groups_per_block(gran)
            assert np.array_equal(ks[h, b * tps:(b + 1) * tps, :ng], r.scales)
            if smooth_k:
                assert np.array_equal(km[b, h], r.mu)
            rv = oracle.quant_v(pb.v[b][h])
            g = v8[h, b * tps:(b + 1) * tps].reshape(-1, D)
            assert np.array_equal(g[:S], rv.codes), (b, h)
            assert np.all(g[S:] == 0)
            assert np.array_equal(vs[b, h], rv.scales)


@pytest.mark.parametrize("D,S,gran,dtype,layout", [
    (128, 300, "per_block", "fp16", "HND"),
    (64, 257, "per_thread", "bf16", "NHD"),
])
@pytest.mark.parametrize("path", ["two_launch", "one_pass"])
def test_prepass_smooth_q_bit_exact(D, S, gran, dtype, layout, path):
    """Smooth Q: block means, INT8 codes of Q - mean, and the per-key score
    corrections (fp64 sum in channel order, rounded to float once)."""
    Hq, Hkv, B = 4, 2, 2
    sp = synth.Spec("t", Hq=Hq, Hkv=Hkv, D=D, B=B, S=S, dtype=dtype, layout=layout, k_bias_std=3.0,
                    q_block_offset_std=1.0, seed=35)
    q, k, v = synth.make(sp)
    ws = torch.zeros(sage.sage_workspace_bytes(B, Hq, Hkv, S, D, 0, 1), dtype=torch.uint8, device="cuda")
    with prepass_path(path):
        sage.quant_qk(_dev(q), _dev(k), ws, layout, gran, smooth_k=True, smooth_q=True)
    assert sage.get_device_error(ws) == (0, 0)
    L = sage.workspace_layout(B, B * S, B * S, S, Hq, Hkv, D, smooth_q=1)
    W = _ws_bytes(ws)
    tps = (S + 127) // 128
    tq = L["tiles_q"]
    qc = wsdecode.codes_int8(W, L, "q_codes", Hq, tq, D)
    qs = wsdecode.scales(W, L, "q_scale", Hq, tq, 128)
    qm = wsdecode.f32(W, L, "q_mean", Hq * tq * D).reshape(Hq, tq, D)
    qb = wsdecode.f32(W, L, "q_bias", Hq * tq * tps * 128).reshape(Hq, tq, tps * 128)
    pb = oracle.problem(q, k, v, layout)
    ng = oracle.q_groups_per_block(gran)
    for b in range(B):
        for h in range(Hq):
            r = oracle.quant_q(pb.q[b][h], gran, True)
            sl = slice(b * tps, (b + 1) * tps)
            assert np.array_equal(qm[h, sl], r.mu_blk), (b, h)
            assert np.array_equal(qc[h, sl].reshape(-1, D)[:S], r.codes), (b, h)
            assert np.array_equal(qs[h, sl, :ng], r.scales), (b, h)
            kq = oracle.quant_k(pb.k[b][h // (Hq // Hkv)], gran, True, dtype == "fp16")
            ref = oracle.smooth_q_bias(r, kq).astype(np.float32)
            assert np.array_equal(qb[h, sl, :S], ref), (b, h)


@pytest.mark.parametrize("D,S,dtype,layout", [(128, 300, "fp16", "HND"), (64, 517, "bf16", "NHD")])
@pytest.mark.parametrize("path", ["two_launch", "one_pass"])
def test_prepass_smooth_v_bit_exact(D, S, dtype, layout, path):
    """Smooth V: channel mean (exact sum), E4M3 codes of V - mean and the
    scales, against the oracle; keys past the sequence stay 0."""
    Hq, Hkv, B = 2, 2, 2
    sp = synth.Spec("t", Hq=Hq, Hkv=Hkv, D=D, B=B, S=S, dtype=dtype, layout=layout, seed=36)
    q, k, v = synth.make(sp)
    v = v + torch.from_numpy(np.random.default_rng(7).normal(0, 8, D).astype(np.float32)).to(v.dtype)
    ws = torch.zeros(sage.sage_workspace_bytes(B, Hq, Hkv, S, D, 2, 0), dtype=torch.uint8, device="cuda")
    with prepass_path(path):
        sage.quant_v(_dev(v), ws, layout, "fp8_smooth_v")
    assert sage.get_device_error(ws) == (0, 0)
    L = sage.workspace_layout(B, B * S, B * S, S, Hq, Hkv, D, pv=2)
    W = _ws_bytes(ws)
    tps = (S + 127) // 128
    v8 = wsdecode.v_fp8(W, L, Hkv, L["tiles_k"], D)
    vs = wsdecode.f32(W, L, "v_scale", B * Hkv * D).reshape(B, Hkv, D)
    vm = wsdecode.f32(W, L, "v_mean", B * Hkv * D).reshape(B, Hkv, D)
    pb = oracle.problem(q, k, v, layout)
    for b in range(B):
        for h in range(Hkv):
            rv = oracle.quant_v(pb.v[b][h], smooth=True, is_fp16=dtype == "fp16")
            g = v8[h, b * tps:(b + 1) * tps].reshape(-1, D)
            assert np.array_equal(vm[b, h], rv.mu), (b, h)
            assert np.array_equal(vs[b, h], rv.scales), (b, h)
            assert np.array_equal(g[:S], rv.codes), (b, h)
            assert np.all(g[S:] == 0)


def _outputs_region(ws, L) -> np.ndarray:
    """The workspace bytes the attention kernel reads (means, scales, codes),
    i.e. everything past the pre-pass accumulators."""
    return _ws_bytes(ws)[L["k_mean"]:L["total"]]


@pytest.mark.parametrize("D,S,B,dtype,layout,pv", [
    (128, 8000, 1, "fp16", "HND", "fp8"),           # 63 tiles: 16-CTA clusters, 4 tiles per CTA
    (128, 4096, 2, "bf16", "NHD", "fp8_smooth_v"),  # 32 tiles: 16 x 2, the benchmark's shape class
    (64, 16000, 1, "bf16", "HND", "fp8"),           # 125 tiles: 16 x 8
    (64, 1000, 3, "fp16", "NHD", "fp16"),           # 8 tiles: 4 x 2
    (128, 129, 2, "fp16", "HND", "fp8"),            # 2 tiles: one CTA per head
])
def test_prepass_paths_write_identical_bytes(D, S, B, dtype, layout, pv):
    """Q, K and V through the one-pass cluster path and through the
    two-launch path: every byte the attention kernel reads is the same, at
    cluster shapes the CASES sizes do not reach (up to 16 CTAs x 8 tiles)."""
    Hq, Hkv = 2, 2
    sp = synth.Spec("t", Hq=Hq, Hkv=Hkv, D=D, B=B, S=S, dtype=dtype, layout=layout, k_bias_std=3.0, seed=37)
    q, k, v = (_dev(t) for t in synth.make(sp))
    code = {"fp8": 0, "fp16": 1, "fp8_smooth_v": 2}[pv]
    L = sage.workspace_layout(B, B * S, B * S, S, Hq, Hkv, D, pv=code)
    got = {}
    for path in ("two_launch", "one_pass"):
        ws = torch.zeros(sage.sage_workspace_bytes(B, Hq, Hkv, S, D, code, 0), dtype=torch.uint8, device="cuda")
        with prepass_path(path):
            sage.quant_qkv(q, k, v, ws, layout, "per_thread", pv)
            taken = sage.debug_last_prepass_path()
        assert sage.get_device_error(ws) == (0, 0)
        assert taken == path, (path, taken)
        got[path] = _outputs_region(ws, L)
    assert np.array_equal(got["one_pass"], got["two_launch"])


@pytest.mark.parametrize("pv,smooth_v", [("fp8", False), ("fp8", True), ("fp16", False)])
def test_varlen_prepass_paths_agree(pv, smooth_v):
    """Varlen with empty, one-token and ragged sequences: both K / V paths of
    the pre-pass give the same attention output, bit for bit, and the
    one-pass result matches the oracle."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=64, seqlens=[200, 1, 0, 129, 1100, 77], causal=True, seed=51)
    q, k, v = synth.make(sp)
    cu = sp.cu_seqlens()
    cu_d = torch.from_numpy(cu).cuda()
    outs = {}
    for path in ("two_launch", "one_pass"):
        with prepass_path(path):
            outs[path] = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), cu_d, cu_d, max(sp.seqlens), True,
                                              pv_dtype=pv, pv_accum_dtype="fp32", smooth_v=smooth_v)
            assert sage.debug_last_prepass_path() == path
    torch.cuda.synchronize()
    assert torch.equal(outs["one_pass"], outs["two_launch"])
    ref = oracle.attention(q, k, v, causal=True, pv=pv, smooth_v=smooth_v, cu_seqlens=cu, with_allowance=True)
    _assert_close(outs["one_pass"], ref, "fp16", "varlen one-pass pre-pass vs oracle")


def test_prepass_v16_layout():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=200, dtype="bf16", seed=32)
    q, k, v = synth.make(sp)
    ws = torch.zeros(sage.sage_workspace_bytes(1, 2, 2, 200, 128, 1, 0), dtype=torch.uint8, device="cuda")
    sage.quant_v(_dev(v), ws, "HND", "fp16")
    L = sage.workspace_layout(1, 200, 200, 200, 2, 2, 128, pv=1)
    g = wsdecode.v_16(_ws_bytes(ws), L, 2, L["tiles_k"], 128).reshape(2, -1, 128)
    ref = v[0].view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(g[:, :200], ref)
    assert np.all(g[:, 200:] == 0)


@pytest.mark.parametrize("D", [64, 128])
def test_qk_tile_scores_bit_exact(D):
    S = 384
    sp = synth.Spec("t", Hq=2, Hkv=1, D=D, B=1, S=S, k_bias_std=3.0, seed=33)
    q, k, v = synth.make(sp)
    ws = torch.zeros(sage.sage_workspace_bytes(1, 2, 1, S, D, 0, 0), dtype=torch.uint8, device="cuda")
    sage.quant_qk(_dev(q), _dev(k), ws, "HND", "per_thread")
    pb = oracle.problem(q, k, v)
    kc = oracle.quant_k(pb.k[0][0], "per_thread", True, True).codes
    for h in range(2):
        qc = oracle.quant_q(pb.q[0][h], "per_thread", False).codes
        ref = oracle.scores_int32(qc, kc)
        for qt, kt in [(0, 0), (1, 2), (2, 1)]:
            s = sage.debug_qk_tile(ws, 1, 2, 1, S, D, 0, h, qt, kt).cpu().numpy()
            assert np.array_equal(s, ref[qt * 128:(qt + 1) * 128, kt * 128:(kt + 1) * 128]), (h, qt, kt)
    assert sage.get_device_error(ws) == (0, 0)


# ----------------------------------------------------------------------------- attention
CASES = [
    # D, S, Hq, Hkv, causal, gran, pv, acc, dtype, layout
    (64, 256, 2, 2, False, "per_block", "fp8", "fp32+fp32", "fp16", "HND"),
    (64, 256, 2, 2, False, "per_block", "fp8", "fp32", "fp16", "HND"),
    (128, 300, 4, 2, False, "per_warp", "fp8", "fp32", "fp16", "NHD"),
    (128, 300, 4, 2, True, "per_thread", "fp8", "fp32+fp32", "fp16", "HND"),
    (128, 520, 2, 1, True, "per_block", "fp8", "fp32", "bf16", "HND"),
    (128, 640, 2, 2, False, "per_block", "fp16", "fp32", "fp16", "HND"),
    (128, 333, 2, 2, True, "per_warp", "fp16", "fp32+fp32", "bf16", "NHD"),
    (64, 700, 4, 1, True, "per_thread", "fp16", "fp32", "fp16", "HND"),
    (64, 129, 2, 2, False, "per_thread", "fp8", "fp32+fp32", "bf16", "NHD"),
    (128, 1, 2, 2, False, "per_block", "fp8", "fp32", "fp16", "HND"),
    (128, 127, 2, 2, True, "per_block", "fp8", "fp32+fp32", "fp16", "HND"),
    (128, 400, 4, 2, True, "per_token", "fp8", "fp32", "fp16", "HND"),
    (64, 300, 2, 2, False, "per_token", "fp16", "fp32+fp32", "bf16", "NHD"),
    (64, 256, 2, 2, False, "per_block", "fp8", "fp32+fp16", "fp16", "HND"),
    (128, 300, 4, 2, True, "per_thread", "fp8", "fp32+fp16", "bf16", "NHD"),
    (128, 520, 2, 1, False, "per_warp", "fp8", "fp32+fp16", "fp16", "HND"),
]


@pytest.mark.parametrize("D,S,Hq,Hkv,causal,gran,pv,acc,dtype,layout", CASES)
def test_attention_matches_oracle(D, S, Hq, Hkv, causal, gran, pv, acc, dtype, layout):
    sp = synth.Spec("t", Hq=Hq, Hkv=Hkv, D=D, B=2, S=S, dtype=dtype, layout=layout, causal=causal,
                    k_bias_std=3.0, seed=40 + S)
    q, k, v = synth.make(sp)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), layout, causal, qk_quant_gran=gran, pv_dtype=pv,
                        pv_accum_dtype=acc)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, layout, causal, gran=gran, pv=pv, with_allowance=True, acc=acc)
    _assert_close(out, ref, dtype, "vs oracle")
    _check_accuracy(out, oracle.attention_exact(q, k, v, layout, causal), ref[0], pv, "vs fp64")


def _random_cases(n=48, seed=2024):
    """Seeded random configurations across the options the API takes:
    shapes with ragged S, GQA ratios, layouts, types, granularities, P~V
    modes, accumulation modes (lazy included), sm_scale and smooth_k."""
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        D = int(rng.choice([64, 128]))
        Hq, Hkv = [(2, 2), (4, 2), (4, 1), (3, 3), (6, 2)][int(rng.integers(5))]
        pv = str(rng.choice(["fp8", "fp16"]))
        accs = ["fp32", "fp32+fp32", "fp32_lazy"] + (["fp32+fp16"] if pv == "fp8" else [])
        cases.append(dict(D=D, S=int(rng.integers(1, 600)), B=int(rng.integers(1, 4)), Hq=Hq, Hkv=Hkv,
                          causal=bool(rng.integers(2)), gran=str(rng.choice(["per_block", "per_warp", "per_thread",
                                                                             "per_token"])),
                          pv=pv, acc=str(rng.choice(accs)), dtype=str(rng.choice(["fp16", "bf16"])),
                          layout=str(rng.choice(["HND", "NHD"])),
                          sm_scale=None if rng.integers(2) else float(rng.uniform(0.03, 0.2)),
                          smooth_k=bool(rng.integers(4) > 0), seed=1000 + i))
    return cases


@pytest.mark.parametrize("c", _random_cases(), ids=lambda c: f"seed{c['seed']}")
def test_attention_random_configurations_match_oracle(c):
    """Element-wise parity and accuracy on seeded random configurations, so
    that option combinations outside the hand-picked cases are covered too."""
    # outlier K channels only where K is smoothed: without smoothing they are
    # the error the method's smoothing step exists to remove
    sp = synth.Spec("t", Hq=c["Hq"], Hkv=c["Hkv"], D=c["D"], B=c["B"], S=c["S"], dtype=c["dtype"],
                    layout=c["layout"], causal=c["causal"], k_bias_std=3.0 if c["smooth_k"] else 0.0,
                    seed=c["seed"])
    q, k, v = synth.make(sp)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), c["layout"], c["causal"], sm_scale=c["sm_scale"],
                        qk_quant_gran=c["gran"], pv_dtype=c["pv"], pv_accum_dtype=c["acc"], smooth_k=c["smooth_k"])
    torch.cuda.synchronize()
    lazy = c["acc"] == "fp32_lazy"
    tau = (2 if c["pv"] == "fp8" else 8) if lazy else 0
    ref = oracle.attention(q, k, v, c["layout"], c["causal"], sm_scale=c["sm_scale"], gran=c["gran"], pv=c["pv"],
                           smooth_k=c["smooth_k"], lazy_tau=tau, with_allowance=True,
                           acc="fp32" if lazy else c["acc"])
    _assert_close(out, ref, c["dtype"], f"vs oracle {c}")
    _check_accuracy(out, oracle.attention_exact(q, k, v, c["layout"], c["causal"], sm_scale=c["sm_scale"]), ref[0],
                    c["pv"], f"vs fp64 {c}")


@pytest.mark.parametrize("D,S,causal,gran,pv,acc,dtype,layout", [
    (128, 384, False, "per_block", "fp8", "fp32", "fp16", "HND"),
    (128, 300, True, "per_thread", "fp8", "fp32+fp32", "bf16", "NHD"),
    (64, 257, False, "per_warp", "fp16", "fp32", "fp16", "HND"),
    (64, 200, True, "per_block", "fp16", "fp32+fp32", "bf16", "HND"),
])
def test_attention_smooth_q_matches_oracle(D, S, causal, gran, pv, acc, dtype, layout):
    """Smooth Q (Q less its block mean, the lost scores restored per key) on
    inputs whose Q carries per-block offsets, as in the video-DiT workload."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=D, B=2, S=S, dtype=dtype, layout=layout, causal=causal, k_bias_std=3.0,
                    q_block_offset_std=1.0, seed=60 + S)
    q, k, v = synth.make(sp)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), layout, causal, qk_quant_gran=gran, pv_dtype=pv,
                        pv_accum_dtype=acc, smooth_q=True)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, layout, causal, gran=gran, pv=pv, smooth_q=True, with_allowance=True)
    _assert_close(out, ref, dtype, "smooth Q vs oracle")
    _check_accuracy(out, oracle.attention_exact(q, k, v, layout, causal), ref[0], pv, "smooth Q vs fp64")


@pytest.mark.parametrize("D,S,causal,acc,dtype,layout", [
    (128, 384, False, "fp32", "fp16", "HND"),
    (128, 300, True, "fp32+fp32", "bf16", "NHD"),
    (64, 257, False, "fp32", "bf16", "HND"),
])
def test_attention_smooth_v_matches_oracle(D, S, causal, acc, dtype, layout):
    """Smooth V on inputs whose V carries large per-channel offsets."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=D, B=2, S=S, dtype=dtype, layout=layout, causal=causal, k_bias_std=3.0,
                    seed=80 + S)
    q, k, v = synth.make(sp)
    v = v + torch.from_numpy(np.random.default_rng(8).normal(0, 8, D).astype(np.float32)).to(v.dtype)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), layout, causal, pv_dtype="fp8", pv_accum_dtype=acc,
                        smooth_v=True)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, layout, causal, pv="fp8", smooth_v=True, with_allowance=True)
    _assert_close(out, ref, dtype, "smooth V vs oracle")
    _check_accuracy(out, oracle.attention_exact(q, k, v, layout, causal), ref[0], "fp8", "smooth V vs fp64")


def test_varlen_smooth_v_matches_oracle():
    sp = synth.Spec("t", Hq=4, Hkv=2, D=128, seqlens=[200, 77, 512], causal=True, seed=90)
    q, k, v = synth.make(sp)
    v = v + torch.from_numpy(np.random.default_rng(9).normal(0, 8, 128).astype(np.float32)).to(v.dtype)
    cu = sp.cu_seqlens()
    cu_d = torch.from_numpy(cu).cuda()
    out = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), cu_d, cu_d, max(sp.seqlens), True, pv_dtype="fp8",
                               pv_accum_dtype="fp32", smooth_v=True)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, causal=True, pv="fp8", smooth_v=True, cu_seqlens=cu, with_allowance=True)
    _assert_close(out, ref, "fp16", "varlen smooth V vs oracle")


@pytest.mark.parametrize("D,S,causal,gran,pv,dtype,layout", [
    (128, 640, False, "per_block", "fp8", "fp16", "HND"),
    (128, 300, True, "per_thread", "fp8", "bf16", "NHD"),
    (64, 517, False, "per_token", "fp16", "fp16", "HND"),
    (128, 384, True, "per_warp", "fp16", "bf16", "HND"),
])
def test_attention_lazy_rescale_matches_oracle(D, S, causal, gran, pv, dtype, layout):
    """Conditional rescaling (tau = 2 with FP8 P~V, 8 with 16-bit)."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=D, B=2, S=S, dtype=dtype, layout=layout, causal=causal, k_bias_std=3.0,
                    seed=100 + S)
    q, k, v = synth.make(sp)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), layout, causal, qk_quant_gran=gran, pv_dtype=pv,
                        pv_accum_dtype="fp32_lazy")
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, layout, causal, gran=gran, pv=pv, lazy_tau=2 if pv == "fp8" else 8,
                           with_allowance=True)
    _assert_close(out, ref, dtype, "lazy rescale vs oracle")
    _check_accuracy(out, oracle.attention_exact(q, k, v, layout, causal), ref[0], pv, "lazy vs fp64")


def test_tiny_config():
    sp = synth.CONFIGS["tiny"]
    q, k, v = synth.make(sp)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), "HND", False)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, with_allowance=True)
    _assert_close(out, ref, "fp16", "tiny")
    _check_accuracy(out, oracle.attention_exact(q, k, v), ref[0], "fp8", "tiny vs fp64")


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("pv,acc", [("fp8", "fp32+fp32"), ("fp16", "fp32")])
def test_varlen_gqa_matches_oracle(causal, pv, acc):
    sp = synth.Spec("t", Hq=4, Hkv=2, D=128, seqlens=[200, 1, 0, 129, 384, 77], causal=causal, seed=50)
    q, k, v = synth.make(sp)
    cu = sp.cu_seqlens()
    cu_d = torch.from_numpy(cu).cuda()
    out = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), cu_d, cu_d, max(sp.seqlens), causal, pv_dtype=pv,
                               pv_accum_dtype=acc)
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, causal=causal, pv=pv, cu_seqlens=cu, with_allowance=True)
    _assert_close(out, ref, "fp16", "varlen")


def test_varlen_single_sequence_equals_dense():
    sp = synth.Spec("t", Hq=4, Hkv=2, D=128, B=1, S=300, layout="NHD", seed=51)
    q, k, v = synth.make(sp)
    dense = sage.sageattn(_dev(q), _dev(k), _dev(v), "NHD", True)
    cu = torch.tensor([0, 300], dtype=torch.int32, device="cuda")
    var = sage.sageattn_varlen(_dev(q[0]), _dev(k[0]), _dev(v[0]), cu, cu, 300, True)
    torch.cuda.synchronize()
    assert torch.equal(dense[0], var)


def test_repeated_calls_are_deterministic():
    sp = synth.Spec("t", Hq=4, Hkv=4, D=128, B=1, S=512, seed=52)
    q, k, v = (_dev(t) for t in synth.make(sp))
    a = sage.sageattn(q, k, v)
    b = sage.sageattn(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@contextlib.contextmanager
def out_map(on):
    """Run the block with the tensor-map output stores of dense one-level
    attention on (the default) or off (per-warp stores everywhere)."""
    sage.debug_set_out_map(on)
    try:
        yield
    finally:
        sage.debug_set_out_map(True)


@pytest.mark.parametrize("D,S,B,Hq,causal,pv,acc,dtype,layout", [
    (128, 4096, 1, 2, False, "fp8", "fp32", "fp16", "HND"),
    (128, 1000, 2, 3, True, "fp16", "fp32", "bf16", "NHD"),
    (64, 777, 2, 2, True, "fp8", "fp32_lazy", "fp16", "NHD"),
    (64, 160, 1, 4, False, "fp16", "fp32_lazy", "bf16", "HND"),
    (128, 33, 3, 2, True, "fp8", "fp32", "bf16", "HND"),
])
def test_output_store_paths_write_identical_bytes(D, S, B, Hq, causal, pv, acc, dtype, layout):
    """Dense one-level attention writes its output through the tensor map by
    default; per-warp stores of the same staged rows give the same bytes, also
    for ragged last tiles and both layouts."""
    sp = synth.Spec("t", Hq=Hq, Hkv=Hq, D=D, B=B, S=S, dtype=dtype, layout=layout, seed=61)
    q, k, v = (_dev(t) for t in synth.make(sp))
    a = sage.sageattn(q, k, v, layout, causal, pv_dtype=pv, pv_accum_dtype=acc)
    torch.cuda.synchronize()
    assert sage.debug_last_out_path() == "tensor_map"
    with out_map(False):
        b = sage.sageattn(q, k, v, layout, causal, pv_dtype=pv, pv_accum_dtype=acc)
        torch.cuda.synchronize()
        assert sage.debug_last_out_path() == "warp_stores"
    assert torch.equal(a, b)


def test_two_level_and_varlen_use_warp_stores():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=256, layout="NHD", seed=62)
    q, k, v = (_dev(t) for t in synth.make(sp))
    sage.sageattn(q, k, v, "NHD", False, pv_dtype="fp8", pv_accum_dtype="fp32+fp32")
    torch.cuda.synchronize()
    assert sage.debug_last_out_path() == "warp_stores"
    cu = torch.tensor([0, 256], dtype=torch.int32, device="cuda")
    sage.sageattn_varlen(q[0], k[0], v[0], cu, cu, 256, False, pv_accum_dtype="fp32")
    torch.cuda.synchronize()
    assert sage.debug_last_out_path() == "warp_stores"


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_one_level_accumulation_as_accurate_as_two_level(pv):
    """The two accumulation modes see the same P~ and V codes; they differ in
    where each tile's partial sums are added: inside the tensor core's
    accumulator (fp32) or into a separate FP32 register buffer (fp32+fp32).
    The oracle adds the same products in fp64.  Over 256 key tiles, an inner
    accumulator narrower than FP32 (the "FP22" of the pages' Hopper kernels,
    SageAttention2 summary) would make the one-level mode measurably worse;
    on B200 both must be equally close to the oracle."""
    S = 32768
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=S, k_bias_std=4.0, seed=61)
    q, k, v = synth.make(sp)
    qd, kd, vd = (t.cuda() for t in (q, k, v))
    a = sage.sageattn(qd, kd, vd, "HND", False, pv_dtype=pv, pv_accum_dtype="fp32").double().cpu().numpy()
    b = sage.sageattn(qd, kd, vd, "HND", False, pv_dtype=pv, pv_accum_dtype="fp32+fp32").double().cpu().numpy()
    torch.cuda.synchronize()
    errs = {"fp32": [], "fp32+fp32": []}
    for h in range(2):
        for r0 in (0, S - 128):
            ref = oracle.attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], pv=pv,
                                   q_rows={(0, 0): (r0, r0 + 128)})[0, 0, r0:r0 + 128]
            errs["fp32"].append(np.abs(a[0, h, r0:r0 + 128] - ref))
            errs["fp32+fp32"].append(np.abs(b[0, h, r0:r0 + 128] - ref))
    e1 = float(np.mean(np.concatenate(errs["fp32"])))
    e2 = float(np.mean(np.concatenate(errs["fp32+fp32"])))
    print(f"mean |gpu - oracle|: fp32 {e1:.3e}, fp32+fp32 {e2:.3e}")
    assert e1 <= 1.1 * e2 + 1e-7, (e1, e2)


# ----------------------------------------------------------------------------- persistent grid
@pytest.mark.parametrize("n_ctas", [1, 3])
@pytest.mark.parametrize("D,S,causal,pv,acc,gran,dtype,layout", [
    (128, 600, False, "fp8", "fp32", "per_block", "fp16", "HND"),
    (128, 600, True, "fp8", "fp32", "per_warp", "bf16", "NHD"),
    (64, 520, True, "fp16", "fp32", "per_block", "fp16", "HND"),
    (128, 300, True, "fp8", "fp32+fp32", "per_thread", "fp16", "HND"),
    (64, 700, False, "fp16", "fp32+fp32", "per_token", "bf16", "NHD"),
    (128, 600, True, "fp8", "fp32+fp16", "per_block", "fp16", "HND"),
])
def test_persistent_items_match_oracle(n_ctas, D, S, causal, pv, acc, gran, dtype, layout):
    """A capped grid, so that each CTA walks many items one after the other:
    the mbarrier phases, the K/V ring, the Q reloads and the FP8 token run on
    across items, including tail items whose second query tile is empty."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=D, B=2, S=S, dtype=dtype, layout=layout, causal=causal, k_bias_std=3.0,
                    seed=120 + S)
    q, k, v = synth.make(sp)
    with max_ctas(n_ctas):
        out = sage.sageattn(_dev(q), _dev(k), _dev(v), layout, causal, qk_quant_gran=gran, pv_dtype=pv,
                            pv_accum_dtype=acc)
        torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, layout, causal, gran=gran, pv=pv, with_allowance=True, acc=acc)
    _assert_close(out, ref, dtype, f"{n_ctas} CTAs vs oracle")


@pytest.mark.parametrize("pv,acc", [("fp8", "fp32"), ("fp16", "fp32"), ("fp8", "fp32+fp32"), ("fp8", "fp32+fp16")])
def test_persistent_varlen_gqa_matches_oracle(pv, acc):
    """Two CTAs over the items of six sequences (one empty, one of a single
    token), causal, grouped heads."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=128, seqlens=[200, 1, 0, 129, 384, 77], causal=True, seed=52)
    q, k, v = synth.make(sp)
    cu = sp.cu_seqlens()
    cu_d = torch.from_numpy(cu).cuda()
    with max_ctas(2):
        out = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), cu_d, cu_d, max(sp.seqlens), True, pv_dtype=pv,
                                   pv_accum_dtype=acc)
        torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, causal=True, pv=pv, cu_seqlens=cu, with_allowance=True, acc=acc)
    _assert_close(out, ref, "fp16", "varlen, 2 CTAs")


@pytest.mark.parametrize("acc", ["fp32", "fp32+fp32", "fp32_lazy", "fp32+fp16"])
def test_persistent_smooth_qv_matches_oracle(acc):
    """Smooth Q (its per-key corrections ride with each V tile through the
    ring) and smooth V with one CTA walking all items."""
    sp = synth.Spec("t", Hq=4, Hkv=2, D=128, B=2, S=400, dtype="fp16", layout="HND", causal=False, k_bias_std=3.0,
                    q_block_offset_std=1.0, seed=130)
    q, k, v = synth.make(sp)
    v = v + torch.from_numpy(np.random.default_rng(13).normal(0, 8, 128).astype(np.float32)).to(v.dtype)
    with max_ctas(1):
        out = sage.sageattn(_dev(q), _dev(k), _dev(v), "HND", False, pv_dtype="fp8", pv_accum_dtype=acc,
                            smooth_q=True, smooth_v=True)
        torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, "HND", False, pv="fp8", smooth_q=True, smooth_v=True,
                           lazy_tau=2 if acc == "fp32_lazy" else 0, with_allowance=True, acc=acc)
    _assert_close(out, ref, "fp16", "smooth Q+V, 1 CTA")


@pytest.mark.parametrize("n_ctas", [0, 2])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("pv,acc", [("fp8", "fp32"), ("fp16", "fp32"), ("fp8", "fp32+fp32")])
def test_varlen_cross_length_matches_oracle(n_ctas, causal, pv, acc):
    """Queries and keys with their own sequence boundaries (more keys, fewer
    keys, no queries, no keys), grouped heads; a sequence without keys gives
    zero rows."""
    rng = np.random.default_rng(7)
    H, Hk, D = 4, 2, 128
    lq, lk = [150, 40, 0, 200, 17, 300], [90, 300, 10, 0, 17, 260]
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    q = torch.from_numpy(rng.normal(size=(cq[-1], H, D)).astype(np.float16))
    k = torch.from_numpy((rng.normal(size=(ck[-1], Hk, D)) + rng.normal(0, 3, size=(1, Hk, D))).astype(np.float16))
    v = torch.from_numpy(rng.normal(size=(ck[-1], Hk, D)).astype(np.float16))
    with max_ctas(n_ctas):
        out = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), torch.from_numpy(cq).cuda(),
                                   torch.from_numpy(ck).cuda(), max(max(lq), max(lk)), causal, pv_dtype=pv,
                                   pv_accum_dtype=acc)
        torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, causal=causal, pv=pv, cu_seqlens=cq, cu_seqlens_k=ck, with_allowance=True)
    _assert_close(out, ref, "fp16", "cross-length varlen vs oracle")
    b = lk.index(0)
    assert torch.count_nonzero(out[cq[b]:cq[b + 1]]).item() == 0


def _random_varlen_cases(n=16, seed=77):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        ns = int(rng.integers(1, 7))
        same = bool(rng.integers(2))
        lq = [int(x) for x in rng.choice([0, 1, 17, 128, 129, 300, 513], size=ns)]
        lk = lq if same else [int(x) for x in rng.choice([0, 1, 40, 128, 255, 400], size=ns)]
        pv = str(rng.choice(["fp8", "fp16"]))
        accs = ["fp32", "fp32+fp32"] + (["fp32+fp16"] if pv == "fp8" else [])
        Hq, Hkv = [(2, 2), (4, 2), (8, 2), (3, 1)][int(rng.integers(4))]
        cases.append(dict(lq=lq, lk=lk, Hq=Hq, Hkv=Hkv, D=int(rng.choice([64, 128])), causal=bool(rng.integers(2)),
                          pv=pv, acc=str(rng.choice(accs)), gran=str(rng.choice(["per_block", "per_warp", "per_thread"])),
                          dtype=str(rng.choice(["fp16", "bf16"])), seed=2000 + i))
    return cases


@pytest.mark.parametrize("c", _random_varlen_cases(), ids=lambda c: f"seed{c['seed']}")
def test_varlen_random_configurations_match_oracle(c):
    """Seeded random packed batches: own query and key boundaries (empty,
    one-token and ragged sequences), grouped heads, both P~V modes, the
    accumulation modes and granularities, fp16 and bf16."""
    rng = np.random.default_rng(c["seed"])
    lq, lk, H, Hk, D = c["lq"], c["lk"], c["Hq"], c["Hkv"], c["D"]
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    tdt = torch.float16 if c["dtype"] == "fp16" else torch.bfloat16
    q = torch.from_numpy(rng.normal(size=(cq[-1], H, D)).astype(np.float32)).to(tdt)
    k = torch.from_numpy((rng.normal(size=(ck[-1], Hk, D)) + rng.normal(0, 3, size=(1, Hk, D))).astype(np.float32)).to(tdt)
    v = torch.from_numpy(rng.normal(size=(ck[-1], Hk, D)).astype(np.float32)).to(tdt)
    mx = max(max(lq), max(lk), 1)
    out = sage.sageattn_varlen(_dev(q), _dev(k), _dev(v), torch.from_numpy(cq).cuda(), torch.from_numpy(ck).cuda(),
                               mx, c["causal"], qk_quant_gran=c["gran"], pv_dtype=c["pv"], pv_accum_dtype=c["acc"])
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, causal=c["causal"], gran=c["gran"], pv=c["pv"], cu_seqlens=cq, cu_seqlens_k=ck,
                           with_allowance=True, acc=c["acc"])
    _assert_close(out, ref, c["dtype"], f"varlen vs oracle {c}")
    for b in range(len(lq)):                   # a sequence without keys gives zero rows
        if lk[b] == 0:
            assert torch.count_nonzero(out[cq[b]:cq[b + 1]].float()).item() == 0


# ----------------------------------------------------------------------------- fp32+fp16 accumulation
def test_fp16_accumulation_partials_round_like_the_oracle():
    """Q = 0 makes every P~ exactly 1 (the scale-1 code); V of E4M3 integers
    with channel maximum 448 makes V's codes V itself.  Each 32-key chunk's
    sum is an integer and the tile's binary16 partial is the chain of
    roundings the oracle computes: the GPU must agree within one binary16
    ulp per rounding (the oracle's allowance), and the rounding must show."""
    S, D = 512, 128
    rng = np.random.default_rng(42)
    vals = np.array([448, 416, 352, 320, 13, 11, 9, 7, 3, 1, 0, -1, -5, -15, -448], np.float64)
    vv = vals[rng.integers(0, len(vals), (S, D))]
    vv[0, :] = 448.0
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(2)).half()
    v = torch.from_numpy(vv.astype(np.float16)).view(1, 1, S, D)
    out = sage.sageattn(_dev(q), _dev(k), _dev(v), "HND", False, pv_dtype="fp8", pv_accum_dtype="fp32+fp16")
    torch.cuda.synchronize()
    ref = oracle.attention(q, k, v, pv="fp8", acc="fp32+fp16", with_allowance=True)
    _assert_close(out, ref, "fp16", "fp16 partials")
    exact_mean = vv.mean(axis=0)
    assert np.max(np.abs(ref[0][0, 0, 0] - exact_mean)) > 1e-3          # the binary16 rounding is visible


def test_fp16_accumulation_unsupported_with_16bit_pv():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=128, seed=5)
    q, k, v = (_dev(t) for t in synth.make(sp))
    with pytest.raises(ValueError):
        sage.sageattn(q, k, v, pv_dtype="fp16", pv_accum_dtype="fp32+fp16")


# ----------------------------------------------------------------------------- device timeout path
@pytest.mark.parametrize("acc", ["fp32", "fp32+fp32"])
def test_device_timeout_is_reported_and_the_context_recovers(acc):
    """CTA 0 withholds one K tile (host-selected debug switch): the MMA's
    bounded wait for it runs out after about 2 s, the CTA tears down through
    the abort path (copies in flight drained, MMAs committed, tensor memory
    freed), and the error word reports the timeout.  No GPU fault is
    involved.  The next normal call, on the same workspace after the error
    word was read and on a fresh one, must match the oracle."""
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=1024, k_bias_std=3.0, seed=140)
    q, k, v = synth.make(sp)
    qd, kd, vd = _dev(q), _dev(k), _dev(v)
    ws = torch.zeros(sage.sage_workspace_bytes(1, 2, 2, 1024, 128, 0, 0), dtype=torch.uint8, device="cuda")
    sage.debug_set_max_ctas(1)
    sage.debug_withhold_k_tile(3)
    try:
        sage.sageattn(qd, kd, vd, "HND", False, pv_accum_dtype=acc, workspace=ws)
        st, bits = sage.get_device_error(ws)
    finally:
        sage.debug_withhold_k_tile(-1)
        sage.debug_set_max_ctas(0)
    assert st == sage.ERR_TIMEOUT, (st, hex(bits))
    # the first of the attention kernel's waits to run out: the MMA issuer's
    # (for the K tile) or the loader's (for the ring slot that tile holds)
    assert bits & 0xF and not bits & ~0xF, hex(bits)
    assert sage.get_device_error(ws) == (0, 0)           # reading cleared it
    ref = oracle.attention(q, k, v, with_allowance=True)
    for w in (ws, torch.zeros_like(ws)):
        out = sage.sageattn(qd, kd, vd, "HND", False, pv_accum_dtype=acc, workspace=w)
        torch.cuda.synchronize()
        assert sage.get_device_error(w) == (0, 0)
        _assert_close(out, ref, "fp16", "after a timeout")
