"""Pins of the CPU oracle against things other than itself.

Each test checks one routine of the oracle against a library routine, a
closed form, an invariant of attention, or brute force on tiny inputs.  The
pins are chosen so that a plausible mistake (a dropped term, a wrong index or
group, a transposed operand, a wrong rounding) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- E4M3 codec
def _golden_points():
    pts = []
    for line in open(os.path.join(GOLDEN, "e4m3_ocp_points.txt")):
        line = line.split("#")[0].strip()
        if line:
            c, v = line.split()
            pts.append((int(c, 16), float(v)))
    return pts


def test_e4m3_decode_matches_ocp_points():
    for code, val in _golden_points():
        got = float(oracle.e4m3_decode(np.array([code], np.uint8))[0])
        if math.isnan(val):
            assert math.isnan(got), hex(code)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(ours[ok].view(np.uint32), ref[ok].view(np.uint32))


def test_e4m3_encode_matches_torch_rne_inside_range():
    # torch's float8_e4m3fn cast is round-to-nearest-even without saturation,
    # so it is a reference for |x| <= 464 (the tie point above 448).
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(40),
        (rng.random(100000).astype(np.float32) * np.float32(2 ** -5)),          # subnormals
        rng.uniform(-464, 464, 100000).astype(np.float32),
    ])
    # every exact midpoint between neighbouring finite codes (ties -> even)
    vals = np.sort(oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64))
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.float32([464.0, -464.0])])
    ours = oracle.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_saturates_and_keeps_nan():
    x = np.float32([465.0, 480.0, 1e6, np.inf, -500.0, -np.inf, np.nan])
    c = oracle.e4m3_encode(x)
    assert list(c[:4]) == [0x7E] * 4 and list(c[4:6]) == [0xFE, 0xFE]
    assert (c[6] & 0x7F) == 0x7F


def test_e4m3_roundtrip_every_code():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_16bit_rounding_matches_library():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.random(20000), rng.random(2000) * 1e-6, [1.0, 0.5, 2 ** -24, 0.0]])
    L = oracle.lib()
    f16 = np.array([L.orc_round_f16(float(np.float32(v))) for v in x])
    assert np.array_equal(f16, np.float32(x).astype(np.float16).astype(np.float64))
    bf = np.array([L.orc_round_bf16(float(v)) for v in x])
    ref = torch.from_numpy(np.float32(x)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(bf, ref)


# ----------------------------------------------------------------------------- smoothing
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_channel_mean_is_the_exact_mean(dtype):
    sp = synth.Spec("t", Hq=1, Hkv=1, D=64, B=1, S=1000, dtype=dtype, k_bias_std=3.0, seed=7)
    _, k, _ = synth.make(sp)
    x = k[0, 0].double().numpy()
    mu = np.empty(64, np.float32)
    oracle.lib().orc_channel_mean(oracle._p(x), 1000, 64, int(dtype == "fp16"), oracle._p(mu))
    # math.fsum is an exactly rounded sum: the reference for "exact mean"
    ref = np.float32([math.fsum(x[:, c]) / 1000.0 for c in range(64)])
    assert np.array_equal(mu, ref)


def test_fp16_channel_mean_exact_with_cancellation():
    # large values that cancel plus tiny ones: an fp32/fp64 running sum would
    # lose the tiny part, the exact fixed-point sum must not
    x = np.zeros((4, 1), dtype=np.float64)
    x[:, 0] = [60000.0, -60000.0, 2.0 ** -24, 2.0 ** -24]
    mu = np.empty(1, np.float32)
    oracle.lib().orc_channel_mean(oracle._p(x), 4, 1, 1, oracle._p(mu))
    assert mu[0] == np.float32(2.0 ** -25)


def test_smooth_q_block_means():
    rng = np.random.default_rng(3)
    L, D = 300, 64
    x = np.float16(rng.standard_normal((L, D))).astype(np.float64)
    mu = np.empty((3, D), np.float32)
    xs = np.empty((L, D), np.float32)
    oracle.lib().orc_smooth_q_blocks(oracle._p(x), L, D, oracle._p(mu), oracle._p(xs))
    for b, (t0, t1) in enumerate([(0, 128), (128, 256), (256, 300)]):
        ref = np.float32([math.fsum(x[t0:t1, c]) / (t1 - t0) for c in range(D)])
        assert np.array_equal(mu[b], ref)
        assert np.array_equal(xs[t0:t1], np.float32(x[t0:t1]) - ref)


# ----------------------------------------------------------------------------- INT8 quantizer
@pytest.mark.parametrize("gran", ["per_block", "per_warp", "per_thread"])
@pytest.mark.parametrize("is_q", [True, False])
def test_int8_quantizer_bounds(gran, is_q):
    rng = np.random.default_rng(4)
    L, D = 300, 64                              # two full blocks and a ragged one
    xs = (rng.standard_normal((L, D)) * rng.uniform(0.1, 10, (L, 1))).astype(np.float32)
    r = oracle._quant_int8(xs, is_q, gran, None)
    assert r.codes.min() >= -127 and r.codes.max() <= 127
    err = np.abs(xs.astype(np.float64) - r.row_scales[:, None].astype(np.float64) * r.codes)
    # |x - delta*code| <= delta/2 up to the float32 rounding of x*(127/amax)
    assert np.all(err <= r.row_scales[:, None] * (0.5 + 1e-5) + 1e-30)
    # within every group the absolute maximum maps to +-127
    for t in range(L):
        g_rows = [u for u in range((t // 128) * 128, min(L, (t // 128) * 128 + 128))
                  if (oracle.q_group if is_q else oracle.k_group)(gran, u % 128)
                  == (oracle.q_group if is_q else oracle.k_group)(gran, t % 128)]
        if t == g_rows[0]:
            sub = np.abs(xs[g_rows])
            i = np.unravel_index(np.argmax(sub), sub.shape)
            assert abs(int(r.codes[g_rows[i[0]], i[1]])) == 127
            assert r.row_scales[t] == np.float32(sub.max()) / np.float32(127)


@pytest.mark.parametrize("gran", ["per_block", "per_warp", "per_thread", "per_token"])
@pytest.mark.parametrize("is_q", [True, False])
def test_int8_group_membership_by_brute_force(gran, is_q):
    """Blowing up one token must change the scale of exactly the tokens that
    the group definition puts in its group -- checked for every token."""
    L, D = 256, 64
    base = np.ones((L, D), np.float32)
    ref = oracle._quant_int8(base, is_q, gran, None).row_scales
    expect_groups = {"per_block": (1, 2), "per_warp": (4, 2), "per_thread": (32, 16), "per_token": (128, 2)}[gran]
    ng = expect_groups[0] if is_q else expect_groups[1]
    assert (oracle.q_groups_per_block if is_q else oracle.k_groups_per_block)(gran) == ng
    for t in range(0, L, 7):
        x = base.copy()
        x[t, 3] = 1000.0
        rs = oracle._quant_int8(x, is_q, gran, None).row_scales
        changed = set(np.nonzero(rs != ref)[0])
        blk = t // 128
        r = t % 128
        if gran == "per_token":
            size = 1 if is_q else 64
            members = {u for u in range(L) if u // 128 == blk and (u % 128) // size == r // size}
        elif gran == "per_block":
            size = 128 if is_q else 64
            members = {u for u in range(L) if u // 128 == blk and (u % 128) // size == r // size}
        elif gran == "per_warp":
            size = 32 if is_q else 64
            members = {u for u in range(L) if u // 128 == blk and (u % 128) // size == r // size}
        else:
            size = 32 if is_q else 64
            members = {u for u in range(L) if u // 128 == blk and (u % 128) // size == r // size
                       and u % 8 == t % 8}
        assert changed == members, (t, sorted(changed)[:8], sorted(members)[:8])


def test_int8_per_token_scale_is_the_row_maximum():
    """Per-token Q: every row's scale is its own |max| / 127 (closed form),
    and its largest element gets code +-127."""
    rng = np.random.default_rng(11)
    L, D = 300, 64
    xs = (rng.standard_normal((L, D)) * rng.uniform(0.01, 50, (L, 1))).astype(np.float32)
    r = oracle._quant_int8(xs, True, "per_token", None)
    am = np.abs(xs).max(axis=1)
    assert np.array_equal(r.row_scales, (am / np.float32(127)).astype(np.float32))
    assert np.all(np.abs(r.codes).max(axis=1) == 127)


def test_int8_zero_group():
    xs = np.zeros((128, 64), np.float32)
    r = oracle._quant_int8(xs, True, "per_block", None)
    assert np.all(r.codes == 0) and np.all(r.scales == 0)


def test_int8_rounding_is_ties_to_even():
    # amax 127 -> scale 1, inv 1: codes are rne(x)
    xs = np.zeros((1, 64), np.float32)
    xs[0, :6] = [127.0, 0.5, 1.5, 2.5, -0.5, -1.5]
    r = oracle._quant_int8(xs, True, "per_block", None)
    assert list(r.codes[0, :6]) == [127, 0, 2, 2, 0, -2]


def test_v_fp8_per_channel():
    rng = np.random.default_rng(5)
    v = np.float16(rng.standard_normal((200, 64)) * rng.uniform(0.01, 20, 64)).astype(np.float64)
    q = oracle.quant_v(v)
    amax = np.abs(v).max(axis=0).astype(np.float32)
    assert np.array_equal(q.scales, amax / np.float32(448))
    deq = oracle.e4m3_decode(q.codes).astype(np.float64) * q.scales[None, :]
    # E4M3 keeps 3 fraction bits: relative error <= 2^-4 for normal codes,
    # absolute <= 2^-10 * delta for subnormal codes
    err = np.abs(deq - v)
    assert np.all(err <= np.maximum(np.abs(v) * 2 ** -4, 2 ** -10 * q.scales[None, :]) * 1.0001)
    # the channel maximum lands exactly on +-448
    idx = np.argmax(np.abs(v), axis=0)
    assert np.all(np.abs(oracle.e4m3_decode(q.codes[idx, np.arange(64)])) == 448.0)


def test_scores_int32_match_integer_matmul():
    rng = np.random.default_rng(6)
    a = rng.integers(-127, 128, (70, 128), dtype=np.int8)
    b = rng.integers(-127, 128, (90, 128), dtype=np.int8)
    ref = a.astype(np.int64) @ b.astype(np.int64).T
    assert np.array_equal(oracle.scores_int32(a, b), ref.astype(np.int32))


# ----------------------------------------------------------------------------- attention
def _sdpa64(q, k, v, causal, scale, layout="HND"):
    q, k, v = (t.double() for t in (q, k, v))
    if layout == "NHD":
        q, k, v = (t.transpose(1, 2) for t in (q, k, v))
    rep = q.shape[1] // k.shape[1]
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=scale)
    if layout == "NHD":
        o = o.transpose(1, 2)
    return o.numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("layout", ["HND", "NHD"])
def test_exact_attention_matches_torch_sdpa(causal, layout):
    sp = synth.Spec("t", Hq=4, Hkv=2, D=64, B=2, S=200, layout=layout, causal=causal, seed=11)
    q, k, v = synth.make(sp)
    ours = oracle.attention_exact(q, k, v, layout, causal)
    ref = _sdpa64(q, k, v, causal, 1.0 / math.sqrt(64), layout)
    # oracle passes the float32 default scale; allow for that rounding only
    assert np.allclose(ours, ref, rtol=1e-6, atol=1e-7)


def _accuracy(out, ref):
    o, r = out.ravel(), ref.ravel()
    cos = float(o @ r / (np.linalg.norm(o) * np.linalg.norm(r)))
    rl1 = float(np.abs(o - r).sum() / np.abs(r).sum())
    return cos, rl1


@pytest.mark.parametrize("gran", ["per_block", "per_warp", "per_thread"])
@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_quantized_attention_accuracy_tiny_config(gran, pv):
    sp = synth.CONFIGS["tiny"]
    q, k, v = synth.make(sp)
    out = oracle.attention(q, k, v, gran=gran, pv=pv)
    ref = oracle.attention_exact(q, k, v)
    cos, rl1 = _accuracy(out, ref)
    # 16-bit P~V: the INT8 QK^T error alone, well inside rel-L1 0.02.
    # FP8 P~V: E4M3 keeps 3 fraction bits, so each of P~ and V carries ~2.5 %
    # RMS relative rounding error (uniform error over steps of 2^-4..2^-3 of
    # the value); the output, a zero-mean weighted sum, inherits it: ~3.5 %
    # rel-L1 for both operands together, whatever the implementation.
    assert cos >= 0.999, cos
    assert rl1 <= (0.02 if pv == "fp16" else 0.045), rl1


def test_smoothing_k_is_what_keeps_outlier_channels_accurate():
    # K with strong per-channel offsets: without smoothing the INT8 grid is
    # spent on the offset; with it the error drops by a large factor.
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=256, k_bias_std=30.0, seed=13)
    q, k, v = synth.make(sp)
    ref = oracle.attention_exact(q, k, v)
    _, e_s = _accuracy(oracle.attention(q, k, v, smooth_k=True), ref)
    _, e_n = _accuracy(oracle.attention(q, k, v, smooth_k=False), ref)
    assert e_s * 3 < e_n, (e_s, e_n)


def test_smooth_q_keeps_attention_and_helps_offset_queries():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=256, q_block_offset_std=8.0, seed=14)
    q, k, v = synth.make(sp)
    ref = oracle.attention_exact(q, k, v)
    cos, rl1 = _accuracy(oracle.attention(q, k, v, smooth_q=True), ref)
    assert cos >= 0.999 and rl1 <= 0.045          # FP8 P~V bound, see above
    _, e_plain = _accuracy(oracle.attention(q, k, v, smooth_q=False), ref)
    assert rl1 < e_plain


def test_k_shift_leaves_exact_attention_unchanged():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=200, k_bias_std=3.0, seed=15)
    q, k, v = synth.make(sp)
    ks = (k.double() - k.double().mean(dim=2, keepdim=True))
    a = oracle.attention_exact(q, k, v)
    b = oracle.attention_exact(q.double(), ks, v.double())
    assert np.max(np.abs(a - b)) < 1e-12


def test_softmax_rows_sum_to_one():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=200, seed=16)
    q, k, _ = synth.make(sp)
    ones = torch.ones(1, 2, 200, 64, dtype=torch.float16)
    for causal in (False, True):
        assert np.max(np.abs(oracle.attention_exact(q, k, ones, causal=causal) - 1.0)) < 1e-13
        assert np.max(np.abs(oracle.attention(q, k, ones, causal=causal, pv="fp16") - 1.0)) < 1e-3


def test_constant_v_gives_the_constant():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=300, seed=17)
    q, k, _ = synth.make(sp)
    v0 = torch.linspace(-3, 3, 64, dtype=torch.float16)
    v = v0.view(1, 1, 1, 64).expand(1, 2, 300, 64).contiguous()
    out = oracle.attention(q, k, v, pv="fp8")
    ref = v0.double().numpy()
    # every V code is +-448, so out = v0 * (sum P8 / 448) / l with l the sum of
    # the unrounded P~: within one E4M3 step (2^-4 relative) of v0
    assert np.all(np.abs(out - ref) <= np.abs(ref) * 2 ** -4 + 1e-12)
    # and the same ratio (sum P8 / 448) / l multiplies every channel of a row
    ratio = out[..., -1:] / ref[-1]
    assert np.allclose(out, ratio * ref, rtol=1e-6, atol=1e-9)


def test_equal_scores_give_the_mean_of_v():
    # Q = 0 -> every score is 0 -> P~ = 1 -> P8 = 448 exactly.  V values on
    # the E4M3 grid of their channel scale dequantize exactly, so the output
    # is the plain mean of V over the keys.
    S, D = 256, 64
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(0)).half()
    # x * 448 lies on the E4M3 grid for each of these (448, 224, 112, 56)
    vals = torch.tensor([1.0, -1.0, 0.5, 0.0, -0.25, 0.125], dtype=torch.float16)
    idx = torch.randint(0, 6, (S, D), generator=torch.Generator().manual_seed(1))
    v = vals[idx].view(1, 1, S, D).clone()
    v[0, 0, 0, :] = 1.0                      # channel max = 1 -> scale 1/448
    out = oracle.attention(q, k, v, pv="fp8")
    # (the stored scale is float32(1/448), hence the 1e-6)
    assert np.max(np.abs(out[0, 0] - v[0, 0].double().mean(dim=0).numpy())) < 1e-6


def test_causal_rows_ignore_future_keys():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=300, causal=True, seed=18)
    q, k, v = synth.make(sp)
    # exact path: arbitrary new future keys/values leave rows < 150 unchanged
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 150:] = torch.randn(1, 2, 150, 64, generator=torch.Generator().manual_seed(3)).half()
    v2[:, :, 150:] = 7.0
    assert np.max(np.abs(oracle.attention_exact(q, k, v, causal=True)[:, :, :150]
                         - oracle.attention_exact(q, k2, v2, causal=True)[:, :, :150])) == 0
    # quantized path: future tokens reach a row only through the statistics
    # shared along the whole sequence (K mean, V channel max).  Permuting the
    # tokens 150..299 keeps those, so rows whose visible keys all lie in the
    # first 128-key block must come out bit-identical.
    perm = torch.randperm(150, generator=torch.Generator().manual_seed(4)) + 150
    k3, v3 = k.clone(), v.clone()
    k3[:, :, 150:] = k[:, :, perm]
    v3[:, :, 150:] = v[:, :, perm]
    for gran in ("per_block", "per_thread"):
        a = oracle.attention(q, k, v, causal=True, gran=gran)
        b = oracle.attention(q, k3, v3, causal=True, gran=gran)
        assert np.array_equal(a[:, :, :128], b[:, :, :128])
        assert not np.array_equal(a[:, :, 150:], b[:, :, 150:])


def test_gqa_equals_mha_with_repeated_kv():
    sp = synth.Spec("t", Hq=4, Hkv=2, D=64, B=1, S=200, seed=19)
    q, k, v = synth.make(sp)
    a = oracle.attention(q, k, v)
    b = oracle.attention(q, k.repeat_interleave(2, dim=1), v.repeat_interleave(2, dim=1))
    assert np.array_equal(a, b)


def test_varlen_equals_dense_per_sequence():
    sp = synth.Spec("t", Hq=4, Hkv=2, D=64, seqlens=[130, 77, 256], causal=True, seed=20)
    q, k, v = synth.make(sp)
    cu = sp.cu_seqlens()
    a = oracle.attention(q, k, v, causal=True, cu_seqlens=cu)
    for b in range(3):
        s0, s1 = cu[b], cu[b + 1]
        d = oracle.attention(*(t[s0:s1].transpose(0, 1).unsqueeze(0) for t in (q, k, v)),
                             causal=True)
        assert np.array_equal(a[s0:s1], d[0].transpose(1, 0, 2))


def test_layouts_agree():
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=2, S=150, layout="NHD", seed=21)
    q, k, v = synth.make(sp)
    a = oracle.attention(q, k, v, layout="NHD")
    b = oracle.attention(*(t.transpose(1, 2).contiguous() for t in (q, k, v)), layout="HND")
    assert np.array_equal(a, b.transpose(0, 2, 1, 3))


def test_row_subset_matches_full():
    sp = synth.Spec("t", Hq=1, Hkv=1, D=64, B=1, S=300, seed=22)
    q, k, v = synth.make(sp)
    full = oracle.attention(q, k, v)
    part = oracle.attention(q, k, v, q_rows={(0, 0): (128, 256)})
    assert np.array_equal(part[0, 0, 128:256], full[0, 0, 128:256])
    assert np.all(part[0, 0, :128] == 0)


# ----------------------------------------------------------------------------- ambiguity allowance
def test_ambiguous_rounding_steps():
    L = oracle.lib()
    rel = 2.0 ** -19
    # E4M3 neighbours 416 and 448 have midpoint 432; 112 and 120 have 116
    assert L.orc_e4m3_alt_step(432.0, rel) == 32.0
    assert L.orc_e4m3_alt_step(432.0 * (1 + 2 ** -20), rel) == 32.0
    assert L.orc_e4m3_alt_step(432.0 * (1 + 2 ** -18), rel) == 0.0      # outside the band
    assert L.orc_e4m3_alt_step(116.0 * (1 - 2 ** -20), rel) == 8.0
    assert L.orc_e4m3_alt_step(116.0 * (1 - 2 ** -18), rel) == 0.0
    assert L.orc_e4m3_alt_step(430.0, rel) == 0.0
    assert L.orc_e4m3_alt_step(448.0, rel) == 0.0              # saturated: no neighbour above
    assert L.orc_e4m3_alt_step(2.0 ** -10, rel) == 2.0 ** -9   # subnormal tie 0 / 2^-9
    # fp16: 1 and 1 + 2^-10 (midpoint 1 + 2^-11); below 1 the spacing halves
    assert L.orc_h16_alt_step(1 + 2 ** -11, 0, rel) == 2.0 ** -10
    assert L.orc_h16_alt_step(1 - 2 ** -12, 0, rel) == 2.0 ** -11
    assert L.orc_h16_alt_step(0.7, 0, rel) == 0.0
    assert L.orc_h16_alt_step(2.0 ** -25, 0, rel) == 2.0 ** -24        # fp16 tie 0 / smallest subnormal
    # bf16: 7 fraction bits
    assert L.orc_h16_alt_step(1 + 2 ** -8, 1, rel) == 2.0 ** -7


def _r32(x):
    """Exact rational x rounded to the nearest float32 (ties to even), as a
    Fraction: an independent statement of float32 rounding for the test."""
    from fractions import Fraction
    x = Fraction(x)
    if x == 0:
        return x
    sgn = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, -126)
    scaled = a / Fraction(2) ** (e - 23)          # 24-bit significand units
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sgn * n * Fraction(2) ** (e - 23)


@pytest.mark.parametrize("fold,tau", [(1, 0), (1, 2), (0, 0)])
def test_p_band_covers_float32_kernel_arithmetic(fold, tau):
    """The derived band against a brute-force emulation of a kernel that holds
    S*c exact in one fused multiply-add, folds float(log2 448) (+ tau) into the
    subtracted maximum with float32 roundings, rounds the exponent once and
    evaluates 2^x with relative error up to +-2^-22 (both extremes tried).
    Every emulated P~ must lie within orc_p_band of the oracle's exact value;
    the band must also not be loose by more than a small factor."""
    from fractions import Fraction
    L = oracle.lib()
    rng = np.random.default_rng(41)
    L8 = float(np.float32(6.0 + math.log2(7.0)))
    worst = 0.0
    for it in range(3000):
        S = int(rng.integers(-2 ** 21, 2 ** 21))
        c = float(np.float32(abs(rng.normal()) * 10.0 ** rng.uniform(-6, -3)))
        sf = float(_r32(Fraction(S) * Fraction(c)))
        m = sf + float(np.float32(abs(rng.normal()) * 10.0 ** rng.uniform(-3, 1.3)))
        m = float(np.float32(m))
        if fold:
            nb = -_r32(_r32(Fraction(m) - Fraction(L8)) + tau)
            ref = 2.0 ** (sf - m + 6.0 + math.log2(7.0) - tau)
        else:
            nb = -Fraction(m)
            ref = 2.0 ** (sf - m)
        arg = float(_r32(Fraction(S) * Fraction(c) + nb))
        band = L.orc_p_band(sf, m, fold, tau, 0.0)
        for eps in (-2.0 ** -22, 2.0 ** -22):
            yk = 2.0 ** arg * (1 + eps)
            d = abs(yk / ref - 1)
            assert d <= band, (S, c, m, d, band)
            worst = max(worst, d / band)
    assert worst > 0.25, worst


def test_p_band_size():
    """At the magnitudes of typical scores (|s|, |m| < 8) the band is about
    2^-20.5; it grows with the scores' magnitude (their float32 ulps)."""
    L = oracle.lib()
    b = L.orc_p_band(3.0, 5.5, 1, 0, 0.0)
    assert 2.0 ** -21.5 < b < 2.0 ** -20, math.log2(b)
    assert L.orc_p_band(300.0, 305.5, 1, 0, 0.0) > 8 * b
    # a P~*448 value 2^-22 off a midpoint is ambiguous, one 2^-19 off is not
    assert L.orc_e4m3_alt_step(432.0 * (1 + 2 ** -22), b) == 32.0
    assert L.orc_e4m3_alt_step(432.0 * (1 + 2 ** -19), b) == 0.0


def test_allowance_zero_when_no_rounding_is_ambiguous():
    S, D = 256, 64
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)          # every P~ = 1 -> 448, exact
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(0)).half()
    v = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(1)).half()
    _, allow = oracle.attention(q, k, v, with_allowance=True)
    assert np.all(allow == 0)


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_allowance_is_sparse_and_bounded(pv):
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=512, causal=True, seed=23)
    q, k, v = synth.make(sp)
    out, allow = oracle.attention(q, k, v, causal=True, pv=pv, with_allowance=True)
    assert np.all(allow >= 0)
    # E4M3 steps are 2^-4..2^-3 relative and the band ~2^-20.5, so few P~
    # fall in it; 16-bit steps are 2^-10 relative, each flip tiny
    if pv == "fp8":
        assert np.mean(allow > 0) < 0.05
    else:
        assert np.max(allow) < 1e-3
    # a single ambiguous P~ moves an output by at most one rounding step of
    # that P~ times |v| / l; l >= 1 (the row maximum contributes P~ = 1)
    step = 32.0 / 448 if pv == "fp8" else 2 ** -11
    vmax = float(v.abs().max())
    assert np.max(allow) <= 512 * step * vmax


def test_allowance_within_gate_on_the_tiny_workload():
    """On the tiny workload (and the non-causal D=64 S=256 case) the
    allowance stays far below the 2e-3 gate."""
    sp = synth.CONFIGS["tiny"]
    q, k, v = synth.make(sp)
    _, allow = oracle.attention(q, k, v, with_allowance=True)
    assert np.max(allow) < 2e-3 and np.mean(allow > 0) < 0.05, (np.max(allow), np.mean(allow > 0))


# ----------------------------------------------------------------------------- identity quantizers
@pytest.mark.parametrize("tau", [0, 1, 2, 8, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_identity_quantizers_equal_exact_attention(tau, causal):
    """The quantized routine's own loop with its identity-quantizer switch
    (unquantized fp64 scores, P~ and V): with the tiling removed it is softmax
    attention, so it must equal the one-pass fp64 reference -- for the plain
    online softmax and for the conditional-rescaling bookkeeping, for any tau
    (1000: the reference never moves after the first tile)."""
    sp = synth.Spec("t", Hq=2, Hkv=2, D=64, B=1, S=333, causal=causal, k_bias_std=3.0, seed=13)
    q, k, v = synth.make(sp)
    pb = oracle.problem(q, k, v)
    sc = oracle.default_scale(64, None)
    for h in range(2):
        a = oracle.attn_exact_head(pb.q[0][h], pb.k[0][h], pb.v[0][h], causal, sc)
        b = oracle.attn_tiled_fp64_head(pb.q[0][h], pb.k[0][h], pb.v[0][h], causal, sc, lazy_tau=tau)
        assert np.max(np.abs(a - b)) < 1e-12


def test_identity_quantizers_whole_problem():
    sp = synth.Spec("t", Hq=4, Hkv=2, D=64, B=2, S=300, causal=True, k_bias_std=3.0, seed=12)
    q, k, v = synth.make(sp)
    a = oracle.attention_exact(q, k, v, "HND", True)
    b = oracle.attention_exact(q, k, v, "HND", True, tiled=True)
    assert np.max(np.abs(a - b)) < 1e-12


# ----------------------------------------------------------------------------- fp32+fp16 accumulation
def test_fp16_accumulation_closed_form_chunk_rounding():
    """Q = 0 makes every P~ 1 (E4M3 code of 1.0 with the scale-1 reading).
    V holds E4M3 integers with channel maximum 448, so V's scale is 1 and its
    codes are V itself.  Each 32-key chunk's sum is then an integer, and the
    binary16 partial of the tile is the chain of round-to-nearest-even
    additions, computed here with numpy's float16."""
    S, D = 128, 64
    rng = np.random.default_rng(42)
    vals = np.array([448, 416, 352, 320, 13, 11, 9, 7, 3, 1, 0, -1, -5, -15, -448], np.float64)
    vv = vals[rng.integers(0, len(vals), (S, D))]
    vv[0, :] = 448.0
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(2)).half()
    v = torch.from_numpy(vv.astype(np.float16)).view(1, 1, S, D)
    out = oracle.attention(q, k, v, pv="fp8", acc="fp32+fp16")
    expect = np.zeros(D)
    for c in range(D):
        acc = np.float16(0)
        for c0 in range(0, S, 32):
            acc = np.float16(float(acc) + float(vv[c0:c0 + 32, c].sum()))
        expect[c] = float(acc) / S
    np.testing.assert_array_equal(out[0, 0, 0], expect)
    assert not np.array_equal(expect, vv.mean(axis=0))      # the rounding is visible


def test_fp16_accumulation_exact_when_partials_representable():
    """V values whose codes are multiples of 8 with partial sums below 2^14
    are exact in binary16: the result is the plain mean of V."""
    S, D = 256, 64
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(0)).half()
    vals = torch.tensor([0.125, -0.125, 0.25, 0.0], dtype=torch.float16)
    idx = torch.randint(0, 4, (S, D), generator=torch.Generator().manual_seed(1))
    v = vals[idx].view(1, 1, S, D).clone()
    v[0, 0, 0, :] = 1.0
    out = oracle.attention(q, k, v, pv="fp8", acc="fp32+fp16")
    assert np.max(np.abs(out[0, 0] - v[0, 0].double().mean(dim=0).numpy())) < 1e-6


def test_fp16_accumulation_no_overflow_at_the_bound():
    """The largest tile partial the scale-1 reading allows, 128 keys of P~ = 1
    times the code 448, is 57344 <= 65504: no overflow, output = V."""
    S, D = 128, 64
    q = torch.zeros(1, 1, S, D, dtype=torch.float16)
    k = torch.randn(1, 1, S, D, generator=torch.Generator().manual_seed(0)).half()
    v = torch.full((1, 1, S, D), 3.0, dtype=torch.float16)
    out, allow = oracle.attention(q, k, v, pv="fp8", acc="fp32+fp16", with_allowance=True)
    assert np.all(np.isfinite(out)) and np.allclose(out, 3.0, rtol=1e-6)


def test_fp16_accumulation_accuracy_and_allowance():
    """Against exact attention the binary16 inner level keeps cosine >= 0.999;
    its difference from the exact per-tile sums stays inside the allowance
    the oracle reports for it."""
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=1024, k_bias_std=3.0, seed=43)
    q, k, v = synth.make(sp)
    ex = oracle.attention_exact(q, k, v)
    o16, a16 = oracle.attention(q, k, v, pv="fp8", acc="fp32+fp16", with_allowance=True)
    cos, rl1 = _accuracy(o16, ex)
    assert cos >= 0.999, cos
    assert rl1 <= 0.06, rl1
    assert np.all(a16 > 0) and np.max(a16) < 2e-3, np.max(a16)


# ----------------------------------------------------------------------------- smooth V
def test_smooth_v_constant_channels_are_exact():
    """Smooth V with V constant per channel: V - mean is exactly 0, so every
    code and scale is 0 and the output is the mean itself, exactly."""
    rng = np.random.default_rng(21)
    B, H, S, D = 1, 2, 200, 64
    q = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    k = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    v0 = rng.standard_normal((1, H, 1, D)).astype(np.float16)
    v = torch.from_numpy(np.broadcast_to(v0, (B, H, S, D)).copy())
    pb = oracle.problem(q, k, v)
    r = oracle.quant_v(pb.v[0][0], smooth=True, is_fp16=True)
    assert np.all(r.codes == 0) and np.all(r.scales == 0)
    assert np.array_equal(r.mu, v0[0, 0, 0].astype(np.float32))
    out = oracle.attention(q, k, v, pv="fp8", smooth_v=True)
    assert np.array_equal(out, np.broadcast_to(v0.astype(np.float64), out.shape))


def test_smooth_v_reduces_error_on_channel_offsets():
    """The method's purpose: with large per-channel V offsets, FP8 V carries
    the offset's rounding error; smoothing V removes it (reading of the
    page's optional smooth-V step).  Error against exact fp64 attention."""
    rng = np.random.default_rng(22)
    B, H, S, D = 1, 2, 384, 64
    q = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    k = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    v = (rng.standard_normal((B, H, S, D)) + rng.normal(0, 20, (1, H, 1, D))).astype(np.float16)
    v = torch.from_numpy(v)
    ex = oracle.attention_exact(q, k, v)
    plain = oracle.attention(q, k, v, pv="fp8")
    smooth = oracle.attention(q, k, v, pv="fp8", smooth_v=True)
    e_plain = np.abs(plain - ex).mean()
    e_smooth = np.abs(smooth - ex).mean()
    assert e_smooth < 0.5 * e_plain, (e_smooth, e_plain)


# ----------------------------------------------------------------------------- lazy rescaling
def test_lazy_without_moves_equals_plain_16bit():
    """Every row's maximum in the first key tile (K zero except key 0, so all
    later scores are 0 <= that maximum): the reference never moves, and with
    16-bit P~ the lazy result equals the plain online softmax exactly."""
    rng = np.random.default_rng(31)
    B, H, S, D = 1, 2, 300, 64
    q = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    kk = np.zeros((B, H, S, D), np.float16)
    kk[:, :, 0] = rng.standard_normal((B, H, D)) * 3
    k = torch.from_numpy(kk)
    v = torch.from_numpy(rng.standard_normal((B, H, S, D)).astype(np.float16))
    plain = oracle.attention(q, k, v, pv="fp16", smooth_k=False)
    lazy = oracle.attention(q, k, v, pv="fp16", smooth_k=False, lazy_tau=8)
    assert np.array_equal(plain, lazy)


def test_lazy_fp8_accuracy():
    """FP8 P~ with the 448 * 2^-2 scale the lazy mode needs keeps the
    method's accuracy against exact attention."""
    sp = synth.Spec("t", Hq=2, Hkv=2, D=128, B=1, S=1024, k_bias_std=3.0, seed=14)
    q, k, v = synth.make(sp)
    ex = oracle.attention_exact(q, k, v)
    plain = oracle.attention(q, k, v, pv="fp8")
    lazy = oracle.attention(q, k, v, pv="fp8", lazy_tau=2)
    cos_l, rl1_l = _accuracy(lazy, ex)
    cos_p, rl1_p = _accuracy(plain, ex)
    assert cos_l >= 0.999, cos_l
    assert rl1_l <= 1.5 * rl1_p, (rl1_l, rl1_p)


def _cross_problem(seed=3, D=64):
    """Packed q with its own sequence lengths and packed k/v with others:
    longer and shorter key sets, an empty query set, an empty key set."""
    rng = np.random.default_rng(seed)
    H, Hk = 4, 2
    lq, lk = [150, 40, 0, 200, 17], [90, 300, 10, 0, 17]
    cq = np.concatenate([[0], np.cumsum(lq)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lk)]).astype(np.int32)
    q = torch.from_numpy(rng.normal(size=(cq[-1], H, D)).astype(np.float16))
    k = torch.from_numpy((rng.normal(size=(ck[-1], Hk, D)) + rng.normal(0, 3, size=(1, Hk, D))).astype(np.float16))
    v = torch.from_numpy(rng.normal(size=(ck[-1], Hk, D)).astype(np.float16))
    return q, k, v, lq, lk, cq, ck


@pytest.mark.parametrize("causal", [False, True])
def test_cross_length_varlen_pins(causal):
    """Queries and keys with their own sequence boundaries: each sequence
    agrees with exact fp64 attention (cosine >= 0.999); a sequence without
    keys gives zero rows; equal boundaries passed twice change nothing."""
    q, k, v, lq, lk, cq, ck = _cross_problem()
    o = oracle.attention(q, k, v, causal=causal, cu_seqlens=cq, cu_seqlens_k=ck)
    e = oracle.attention_exact(q, k, v, causal=causal, cu_seqlens=cq, cu_seqlens_k=ck)
    for b in range(len(lq)):
        a, x = o[cq[b]:cq[b + 1]].ravel(), e[cq[b]:cq[b + 1]].ravel()
        if a.size == 0:
            continue
        if lk[b] == 0:
            assert np.all(a == 0) and np.all(x == 0)
            continue
        assert a @ x / (np.linalg.norm(a) * np.linalg.norm(x)) >= 0.999
    # same boundaries for both: identical to the single-boundary call
    lq2 = [130, 64, 201]
    cu = np.concatenate([[0], np.cumsum(lq2)]).astype(np.int32)
    rng = np.random.default_rng(4)
    q2, k2, v2 = (torch.from_numpy(rng.normal(size=(cu[-1], 2, 64)).astype(np.float16)) for _ in range(3))
    np.testing.assert_array_equal(oracle.attention(q2, k2, v2, causal=causal, cu_seqlens=cu),
                                  oracle.attention(q2, k2, v2, causal=causal, cu_seqlens=cu, cu_seqlens_k=cu))


def test_cross_length_causal_reduces_to_full_past_the_keys():
    """Causal with fewer keys than queries: from query row Lk - 1 on every
    key is visible, so those rows equal the non-causal rows exactly."""
    q, k, v, lq, lk, cq, ck = _cross_problem(seed=5)
    oc = oracle.attention(q, k, v, causal=True, cu_seqlens=cq, cu_seqlens_k=ck)
    on = oracle.attention(q, k, v, causal=False, cu_seqlens=cq, cu_seqlens_k=ck)
    b = 0                                                   # 150 queries, 90 keys
    assert lk[b] < lq[b]
    np.testing.assert_array_equal(oc[cq[b] + lk[b] - 1:cq[b + 1]], on[cq[b] + lk[b] - 1:cq[b + 1]])
    assert not np.array_equal(oc[cq[b]:cq[b] + lk[b] - 1], on[cq[b]:cq[b] + lk[b] - 1])


def test_cross_length_smooth_v_rows_without_keys_are_zero():
    """Smooth V adds the channel mean back only where there are keys: a
    sequence without keys still gives zero rows, the others stay finite."""
    q, k, v, lq, lk, cq, ck = _cross_problem(seed=6)
    o = oracle.attention(q, k, v, causal=True, cu_seqlens=cq, cu_seqlens_k=ck, smooth_v=True)
    b = lk.index(0)
    assert np.all(o[cq[b]:cq[b + 1]] == 0)
    assert np.all(np.isfinite(o))
