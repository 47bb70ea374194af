"""Host-side checks of the C ABI: the library loads, exports exactly what
include/sage.h declares, plans workspaces, and rejects bad arguments before
launching anything (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest

import quantized_attention_token_b200 as sage
from quantized_attention_token_b200 import build as sage_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    sage_build.build()
    return sage.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "sage.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b(sage_[a-z0-9_]+)\s*\(", src))


def test_exports_match_header(L):
    out = subprocess.run(["nm", "-D", "--defined-only", sage.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("sage_")}
    assert exported == _declared()


def test_workspace_planner(L):
    b = sage.sage_workspace_bytes(2, 32, 32, 4096, 128, 0, 0)
    lay = sage.workspace_layout(2, 8192, 8192, 4096, 32, 32, 128)
    assert b == lay["total"] and lay["tiles_q"] == 64 and lay["tiles_k"] == 64
    # every region 256-byte aligned, tile regions 1024-byte aligned, disjoint and ordered
    keys = ["err", "k_stat", "v_stat", "k_mean", "v_scale", "k_codes", "k_scale", "v_codes", "q_codes", "q_scale"]
    offs = [lay[k] for k in keys]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert all(lay[k] % 1024 == 0 for k in ("k_codes", "v_codes", "q_codes"))
    assert lay["q_codes"] - lay["v_codes"] >= 32 * 64 * 128 * 128 * 2
    assert b >= 32 * 64 * 128 * 128 * 4      # Q and K codes + 16-bit V at least
    # GQA shrinks the K/V part only; Hq does not move the K/V regions
    g = sage.workspace_layout(2, 8192, 8192, 4096, 32, 8, 128)
    assert g["total"] < b
    h = sage.workspace_layout(2, 8192, 8192, 4096, 8, 8, 128)
    assert h["v_codes"] == g["v_codes"] and h["k_codes"] == g["k_codes"]
    # varlen: tiles bounded by total/128 + n
    v = sage.workspace_layout(4, 27648, 27648, 16384, 32, 8, 128, varlen=1)
    assert v["tiles_q"] == 27648 // 128 + 4
    assert sage.sage_varlen_workspace_bytes(4, 27648, 27648, 16384, 32, 8, 128) == v["total"]


@pytest.mark.parametrize("args,expect", [
    (dict(D=96), sage.ERR_UNSUPPORTED),
    (dict(Hkv=5), sage.ERR_UNSUPPORTED),
    (dict(S=0), sage.ERR_INVALID_ARG),
    (dict(q=0), sage.ERR_INVALID_ARG),
    (dict(q=0x1008), sage.ERR_INVALID_ARG),          # misaligned
    (dict(ws=0x1010), sage.ERR_INVALID_ARG),         # ws must be 256-byte aligned
    (dict(gran=7), sage.ERR_INVALID_ARG),
    (dict(pv=3), sage.ERR_INVALID_ARG),
    (dict(acc=4), sage.ERR_INVALID_ARG),
    (dict(acc=3, pv=1), sage.ERR_UNSUPPORTED),       # binary16 inner accumulation needs FP8 P~V
    (dict(layout=2), sage.ERR_INVALID_ARG),
    (dict(dtype=2), sage.ERR_INVALID_ARG),
    (dict(ws_bytes=1000), sage.ERR_WORKSPACE),
    (dict(scale=float("nan")), sage.ERR_INVALID_ARG),
])
def test_attn_fwd_rejects_bad_arguments(L, args, expect):
    a = dict(q=0x10000, k=0x20000, v=0x30000, out=0x40000, dtype=0, B=1, Hq=4, Hkv=2, S=256, D=128, layout=0,
             causal=0, scale=0.0, gran=0, pv=0, acc=1, sk=1, sq=0, ws=0x100000, ws_bytes=1 << 30)
    a.update(args)
    st = L.sage_attn_fwd(a["q"], a["k"], a["v"], a["out"], a["dtype"], a["B"], a["Hq"], a["Hkv"], a["S"], a["D"],
                         a["layout"], a["causal"], a["scale"], a["gran"], a["pv"], a["acc"], a["sk"], a["sq"],
                         a["ws"], a["ws_bytes"], None)
    assert st == expect


def test_valid_arguments_without_a_gpu_report_cuda_error(L):
    # everything validates; the device check then fails on a GPU-less host,
    # and nothing is launched
    import torch
    if torch.cuda.is_available():
        pytest.skip("host has a GPU")
    st = L.sage_attn_fwd(0x10000, 0x20000, 0x30000, 0x40000, 0, 1, 4, 2, 256, 128, 0, 0, 0.0, 0, 0, 1, 1, 0,
                         0x100000, 1 << 30, None)
    assert st in (sage.ERR_CUDA, sage.ERR_UNSUPPORTED)
    if st == sage.ERR_CUDA:        # the runtime's reason is kept for the caller
        assert L.sage_last_cuda_error() != 0
        assert L.sage_last_cuda_error_name().decode().startswith("cudaError")


def test_varlen_rejects_bad_arguments(L):
    base = [0x10000, 0x20000, 0x30000, 0x40000, 0, 0x50000, 0x50100, 4, 1024, 1024, 512, 8, 2, 128, 1, 0.0, 0, 0, 1,
            1, 0x100000, 1 << 30, None]
    assert L.sage_attn_varlen_fwd(*base) in (sage.ERR_CUDA, sage.ERR_UNSUPPORTED)
    bad = list(base); bad[5] = 0
    assert L.sage_attn_varlen_fwd(*bad) == sage.ERR_INVALID_ARG
    bad = list(base); bad[12] = 3
    assert L.sage_attn_varlen_fwd(*bad) == sage.ERR_UNSUPPORTED
    bad = list(base); bad[21] = 4096
    assert L.sage_attn_varlen_fwd(*bad) == sage.ERR_WORKSPACE


def test_debug_settings_validate_and_reset(L):
    assert L.sage_debug_set_max_ctas(-1) == sage.ERR_INVALID_ARG
    assert L.sage_debug_withhold_k_tile(-2) == sage.ERR_INVALID_ARG
    assert L.sage_debug_set_max_ctas(3) == sage.OK and L.sage_debug_set_max_ctas(0) == sage.OK
    assert L.sage_debug_withhold_k_tile(5) == sage.OK and L.sage_debug_withhold_k_tile(-1) == sage.OK
    assert L.sage_debug_set_prepass_one_pass(2) == sage.ERR_INVALID_ARG
    assert L.sage_debug_set_prepass_one_pass(1) == sage.OK and L.sage_debug_set_prepass_one_pass(0) == sage.OK
    assert L.sage_debug_last_prepass_path() in (0, 1, 2)
    assert L.sage_debug_set_out_map(2) == sage.ERR_INVALID_ARG
    assert L.sage_debug_set_out_map(0) == sage.OK and L.sage_debug_set_out_map(1) == sage.OK
    assert L.sage_debug_last_out_path() in (0, 1, 2)


def test_library_reads_no_environment():
    """Behaviour is selected through arguments and the debug entry points
    only: no source of the library reads the process environment."""
    csrc = os.path.join(ROOT, "quantized_attention_token_b200", "csrc")
    for f in os.listdir(csrc):
        src = open(os.path.join(csrc, f)).read()
        assert "getenv" not in src, f


def test_status_strings(L):
    for s in range(6):
        assert L.sage_status_string(s)


def test_varlen_layout_with_separate_query_and_key_tokens(L):
    """Queries and keys with their own token counts: Q tiles follow total_q,
    K/V tiles total_k; the K means, V scales and V means (zeroed before a
    varlen pre-pass, one contiguous range for the V part) sit in that order
    inside the workspace."""
    n, Tq, Tk, mx, Hq, Hkv, D = 6, 707, 677, 300, 4, 2, 128
    lay = sage.workspace_layout(n, Tq, Tk, mx, Hq, Hkv, D, varlen=1)
    assert lay["tiles_q"] <= Tq // 128 + n and lay["tiles_k"] <= Tk // 128 + n
    assert lay["tiles_q"] >= -(-Tq // 128) and lay["tiles_k"] >= -(-Tk // 128)
    nd = n * Hkv * D
    assert lay["k_mean"] + 4 * nd <= lay["v_scale"] and lay["v_scale"] + 4 * nd <= lay["v_mean"]
    assert lay["v_mean"] + 4 * nd <= lay["total"]
    assert sage.sage_varlen_workspace_bytes(n, Tq, Tk, mx, Hq, Hkv, D) == lay["total"]
    more_k = sage.workspace_layout(n, Tq, 4 * Tk, mx, Hq, Hkv, D, varlen=1)
    assert more_k["tiles_q"] == lay["tiles_q"] and more_k["tiles_k"] > lay["tiles_k"]
