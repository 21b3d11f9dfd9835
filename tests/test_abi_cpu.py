"""The C-ABI library on the CPU: it builds, loads, exports every declared symbol,
and its host-side logic (capacity, workspace sizing, argument validation)
behaves as documented.  No kernel is launched here."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    swl_build.build()
    return swl.lib()


def _declared():
    txt = open(os.path.join(ROOT, "include", "switch_layer.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(switch_layer_\w+)\s*\(", txt)))


def test_exports_every_declared_symbol(L):
    decl = _declared()
    assert decl == sorted(swl.EXPORTS)
    for name in decl:
        assert hasattr(L, name), name
    assert L.switch_layer_stage_name(0).decode() == "router_logits"
    assert L.switch_layer_stage_name(swl.SWL_NUM_STAGES) is None


def test_capacity_matches_oracle(L):
    rng = np.random.default_rng(0)
    for _ in range(3000):
        T = int(rng.integers(0, 1 << 20))
        N = int(rng.integers(1, 5000))
        cf = float(rng.choice([0.1, 0.25, 1.0, 1.1, 1.25, 2.0, 3.3])) * float(rng.uniform(0.5, 2))
        assert swl.switch_layer_capacity(T, N, cf) == oracle.capacity(T, N, cf), (T, N, cf)
    for T, N, cf, C in ((64, 4, 1.0, 16), (4096, 64, 1.25, 80), (16384, 128, 1.0, 128),
                        (32768, 64, 2.0, 1024), (65536, 2048, 1.0, 32), (10, 4, 1.0, 3),
                        (1, 1000, 1e-300, 1)):
        assert swl.switch_layer_capacity(T, N, cf) == C
    for bad in ((5, 0, 1.0), (-1, 3, 1.0), (5, 3, 0.0), (5, 3, -2.0), (5, 3, math.inf),
                (5, 3, math.nan)):
        assert swl.switch_layer_capacity(*bad) == -1
    assert swl.switch_layer_capacity(1 << 30, 1, 1e300) == 2 ** 63 - 1   # saturates


def test_workspace_size_and_validation(L):
    n = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
    # the packed expert input / hidden buffers dominate
    assert n >= 4096 * (768 + 3072) * 2
    n2 = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25,
                                         swl.SWL_WS_HOST_IO)
    assert n2 > n
    for args, code in (((10, 12, 16, 2, swl.SWL_BF16, 1.0), 2),   # d % 8
                       ((10, 16, 12, 2, swl.SWL_BF16, 1.0), 2),   # d_ff % 8
                       ((10, 12, 16, 2, 7, 1.0), 1),               # dtype
                       ((10, 12, 16, 0, 0, 1.0), 1),               # N
                       ((-1, 12, 16, 2, 0, 1.0), 1),               # T
                       ((10, 12, 16, 2, 0, 0.0), 1)):              # cf
        with pytest.raises(swl.SwitchLayerError) as ei:
            swl.switch_layer_workspace_size(*args)
        assert ei.value.status == code
    assert swl.switch_layer_workspace_size(0, 8, 8, 2, swl.SWL_F32, 1.0) > 0


def _fwd_raw(L, T=16, d=8, d_ff=8, N=2, dtype=0, ptr=0x1000, ws=0x10000, ws_bytes=1 << 30,
             null=None, cf=1.0):
    p = [ptr] * 11
    if null is not None:
        p[null] = None
    return L.switch_layer_forward(T, d, d_ff, N, dtype, p[0], p[1], p[2], p[3], p[4], p[5], cf,
                                  p[6], p[7], p[8], p[9], p[10], None, ws, ws_bytes, None)


def test_forward_rejects_bad_arguments_without_launching(L):
    before = L.switch_layer_launch_count()
    for i in range(11):
        assert _fwd_raw(L, null=i) == 1
    assert _fwd_raw(L, ws=None) == 1
    assert _fwd_raw(L, ws_bytes=16) == 3                       # workspace too small
    assert _fwd_raw(L, ws=0x10010) == 2                         # workspace not 256-B aligned
    assert _fwd_raw(L, dtype=1, ptr=0x1002) == 2                # bf16 needs 16-B aligned rows
    assert _fwd_raw(L, d=12, dtype=1) == 2                      # bf16 d % 8
    assert _fwd_raw(L, cf=-1.0) == 1
    assert _fwd_raw(L, T=-3) == 1
    assert L.switch_layer_launch_count() == before
    assert L.switch_layer_forward_timed(16, 8, 8, 2, 0, *([0x1000] * 6), 1.0, *([0x1000] * 5),
                                        None, 0x10000, 1 << 30, None, None) == 1
    assert swl.switch_layer_status_string(3) == "workspace too small"


def test_router_mode_switch(L):
    assert swl.switch_layer_router_mode() == swl.SWL_ROUTER_TENSOR
    n_tensor = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_FFMA)
    try:
        assert swl.switch_layer_router_mode() == swl.SWL_ROUTER_FFMA
        n_ffma = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
        # the tensor-core router keeps the three bf16 pieces of W_r in the workspace
        assert n_tensor - n_ffma >= 3 * 64 * 768 * 2
        # fp32 layers use the FFMA router in both modes
        assert (swl.switch_layer_workspace_size(64, 32, 64, 4, swl.SWL_F32, 1.0) ==
                swl.switch_layer_workspace_size(64, 32, 64, 4, swl.SWL_F32, 1.0))
    finally:
        swl.switch_layer_set_router_mode(swl.SWL_ROUTER_TENSOR)
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.switch_layer_set_router_mode(7)
    assert ei.value.status == 1
    assert swl.switch_layer_router_mode() == swl.SWL_ROUTER_TENSOR


# Each GPU parity case is named for the kernel variant it exercises; the host's
# plan (host logic only, no device) confirms that the shape takes that variant.
_PLAN_CASES = [
    # workloads
    ("base_T4096_d768_N64", None, {"router": "tc", "ksplit": 4, "router_stages": 4,
                                   "dispatch": "fused", "ffn": "sm100", "accumulators": 4,
                                   "gemm2_split": 1}),
    ("large_T16384_d1024_N128", None, {"router": "tc", "ksplit": 1, "router_stages": 3,
                                       "dispatch": "two_kernel", "tile_rows": 128,
                                       "accumulators": 4}),
    ("skewed_T32768_d2048_N64", None, {"router": "tc", "ksplit": 1, "router_stages": 2,
                                       "dispatch": "two_kernel", "tile_rows": 256,
                                       "accumulators": 2, "gemm2_split": 4}),
    ("many_T65536_d1024_N2048", None, {"router": "tc_wide", "softmax": "stream",
                                       "dispatch": "two_kernel", "tokens_per_block": 111}),
    ("tiny_f32_T64_d32_N4", None, {"router": "ffma_warpsplit", "ffn": "f32", "dispatch": "fused"}),
    # test_kernel_variant_shapes
    ("tc_np96_s4", (1000, 1024, 256, 80, 1.25, "bf16"), {"router": "tc", "ksplit": 4}),
    ("tc_np128_s2", (2000, 256, 128, 128, 1.25, "bf16"), {"router": "tc", "ksplit": 2}),
    ("tc_wide_ragged", (700, 256, 128, 200, 2.0, "bf16"), {"router": "tc_wide",
                                                            "softmax": "stream"}),
    ("tc_wide_rows", (500, 128, 64, 202, 2.0, "bf16"), {"router": "tc_wide",
                                                         "softmax": "rows"}),
    ("tc_wide_threepass", (300, 64, 64, 2100, 8.0, "bf16"), {"router": "tc_wide",
                                                              "softmax": "wide"}),
    ("ffma_wide", (300, 48, 40, 150, 2.0, "f32"), {"router": "ffma_wide", "softmax": "rows"}),
    ("ffma_tile", (25700, 32, 32, 48, 1.0, "f32"), {"router": "ffma_tile"}),
    ("two_kernel_dispatch", (20000, 256, 32, 8, 1.0, "f32"), {"dispatch": "two_kernel"}),
    ("two_accumulators", (900, 64, 64, 4, 1.0, "bf16"), {"ffn": "sm100", "accumulators": 2}),
    ("gemm2_split_mixed", (12288, 768, 4096, 8, 1.0, "bf16"),
     {"dispatch": "two_kernel", "tile_rows": 256, "gemm2_split": 4}),
    # streaming softmax: token blocks sized so every persistent CTA takes as many
    ("stream_full_warp_row", (6600, 128, 64, 1024, 2.0, "bf16"),
     {"router": "tc_wide", "softmax": "stream", "tokens_per_block": 45}),
    ("stream_pair_ragged", (5400, 128, 64, 1500, 2.0, "bf16"),
     {"router": "tc_wide", "softmax": "stream", "tokens_per_block": 37}),
    # test_router_bias_paths
    ("tc_s1_bias_padded", (6000, 128, 64, 50, 1.25, "bf16"),
     {"router": "tc", "ksplit": 1, "router_stages": 4}),
    ("tc_s1_two_per_sm", (20000, 256, 64, 50, 1.25, "bf16"),
     {"router": "tc", "ksplit": 1, "router_stages": 2}),
    ("tc_s2_bias_np128", (3000, 256, 64, 100, 1.0, "bf16"), {"router": "tc", "ksplit": 2}),
    ("tc_s4_bias_padded", (1000, 1024, 64, 40, 1.25, "bf16"), {"router": "tc", "ksplit": 4}),
    ("tc_wide_stream_bias", (3000, 256, 64, 300, 1.25, "bf16"),
     {"router": "tc_wide", "softmax": "stream"}),
]


@pytest.mark.parametrize("case", _PLAN_CASES, ids=lambda c: c[0])
def test_parity_cases_take_their_kernel_variant(case):
    name, shape, want = case
    if shape is None:
        w = synth.WORKLOADS[name]
        shape = (w.T, w.d, w.d_ff, w.N, w.cf, w.dtype)
    T, d, d_ff, N, cf, dt = shape
    code = swl.SWL_BF16 if dt == "bf16" else swl.SWL_F32
    plan = swl.switch_layer_describe_plan(T, d, d_ff, N, code, cf, num_sms=148)
    assert {k: plan[k] for k in want} == want, plan


def test_describe_plan_router_mode_and_errors(L):
    base = (4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_FFMA)
    try:
        plan = swl.switch_layer_describe_plan(*base)
        assert plan["router"].startswith("ffma_") and plan["router_stages"] == 0
    finally:
        swl.switch_layer_set_router_mode(swl.SWL_ROUTER_TENSOR)
    # fewer SMs than one-CTA router tiles: two stages per CTA (two CTAs per SM)
    assert swl.switch_layer_describe_plan(16384, 1024, 64, 64, swl.SWL_BF16, 1.25,
                                          num_sms=100)["router_stages"] == 2
    assert swl.switch_layer_describe_plan(16384, 1024, 64, 64, swl.SWL_BF16, 1.25,
                                          num_sms=148)["router_stages"] == 4
    small = ctypes.create_string_buffer(8)
    assert L.switch_layer_describe_plan(*base, 148, small, len(small)) == 1   # too small
    big = ctypes.create_string_buffer(256)
    assert L.switch_layer_describe_plan(*base, 0, big, len(big)) == 1         # no SMs
    assert L.switch_layer_describe_plan(*base, 148, None, 256) == 1           # no buffer
    assert L.switch_layer_describe_plan(4096, 0, 3072, 64, swl.SWL_BF16, 1.25, 148, big,
                                        len(big)) == 1                         # d = 0
    assert L.switch_layer_describe_plan(4096, 764, 3072, 64, swl.SWL_BF16, 1.25, 148, big,
                                        len(big)) != 0                         # d % 8 != 0


def test_checked_build_exports_the_same_symbols():
    """The range-checked variant (SWL_CHECKED) builds and exports every symbol
    the header declares."""
    import ctypes
    path = swl_build.build(checked=True)
    assert path.endswith("libswitchlayer_checked.so")
    L2 = ctypes.CDLL(path)
    for name in swl.EXPORTS:
        assert hasattr(L2, name), name


def test_top2_workspace_and_validation(L):
    """Top-2 workspaces hold twice the packed rows plus the per-assignment output
    rows; one expert, or top-2 beyond 2048 experts, is refused on the host."""
    import ctypes
    n1 = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
    n2 = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25, swl.SWL_WS_TOP2)
    assert n2 > n1 + 4096 * (768 + 3072 + 768) * 2
    n = ctypes.c_size_t(0)
    assert L.switch_layer_workspace_size(64, 32, 32, 1, swl.SWL_BF16, 1.0, swl.SWL_WS_TOP2,
                                         ctypes.byref(n)) == 1
    assert L.switch_layer_workspace_size(64, 32, 32, 4096, swl.SWL_BF16, 1.0, swl.SWL_WS_TOP2,
                                         ctypes.byref(n)) == 2
    assert L.switch_layer_workspace_size(64, 32, 32, 4, swl.SWL_BF16, 1.0,
                                         swl.SWL_WS_TOP2 | swl.SWL_WS_HOST_IO,
                                         ctypes.byref(n)) == 1


def test_ntlb_workspace_and_validation(L):
    """No-Token-Left-Behind workspaces hold one packed row per token (not two),
    the top-2 router's block arrays and the stage-2 scratch; the flag combines
    with no other; one expert is refused."""
    import ctypes
    n1 = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25)
    n2 = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25, swl.SWL_WS_TOP2)
    nn = swl.switch_layer_workspace_size(4096, 768, 3072, 64, swl.SWL_BF16, 1.25, swl.SWL_WS_NTLB)
    assert n1 < nn < n2
    n = ctypes.c_size_t(0)
    for flags in (swl.SWL_WS_NTLB | swl.SWL_WS_TOP2, swl.SWL_WS_NTLB | swl.SWL_WS_HOST_IO, 8):
        assert L.switch_layer_workspace_size(64, 32, 32, 4, swl.SWL_BF16, 1.0, flags,
                                             ctypes.byref(n)) == 1, flags
    assert L.switch_layer_workspace_size(64, 32, 32, 1, swl.SWL_BF16, 1.0, swl.SWL_WS_NTLB,
                                         ctypes.byref(n)) == 1
