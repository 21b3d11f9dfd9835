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
