"""switch_layer_forward_noalloc: the forward pass for callers that cannot call
cudaMalloc (code inside a host framework that owns all device memory, or a
latency-critical loop that must not allocate).  Its scratch is a fixed static
device array inside the library, so these checks run it through the C ABI and
compare it with switch_layer_forward, which uses a caller-provided workspace,
on two calls in a row (the second call reuses the array's old contents).

This file is collected last so that a failure here does not hide the other
tests in a run that stops at the first failure.
"""
import ctypes

import pytest
import torch

import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    return swl.lib()


def _noalloc(L, ig, cf, o):
    x, W1 = ig["x"], ig["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    p = lambda t: None if t is None else t.data_ptr()
    return L.switch_layer_forward_noalloc(
        T, d, d_ff, N, swl.dtype_code(x.dtype), p(x), p(ig["W_r"]), p(W1), p(ig["b1"]),
        p(ig["W2"]), p(ig["b2"]), float(cf), p(o["out"]), p(o["expert_idx"]), p(o["gate"]),
        p(o["pos_in_expert"]), p(o["aux_loss"]), p(ig.get("b_r")),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("name", ["tiny_f32_T64_d32_N4", "base_T4096_d768_N64"])
def test_noalloc_matches_workspace_entry_point(L, name):
    spec = synth.WORKLOADS[name]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(name))
    ref = swl.forward(ig, spec.cf)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream().cuda_stream
    outs = [swl.alloc_outputs(spec.T, spec.d, ig["x"].dtype) for _ in range(2)]
    for call in range(2):
        o = outs[call]
        for k in o:
            o[k].fill_(7)                       # stale values must be overwritten
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the results are bit-identical to
        # the workspace entry point's (a fortiori within the tests' tolerance)
        free_before = torch.cuda.mem_get_info()[0]
        assert _noalloc(L, ig, spec.cf, o) == 0
        assert L.switch_layer_noalloc_status(ctypes.c_void_p(stream)) == 0, call
        free_after = torch.cuda.mem_get_info()[0]
        if call == 1:
            # the first call has loaded the library's device code; from then on a
            # call takes no device memory at all
            assert free_after == free_before, (free_before, free_after)
        for k in ref:
            assert torch.equal(o[k], ref[k]), (call, k)


def test_noalloc_rejects_shapes_beyond_its_scratch(L):
    spec = synth.WORKLOADS["large_T16384_d1024_N128"]    # needs ~180 MB of scratch
    need = swl.switch_layer_workspace_size(spec.T, spec.d, spec.d_ff, spec.N, swl.SWL_BF16,
                                           spec.cf)
    assert need > swl.SWL_NOALLOC_MAX_BYTES
    x = torch.empty((spec.T, spec.d), dtype=torch.bfloat16, device="cuda")
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    o = swl.alloc_outputs(spec.T, spec.d, torch.bfloat16)
    before = L.switch_layer_launch_count()
    p = lambda t: t.data_ptr()
    st = L.switch_layer_forward_noalloc(
        spec.T, spec.d, spec.d_ff, spec.N, swl.SWL_BF16, p(x), p(dummy), p(dummy), p(dummy),
        p(dummy), p(dummy), spec.cf, p(o["out"]), p(o["expert_idx"]), p(o["gate"]),
        p(o["pos_in_expert"]), p(o["aux_loss"]), None, torch.cuda.current_stream().cuda_stream)
    assert st == 3                                      # SWL_ERR_WORKSPACE
    assert L.switch_layer_launch_count() == before      # nothing was enqueued
