"""CUDA path (through the C ABI) against the fp64 oracle, on seeded inputs.

Routing (expert_idx, pos_in_expert, drop mask) must match bit for bit; gate,
aux loss and outputs within the stated tolerances (see helpers.py).  The five
named workloads run at full size, in the launch configuration the bench uses;
the two largest regenerate each expert's weights on demand in the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import check_close, check_routing, gap_redraws

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _run(inputs_gpu, cf):
    out = swl.forward(inputs_gpu, cf)
    torch.cuda.synchronize()
    return out


def _np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def _full_parity(spec: synth.LayerSpec, redraws, seed=0):
    ig = synth.make_layer_inputs(spec, seed, device="cuda", redraws=redraws)
    got = _run(ig, spec.cf)
    ic = synth.make_layer_inputs(spec, seed, device="cpu", redraws=redraws)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf, b_r=ic["b_r"])
    C = oracle.capacity(spec.T, spec.N, spec.cf)
    assert swl.switch_layer_capacity(spec.T, spec.N, spec.cf) == C
    check_routing(got, ref, C, spec.T)
    check_close(_np(got["out"]), ref["out"], spec.dtype)
    return got, ref


# ------------------------------------------------------------------ generator
def test_generator_gpu_equals_cpu():
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    rd = synth.load_gap_redraws(spec.name)
    xg = synth.make_x(spec, device="cuda", redraws=rd).cpu()
    xc = synth.make_x(spec, device="cpu", redraws=rd)
    assert torch.equal(xg, xc)
    eg = synth.expert_slice(spec, [0, 17, 63], device="cuda")
    ec = synth.expert_slice(spec, [0, 17, 63], device="cpu")
    for k in eg:
        assert torch.equal(eg[k].cpu(), ec[k]), k
    rg = synth.make_router(spec, device="cuda")
    assert torch.equal(rg["W_r"].cpu(), synth.make_router(spec)["W_r"])


# ------------------------------------------------------------------ named workloads, full size
@pytest.mark.parametrize("name", ["tiny_f32_T64_d32_N4", "base_T4096_d768_N64",
                                  "large_T16384_d1024_N128"])
def test_named_workload_full(name):
    spec = synth.WORKLOADS[name]
    rd = synth.load_gap_redraws(spec.name)
    got, ref = _full_parity(spec, rd)
    assert (~ref["kept"]).sum() >= 0


def _every_token_parity(spec: synth.LayerSpec, seed=0):
    """Full-size parity for layers whose fp64 weights would not fit in host
    memory at once: the oracle routes every token, then computes the output row
    of every kept token one expert at a time (dropped rows must be zero).  Each
    expert's weights are the seeded inputs themselves, copied from the device
    one expert at a time (the generator is bit-identical on CPU and GPU; see
    test_generator_gpu_equals_cpu)."""
    rd = synth.load_gap_redraws(spec.name)
    ig = synth.make_layer_inputs(spec, seed, device="cuda", redraws=rd)
    got = _run(ig, spec.cf)

    def weights(e):
        return {k: ig[k][e].cpu() for k in ("W1", "b1", "W2", "b2")}

    x = ig["x"].cpu()
    b_r = ig["b_r"].cpu() if ig["b_r"] is not None else None
    ref = oracle.switch_forward_sampled(x, ig["W_r"].cpu(), spec.cf, range(spec.T), weights,
                                        b_r=b_r)
    check_routing(got, ref, ref["capacity"], spec.T)
    out = got["out"]
    kept = ref["kept"]
    # every dropped row is exactly zero; every kept row within tolerance
    dropped = torch.from_numpy(np.nonzero(~kept)[0]).to(out.device)
    assert not out[dropped].any(), "a dropped token has a non-zero output row"
    toks = np.nonzero(kept)[0]
    want = np.stack([ref["out_rows"][int(t)] for t in toks])
    check_close(_np(out[torch.from_numpy(toks).to(out.device)]), want, spec.dtype)
    # every touched expert contributes compared rows, first and last kept ones included
    touched = np.unique(ref["expert_idx"][kept])
    assert len(touched) == len(np.unique(ref["expert_idx"]))
    return got, ref


def test_skewed_workload_every_token():
    spec = synth.WORKLOADS["skewed_T32768_d2048_N64"]
    got, ref = _every_token_parity(spec)
    C = ref["capacity"]
    zero = np.nonzero(ref["expert_idx"] == 0)[0]
    # expert 0 overflows: its last kept and first dropped tokens are in the comparison
    assert len(zero) > C and ref["kept"][zero[C - 1]] and not ref["kept"][zero[C]]
    assert (~ref["kept"]).sum() > 0


def test_many_expert_workload_every_token():
    spec = synth.WORKLOADS["many_T65536_d1024_N2048"]
    got, ref = _every_token_parity(spec)
    assert len(np.unique(ref["expert_idx"][ref["kept"]])) == spec.N


# ------------------------------------------------------------------ random shapes, ragged tails
def _random_specs():
    rng = np.random.default_rng(2024)
    specs = []
    for i in range(10):
        specs.append(synth.random_spec(rng, "rand_bf16_%d" % i, "bf16"))
    for i in range(5):
        specs.append(synth.random_spec(rng, "rand_f32_%d" % i, "f32", max_T=300))
    return specs


@pytest.mark.parametrize("spec", _random_specs(), ids=lambda s: "%s_T%d_d%d_f%d_N%d_cf%g" % (
    s.name, s.T, s.d, s.d_ff, s.N, s.cf))
def test_random_shapes(spec):
    _full_parity(spec, gap_redraws(spec))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", ["one_token", "one_expert", "tiny_capacity", "no_drops",
                                  "ragged_tiles", "wide_ffn"])
def test_edge_cases(dtype, case):
    shapes = {
        "one_token": (1, 64, 128, 4, 1.0),
        "one_expert": (300, 64, 128, 1, 1.0),       # dense FFN, gate 1
        "tiny_capacity": (257, 64, 64, 3, 0.01),    # C = 1
        "no_drops": (300, 48, 80, 5, 5.0),          # C = T
        "ragged_tiles": (333, 200, 136, 6, 1.5),    # d, d_ff not multiples of 64 / 128
        "wide_ffn": (130, 128, 1032, 2, 2.0),
    }
    T, d, d_ff, N, cf = shapes[case]
    spec = synth.LayerSpec("edge_%s_%s" % (case, dtype), T, d, d_ff, N, cf, dtype, bias_std=0.05)
    _full_parity(spec, gap_redraws(spec))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_collapse_multi_tile_expert(dtype):
    """Every token picks expert 0 (router bias), C = T: one expert with several
    256-row token tiles, the others empty."""
    T, d, d_ff, N = 700, 64, 192, 4
    spec = synth.LayerSpec("collapse_%s" % dtype, T, d, d_ff, N, float(N), dtype, bias_std=0.05)
    rd = gap_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    b_r = torch.tensor([30.0] + [0.0] * (N - 1), dtype=torch.float32)
    ig["b_r"], ic["b_r"] = b_r.cuda(), b_r
    got = _run(ig, spec.cf)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf, b_r=b_r)
    assert np.all(ref["expert_idx"] == 0) and ref["kept"].all()
    check_routing(got, ref, oracle.capacity(T, N, spec.cf), T)
    check_close(_np(got["out"]), ref["out"], dtype)


def test_empty_batch():
    spec = synth.LayerSpec("empty", 0, 16, 16, 3, 1.0, "bf16")
    ig = synth.make_layer_inputs(spec, device="cuda")
    got = _run(ig, 1.0)
    assert float(got["aux_loss"].cpu()[0]) == 0.0


# ------------------------------------------------------------------ API variants and status
def test_host_io_and_timed_variants_match():
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(spec.name))
    a = _run(ig, spec.cf)
    b = _run(ig, spec.cf)                  # repeat: deterministic
    for k in a:
        assert torch.equal(a[k], b[k]), k
    T, d = ig["x"].shape
    N, d_ff, _ = ig["W1"].shape
    ws = swl.alloc_workspace(T, d, d_ff, N, ig["x"].dtype, spec.cf, host_io=True)
    xh = ig["x"].cpu().pin_memory()
    oh = {"out": torch.empty((T, d), dtype=ig["x"].dtype).pin_memory(),
          "expert_idx": torch.empty(T, dtype=torch.int32).pin_memory(),
          "gate": torch.empty(T, dtype=torch.float32).pin_memory(),
          "pos_in_expert": torch.empty(T, dtype=torch.int32).pin_memory(),
          "aux_loss": torch.empty(1, dtype=torch.float32).pin_memory()}
    swl.switch_layer_forward_host_io(xh, ig["W_r"], ig["W1"], ig["b1"], ig["W2"], ig["b2"],
                                     spec.cf, oh["out"], oh["expert_idx"], oh["gate"],
                                     oh["pos_in_expert"], oh["aux_loss"], b_r=ig["b_r"],
                                     workspace=ws)
    torch.cuda.synchronize()
    assert swl.switch_layer_device_status(ws) == 0
    for k in a:
        assert torch.equal(a[k].cpu(), oh[k]), k
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(swl.SWL_NUM_STAGES + 1)]
    c = swl.alloc_outputs(T, d, ig["x"].dtype)
    ws2 = swl.alloc_workspace(T, d, d_ff, N, ig["x"].dtype, spec.cf)
    swl.switch_layer_forward(ig["x"], ig["W_r"], ig["W1"], ig["b1"], ig["W2"], ig["b2"], spec.cf,
                             c["out"], c["expert_idx"], c["gate"], c["pos_in_expert"],
                             c["aux_loss"], b_r=ig["b_r"], workspace=ws2, stage_events=evs)
    torch.cuda.synchronize()
    for k in a:
        assert torch.equal(a[k], c[k]), k
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(swl.SWL_NUM_STAGES)]
    assert all(t >= 0 for t in times)


def test_small_workspace_is_rejected():
    spec = synth.WORKLOADS["tiny_f32_T64_d32_N4"]
    ig = synth.make_layer_inputs(spec, device="cuda")
    o = swl.alloc_outputs(spec.T, spec.d, ig["x"].dtype)
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    before = swl.switch_layer_launch_count()
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.switch_layer_forward(ig["x"], ig["W_r"], ig["W1"], ig["b1"], ig["W2"], ig["b2"],
                                 spec.cf, o["out"], o["expert_idx"], o["gate"],
                                 o["pos_in_expert"], o["aux_loss"], workspace=ws)
    assert ei.value.status == 3
    assert swl.switch_layer_launch_count() == before


def test_nonfinite_router_input_reports_device_status():
    spec = synth.LayerSpec("nan_row", 200, 32, 64, 4, 1.0, "bf16")
    ig = synth.make_layer_inputs(spec, device="cuda")
    ig["x"][7] = float("nan")
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.forward(ig, spec.cf)
    assert ei.value.status == 5
    # the context is still usable
    ig["x"][7] = 0.5
    swl.forward(ig, spec.cf)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N", [4, 200])
def test_infinite_router_weight_reports_device_status(dtype, N):
    """An infinite router weight gives tokens an infinite maximum logit (+inf
    minus +inf in the softmax would make the gate NaN): the call reports
    SWL_ERR_DEVICE, and the context stays usable.  N = 200 takes the wide
    router with its separate softmax kernel."""
    spec = synth.LayerSpec("inf_wr_%s_N%d" % (dtype, N), 300, 64, 64, N, 1.0, dtype)
    ig = synth.make_layer_inputs(spec, device="cuda")
    w = ig["W_r"][2, 0].item()
    ig["W_r"][2, 0] = float("inf")
    with pytest.raises(swl.SwitchLayerError) as ei:
        swl.forward(ig, spec.cf)
    assert ei.value.status == 5
    ig["W_r"][2, 0] = w
    swl.forward(ig, spec.cf)


@pytest.mark.parametrize("dtype,N", [("bf16", 8), ("f32", 8), ("bf16", 200)])
def test_router_decision_needs_float32_weights(dtype, N):
    """The router works in float32 (selective precision).  Experts 0 and 1 have
    weights 1 + 2^-9 and 1 + 2^-9 + 2^-17: equal in bfloat16, and equal after
    the first two bf16 pieces of an fp32 split (the 2^-17 lives only in the third
    piece).  Their logits for x = c * ones(64) differ by c * 64 * 2^-17, about 64
    ulps of the logit, far above the worst-case fp32 accumulation error
    (64 * ulp/2), so a float32 router sends every token with c > 0 to expert 1,
    while any router that drops the low piece ties them and takes expert 0.
    N = 200 takes the wide tensor-core logits kernel (all pieces in one
    accumulator) and the separate softmax."""
    T, d, d_ff, cf = 256, 64, 64, float(8)
    spec = synth.LayerSpec("fp32_router_%s_N%d" % (dtype, N), T, d, d_ff, N, cf, dtype)
    ic = synth.make_layer_inputs(spec, device="cpu")
    scale = torch.tensor([0.5, 1.0, 2.0, 4.0, -1.0])[torch.arange(T) % 5]
    ic["x"] = (scale[:, None] * torch.ones(T, d)).to(ic["x"].dtype)
    W_r = torch.zeros(N, d, dtype=torch.float32)
    W_r[0] = 1.0 + 2.0 ** -9
    W_r[1] = 1.0 + 2.0 ** -9 + 2.0 ** -17
    assert float(W_r[1, 0]) - float(W_r[0, 0]) == 2.0 ** -17      # exact in fp32
    assert torch.equal(W_r[0].to(torch.bfloat16), W_r[1].to(torch.bfloat16))
    ic["W_r"], ic["b_r"] = W_r, None
    ig = {k: (v.cuda() if v is not None else None) for k, v in ic.items()}
    got = _run(ig, cf)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"], cf)
    pos = (scale > 0).numpy()
    assert np.all(ref["expert_idx"][pos] == 1)
    check_routing(got, ref, oracle.capacity(T, N, cf), T)
    check_close(_np(got["out"]), ref["out"], dtype)


# Shapes chosen to reach each kernel variant of the path (see the router plan,
# the dispatch choice and the expert FFN accumulator count in csrc/):
#   bf16 N = 80 (96-expert router tiles), K split over a 4-CTA cluster
#   bf16 N = 128, K split over a 2-CTA cluster
#   bf16 N = 200: tensor-core logits tiles with a ragged last expert tile + streaming softmax
#   bf16 N = 202 (not a multiple of 4): softmax with the row held in registers
#   bf16 N = 2100 (beyond the register row): three-pass softmax
#   fp32 N = 150: FFMA logits with K slices + softmax kernel
#   fp32 N = 48, ~100 big router tiles: FFMA tile router, fused dispatch
#   fp32 N = 8, x > 16 MiB: warp-split router, two-kernel dispatch (scan + gather)
#   bf16 N = 4, capacity > 128 rows: two 256-column TMEM accumulators
#   bf16 x > 48 MiB, cf = 0.25: two-kernel dispatch, most tokens dropped
_VARIANT_SHAPES = [
    ("tc_np96_s4", 1000, 1024, 256, 80, 1.25, "bf16"),
    ("tc_np128_s2", 2000, 256, 128, 128, 1.25, "bf16"),
    ("tc_wide_ragged", 700, 256, 128, 200, 2.0, "bf16"),
    ("tc_wide_rows", 500, 128, 64, 202, 2.0, "bf16"),
    ("tc_wide_threepass", 300, 64, 64, 2100, 8.0, "bf16"),
    ("ffma_wide", 300, 48, 40, 150, 2.0, "f32"),
    ("ffma_tile", 25700, 32, 32, 48, 1.0, "f32"),
    ("two_kernel_dispatch", 20000, 256, 32, 8, 1.0, "f32"),
    ("two_accumulators", 900, 64, 64, 4, 1.0, "bf16"),
    # GEMM2 split over K on the first experts, unsplit tiles on the rest
    ("gemm2_split_mixed", 12288, 768, 4096, 8, 1.0, "bf16"),
    # d_ff = 4160: K chunks of 17 k-blocks (1088 features), so GEMM1 feature tiles
    # 8 and 25 straddle two chunks and count in both
    ("gemm2_split_straddle", 12288, 768, 4160, 8, 1.0, "bf16"),
    # streaming softmax: a warp per row at full width (N = 1024), a warp pair per row
    # with a ragged second half (N = 1500); token blocks of 45 and 37 tokens
    ("stream_full_warp_row", 6600, 128, 64, 1024, 2.0, "bf16"),
    ("stream_pair_ragged", 5400, 128, 64, 1500, 2.0, "bf16"),
    # x above 48 MiB with most tokens dropped: the gather reads only the kept
    # tokens' rows (no early row loads) and zeroes the dropped tokens' rows
    ("gather_mostly_dropped", 25000, 1024, 64, 16, 0.25, "bf16"),
]


@pytest.mark.parametrize("shape", _VARIANT_SHAPES, ids=lambda s: s[0])
def test_kernel_variant_shapes(shape):
    name, T, d, d_ff, N, cf, dtype = shape
    spec = synth.LayerSpec("variant_" + name, T, d, d_ff, N, cf, dtype, bias_std=0.05)
    _full_parity(spec, gap_redraws(spec))


# Router bias on each tensor-core router path: one CTA per 128-token tile (bias
# added at the TMEM read-out; d = 128 leaves K too short to split; with more
# tiles than SMs, two CTAs of two stages each per SM), 2- and 4-CTA
# clusters (bias added after the rank-ordered sum of the partial logits).  N is
# not a multiple of 32 in two of them (padded expert columns), and every batch
# ends in a ragged tile.  A mild bias (0.1 ln(1/(i+1))) keeps most experts in use.
_ROUTER_BIAS_SHAPES = [
    ("tc_s1_bias_padded", 6000, 128, 64, 50, 1.25),
    ("tc_s1_two_per_sm", 20000, 256, 64, 50, 1.25),   # 157 one-CTA tiles > 148 SMs: 2 stages
    ("tc_s2_bias_np128", 3000, 256, 64, 100, 1.0),
    ("tc_s4_bias_padded", 1000, 1024, 64, 40, 1.25),
    ("tc_wide_stream_bias", 3000, 256, 64, 300, 1.25),   # bias added by the streaming softmax
]


@pytest.mark.parametrize("shape", _ROUTER_BIAS_SHAPES, ids=lambda s: s[0])
def test_router_bias_paths(shape):
    name, T, d, d_ff, N, cf = shape
    spec = synth.LayerSpec("rbias_" + name, T, d, d_ff, N, cf, "bf16", bias_std=0.05,
                           router_bias="zipf0.1")
    _full_parity(spec, gap_redraws(spec))


# ------------------------------------------------------------------ FFMA router for bf16 layers
@pytest.fixture
def ffma_router():
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_FFMA)
    yield
    swl.switch_layer_set_router_mode(swl.SWL_ROUTER_TENSOR)


def test_base_workload_ffma_router(ffma_router):
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    _full_parity(spec, synth.load_gap_redraws(spec.name))


@pytest.mark.parametrize("spec", _random_specs()[:5], ids=lambda s: s.name)
def test_random_shapes_ffma_router(spec, ffma_router):
    _full_parity(spec, gap_redraws(spec))


def test_router_decision_needs_float32_weights_ffma(ffma_router):
    test_router_decision_needs_float32_weights("bf16", 8)


# ------------------------------------------------------------------ failure path (bounded waits)
def test_wait_that_runs_out_reports_device_status_and_context_survives():
    """The expert FFN is made to wait for a GEMM1 epilogue warp that does not
    exist (test hook): the wait gives up after its (shortened) limit, the call
    reports SWL_ERR_DEVICE, and the next normal call on the same context passes
    parity."""
    spec = synth.LayerSpec("stall_wait", 600, 128, 256, 4, 1.25, "bf16", bias_std=0.05)
    rd = gap_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    swl.switch_layer_set_wait_limit_ns(1_000_000)          # 1 ms
    swl.switch_layer_set_stall_test(True)
    try:
        with pytest.raises(swl.SwitchLayerError) as ei:
            swl.forward(ig, spec.cf)
        assert ei.value.status == 5
    finally:
        swl.switch_layer_set_stall_test(False)
        swl.switch_layer_set_wait_limit_ns(0)
    _full_parity(spec, rd)
