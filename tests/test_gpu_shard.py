"""One global batch sharded by contiguous token ranges, through the C ABI's
shard entry points, with the ranks emulated one after another on one GPU (no
kernel of one rank waits for another's: the records are gathered on the host
side between the two steps, as an all-gather would).

The ranks together must give the unsharded batch's routing bit for bit
(expert_idx, pos_in_expert, drop mask), its outputs within the stated
tolerances of the fp64 oracle, and one aux loss, the same on every rank."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
import sparse_mixture_experts_argmax_b200 as swl
from sparse_mixture_experts_argmax_b200 import build as swl_build

from helpers import AUX_RTOL, check_close, check_routing, gap_redraws

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    swl_build.build()
    swl.lib()


def _sharded_run(ig, cf, bounds):
    """Both steps of every rank; returns the global outputs and each rank's aux."""
    x = ig["x"]
    T, d = x.shape
    N, d_ff, _ = ig["W1"].shape
    world = len(bounds) - 1
    out = swl.alloc_outputs(T, d, x.dtype)
    R = swl.switch_layer_shard_record_bytes(N)
    recs = torch.empty(world * R, dtype=torch.uint8, device="cuda")
    works, auxes = [], []
    for g in range(world):
        a, b = bounds[g], bounds[g + 1]
        works.append(swl.alloc_workspace(max(b - a, 1), d, d_ff, N, x.dtype, cf))
        swl.switch_layer_forward_shard_begin(
            x[a:b], ig["W_r"], cf, T, out["expert_idx"][a:b], out["gate"][a:b],
            out["pos_in_expert"][a:b], recs[g * R:(g + 1) * R], d_ff, b_r=ig.get("b_r"),
            workspace=works[g])
    gathered = recs.clone()            # the all-gather, in rank order
    for g in range(world):
        a, b = bounds[g], bounds[g + 1]
        aux = torch.empty(1, dtype=torch.float32, device="cuda")
        swl.switch_layer_forward_shard_end(
            x[a:b], ig["W1"], ig["b1"], ig["W2"], ig["b2"], cf, T, g, world, gathered,
            out["out"][a:b], out["expert_idx"][a:b], out["gate"][a:b],
            out["pos_in_expert"][a:b], aux, workspace=works[g])
        auxes.append(aux)
    torch.cuda.synchronize()
    for w in works:
        assert swl.switch_layer_device_status(w) == 0
    out["aux_loss"] = auxes[0]
    return out, [float(a.item()) for a in auxes]


_CASES = [
    # name, spec, rank boundaries
    ("base_two", synth.WORKLOADS["base_T4096_d768_N64"], [0, 1000, 4096]),
    ("base_three_one_empty", synth.WORKLOADS["base_T4096_d768_N64"], [0, 1500, 1500, 4096]),
    ("tiny_f32_two", synth.WORKLOADS["tiny_f32_T64_d32_N4"], [0, 23, 64]),
    ("wide_bias_four", synth.LayerSpec("shard_wide_bias", 3000, 256, 64, 300, 1.25, "bf16",
                                       bias_std=0.05, router_bias="zipf0.1"),
     [0, 700, 1400, 2000, 3000]),
    ("ragged_two", synth.LayerSpec("shard_ragged", 333, 200, 136, 6, 1.5, "bf16",
                                   bias_std=0.05), [0, 111, 333]),
]


@pytest.mark.parametrize("case", _CASES, ids=lambda c: c[0])
def test_sharded_batch_matches_oracle_and_unsharded_run(case):
    name, spec, bounds = case
    rd = synth.load_gap_redraws(spec.name) if spec.name in synth.WORKLOADS else gap_redraws(spec)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got, auxes = _sharded_run(ig, spec.cf, bounds)
    assert len(set(auxes)) == 1, auxes          # every rank computes the same aux loss
    ic = synth.make_layer_inputs(spec, device="cpu", redraws=rd)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf, b_r=ic["b_r"])
    check_routing(got, ref, ref["capacity"], spec.T)
    check_close(got["out"].double().cpu().numpy(), ref["out"], spec.dtype)
    one = swl.forward(ig, spec.cf)
    for k in ("expert_idx", "pos_in_expert"):
        assert torch.equal(got[k], one[k]), k
    a1 = float(one["aux_loss"].item())
    assert abs(auxes[0] - a1) <= AUX_RTOL * abs(a1)


def test_many_expert_workload_two_ranks():
    spec = synth.WORKLOADS["many_T65536_d1024_N2048"]
    rd = synth.load_gap_redraws(spec.name)
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=rd)
    got, auxes = _sharded_run(ig, spec.cf, [0, 32768, 65536])
    one = swl.forward(ig, spec.cf)
    assert len(set(auxes)) == 1
    for k in ("expert_idx", "pos_in_expert"):
        assert torch.equal(got[k], one[k]), k
    assert abs(auxes[0] - float(one["aux_loss"].item())) <= AUX_RTOL * float(one["aux_loss"])
    # both runs compute each output row from the same weights and row: they agree
    # within the bf16 tolerance (the unsharded run is itself checked against the
    # oracle on every token in test_gpu_parity.py)
    check_close(got["out"].double().cpu().numpy(), one["out"].double().cpu().numpy(), "bf16")


def test_records_that_do_not_add_up_report_device_status():
    """A record set whose counts do not add up to T_total (here one rank told
    the batch has one token more than it does) raises the device status; the
    context stays usable."""
    spec = synth.WORKLOADS["tiny_f32_T64_d32_N4"]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(spec.name))
    T, d = ig["x"].shape
    N, d_ff, _ = ig["W1"].shape
    out = swl.alloc_outputs(T, d, ig["x"].dtype)
    R = swl.switch_layer_shard_record_bytes(N)
    rec = torch.empty(R, dtype=torch.uint8, device="cuda")
    w = swl.alloc_workspace(T + 1, d, d_ff, N, ig["x"].dtype, spec.cf)
    swl.switch_layer_forward_shard_begin(ig["x"], ig["W_r"], spec.cf, T + 1, out["expert_idx"],
                                         out["gate"], out["pos_in_expert"], rec, d_ff,
                                         workspace=w)
    swl.switch_layer_forward_shard_end(ig["x"], ig["W1"], ig["b1"], ig["W2"], ig["b2"], spec.cf,
                                       T + 1, 0, 1, rec.clone(), out["out"], out["expert_idx"],
                                       out["gate"], out["pos_in_expert"], out["aux_loss"],
                                       workspace=w)
    assert swl.switch_layer_device_status(w) == 5
    swl.forward(ig, spec.cf)


def test_world_of_one_equals_forward():
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    ig = synth.make_layer_inputs(spec, device="cuda", redraws=synth.load_gap_redraws(spec.name))
    got = swl.forward_shard(ig, spec.cf, spec.T, 0, 1, lambda r: r.clone())
    one = swl.forward(ig, spec.cf)
    for k in ("out", "expert_idx", "gate", "pos_in_expert"):
        assert torch.equal(got[k], one[k]), k
    # the aux loss sums the same fp32 block sums in another fp64 order
    a1 = float(one["aux_loss"].item())
    assert abs(float(got["aux_loss"].item()) - a1) <= AUX_RTOL * abs(a1)
