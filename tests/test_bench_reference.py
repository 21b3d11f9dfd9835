"""The reference arm of bench.py on the host (no GPU): one JSON line carrying
the contract's keys, with the fp64 oracle as the timed program; under a
multi-rank launch, ranks other than 0 print nothing and exit 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, *args):
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    env.update(env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           *args], cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)


def test_reference_arm_line():
    r = _run({}, "--workload", "base_T4096_d768_N64", "--steps", "1", "--warmup", "0",
             "--cpu-budget", "0.5")
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 1 and d["warmup"] == 3          # at least three warm-up steps
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == "base_T4096_d768_N64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1
    assert "oracle" in cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    r = _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}, "--steps", "1")
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_default_workload_is_the_largest_single_gpu_layer():
    sys.path.insert(0, ROOT)
    import bench
    import synth
    big = max(synth.WORKLOADS.values(), key=lambda w: w.T * w.d + 2 * w.N * w.d * w.d_ff)
    assert bench.DEFAULT_WORKLOAD == big.name == "many_T65536_d1024_N2048"


def test_algorithmic_bytes_of_base_workload():
    """The roofline's byte count for base_T4096_d768_N64: the oracle's routing of the
    seeded batch keeps 4087 tokens over all 64 experts, and the FFN launch needs
    9 444 864 B per touched expert (weights and biases) plus 3 080 B per kept token
    (its input row in, its output row out, destination index and gate):
    617 059 256 B.  The hidden rows between the GEMMs are not counted."""
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import synth
    import numpy as np
    spec = synth.WORKLOADS["base_T4096_d768_N64"]
    ic = synth.make_layer_inputs(spec, 0, device="cpu", redraws=synth.load_gap_redraws(spec.name))
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf, b_r=ic["b_r"])
    C = oracle.capacity(spec.T, spec.N, spec.cf)
    e = np.asarray(ref["expert_idx"])
    kept = int((np.asarray(ref["pos_in_expert"]) < C).sum())
    touched = int((np.bincount(e, minlength=spec.N) > 0).sum())
    assert (touched, kept) == (64, 4087)
    ffn, layer = bench.algorithmic_bytes(spec.T, spec.d, spec.d_ff, spec.N, 2, touched, kept)
    assert ffn == 64 * 9_444_864 + 4087 * 3_080 == 617_059_256
    # the layer adds the router's and the dispatch's bytes to the FFN's
    assert ffn < layer < ffn + 4 * spec.T * spec.d * 2 + spec.N * spec.d * 4 + 16 * spec.T
