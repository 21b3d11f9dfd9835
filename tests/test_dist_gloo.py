"""Multi-rank host logic of bench.py on two gloo ranks (CPU): process-group
setup from the torchrun environment, barrier, max over ranks of the timed
region, whole-job throughput, and one seed per rank."""
import os
import socket
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = textwrap.dedent("""
    import sys, json
    sys.path.insert(0, %r)
    from sparse_mixture_experts_argmax_b200 import dist as d
    info = d.init("gloo", timeout_s=60)
    d.barrier(info)
    local_ms = 10.0 + 5.0 * info.rank          # rank 1 is the slower one
    mx = d.max_over_ranks(info, local_ms)
    thr = d.aggregate_throughput(info, units_per_rank=4096, steps=20, max_total_ms=mx)
    print(json.dumps({"rank": info.rank, "world": info.world_size, "max": mx, "thr": thr,
                      "seed": d.rank_seed(info, 7)}), flush=True)
    d.finalize(info)
""") % ROOT


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_two_gloo_ranks():
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    import json
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        outs.append(json.loads(out.strip().splitlines()[-1]))
    outs.sort(key=lambda o: o["rank"])
    assert [o["world"] for o in outs] == [2, 2]
    assert all(o["max"] == 15.0 for o in outs)               # the slower rank decides
    assert all(abs(o["thr"] - 2 * 4096 * 20 / 0.015) < 1e-6 for o in outs)
    assert [o["seed"] for o in outs] == [7, 8]


def test_single_rank_defaults():
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK")}
    code = ("import sys; sys.path.insert(0, %r)\n"
            "from sparse_mixture_experts_argmax_b200 import dist as d\n"
            "i = d.init('gloo'); assert not i.distributed\n"
            "assert d.max_over_ranks(i, 3.5) == 3.5\n"
            "assert d.aggregate_throughput(i, 100, 2, 1000.0) == 200.0\n" % ROOT)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0, r.stderr


# ---------------------------------------------------------------------------
# one global batch sharded by token ranges: the oracle on each rank's range plus
# the record all-gather gives the unsharded batch's routing
# ---------------------------------------------------------------------------
SHARD_WORKER = textwrap.dedent("""
    import sys, json
    sys.path.insert(0, %r)
    sys.path.insert(0, %r)
    import numpy as np, torch
    import oracle, synth
    from sparse_mixture_experts_argmax_b200 import dist as d
    info = d.init("gloo", timeout_s=60)
    spec = synth.LayerSpec("shard_gloo", 901, 24, 16, 7, 1.0, "f32", bias_std=0.05)
    x = synth.make_x(spec)
    W_r = synth.make_router(spec)["W_r"]
    bounds = [0, 300, 901] if info.world_size == 2 else [0, 0, 450, 901]
    a, b = bounds[info.rank], bounds[info.rank + 1]
    # this rank's routing, by the oracle's steps on its own tokens
    p = oracle.router_probs(oracle.router_logits(x[a:b], W_r)) if b > a else np.zeros((0, 7))
    e, g = oracle.top1(p) if b > a else (np.zeros(0, np.int64), np.zeros(0))
    counts = np.bincount(e, minlength=spec.N).astype(np.int32)
    psum = p.sum(axis=0) if b > a else np.zeros(spec.N)
    # the exchange record: int32 counts, fp64 sums at the next 16-byte boundary
    off = (4 * spec.N + 15) // 16 * 16
    rec = np.zeros((off + 8 * spec.N + 15) // 16 * 16, dtype=np.uint8)
    rec[:4 * spec.N] = counts.view(np.uint8)
    rec[off:off + 8 * spec.N] = psum.view(np.uint8)
    gathered = d.exchange_records(info, torch.from_numpy(rec)).numpy()
    R = rec.size
    cnt = np.stack([gathered[g0 * R:g0 * R + 4 * spec.N].view(np.int32)
                    for g0 in range(info.world_size)])
    ps = np.stack([gathered[g0 * R + off:g0 * R + off + 8 * spec.N].view(np.float64)
                   for g0 in range(info.world_size)])
    before = cnt[:info.rank].sum(axis=0)
    pos = before[e] + oracle.positions(e, spec.N)
    T_total = int(cnt.sum())
    C = oracle.capacity(T_total, spec.N, spec.cf)
    f = cnt.sum(axis=0) / T_total
    P = np.zeros(spec.N)
    for g0 in range(info.world_size):
        P = P + ps[g0]
    aux = oracle.aux_loss(f, P / T_total)
    print(json.dumps({"rank": info.rank, "range": [a, b], "e": e.tolist(), "pos": pos.tolist(),
                      "kept": (pos < C).tolist(), "C": C, "aux": aux}), flush=True)
    d.finalize(info)
""") % (ROOT, os.path.join(ROOT, "tests"))


def _run_ranks(code, world):
    import json
    port = _free_port()
    procs = []
    for rank in range(world):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=180)
        assert p.returncode == 0, err[-3000:]
        outs.append(json.loads(out.strip().splitlines()[-1]))
    return sorted(outs, key=lambda o: o["rank"])


import pytest  # noqa: E402


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_batch_routing_equals_unsharded(world):
    """Ranks holding contiguous token ranges (one of them empty for world = 3)
    exchange per-expert counts and sums of p and get the unsharded batch's
    expert choices, positions, drop mask and capacity exactly, and its aux loss
    up to the order of the fp64 sums (the same value on every rank)."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    import synth
    outs = _run_ranks(SHARD_WORKER, world)
    spec = synth.LayerSpec("shard_gloo", 901, 24, 16, 7, 1.0, "f32", bias_std=0.05)
    ic = synth.make_layer_inputs(spec)
    ref = oracle.switch_forward(ic["x"], ic["W_r"], ic["W1"], ic["b1"], ic["W2"], ic["b2"],
                                spec.cf)
    e = np.concatenate([o["e"] for o in outs]).astype(np.int64)
    pos = np.concatenate([o["pos"] for o in outs]).astype(np.int64)
    kept = np.concatenate([o["kept"] for o in outs]).astype(bool)
    assert [o["range"] for o in outs][0][0] == 0 and outs[-1]["range"][1] == spec.T
    assert np.array_equal(e, ref["expert_idx"])
    assert np.array_equal(pos, ref["pos_in_expert"])
    assert np.array_equal(kept, ref["kept"]) and (~kept).any()
    assert all(o["C"] == ref["capacity"] for o in outs)
    assert len({o["aux"] for o in outs}) == 1
    assert abs(outs[0]["aux"] - ref["aux"]) <= 1e-13 * ref["aux"]


# ---------------------------------------------------------------------------
# expert parallelism: per-peer row counts from the gathered records, and the
# row all-to-all that carries kept tokens to the owners of their experts
# ---------------------------------------------------------------------------
EP_WORKER = textwrap.dedent("""
    import sys, json
    sys.path.insert(0, %r)
    import numpy as np, torch
    import sparse_mixture_experts_argmax_b200 as swl
    from sparse_mixture_experts_argmax_b200 import dist as d
    info = d.init("gloo", timeout_s=60)
    W, N, cf = info.world_size, 6, 1.0
    rng = np.random.default_rng(5)
    counts = rng.integers(0, 9, size=(W, N)).astype(np.int32)     # every rank's record
    T_total = int(counts.sum())
    R = swl.switch_layer_shard_record_bytes(N)
    rec = np.zeros(R, dtype=np.uint8)
    rec[:4 * N] = counts[info.rank].view(np.uint8)
    gathered = d.exchange_records(info, torch.from_numpy(rec))
    send, recv = swl.switch_layer_ep_counts(N, W, info.rank, T_total, cf, gathered)
    # rows labelled (source rank, expert, global position), packed by expert
    C = swl.switch_layer_capacity(T_total, N, cf)
    before = counts[:info.rank].sum(axis=0)
    labels = []
    for e in range(N):
        m = max(0, min(int(counts[info.rank, e]), C - int(before[e])))
        labels += [[info.rank, e, int(before[e]) + j] for j in range(m)]
    rows = torch.tensor(labels, dtype=torch.int64).reshape(-1, 3)
    got = d.alltoall_rows(info, rows, send, recv)
    print(json.dumps({"rank": info.rank, "send": send, "recv": recv, "got": got.tolist(),
                      "C": C, "counts": counts.tolist()}), flush=True)
    d.finalize(info)
""") % ROOT


@pytest.mark.parametrize("world", [2, 3])
def test_expert_parallel_counts_and_row_exchange(world):
    """Every rank's send count to a peer equals that peer's receive count from
    it, and each owner receives exactly the kept (expert, position) pairs of
    its experts, source by source, positions ascending: the global position
    order of the unsharded layer once permuted per expert."""
    outs = _run_ranks(EP_WORKER, world)
    N = 6
    L = N // world
    counts = outs[0]["counts"]
    C = outs[0]["C"]
    for g in range(world):
        for r in range(world):
            assert outs[g]["send"][r] == outs[r]["recv"][g]
    for r in range(world):
        got = outs[r]["got"]
        want = []
        for g in range(world):
            for e in range(r * L, r * L + L):
                before = sum(counts[h][e] for h in range(g))
                m = max(0, min(counts[g][e], C - before))
                want += [[g, e, before + j] for j in range(m)]
        assert got == want
