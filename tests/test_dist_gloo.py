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
