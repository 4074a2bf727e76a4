"""The multi-rank path of bench.py on CPU: two gloo ranks, as torchrun would
start them (RANK, WORLD_SIZE, MASTER_ADDR=127.0.0.1).  Each rank decides its
own independent problems (weak scaling); the only collectives are the barrier
and the max-over-ranks timing reduction."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    import oracle
    from moe_expert_load_bf16_b200 import workloads
    try:
        w, r, _ = bench.dist_setup("gloo")
        assert (w, r) == (world, rank)
        wl = bench.rank_workload(workloads.WORKLOADS["tiny"], rank)
        # this rank's own problem, decided on the host oracle (no exchange)
        hid = workloads.hidden_chain(wl, 2)
        Wt = workloads.gate_weights(wl, 1)[0]
        b = workloads.biases(wl, 1)[0].numpy()
        _, ids = oracle.gate(workloads.bf16_bits(hid[1]), workloads.bf16_bits(Wt), b, wl.k)
        cnt = oracle.count(ids, wl.G, wl.E)
        bench.barrier(w)
        t = bench.max_over_ranks(10.0 + rank, w)          # rank 1 is the slower one
        rate = bench.whole_job_rate(wl.T * wl.k, w, t)
        q.put((rank, t, wl.seed, rate, cnt.tolist()))
        torch.distributed.destroy_process_group()
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e)))


def test_two_gloo_ranks_timing_and_independent_problems():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        item = q.get(timeout=240)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(res[r][1] != "error" for r in res), res
    # max over ranks seen identically by both
    assert res[0][1] == res[1][1] == 11.0
    # whole-job rate counts both ranks' assignments against the slowest rank
    assert res[0][3] == res[1][3] == 256 * 2 * 2 / 11e-3
    # independent problems: different seeds, different counts
    assert res[0][2] != res[1][2]
    assert not np.array_equal(np.array(res[0][4]), np.array(res[1][4]))


def test_reference_arm_under_two_ranks_only_rank0_prints():
    outs = []
    for rank in (1, 0):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(_free_port()))
        p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                            "--steps", "1", "--warmup", "1", "--cpu-budget", "0.3"],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
        assert p.returncode == 0, p.stderr
        outs.append(p.stdout.strip())
    assert outs[0] == ""                       # rank 1: no work, no line
    line = json.loads(outs[1])                 # rank 0: one JSON line
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
