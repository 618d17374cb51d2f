"""The multi-rank host path of bench.py on CPU: two gloo ranks, no GPU.

One process per GPU is the bench's layout for N > 1 (replicas of the workload, no
data-path collective); what it needs from torch.distributed is the process group,
the maximum of the step time over ranks and a barrier.  Here two ranks run that
plumbing over gloo, and the reference arm runs under torchrun with two ranks:
rank 0 alone prints the JSON line, the other rank exits 0 without work.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    try:
        w, r, _ = bench.dist_setup()
        # each rank's "step time" differs; every rank must see the slowest
        m = bench.reduce_max(10.0 + 5.0 * r, torch.device("cpu"))
        bench.barrier()
        out_q.put((r, w, dist.get_backend(), m))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_share_the_max_step_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == 2 and g[2] == "gloo" and g[3] == 15.0 for g in got), got


def test_reduce_max_without_a_process_group_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25, torch.device("cpu")) == 3.25
    bench.barrier()   # no group: a no-op


def test_reference_arm_under_torchrun_prints_once():
    env = dict(os.environ, GATTN_REF_BUDGET_S="1", OMP_NUM_THREADS="1")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
           "--workload", "gemma2_2b_local_s256"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["n_gpus"] == 2 and res["steps"] == 3
    assert res["value"] > 0 and res["e2e"]["h2d_bytes_per_step"] == 0
    assert res["cpu_baseline"]["kind"] == "oracle"


def test_sweep_appends_each_workload_once_and_resumes(tmp_path):
    out = tmp_path / "sweep.jsonl"
    env = dict(os.environ, GATTN_REF_BUDGET_S="1", OMP_NUM_THREADS="1")

    def run(names):
        cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "3", "--warmup", "3",
               "--sweep", str(out), "--sweep-workloads", names]
        r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode == 0, r.stderr[-2000:]
        return r

    run("gemma2_2b_local_s256,gemma4_12b_decode_local_b64")
    lines = out.read_text().splitlines()
    assert [json.loads(ln)["config"]["workload"] for ln in lines] == ["gemma2_2b_local_s256",
                                                                     "gemma4_12b_decode_local_b64"]
    # an interrupted run's partial line is ignored; done workloads are skipped
    with open(out, "a") as f:
        f.write('{"metric": "cut sho')
    r = run("gemma2_2b_local_s256,gemma4_12b_decode_local_b64,gemma3_1b_global_b8_chunk1024_prefix7168")
    assert r.stderr.count("skipped") == 2
    recs = []
    for ln in out.read_text().splitlines():
        try:
            recs.append(json.loads(ln))
        except ValueError:
            pass
    assert [x["config"]["workload"] for x in recs][-1] == "gemma3_1b_global_b8_chunk1024_prefix7168"
    assert len(recs) == 3 and all(x["impl"] == "reference" for x in recs)
