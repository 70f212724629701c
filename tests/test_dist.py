"""bench.py's multi-rank path on CPU (gloo, world size 2).

Paged decode shards by sequence with no exchange: each rank decodes its own
batch on its own GPU, and the only cross-rank operations are the barrier and
the max over ranks of the device time. These tests run those host-side steps
with two gloo ranks, and run the reference arm under torchrun (rank 0 prints
one line, rank 1 exits 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(world)
    bench.barrier(w)
    slowest = bench.max_over_ranks(10.0 * (r + 1), w)
    out.put((r, w, slowest, torch.distributed.get_backend()))
    torch.distributed.destroy_process_group()


def test_max_over_ranks_and_barrier_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r for r, *_ in results] == [0, 1]
    assert all(w == 2 and slowest == 20.0 and backend == "gloo" for _, w, slowest, backend in results)


def test_reference_arm_under_torchrun_prints_one_line():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--workload", "tiny", "--gpus", "2", "--steps", "2", "--warmup", "1"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "seqs/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_each_rank_decodes_its_own_batch():
    """Weak scaling: rank r builds the workload from seed + r, so ranks never share sequences."""
    sys.path.insert(0, ROOT)
    from paged_kv_cache_372_b200 import workloads
    a = workloads.llama7b(0, num_seqs=4)
    b = workloads.llama7b(1, num_seqs=4)
    assert not torch.equal(a.steps[0].q, b.steps[0].q)
    assert list(a.steps[0].context_lens) != list(b.steps[0].context_lens)
