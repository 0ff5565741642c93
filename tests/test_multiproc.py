"""The N>1 host logic of the benchmark (data-parallel replicas) on CPU with gloo, world size 2:
max-over-ranks timing, per-rank seeds, and the rank-0-only reference arm."""
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    import workloads
    t = bench.max_over_ranks(1.5 + rank, world)
    seed = bench.rank_seed(0, rank)
    cfg = workloads.CONFIGS["tiny_bf16_fwd"]
    d = workloads.make_layer_inputs(cfg, seed=seed)
    bench.barrier(world)
    q.put((rank, t, seed, float(d["x"].float().sum())))
    dist.destroy_process_group()


def test_two_rank_timing_and_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]          # both ranks see the maximum
    assert [r[2] for r in res] == [0, 1]              # distinct seeds per replica
    assert res[0][3] != res[1][3]                     # so distinct batches


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_bf16_fwd"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank0():
    import json
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3", "--workload", "tiny_bf16_fwd", "--reference-tokens", "32"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _grad_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import mixture_experts_grouped_top_b200 as mb
    # each replica's weight gradients (bf16, as the layer produces them): small integers,
    # so their sum is exact in bf16
    dw1 = torch.full((2, 3, 8), float(rank + 1), dtype=torch.bfloat16)
    dw2 = torch.arange(12, dtype=torch.float32).reshape(2, 6).to(torch.bfloat16) * (rank + 1)
    mb.allreduce_grads([dw1, dw2])
    avg = torch.full((4,), float(2 * rank + 2), dtype=torch.float32)
    mb.allreduce_grads([avg], average=True)
    q.put((rank, dw1.float().sum().item(), dw2.float().tolist(), avg.tolist()))
    dist.destroy_process_group()


def test_two_rank_weight_gradient_allreduce():
    """The data-parallel backward's exchange (sum of dw1, dw2 over the replicas)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_grad_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, s1, dw2, avg in res:
        assert s1 == (1 + 2) * 2 * 3 * 8
        assert dw2 == [[3.0 * v for v in range(6)], [3.0 * v for v in range(6, 12)]]
        assert avg == [3.0] * 4
