"""Multi-rank host logic on CPU ranks over gloo.

* bench.py (world size 2): the slowest rank's time is what every rank sees,
  the whole-job value counts every rank's work, and the reference arm does
  its work on rank 0 only.
* The exchange of the multi-GPU form (world sizes 2 and 4): the product's
  all-to-all (video_dit_sequence_b200.nccl_all_to_all, which only uses
  torch.distributed) routes the chunks the way UlyssesRank's phases expect.
  The local phases are played by the oracle (the CUDA kernels need a GPU):
  exchange pack, attention of the received head group, exchange unpack; the
  result must equal the unsharded attention bit for bit after bf16 rounding."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 100.0 + 25.0 * rank          # rank 1 is the slow one
        t_max = bench.max_over_ranks(local_ms, world)
        value = bench.weak_scaling_value(world, 10, 1e12, t_max)
        q.put((rank, t_max, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(100)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, t_max, value in got:
        assert t_max == 125.0
        # 2 ranks x 10 steps x 1 TFLOP in 125 ms
        assert abs(value - 2 * 10 * 1.0 / 0.125) < 1e-9


def test_reference_arm_rank_nonzero_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_single_rank_aggregation_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.weak_scaling_value(1, 4, 2e12, 1000.0) == 8.0


def _ulysses_rank_main(rank, world, port, q, shape_args):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    import video_dit_sequence_b200 as sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, N, H, D = shape_args
        P = world
        cfg = synth.Config("g", synth.Shape(B, N, H, D, 1), seed=21)
        Q, K, V = synth.qkv_logical(cfg)
        xs = [synth.to_seq_shards(x, P)[rank] for x in (Q, K, V)]   # this rank's shard
        a2a = sp.nccl_all_to_all()

        def bf16(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

        def words(t):
            return t.view(torch.int16).numpy().view(np.uint16)

        recv = [words(a2a(bf16(oracle.exchange_pack(x, N, P)))) for x in xs]
        # recv[t] is head group `rank` in rank-major shards [P][B][Nl][Hl][D]
        grp = [synth.from_seq_shards(r, N) for r in recv]          # [B][N][Hl][D]
        O, _ = oracle.attention_full(*grp, scale=1.0 / np.sqrt(D), threads=1)
        o_sh = synth.to_seq_shards(synth.f32_to_bf16(O.astype(np.float32)), P)
        back = words(a2a(bf16(o_sh)))
        out = oracle.exchange_unpack(back, N, H)                    # [B][Nl][H][D]
        full, _ = oracle.attention_full(Q, K, V, threads=1)
        want = synth.to_seq_shards(synth.f32_to_bf16(full.astype(np.float32)), P)[rank]
        q.put((rank, bool(np.array_equal(out, want))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(180)
@pytest.mark.parametrize("world,shape_args", [(2, (2, 37, 4, 16)), (4, (1, 50, 8, 16))])
def test_multi_gpu_exchange_routing_over_gloo(world, shape_args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_ulysses_rank_main, args=(r, world, port, q, shape_args))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(150)
        assert p.exitcode == 0
    got = dict(q.get(timeout=5) for _ in range(world))
    assert all(got[r] for r in range(world)), got


def _dead_peer_main(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import datetime
    import time

    import torch
    import torch.distributed as dist

    import video_dit_sequence_b200 as sp
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # this rank fails between steps: it leaves before the exchange
        q.put((rank, "left"))
        q.close()
        q.join_thread()
        os._exit(0)
    send = torch.zeros((world, 4), dtype=torch.bfloat16)
    t0 = time.monotonic()
    try:
        sp.nccl_all_to_all()(send)
        q.put((rank, "no error"))
    except Exception as e:  # the group's timeout ends the exchange with an error
        q.put((rank, f"error after {time.monotonic() - t0:.1f}s: {type(e).__name__}"))
    q.close()
    q.join_thread()
    os._exit(0)


@pytest.mark.timeout(120)
def test_exchange_with_a_dead_peer_errors_instead_of_hanging():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dead_peer_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode is not None, "a rank hung"
    got = dict(q.get(timeout=5) for _ in range(world))
    assert got[1] == "left"
    assert got[0].startswith("error after"), got[0]
    assert float(got[0].split()[2].rstrip("s:")) < 60
