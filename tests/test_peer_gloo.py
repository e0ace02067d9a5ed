"""Host logic of UlyssesPeerRank (the multi-GPU form with the Q and O
exchanges fused into the attention kernel) on CPU ranks over gloo.

A shared-memory backend stands in for device memory and CUDA IPC: every
rank's Q and O shard is a named shared-memory block that the other ranks map
by name, and the peer step is the kernel's contract played by the oracle:
query token t is read from rank t // Nl, this rank's head group is attended
over the whole sequence, and O rows are stored into rank t // Nl at the
group's head columns.  The test checks the handle exchange, the address
tables in rank order, the K/V exchange that feeds the peer step, and the
closing collective that orders the peers' O stores before a rank reads its
shard: rank 0's peer step is delayed, so a rank that read its shard too
early would miss head group 0.

With kv_exchange="push" the backend also plays sp_exchange_push (rank r
writes its chunk for group j into rank j's received groups at slot r, then
raises rank j's arrival counter for r to the step number) and the waiting
side of sp_attention_ulysses_overlap (the step starts on the received groups
only once every counter shows this step).  Rank P-1 pushes late, so a rank
that did not wait for its chunks would attend stale K/V."""
import math
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _peer_rank_main(rank, world, port, q, shape_args, kv_exchange):
    sys.path.insert(0, ROOT)
    import datetime
    import time
    from multiprocessing import resource_tracker, shared_memory

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    import video_dit_sequence_b200 as sp

    def words(t):
        return t.view(torch.int16).numpy().view(np.uint16)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

    class ShmBackend:
        def __init__(self, shape):
            self.shape = shape
            self.own = {}
            self.maps = []

        def empty(self, shp, dtype=None):
            dtype = dtype or torch.bfloat16
            n = math.prod(shp)
            shm = shared_memory.SharedMemory(create=True,
                                             size=n * torch.empty(0, dtype=dtype).element_size())
            t = torch.frombuffer(shm.buf, dtype=dtype, count=n).view(shp)
            t.zero_()
            self.own[t.data_ptr()] = shm
            return t

        zeros = empty

        def export(self, t):
            return self.own[t.data_ptr()].name, 0   # the whole block

        def open(self, name, offset):
            """A peer's block as raw bytes (the product code only passes it on)."""
            assert offset == 0
            shm = shared_memory.SharedMemory(name=name)
            resource_tracker.unregister(shm._name, "shared_memory")  # the owner unlinks it
            self.maps.append(shm)
            return torch.frombuffer(shm.buf, dtype=torch.uint8, count=shm.size)

        @staticmethod
        def part(x, i, shape):
            if x.dtype == torch.uint8:
                return x.view(torch.bfloat16).view(2, -1)[i]
            return x[i]

        @staticmethod
        def _counts(x):
            return x.view(torch.int64) if x.dtype == torch.uint8 else x

        def push(self, k, v, k_addrs, v_addrs, count_addrs, epoch, r, shape):
            if r == shape.P - 1:
                time.sleep(0.5)                                   # a late pusher
            for x, dst in ((k, k_addrs), (v, v_addrs)):
                send = oracle.exchange_pack(words(x), shape.N, shape.P)   # [P][B][Nl][Hl][D]
                for j in range(shape.P):
                    words(dst[j]).reshape(send.shape)[r] = send[j]
            for j in range(shape.P):
                self._counts(count_addrs[j])[r] = epoch

        def overlap_step(self, q_addrs, k_group, v_group, o_addrs, counts, epoch, j, shape):
            t0 = time.time()
            while int(counts.min()) < epoch:                      # every chunk of this step
                assert time.time() - t0 < 30, "chunks never arrived"
                time.sleep(0.01)
            self.peer_step(q_addrs, k_group, v_group, o_addrs, j, shape)

        def exchange_pack(self, x, send, shape):
            send.copy_(bf16(oracle.exchange_pack(words(x), shape.N, shape.P)))

        def peer_step(self, q_addrs, k_group, v_group, o_addrs, j, shape):
            if j == 0:
                time.sleep(0.5)
            N, H, P = shape.N, shape.H, shape.P
            Hl = H // P
            shard = tuple(shape.rank_shard)
            q_all = np.stack([words(x).reshape(shard) for x in q_addrs])   # [P][B][Nl][H][D]
            qg = synth.from_seq_shards(q_all, N)[:, :, j * Hl:(j + 1) * Hl]
            kg, vg = (synth.from_seq_shards(words(x).reshape(shape.send_chunks), N)
                      for x in (k_group, v_group))
            O, _ = oracle.attention_full(np.ascontiguousarray(qg), kg, vg,
                                         scale=1.0 / np.sqrt(shape.D), threads=1)
            o_sh = synth.to_seq_shards(synth.f32_to_bf16(O.astype(np.float32)), P)
            for r in range(P):
                words(o_addrs[r]).reshape(shard)[:, :, j * Hl:(j + 1) * Hl] = o_sh[r]

        def close(self):
            for shm in self.maps:
                shm.close()
            self.maps = []

        def release(self):
            for shm in self.own.values():
                shm.close()
                shm.unlink()

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, N, H, D = shape_args
        P = world
        shape = sp.Shape(B, N, H, D, P)
        be = ShmBackend(shape)
        pr = sp.UlyssesPeerRank(shape, backend=be, kv_exchange=kv_exchange)
        results = []
        for seed in (31, 32):                                     # two steps, buffers reused
            cfg = synth.Config("p", synth.Shape(B, N, H, D, 1), seed=seed)
            Q, K, V = synth.qkv_logical(cfg)
            qs, ks, vs = (synth.to_seq_shards(x, P)[rank] for x in (Q, K, V))
            out = words(pr.step(bf16(ks), bf16(vs), q=bf16(qs))).copy()
            full, _ = oracle.attention_full(Q, K, V, threads=1)
            want = synth.to_seq_shards(synth.f32_to_bf16(full.astype(np.float32)), P)[rank]
            results.append(bool(np.array_equal(out, want)))
        pr.close()
        be.release()
        q.put((rank, results))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("kv_exchange", ["push", "nccl"])
@pytest.mark.parametrize("world,shape_args", [(2, (1, 100, 4, 16)), (4, (2, 37, 8, 16))])
def test_peer_rank_host_logic(world, shape_args, kv_exchange):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_peer_rank_main, args=(r, world, port, q, shape_args, kv_exchange))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(200)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [r for r, _ in got] == list(range(world))
    for rank, results in got:
        assert results == [True, True], (rank, results)
