"""Multi-rank host logic on CPU: two gloo ranks (spawned processes) shard a
batch and the kv-head groups of an attention problem, compute their shares
(with the fp64 oracle, as there is no GPU here), and check that the shards
partition the work, that the gathered result equals the unsharded one, and
that the timing reduction takes the max over ranks."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from attention_forward_tmem_b200.parallel import shard_heads, shard_range


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("n,world", [(10, 2), (3, 4), (0, 2), (7, 3), (8, 8)])
def test_shard_range_partitions(n, world):
    parts = [shard_range(n, r, world) for r in range(world)]
    assert parts[0][0] == 0 and parts[-1][1] == n
    for (a, b), (c, d) in zip(parts, parts[1:]):
        assert b == c and a <= b
    sizes = [b - a for a, b in parts]
    assert max(sizes) - min(sizes) <= 1


def test_shard_heads_keeps_gqa_groups():
    group, kv = 4, 8
    covered = []
    for r in range(3):
        q0, q1, k0, k1 = shard_heads(kv, group, r, 3)
        assert (q0, q1) == (k0 * group, k1 * group)
        covered += list(range(q0, q1))
    assert covered == list(range(kv * group))


def _worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    import oracle
    from attention_forward_tmem_b200 import parallel
    from attention_forward_tmem_b200 import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hk, L, D = 5, 4, 2, 17, 8
        q, k, v = W.dense_inputs(B, Hq, Hk, L, L, D, D, torch.float32, seed=3)
        b0, b1 = parallel.shard_range(B, rank, world)
        mine = torch.from_numpy(oracle.sdpa(q[b0:b1], k[b0:b1], v[b0:b1], mask_kind="causal",
                                            qk_scale=0.3))
        full = parallel.gather_along(mine, dim=0)
        ref = torch.from_numpy(oracle.sdpa(q, k, v, mask_kind="causal", qk_scale=0.3))
        ok_batch = torch.equal(full, ref)
        q0, q1, k0, k1 = parallel.shard_heads(Hk, Hq // Hk, rank, world)
        mine_h = torch.from_numpy(oracle.sdpa(q[:, q0:q1], k[:, k0:k1], v[:, k0:k1],
                                              mask_kind="causal", qk_scale=0.3,
                                              head_num=q1 - q0, kv_head_num=k1 - k0))
        full_h = parallel.gather_along(mine_h, dim=1)
        ok_heads = torch.equal(full_h, ref)
        mx = parallel.max_over_ranks(10.0 + rank)
        queue.put((rank, ok_batch, ok_heads, mx))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    results = sorted(q.get(timeout=5) for _ in range(world))
    for rank, ok_batch, ok_heads, mx in results:
        assert ok_batch and ok_heads
        assert mx == 10.0 + world - 1
