"""Head sharding of the plan (one rank per GPU holding some heads of a layer).

The plan's one exchange is an all-gather of per-chunk zone statistics; with
sequence-sharded activations an all-to-all each way moves them to head
shards and back.  These tests check the host side (parameter validation, the
helpers over gloo with 2 and 3 ranks) without a GPU.  The GPU test that shards a layer across
ranks emulated in one process is in test_parity_gpu.py.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _params(**kw):
    from dynamic_block_sparse_zone_b200.binding import Params
    base = dict(batch=1, T=16, H=32, W=32, heads=4, head_dim=128, top_k=8, top_p=0.9)
    base.update(kw)
    return Params(**base)


def test_shard_parameters_are_validated_on_the_host():
    from dynamic_block_sparse_zone_b200 import build as b
    b.build()
    from dynamic_block_sparse_zone_b200.binding import prism_plan_bytes
    whole = prism_plan_bytes(_params(heads=8))
    half = prism_plan_bytes(_params(heads=4, heads_total=8, head_offset=4))
    assert whole > 0 and 0 < half < whole
    assert prism_plan_bytes(_params(heads=4, heads_total=8, head_offset=5)) == 0   # past heads_total
    assert prism_plan_bytes(_params(heads=4, heads_total=8, head_offset=-1)) == 0
    assert prism_plan_bytes(_params(heads=3, head_dim=64, heads_total=6, head_offset=3)) == 0  # 192 channels
    assert prism_plan_bytes(_params(heads=2, head_dim=64, heads_total=6, head_offset=2)) > 0   # whole chunks


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from dynamic_block_sparse_zone_b200.binding import exchange_zone_stats
    n = 6
    whole = torch.zeros(world * n, dtype=torch.float64)
    mine = whole[rank * n:(rank + 1) * n]
    mine.copy_(torch.arange(n, dtype=torch.float64) + 100.0 * (rank + 1))
    exchange_zone_stats(whole, mine)
    out[rank] = whole.tolist()
    dist.barrier()
    dist.destroy_process_group()


def test_zone_stat_slices_all_gather_in_rank_order_gloo_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    expect = [100.0 + i for i in range(6)] + [200.0 + i for i in range(6)]
    assert out[0] == expect and out[1] == expect


def _layout_worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from dynamic_block_sparse_zone_b200.binding import gather_sequence, heads_to_sequence, sequence_to_heads
    g = torch.Generator().manual_seed(7)
    B, N, H, D = 2, 24, 6, 4
    full = torch.randn(B, N, H, D, generator=g)
    a_full = torch.randn(B, N, generator=g)
    n, h = N // world, H // world
    mine = full[:, rank * n:(rank + 1) * n].contiguous()
    heads = sequence_to_heads(mine)
    ok = torch.equal(heads, full[:, :, rank * h:(rank + 1) * h])
    back = heads_to_sequence(heads)
    ok = ok and torch.equal(back, mine)
    a = gather_sequence(a_full[:, rank * n:(rank + 1) * n].contiguous())
    ok = ok and torch.equal(a, a_full)
    out[rank] = bool(ok)
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_head_layout_exchange_gloo(world):
    """Sequence-sharded activations to a head shard and back (one all-to-all
    each way) and the token all-gather of the audio norms, against slicing the
    whole tensors."""
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_layout_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert all(out[r] for r in range(world))
