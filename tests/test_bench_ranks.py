"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2).

The path has no exchange step: ranks are independent replicas and the only
collective is the max-over-ranks timing; whole-job throughput counts every
rank's steps against the slowest rank's time.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


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
    import bench
    ms = bench.max_over_ranks(100.0 + 50.0 * rank, world)
    out[rank] = ms
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 150.0


def test_aggregate_value_is_weak_scaling():
    import bench
    one = bench.aggregate_value(352e12, 5, 1, 2500.0)
    two = bench.aggregate_value(352e12, 5, 2, 2500.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(352e12 * 5 / 2.5 / 1e12)


def test_traffic_record_applies_only_to_its_workload():
    """The per-launch DRAM bytes of the committed ncu capture are reported only
    for the workload and size they were taken on, and only while the kernel
    source is the one captured."""
    import bench
    from dynamic_block_sparse_zone_b200.synth import WORKLOADS, scaled
    train = WORKLOADS["latent2k_train_24x96x160"]
    rec = bench.traffic_for("attn_bwd", train)
    assert rec is None or rec > 0
    assert bench.traffic_for("attn_bwd", scaled(train, heads=2)) is None
    assert bench.traffic_for("attn_bwd", WORKLOADS["latent720p_24x48x80"]) is None
    assert bench.traffic_for("attn_fwd", WORKLOADS["tiny_8x16x16"]) is None
    assert bench.traffic_for("no_such_kernel", train) is None


def test_nvidia_smi_id_follows_cuda_visible_devices(monkeypatch):
    """The clock sampler asks nvidia-smi about the GPU the process runs on:
    torch's device i is the i-th entry of CUDA_VISIBLE_DEVICES."""
    import bench
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "3,5")
    assert bench.smi_device_id(0) == "3" and bench.smi_device_id(1) == "5"
    monkeypatch.setenv("CUDA_VISIBLE_DEVICES", "GPU-1b2c, GPU-9f00")
    assert bench.smi_device_id(1) == "GPU-9f00"
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES")
    assert bench.smi_device_id(2) == "2"
