"""Head-sharded plans run as real ranks: two processes on the one GPU, each
holding two of the layer's four heads (needs a B200).

After the zone decisions a layer's heads are independent [Prism guide,
Method sections 1-3]; the decisions need the statistics of every channel.  So
each rank computes its heads' zone statistics, the ranks all-gather them
(PrismPlan.build_sharded; here over gloo through host copies, NCCL over NVLink
on a multi-GPU node), and each finishes the plan for its heads.  The ranks'
kernels never wait on one another: the only exchanges are host-side
collectives between launches.  Every rank's plan and outputs are checked
against the fp64 oracle of the whole layer.

Two layouts are covered: ranks given their heads of every token, and ranks
given a token range of every head (sequence-sharded activations), which move
to head shards and back with one all-to-all each way.
"""
import datetime
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from dynamic_block_sparse_zone_b200.synth import WORKLOADS, bf16_bits, make_inputs, scaled
from test_parity_gpu import assert_close, check_shard_against_oracle, compare_plan, oracle_plan, sample_rows

pytestmark = pytest.mark.gpu

WORLD = 2
SEED = 12


def _workload():
    return scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=4, planted=2, backward=True)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, port, mode, outdir):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=120))
    import dynamic_block_sparse_zone_b200 as P
    from dynamic_block_sparse_zone_b200.binding import gather_sequence, heads_to_sequence, sequence_to_heads
    P.load_library()
    w = _workload()
    inp = make_inputs(w, SEED)
    hs = w.heads // WORLD
    prm = P.params_for(w)
    prm.heads, prm.heads_total, prm.head_offset = hs, w.heads, rank * hs
    plan = P.PrismPlan(prm)
    if mode == "heads":
        sl = slice(rank * hs, (rank + 1) * hs)
        Q, K, V, dO = (x[:, :, sl].contiguous().cuda() for x in (inp.Q, inp.K, inp.V, inp.dO))
        a = inp.a.cuda()
    else:  # tokens [rank n, (rank + 1) n) of every head, moved to this rank's heads of every token
        n = w.N // WORLD
        tok = slice(rank * n, (rank + 1) * n)
        Q, K, V, dO = (sequence_to_heads(x[:, tok].contiguous().cuda()) for x in (inp.Q, inp.K, inp.V, inp.dO))
        a_mine = inp.a.reshape(inp.a.shape[0], w.N)[:, tok].contiguous().cuda()
        a = gather_sequence(a_mine).reshape(inp.a.shape).contiguous()
    plan.build_sharded(Q, K, V, a)
    O, lse = plan.fwd()
    dQ, dK, dV = plan.bwd(O, dO)
    torch.cuda.synchronize()
    plan.check()
    view = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in plan.view().items()}
    out = dict(view=view, lse=lse.cpu())
    if mode == "heads":
        out.update(O=O.cpu(), dQ=dQ.cpu(), dK=dK.cpu(), dV=dV.cpu())
    else:
        out.update({k: heads_to_sequence(x).cpu() for k, x in (("O", O), ("dQ", dQ), ("dK", dK), ("dV", dV))})
    torch.save(out, os.path.join(outdir, f"rank{rank}.pt"))
    plan.close()
    dist.barrier()
    dist.destroy_process_group()


def _run_ranks(mode):
    port = _free_port()
    ctx = mp.get_context("spawn")
    with tempfile.TemporaryDirectory() as d:
        procs = [ctx.Process(target=_rank_main, args=(r, port, mode, d)) for r in range(WORLD)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(300)
        for p in procs:
            if p.is_alive():
                p.kill()
            assert p.exitcode == 0, f"rank exited with {p.exitcode}"
        return [torch.load(os.path.join(d, f"rank{r}.pt")) for r in range(WORLD)]


def test_two_ranks_build_head_shards_through_the_exchange():
    """Each rank holds its two heads of every token: its plan, O, lse, dQ, dK,
    dV against the oracle of the whole layer."""
    w = _workload()
    inp = make_inputs(w, SEED)
    pl, bits = oracle_plan(w, inp)
    dOb = bf16_bits(inp.dO[0])
    outs = _run_ranks("heads")
    hs = w.heads // WORLD
    for r, o in enumerate(outs):
        check_shard_against_oracle(w, pl, bits, dOb, o["view"], o["O"], o["lse"], (o["dQ"], o["dK"], o["dV"]),
                                   r * hs, hs, seed=80 + r)


def test_two_ranks_from_sequence_shards_and_back():
    """Each rank starts from a token range of every head: all-to-all to head
    shards, the sharded plan, forward and backward, all-to-all back.  The
    token ranges put together give the whole layer's O, dQ, dK, dV."""
    w = _workload()
    inp = make_inputs(w, SEED)
    pl, bits = oracle_plan(w, inp)
    dOb = bf16_bits(inp.dO[0])
    outs = _run_ranks("sequence")
    hs = w.heads // WORLD
    for r, o in enumerate(outs):
        heads = list(range(r * hs, (r + 1) * hs))
        from test_parity_gpu import _select_heads
        compare_plan(w, _select_heads(pl, heads), o["view"], heads=heads, view_head0=r * hs, view_heads=hs)
    full = {k: torch.cat([o[k] for o in outs], dim=1) for k in ("O", "dQ", "dK", "dV")}
    for k in full:
        assert full[k].shape == inp.Q.shape
    rs = np.random.default_rng(90)
    req_h, req_t = sample_rows(rs, w, 512)
    O_ref, _ = oracle.attn_fwd_rows(pl, *bits, req_h, req_t)
    assert_close("O(seq shards)", full["O"][0].float().numpy()[req_t, req_h], O_ref)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h[:256], req_t[:256])
    assert_close("dQ(seq shards)", full["dQ"][0].float().numpy()[req_t[:256], req_h[:256]], dQ_ref)
    req_h, req_t = sample_rows(rs, w, 128)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dK(seq shards)", full["dK"][0].float().numpy()[req_t, req_h], dK_ref)
    assert_close("dV(seq shards)", full["dV"][0].float().numpy()[req_t, req_h], dV_ref)
