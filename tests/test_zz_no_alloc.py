"""The allocation-free entry point against the regular plan build (needs a B200).

prism_zone_shapes_noalloc serves callers that cannot call cudaMalloc (an
application whose caching allocator owns all device memory, or a loop that
cannot take cudaMalloc's implicit synchronisation); it takes its scratch from
a fixed array inside the library.  Its zone volumes and shapes must equal the
ones prism_plan_build computes, on two calls in a row (the second call reuses
the scratch the first one left behind).  This file is collected last.
"""
import pytest
import torch

from dynamic_block_sparse_zone_b200.synth import WORKLOADS, make_inputs, scaled

pytestmark = pytest.mark.gpu


def _lib():
    from dynamic_block_sparse_zone_b200 import build as b
    b.build()
    import dynamic_block_sparse_zone_b200 as P
    P.load_library()
    return P


@pytest.mark.parametrize("name", ["dynamic_16x32x32", "tiny_8x16x16", "batch2"])
def test_noalloc_matches_plan_build_twice(name):
    from dynamic_block_sparse_zone_b200.binding import prism_zone_shapes_noalloc
    P = _lib()
    if name == "batch2":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, batch=2)
    else:
        w = WORKLOADS[name]
    inp = make_inputs(w, 5)
    Q, K, V, a = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a))
    params = P.params_for(w, batch=inp.Q.shape[0])
    plan = P.PrismPlan(params)
    plan.build(Q, K, V, a)
    ref = plan.view()
    M = w.N // 512
    for _ in range(2):
        zB = torch.full((params.batch, M), -1, dtype=torch.int32, device="cuda")
        zS = torch.full((params.batch, M), -1, dtype=torch.int32, device="cuda")
        prism_zone_shapes_noalloc(params, V, a, zB, zS)
        torch.cuda.synchronize()
        assert torch.equal(zB, ref["zone_B"]), "zone volumes differ from prism_plan_build"
        assert torch.equal(zS, ref["zone_shape"]), "zone shapes differ from prism_plan_build"
    plan.close()


def test_noalloc_rejects_problems_beyond_its_scratch():
    from dynamic_block_sparse_zone_b200.binding import Params, PrismError, prism_zone_shapes_noalloc
    _lib()
    # 4 samples of a 2K grid with 64 heads of 128 needs more than the fixed scratch;
    # the call is rejected on the host before it touches the (too small) buffers
    p = Params(batch=4, T=24, H=96, W=160, heads=64, head_dim=128, top_k=1, top_p=0.5)
    tiny = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    from dynamic_block_sparse_zone_b200 import binding as B
    import ctypes
    c = p.to_c()
    st = B.load_library().prism_zone_shapes_noalloc(ctypes.byref(c), B._ptr(tiny), B._ptr(tiny), B._ptr(out),
                                                    B._ptr(out), B._stream())
    assert st == 2
    assert b"scratch" in B.load_library().prism_last_error()


def test_noalloc_rejects_a_head_shard():
    """The entry point takes the whole layer: a head shard (head_offset > 0)
    is refused, as prism_plan_create refuses heads outside heads_total."""
    from dynamic_block_sparse_zone_b200.binding import Params, PrismError, prism_zone_shapes_noalloc
    _lib()
    w = WORKLOADS["tiny_8x16x16"]
    inp = make_inputs(w, 5)
    V, a = inp.V.cuda(), inp.a.cuda()
    M = w.N // 512
    zB = torch.zeros((1, M), dtype=torch.int32, device="cuda")
    zS = torch.zeros((1, M), dtype=torch.int32, device="cuda")
    p = Params(batch=1, T=w.T, H=w.H, W=w.W, heads=w.heads, head_dim=w.head_dim, top_k=w.top_k, top_p=w.top_p,
               heads_total=0, head_offset=2)
    with pytest.raises(PrismError) as e:
        prism_zone_shapes_noalloc(p, V, a, zB, zS)
    assert e.value.status == 2
