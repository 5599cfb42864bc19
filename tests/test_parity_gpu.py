"""CUDA path vs the fp64 oracle, through the C ABI (needs a B200).

Plans (zone volumes and shapes, permutation, block table, selected-block CSR)
must match exactly; a mismatch is accepted only where the oracle shows a
near-tie below 1e-6 (two shape distances, the density against a threshold,
the logits at the selection cut, or the cumulative mass against p), and such
cases are counted.  Attention outputs and gradients must be within max-abs
2e-2 and relative-L2 1e-2 of the oracle (bf16 inputs, fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_zone_b200.synth import WORKLOADS, bf16_bits, make_inputs, scaled

pytestmark = pytest.mark.gpu

TIE = 1e-6
ATOL = 2e-2
RTOL_L2 = 1e-2


def _f32(x):
    return float(np.float32(x))


def _lib():
    from dynamic_block_sparse_zone_b200 import build as b
    b.build()
    import dynamic_block_sparse_zone_b200 as P
    P.load_library()
    return P


def run_gpu(w, inp, backward=False, zone_decisions=None):
    """The GPU path on inp; zone_decisions = (zone_B, zone_shape) [batch, M]
    builds from given decisions instead of the zone statistics."""
    P = _lib()
    plan = P.PrismPlan(P.params_for(w, batch=inp.Q.shape[0]))
    Q, K, V, a = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a))
    if zone_decisions is None:
        plan.build(Q, K, V, a)
    else:
        plan.build_with_zones(Q, K, V, zone_decisions[0], zone_decisions[1])
    O, lse = plan.fwd()
    out = dict(O=O, lse=lse)
    if backward:
        dO = inp.dO.cuda()
        out["dQ"], out["dK"], out["dV"] = plan.bwd(O, dO)
    torch.cuda.synchronize()
    plan.check()
    out["view"] = plan.view()
    out["plan"] = plan
    out["_rerun"] = (w, inp, backward)  # what compare_plan needs to rebuild after a near-tie flip
    return out


def oracle_plan(w, inp, b=0, heads=None, zone_decisions=None):
    Qb, Kb, Vb = (bf16_bits(x[b]) for x in (inp.Q, inp.K, inp.V))
    pl = oracle.plan(Qb, Kb, Vb, inp.a[b].cpu().numpy(), w.T, w.H, w.W, w.heads, w.head_dim, w.top_k,
                     _f32(w.top_p), _f32(w.max_frac), fixed_shape=w.fixed_shape, with_select=heads is None,
                     zone_decisions=zone_decisions)
    if heads is not None:  # selection of a few heads only (heads are independent)
        cnt, cols, diag = oracle.select(pl.Qbar[heads], pl.Kbar[heads], w.top_k, _f32(w.top_p), _f32(w.max_frac))
        pl.cnt, pl.cols, pl.diag = cnt, cols, diag
    return pl, (Qb, Kb, Vb)


def valid_selection(w, pl, h, i, g_set):
    """A selection row that differs from the oracle's at a near-tie must still
    be a correct S_i = Top-k U Top-p under the oracle's fp64 pooled scores
    [Prism guide, Method section 3]: a prefix of the order (z descending, j
    ascending) up to ties below 1e-6, at least min(k, N_b) long, its softmax
    mass >= p unless it stops at the cap, and no longer than needed (dropping
    its last block falls below p, unless it is the Top-k prefix)."""
    nb = pl.nb
    z = pl.Qbar[h, i] @ pl.Kbar[h, :nb].T / np.sqrt(w.head_dim)
    P = np.exp(z - z.max())
    P /= P.sum()
    n = len(g_set)
    kk = min(w.top_k, nb)
    cap_ = oracle.cap(nb, w.top_k, _f32(w.max_frac)) if w.max_frac > 0 else nb
    assert np.all(np.diff(g_set) > 0) and np.all((g_set >= 0) & (g_set < nb)), "not an ascending block list"
    assert kk <= n <= cap_, f"{n} blocks, Top-k {kk}, cap {cap_}"
    inside = np.zeros(nb, bool)
    inside[g_set] = True
    if n < nb:
        assert z[inside].min() >= z[~inside].max() - TIE, "not a prefix of the descending order"
    mass = P[inside].sum()
    assert mass >= _f32(w.top_p) - TIE or n == cap_, f"mass {mass} below p"
    if n > kk:
        assert mass - P[inside].min() < _f32(w.top_p) + TIE, "longer than the Top-p prefix"


def _rebuild_with_oracle_decisions(g, pl, b):
    """After a zone decision flipped at an oracle near-tie: rebuild the GPU plan
    from the oracle's decisions for sample b (the GPU's own for the other
    samples), so that everything downstream is still compared."""
    w, inp, backward = g["_rerun"]
    v = g["view"]
    zB = v["zone_B"].cpu().numpy().copy()
    zs = v["zone_shape"].cpu().numpy().copy()
    zB[b], zs[b] = pl.zone_B, pl.zone_shape
    g["plan"].close()
    g.update(run_gpu(w, inp, backward, zone_decisions=(zB, zs)))


def compare_plan(w, pl, g, b=0, heads=None, view_head0=0, view_heads=None):
    """Exact plan parity with counted near-ties.  g is run_gpu's dict (or a bare
    view of a plan that cannot flip: given decisions).  view_head0 / view_heads:
    the view is a head shard holding heads [view_head0, view_head0 + view_heads).
    Returns the tie counters."""
    view = g["view"] if "view" in g else g
    ties = dict(shape=0, rho=0, select=0, rebuilt=0)
    zB = view["zone_B"][b].cpu().numpy()
    zs = view["zone_shape"][b].cpu().numpy()
    bad = np.nonzero((zB != pl.zone_B) | (zs != pl.zone_shape))[0]
    for m in bad:
        assert pl.gap_shape[m] < TIE or pl.gap_rho[m] < TIE, f"zone {m}: gpu {zB[m]}/{zs[m]} oracle " \
            f"{pl.zone_B[m]}/{pl.zone_shape[m]} (gaps {pl.gap_shape[m]}, {pl.gap_rho[m]})"
    ties["shape"] = int(np.sum(pl.gap_shape < TIE))
    ties["rho"] = int(np.sum(pl.gap_rho < TIE))
    if len(bad):
        assert "_rerun" in g, f"{len(bad)} zone decision(s) flipped at a near-tie in a plan that cannot be rebuilt"
        _rebuild_with_oracle_decisions(g, pl, b)
        view = g["view"]
        ties["rebuilt"] = len(bad)
        assert np.array_equal(view["zone_shape"][b].cpu().numpy(), pl.zone_shape)
    assert view["n_blocks"][b] == pl.nb
    np.testing.assert_array_equal(view["blk_off"][b, : pl.nb + 1].cpu().numpy(), pl.blk_off())
    np.testing.assert_array_equal(view["perm"][b].cpu().numpy(), pl.perm)
    rp = view["row_ptr"].cpu().numpy()
    col = view["col_idx"].cpu().numpy()
    nbmax = view["nbmax"]
    vh = w.heads if view_heads is None else view_heads
    hs = range(w.heads) if heads is None else heads
    for hi, h in enumerate(hs):
        for i in range(pl.nb):
            r = (b * vh + (h - view_head0)) * nbmax + i
            g_set = col[rp[r]:rp[r + 1]]
            o_set = pl.cols[hi, i, : pl.cnt[hi, i]]
            if len(g_set) != len(o_set) or np.any(g_set != o_set):
                d = pl.diag[hi, i]
                assert d[0] < TIE or d[1] < TIE, f"head {h} row {i}: selection differs without a near-tie"
                valid_selection(w, pl, h, i, g_set)
                ties["select"] += 1
            assert np.all(np.diff(g_set) > 0)
    return ties


def bf16_half_ulp(x):
    """Half a bf16 unit in the last place at |x| (8 significant bits)."""
    ax = np.abs(x)
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, np.exp2(e - 8), 0.0)


def _err(gpu, ref):
    """(max-abs error beyond the bf16 rounding of the output itself, relative
    L2 error, raw max-abs error).  Outputs are stored in bf16, so a value of
    magnitude in [4, 8) can be off by up to 2^-6 from rounding alone; the
    max-abs bound applies to what the arithmetic adds on top of that."""
    gpu = gpu.astype(np.float64)
    raw = np.abs(gpu - ref)
    diff = np.maximum(raw - bf16_half_ulp(ref), 0.0)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    return float(diff.max()), float(rel), float(raw.max())


def assert_close(name, gpu, ref):
    from conftest import record_error
    mx, rel, raw = _err(gpu, ref)
    record_error(name, raw, mx, rel)
    assert mx <= ATOL and rel <= RTOL_L2, f"{name}: max-abs {mx:.3e} (raw {raw:.3e}) rel-L2 {rel:.3e}"
    return mx, rel


def sample_rows(rs, w, n, heads=None):
    hs = np.arange(w.heads) if heads is None else np.asarray(heads)
    req_h = rs.choice(hs, size=n).astype(np.int32)
    req_t = rs.integers(0, w.N, size=n).astype(np.int32)
    return req_h, req_t


def check_forward(w, inp, g, pl, bits, nrows, heads=None, b=0):
    rs = np.random.default_rng(11)
    req_h, req_t = sample_rows(rs, w, nrows, heads)
    Qb, Kb, Vb = bits
    # the oracle's selection arrays are indexed by position in `heads`
    ho = req_h if heads is None else np.searchsorted(np.asarray(heads), req_h).astype(np.int32)
    pl_h = pl if heads is None else _heads_view(pl, heads)
    O_ref, lse_ref = oracle.attn_fwd_rows(pl_h, *_head_slice(bits, heads), ho, req_t)
    O = g["O"][b].float().cpu().numpy()[req_t, req_h]
    assert_close("O", O, O_ref)
    lse = g["lse"][b].cpu().numpy()[req_h, req_t]
    assert np.max(np.abs(lse - lse_ref)) < 2e-3
    return req_h, req_t


def check_forward_taylor(w, plan, pl, bits, nrows, heads=None, b=0, out=None):
    """prism_attn_fwd_taylor against the oracle's forward with the zeroth-order
    Taylor term for the blocks outside S_i, on sampled rows (out: the (O, lse)
    of an earlier call)."""
    O, lse = plan.fwd(taylor=True) if out is None else out
    torch.cuda.synchronize()
    plan.check()
    rs = np.random.default_rng(12)
    req_h, req_t = sample_rows(rs, w, nrows, heads)
    ho = req_h if heads is None else np.searchsorted(np.asarray(heads), req_h).astype(np.int32)
    pl_h = pl if heads is None else _heads_view(pl, heads)
    O_ref, lse_ref = oracle.attn_fwd_taylor_rows(pl_h, *_head_slice(bits, heads), ho, req_t)
    res = assert_close("O(taylor)", O[b].float().cpu().numpy()[req_t, req_h], O_ref)
    assert np.max(np.abs(lse[b].cpu().numpy()[req_h, req_t] - lse_ref)) < 2e-3
    return res


def _heads_view(pl, heads):
    import copy
    p2 = copy.copy(pl)
    p2.heads = len(heads)
    return p2


def _head_slice(bits, heads):
    if heads is None:
        return bits
    return tuple(np.ascontiguousarray(x[:, heads, :]) for x in bits)


# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny_8x16x16", "dynamic_16x32x32"])
def test_plan_and_forward_parity(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, 0)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    ties = compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 4096 if w.N <= 4096 else 1536)
    print(name, "near-ties", ties)


def test_tiny_forward_all_rows():
    w = WORKLOADS["tiny_8x16x16"]
    inp = make_inputs(w, 3)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    req_h = np.repeat(np.arange(w.heads), w.N).astype(np.int32)
    req_t = np.tile(np.arange(w.N), w.heads).astype(np.int32)
    O_ref, lse_ref = oracle.attn_fwd_rows(pl, *bits, req_h, req_t)
    O = g["O"][0].float().cpu().numpy()[req_t, req_h]
    assert_close("O", O, O_ref)


def pick_dkv_rows(pl, hi, nblocks, per_block, rs, most=False):
    """Key tokens from the `nblocks` key blocks of oracle head index `hi` that
    the fewest query blocks selected (their dK/dV are cheap to compute one by
    one: only those query blocks contribute), or with most=True the ones the
    most query blocks selected (the longest columns of the backward)."""
    counts = np.zeros(pl.nb, np.int64)
    for i in range(pl.nb):
        counts[pl.cols[hi, i, : pl.cnt[hi, i]]] += 1
    cand = np.nonzero(counts)[0]
    order = np.argsort(counts[cand], kind="stable")
    chosen = cand[order[::-1][:nblocks] if most else order[:nblocks]]
    off = pl.blk_off()
    toks = []
    for j in chosen:
        blk = pl.perm[off[j]:off[j + 1]]
        toks.extend(rs.choice(blk, size=min(per_block, len(blk)), replace=False))
    toks = np.asarray(toks, np.int32)
    return np.full(len(toks), hi, np.int32), toks


def _select_heads(pl, heads):
    """The oracle plan with its selection arrays cut to `heads` (a plan whose
    selection covers every head of the layer)."""
    import copy
    p2 = copy.copy(pl)
    p2.cnt, p2.cols, p2.diag = pl.cnt[heads], pl.cols[heads], pl.diag[heads]
    return p2


def check_shard_against_oracle(w, pl, bits, dOb, v, O, lse, grads, head_lo, hs, seed, nrows=384):
    """A head shard holding heads [head_lo, head_lo + hs) of the layer against
    the oracle's plan of the whole layer (pl: every head selected): zone
    decisions, permutation, block table and its heads' selection rows exactly,
    and O, lse and (grads given) dQ, dK, dV on sampled rows within the
    tolerance."""
    heads = list(range(head_lo, head_lo + hs))
    compare_plan(w, _select_heads(pl, heads), v, heads=heads, view_head0=head_lo, view_heads=hs)
    rs = np.random.default_rng(seed)
    req_h, req_t = sample_rows(rs, w, nrows, heads)
    O_ref, lse_ref = oracle.attn_fwd_rows(pl, *bits, req_h, req_t)
    assert_close("O(shard)", O[0].float().cpu().numpy()[req_t, req_h - head_lo], O_ref)
    assert np.max(np.abs(lse[0].cpu().numpy()[req_h - head_lo, req_t] - lse_ref)) < 2e-3
    if grads is None:
        return
    dQ, dK, dV = (x[0].float().cpu().numpy() for x in grads)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h[:256], req_t[:256])
    assert_close("dQ(shard)", dQ[req_t[:256], req_h[:256] - head_lo], dQ_ref)
    req_h, req_t = sample_rows(rs, w, 128, heads)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dK(shard)", dK[req_t, req_h - head_lo], dK_ref)
    assert_close("dV(shard)", dV[req_t, req_h - head_lo], dV_ref)


@pytest.mark.parametrize("name", ["tiny_8x16x16", "dynamic_small_d64", "dynamic_16x32x32"])
def test_backward_parity(name):
    if name == "dynamic_small_d64":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=3, head_dim=64, planted=2)
    else:
        w = WORKLOADS[name]
    w = scaled(w, backward=True)
    inp = make_inputs(w, 1)
    g = run_gpu(w, inp, backward=True)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    dOb = bf16_bits(inp.dO[0])
    rs = np.random.default_rng(5)
    n = 1024 if w.N <= 4096 else 384
    req_h, req_t = sample_rows(rs, w, n)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dQ", g["dQ"][0].float().cpu().numpy()[req_t, req_h], dQ_ref)
    if w.N <= 4096:
        req_h, req_t = sample_rows(rs, w, n // 2)
    else:
        req_h, req_t = pick_dkv_rows(pl, 1, 3, 8, rs)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dK", g["dK"][0].float().cpu().numpy()[req_t, req_h], dK_ref)
    assert_close("dV", g["dV"][0].float().cpu().numpy()[req_t, req_h], dV_ref)
    check_gradient_sums(g, inp)


# ---------------------------------------------------------------------------
# Stage-wise parity: the steps after the zone decisions, fed given decisions
# (prism_plan_build_with_zones), so that a decision flipped at a near-tie
# upstream cannot hide a fault downstream, and every candidate shape is used.
# ---------------------------------------------------------------------------
def _small_d64():
    return scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=3, head_dim=64, planted=2)


def _random_zone_decisions(w, seed):
    """Seeded shapes drawn uniformly over the 16 candidates, one per zone, and
    their volumes."""
    rs = np.random.default_rng(seed)
    table = oracle.shape_table()
    zs = rs.integers(0, len(table), size=w.N // 512).astype(np.int32)
    return (1 << table[zs].sum(axis=1)).astype(np.int32), zs


def run_gpu_given(w, inp, zB, zs, backward=False):
    P = _lib()
    plan = P.PrismPlan(P.params_for(w, batch=1))
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    plan.build_with_zones(Q, K, V, zB[None], zs[None])
    O, lse = plan.fwd()
    out = dict(O=O, lse=lse)
    if backward:
        out["dQ"], out["dK"], out["dV"] = plan.bwd(O, inp.dO.cuda())
    torch.cuda.synchronize()
    plan.check()
    out["view"] = plan.view()
    return out


@pytest.mark.parametrize("name", ["dynamic_16x32x32", "dynamic_small_d64"])
def test_stagewise_plan_from_the_oracle_decisions(name):
    w = WORKLOADS[name] if name in WORKLOADS else _small_d64()
    inp = make_inputs(w, 4)
    pl, bits = oracle_plan(w, inp)
    g = run_gpu_given(w, inp, pl.zone_B, pl.zone_shape)
    compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 1536)


@pytest.mark.parametrize("name,seed", [("dynamic_16x32x32", 31), ("dynamic_small_d64", 32), ("tiny_8x16x16", 33)])
def test_plan_from_random_zone_decisions_forward_backward(name, seed):
    w = scaled(WORKLOADS[name] if name in WORKLOADS else _small_d64(), backward=True)
    inp = make_inputs(w, seed)
    zB, zs = _random_zone_decisions(w, seed)
    pl, bits = oracle_plan(w, inp, zone_decisions=(zB, zs))
    g = run_gpu_given(w, inp, zB, zs, backward=True)
    assert np.array_equal(g["view"]["zone_shape"][0].cpu().numpy(), zs)
    compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 1536)
    dOb = bf16_bits(inp.dO[0])
    rs = np.random.default_rng(seed)
    req_h, req_t = sample_rows(rs, w, 512)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dQ", g["dQ"][0].float().cpu().numpy()[req_t, req_h], dQ_ref)
    req_h, req_t = sample_rows(rs, w, 256)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dK", g["dK"][0].float().cpu().numpy()[req_t, req_h], dK_ref)
    assert_close("dV", g["dV"][0].float().cpu().numpy()[req_t, req_h], dV_ref)


def test_batch_two_from_given_zone_decisions():
    """Two samples with their own given decisions (so their own block counts):
    each sample's plan and forward match the oracle fed that sample's
    decisions."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, batch=2)
    inp = make_inputs(w, 8)
    dec = [_random_zone_decisions(w, 51 + b) for b in range(2)]
    plan = P.PrismPlan(P.params_for(w))
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    plan.build_with_zones(Q, K, V, np.stack([d[0] for d in dec]), np.stack([d[1] for d in dec]))
    O, lse = plan.fwd()
    torch.cuda.synchronize()
    plan.check()
    g = dict(O=O, lse=lse, view=plan.view())
    nbs = []
    for b in range(2):
        pl, bits = oracle_plan(w, inp, b=b, zone_decisions=dec[b])
        compare_plan(w, pl, g, b=b)
        check_forward(w, inp, g, pl, bits, 512, b=b)
        nbs.append(pl.nb)
    assert nbs[0] != nbs[1]  # the samples' block tables differ


def test_build_with_zones_rejections():
    P = _lib()
    w = WORKLOADS["dynamic_16x32x32"]
    inp = make_inputs(w, 2)
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    zB, zs = _random_zone_decisions(w, 3)
    plan = P.PrismPlan(P.params_for(w))
    for mutate in (lambda b, s: b.__setitem__(3, 96),                      # not a volume
                   lambda b, s: b.__setitem__(5, 64 if b[5] != 64 else 128),  # volume differs from the shape's
                   lambda b, s: s.__setitem__(7, 16),                      # outside the table
                   lambda b, s: s.__setitem__(0, -1)):
        b2, s2 = zB.copy(), zs.copy()
        mutate(b2, s2)
        with pytest.raises(P.PrismError) as e:
            plan.build_with_zones(Q, K, V, b2[None], s2[None])
        assert e.value.status == 1 and "zone" in str(e.value)
    with pytest.raises(P.PrismError) as e:  # refused entries build nothing: still no plan
        plan.fwd()
    assert e.value.status == 6
    plan.build_with_zones(Q, K, V, zB[None], zs[None])  # the plan stays usable
    plan.fwd()
    torch.cuda.synchronize()
    plan.check()
    hp = P.PrismPlan(P.params_for(w, hilbert_block=128))
    with pytest.raises(P.PrismError) as e:
        hp.build_with_zones(Q, K, V, zB[None], zs[None])
    assert e.value.status == 6


def test_head_shards_built_from_given_zone_decisions():
    """Head shards built from the same given decisions (no statistics, no
    exchange) hold the whole layer's plan: identical permutation and block
    table, their heads' selections, and bit-identical forward outputs."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=4, planted=2, backward=True)
    inp = make_inputs(w, 6)
    Q, K, V, dO = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.dO))
    zB, zs = _random_zone_decisions(w, 41)
    pl, bits = oracle_plan(w, inp, zone_decisions=(zB, zs))
    dOb = bf16_bits(inp.dO[0])
    whole = P.PrismPlan(P.params_for(w))
    whole.build_with_zones(Q, K, V, zB[None], zs[None])
    O_all, lse_all = whole.fwd()
    v_all = whole.view()
    torch.cuda.synchronize()
    hs = 2
    for r in range(2):
        prm = P.params_for(w)
        prm.heads, prm.heads_total, prm.head_offset = hs, w.heads, r * hs
        plan = P.PrismPlan(prm)
        sl = slice(r * hs, (r + 1) * hs)
        Qr, Kr, Vr = (x[:, :, sl].contiguous() for x in (Q, K, V))
        plan.build_with_zones(Qr, Kr, Vr, zB[None], zs[None])
        O_r, lse_r = plan.fwd()
        grads = plan.bwd(O_r, dO[:, :, sl].contiguous())
        torch.cuda.synchronize()
        plan.check()
        v = plan.view()
        check_shard_against_oracle(w, pl, bits, dOb, v, O_r, lse_r, grads, r * hs, hs, seed=60 + r)
        for key in ("zone_B", "zone_shape", "perm"):
            assert torch.equal(v[key], v_all[key]), key
        nb = int(v["n_blocks"][0])
        assert nb == int(v_all["n_blocks"][0])
        assert torch.equal(v["blk_off"][:, :nb + 1], v_all["blk_off"][:, :nb + 1])
        rp, rp_all = v["row_ptr"].cpu().numpy(), v_all["row_ptr"].cpu().numpy()
        col, col_all = v["col_idx"].cpu().numpy(), v_all["col_idx"].cpu().numpy()
        nbmax = v["nbmax"]
        for hh in range(hs):
            for i in range(nb):
                ra, rb = hh * nbmax + i, (r * hs + hh) * nbmax + i
                assert np.array_equal(col[rp[ra]:rp[ra + 1]], col_all[rp_all[rb]:rp_all[rb + 1]])
        assert torch.equal(O_r, O_all[:, :, sl])
        assert torch.equal(lse_r, lse_all[:, sl])
        plan.close()
    whole.close()


def check_gradient_sums(g, inp, b=0):
    """Properties of softmax attention at any size: for every query the dS row
    sums to zero, so sum_t dK_t = 0; the P row sums to one, so
    sum_t dV_t = sum_q dO_q (per head, over the whole sequence).

    The kernels form Delta_q = dO_q . O_q from the bf16-rounded O, so each dS
    row sums to -dDelta_q instead of 0, with dDelta_q of standard deviation at
    most 2^-8/sqrt(3) |dO_q * O_q|.  Hence sum_t dK_t has standard deviation
    at most scale 2^-8/sqrt(3) sqrt(sum_q |dO_q * O_q|^2 Q_qc^2) per channel;
    the bound is six of those plus 2% of |dK| for the bf16 rounding of dS."""
    dK = g["dK"][b].double()
    dV = g["dV"][b].double()
    dev = dK.device
    dO = inp.dO[b].to(dev).double()
    O = g["O"][b].double()
    Q = inp.Q[b].to(dev).double()
    scale = 1.0 / np.sqrt(Q.shape[-1])
    w2 = ((dO * O) ** 2).sum(-1, keepdim=True)                 # [N, heads, 1]
    sigma = scale * 2.0 ** -8 / np.sqrt(3.0) * torch.sqrt((w2 * Q * Q).sum(0))
    sk = dK.sum(0)
    bound = 6.0 * sigma + 0.02 * dK.norm(dim=0) + 1e-3
    assert torch.all(sk.abs() <= bound), float((sk.abs() / bound).max())
    sv, so = dV.sum(0), dO.sum(0)
    assert torch.all((sv - so).abs() <= 0.02 * dV.norm(dim=0) + 1e-3), float((sv - so).abs().max())


def test_batch_two_samples_are_independent():
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, head_dim=128, planted=2, batch=2)
    inp = make_inputs(w, 4)
    g = run_gpu(w, inp)
    for b in range(2):
        pl, bits = oracle_plan(w, inp, b=b)
        compare_plan(w, pl, g, b=b)
        check_forward(w, inp, g, pl, bits, 512, b=b)


def test_all_blocks_selected_is_dense_attention():
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=16, heads=2, top_k=10 ** 6, planted=1)
    inp = make_inputs(w, 2)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    assert np.all(pl.cnt == pl.nb)
    q, k, v = (x[0].cuda().float().transpose(0, 1) for x in (inp.Q, inp.K, inp.V))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v).transpose(0, 1)
    assert_close("O(dense)", g["O"][0].float().cpu().numpy(), ref.double().cpu().numpy())


@pytest.mark.parametrize("top_p,k", [(1.0, 1), (0.05, 1), (0.5, 3)])
def test_selection_edge_parameters(top_p, k):
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, top_k=k, top_p=top_p, planted=2)
    inp = make_inputs(w, 6)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 512)


def test_constant_inputs_degenerate_zones():
    """Constant V and a = 0: every zone isotropic and coarsest (256, 4x8x8 first)."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=16, heads=2, head_dim=64, planted=0)
    inp = make_inputs(w, 7)
    inp.V = torch.full_like(inp.V, 0.25)
    inp.a = torch.zeros_like(inp.a)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    assert np.all(pl.zone_B == 256)
    compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 512)


@pytest.mark.slow
def test_latent720p_full_size():
    w = WORKLOADS["latent720p_24x48x80"]
    inp = make_inputs(w, 0, device="cuda")
    g = run_gpu(w, inp)
    heads = [0, 13]
    pl, bits = oracle_plan(w, inp, heads=heads)
    ties = compare_plan(w, pl, g, heads=heads)
    check_forward(w, inp, g, pl, bits, 256, heads=heads)
    check_forward_taylor(w, g["plan"], pl, bits, 128, heads=heads)
    print("720p near-ties", ties, "blocks", pl.nb)


@pytest.mark.slow
def test_latent2k_train_full_size_sampled():
    """2K grid, forward and backward in the benchmark's configuration; plan on 2
    heads, outputs and gradients on sampled rows of 1 head."""
    w = WORKLOADS["latent2k_train_24x96x160"]
    inp = make_inputs(w, 0, device="cuda")
    g = run_gpu(w, inp, backward=True)
    heads = [5]
    pl, bits = oracle_plan(w, inp, heads=heads)
    ties = compare_plan(w, pl, g, heads=heads)
    check_forward(w, inp, g, pl, bits, 96, heads=heads)
    dOb = bf16_bits(inp.dO[0])
    rs = np.random.default_rng(9)
    req_t = rs.integers(0, w.N, size=48).astype(np.int32)
    zero = np.zeros(len(req_t), np.int32)
    hb = _head_slice(bits, heads)
    dOs = np.ascontiguousarray(dOb[:, heads, :])
    ph = _heads_view(pl, heads)
    dQ_ref = oracle.attn_bwd_dq_rows(ph, *hb, dOs, zero, req_t)
    assert_close("dQ", g["dQ"][0].float().cpu().numpy()[req_t, heads[0]], dQ_ref)
    req_h, req_t = pick_dkv_rows(ph, 0, 2, 8, rs)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(ph, *hb, dOs, req_h, req_t)
    assert_close("dK", g["dK"][0].float().cpu().numpy()[req_t, heads[0]], dK_ref)
    assert_close("dV", g["dV"][0].float().cpu().numpy()[req_t, heads[0]], dV_ref)
    # and the longest column: 8 tokens of the key block the most query blocks selected
    req_h, req_t = pick_dkv_rows(ph, 0, 1, 8, rs, most=True)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(ph, *hb, dOs, req_h, req_t)
    assert_close("dK(longest)", g["dK"][0].float().cpu().numpy()[req_t, heads[0]], dK_ref)
    assert_close("dV(longest)", g["dV"][0].float().cpu().numpy()[req_t, heads[0]], dV_ref)
    check_gradient_sums(g, inp)
    check_forward_taylor(w, g["plan"], pl, bits, 64, heads=heads)
    print("2K near-ties", ties, "blocks", pl.nb)


def test_bounded_wait_reports_timeout_and_context_stays_usable():
    """A device wait that nothing satisfies gives up, the host reads
    PRISM_ERR_TIMEOUT, the status clears, and the plan keeps working."""
    import time
    from dynamic_block_sparse_zone_b200.binding import PrismError
    w = WORKLOADS["tiny_8x16x16"]
    inp = make_inputs(w, 0)
    g = run_gpu(w, inp)
    plan = g["plan"]
    t0 = time.time()
    plan.selftest_timeout()
    with pytest.raises(PrismError) as ei:
        plan.check()
    assert ei.value.status == 4 and "wait gave up" in str(ei.value)
    assert time.time() - t0 < 60
    plan.check()  # cleared
    Q, K, V, a = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a))
    plan.build(Q, K, V, a)
    O, _ = plan.fwd()
    torch.cuda.synchronize()
    plan.check()
    assert torch.equal(O, g["O"])


EDGE_CASES = {
    # fixed non-cubic shapes (volume 64 and 256) exercise the fixed-shape path
    "fixed_2x4x8": scaled(WORKLOADS["tiny_8x16x16"], fixed_shape=(2, 4, 8)),
    "fixed_8x8x4": scaled(WORKLOADS["tiny_8x16x16"], T=16, fixed_shape=(8, 8, 4), top_k=1),
    # one zone, one head: the smallest problem (8 to 2 blocks)
    "single_zone": scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=8, W=8, heads=1, planted=0, top_k=1, top_p=0.5),
    # cap equal to k (max_frac so small that floor(frac * N_b) < k)
    "cap_is_k": scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, top_k=3, top_p=0.99,
                       max_frac=0.01),
    # cap binding at head_dim 64
    "cap_d64": scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, head_dim=64, planted=2, top_k=2,
                      top_p=0.95, max_frac=0.1),
    # 1280 channels: the permute-and-pool kernel's second 1024-channel slice is a quarter full
    "ragged_channel_slice": scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=10, planted=2),
}


@pytest.mark.parametrize("name", sorted(EDGE_CASES))
def test_edge_case_plans_and_forward(name):
    w = EDGE_CASES[name]
    inp = make_inputs(w, 8)
    g = run_gpu(w, inp)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    if w.max_frac > 0:
        cap = oracle.cap(pl.nb, w.top_k, _f32(w.max_frac))
        assert pl.cnt.max() <= cap
    check_forward(w, inp, g, pl, bits, min(512, w.N * w.heads))


def test_capped_backward():
    w = scaled(EDGE_CASES["cap_is_k"], backward=True)
    inp = make_inputs(w, 9)
    g = run_gpu(w, inp, backward=True)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    dOb = bf16_bits(inp.dO[0])
    rs = np.random.default_rng(3)
    req_h, req_t = sample_rows(rs, w, 256)
    assert_close("dQ", g["dQ"][0].float().cpu().numpy()[req_t, req_h],
                 oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h, req_t))
    req_h, req_t = sample_rows(rs, w, 128)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close("dK", g["dK"][0].float().cpu().numpy()[req_t, req_h], dK_ref)
    assert_close("dV", g["dV"][0].float().cpu().numpy()[req_t, req_h], dV_ref)


def test_plan_reuse_with_new_inputs():
    """prism_plan_update_qkv keeps the plan of the first inputs and attends with
    the second: compare with the oracle's plan of the first inputs applied to
    the second inputs' Q, K, V."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, backward=True)
    first = make_inputs(w, 21)
    second = make_inputs(w, 22)
    P = _lib()
    plan = P.PrismPlan(P.params_for(w))
    plan.build(*(x.cuda() for x in (first.Q, first.K, first.V, first.a)))
    with pytest.raises(P.PrismError):
        plan.bwd(torch.zeros_like(first.Q).cuda(), first.dO.cuda())  # no forward yet
    plan.update_qkv(*(x.cuda() for x in (second.Q, second.K, second.V)))
    O, lse = plan.fwd()
    dQ, dK, dV = plan.bwd(O, second.dO.cuda())
    torch.cuda.synchronize()
    plan.check()
    pl, _ = oracle_plan(w, first)
    compare_plan(w, pl, plan.view())
    bits2 = tuple(bf16_bits(x[0]) for x in (second.Q, second.K, second.V))
    rs = np.random.default_rng(4)
    req_h, req_t = sample_rows(rs, w, 512)
    O_ref, _ = oracle.attn_fwd_rows(pl, *bits2, req_h, req_t)
    assert_close("O", O[0].float().cpu().numpy()[req_t, req_h], O_ref)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits2, bf16_bits(second.dO[0]), req_h[:128], req_t[:128])
    assert_close("dQ", dQ[0].float().cpu().numpy()[req_t[:128], req_h[:128]], dQ_ref)
    # the Taylor term pools the second inputs' keys and values under the first plan
    check_forward_taylor(w, plan, pl, bits2, 512)


def test_host_steps_match_the_device_path():
    """Pipelined steps from page-locked host buffers (prism_step_host) give the
    outputs of prism_plan_build + prism_attn_fwd + prism_attn_bwd on device
    tensors: forward outputs, lse, dK and dV bit for bit (same kernels, same
    order), dQ up to the order of its fp32 reduce-adds.  Ten steps cycle the
    two staging sets and wrap the ring of eight completion events."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, backward=True)
    inputs = [make_inputs(w, seed, with_grad_output=True) for seed in range(3)]
    refs = []
    plan = P.PrismPlan(P.params_for(w))
    for inp in inputs:
        Q, K, V, a, dO = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a, inp.dO))
        plan.build(Q, K, V, a)
        O, lse = plan.fwd()
        dQ, dK, dV = plan.bwd(O, dO)
        refs.append([t.cpu() for t in (O, lse, dQ, dK, dV)])
    torch.cuda.synchronize()
    plan.check()

    shp, lshp = inputs[0].Q.shape, refs[0][1].shape
    pin = [[x.pin_memory() for x in (inp.Q, inp.K, inp.V, inp.a, inp.dO)] for inp in inputs]
    outs, tickets = [], []
    for step in range(10):
        k = step % 3
        bwd = step % 4 != 3  # some forward-only steps
        O = torch.empty(shp, dtype=torch.bfloat16).pin_memory()
        lse = torch.empty(lshp, dtype=torch.float32).pin_memory() if step % 2 == 0 else None
        grads = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(3)] if bwd else [None] * 3
        Q, K, V, a, dO = pin[k]
        tickets.append(plan.step_host(Q, K, V, a, O, lse=lse, dO=dO if bwd else None,
                                      dQ=grads[0], dK=grads[1], dV=grads[2]))
        outs.append((k, bwd, O, lse, grads))
    assert tickets == list(range(1, 11))
    plan.step_wait(tickets[-1])
    plan.check()
    for k, bwd, O, lse, (dQ, dK, dV) in outs:
        rO, rl, rdQ, rdK, rdV = refs[k]
        assert torch.equal(O, rO)
        if lse is not None:
            assert torch.equal(lse, rl)
        if bwd:
            assert torch.equal(dK, rdK) and torch.equal(dV, rdV)
            assert torch.allclose(dQ.float(), rdQ.float(), rtol=1e-2, atol=1e-3)
    with pytest.raises(P.PrismError):
        plan.step_wait(11)
    with pytest.raises(P.PrismError):
        plan.step_wait(0)
    plan.step_wait(1)  # long completed: fine
    # a forward-only step with the Taylor term equals prism_attn_fwd_taylor
    Q, K, V, a, dO = pin[1]
    O = torch.empty(shp, dtype=torch.bfloat16).pin_memory()
    lse = torch.empty(lshp, dtype=torch.float32).pin_memory()
    plan.step_wait(plan.step_host(Q, K, V, a, O, lse=lse, taylor=True))
    plan.build(*(x.cuda() for x in (inputs[1].Q, inputs[1].K, inputs[1].V, inputs[1].a)))
    rO, rl = plan.fwd(taylor=True)
    torch.cuda.synchronize()
    assert torch.equal(O, rO.cpu()) and torch.equal(lse, rl.cpu())
    with pytest.raises(P.PrismError):  # the Taylor forward has no backward
        g = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
        plan.step_host(Q, K, V, a, O, dO=dO, dQ=g[0], dK=g[1], dV=g[2], taylor=True)
    plan.close()


def test_cuda_graph_capture_of_a_training_step():
    """The hot path enqueues only (no host synchronisation, no allocation), so a
    whole step -- plan build, forward, backward -- can be captured once in a
    CUDA graph and replayed on new inputs copied into the captured buffers.
    The replay matches eager calls on the same inputs: O, lse, dK, dV bit for
    bit, dQ up to the order of its fp32 reduce-adds."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, backward=True)
    first, second = (make_inputs(w, seed, with_grad_output=True) for seed in (3, 4))
    plan = P.PrismPlan(P.params_for(w))
    Q, K, V, a, dO = (x.cuda() for x in (first.Q, first.K, first.V, first.a, first.dO))
    O = torch.empty_like(Q)
    lse = torch.empty((w.batch, w.heads, w.N), dtype=torch.float32, device="cuda")
    dQ, dK, dV = (torch.empty_like(Q) for _ in range(3))

    def step():
        plan.build(Q, K, V, a)
        plan.fwd(O, lse)
        plan.bwd(O, dO, dQ, dK, dV)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for x, y in zip((Q, K, V, a, dO), (second.Q, second.K, second.V, second.a, second.dO)):
        x.copy_(y.cuda())
    graph.replay()
    torch.cuda.synchronize()
    plan.check()
    got = [t.clone() for t in (O, lse, dQ, dK, dV)]

    ref = P.PrismPlan(P.params_for(w))
    Q2, K2, V2, a2, dO2 = (x.cuda() for x in (second.Q, second.K, second.V, second.a, second.dO))
    ref.build(Q2, K2, V2, a2)
    rO, rl = ref.fwd()
    rdQ, rdK, rdV = ref.bwd(rO, dO2)
    torch.cuda.synchronize()
    assert torch.equal(got[0], rO) and torch.equal(got[1], rl)
    assert torch.equal(got[3], rdK) and torch.equal(got[4], rdV)
    assert torch.allclose(got[2].float(), rdQ.float(), rtol=1e-2, atol=1e-3)
    del graph
    plan.close()
    ref.close()


def _audio_h(batch, N, C, seed):
    """Synthetic cross-attention outputs: random directions with per-token scales."""
    g = torch.Generator().manual_seed(seed)
    dirs = torch.randn(batch, N, C, generator=g)
    scale = torch.rand(batch, N, 1, generator=g) * 3.0 + 0.01
    return (dirs * scale).to(torch.bfloat16)


def test_audio_norms_against_the_oracle():
    """prism_audio_norms vs the fp64 oracle: the 16-byte path (C = 3072), the
    scalar path (C = 100, and C = 3072 from a misaligned base); relative
    error <= 1e-5 (fp32 sums of exact squares)."""
    from dynamic_block_sparse_zone_b200 import binding as B
    _lib()
    T, H, W = 8, 16, 32
    for C, misalign in ((3072, False), (100, False), (3072, True)):
        h = _audio_h(2, T * H * W, C, seed=C)
        if misalign:
            buf = torch.empty(h.numel() + 1, dtype=torch.bfloat16, device="cuda")
            hd = buf[1:].view(h.shape)
            hd.copy_(h.cuda())
            assert hd.data_ptr() % 16 != 0
        else:
            hd = h.cuda()
        a = B.prism_audio_norms(hd, T, H, W).cpu().numpy().astype(np.float64)
        ref = oracle.audio_norms(bf16_bits(h)).reshape(2, T, H, W)
        assert np.max(np.abs(a / ref - 1)) <= 1e-5, (C, misalign)


def test_audio_norms_feed_the_plan():
    """The producer's a drives prism_plan_build: the plan built on the GPU from
    the kernel's a equals the oracle's plan from the same a."""
    from dynamic_block_sparse_zone_b200 import binding as B
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2)
    inp = make_inputs(w, 0)
    # cross-attention outputs whose norms follow the workload's planted audio field
    C = 3072
    g = torch.Generator().manual_seed(7)
    dirs = torch.randn(1, w.N, C, generator=g)
    dirs = dirs / dirs.norm(dim=-1, keepdim=True)
    h = (dirs * inp.a.reshape(1, w.N, 1)).to(torch.bfloat16)
    a = B.prism_audio_norms(h.cuda(), w.T, w.H, w.W)
    inp.a = a.cpu()
    g_out = run_gpu(w, inp)
    pl, _ = oracle_plan(w, inp)
    compare_plan(w, pl, g_out)


def test_head_sharded_plan_equals_the_whole_layer():
    """A layer's heads split over two ranks (emulated in one process, the
    all-gather done by copies): every rank's zone shapes, permutation and block
    table equal those of an unsharded plan of the whole layer bit for bit, its
    heads' selections equal the whole plan's rows for them, and its forward
    outputs equal the whole plan's for its heads."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=4, planted=2, backward=True)
    inp = make_inputs(w, 0)
    Q, K, V, a, dO = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a, inp.dO))
    pl, bits = oracle_plan(w, inp)
    dOb = bf16_bits(inp.dO[0])
    whole = P.PrismPlan(P.params_for(w))
    whole.build(Q, K, V, a)
    O_all, lse_all = whole.fwd()
    v_all = whole.view()
    torch.cuda.synchronize()

    hs = 2
    ranks = []
    for r in range(2):
        prm = P.params_for(w)
        prm.heads, prm.heads_total, prm.head_offset = hs, w.heads, r * hs
        plan = P.PrismPlan(prm)
        sl = slice(r * hs, (r + 1) * hs)
        Qr, Kr, Vr = (x[:, :, sl].contiguous() for x in (Q, K, V))
        with pytest.raises(P.PrismError):
            plan.build(Qr, Kr, Vr, a)  # a sharded plan needs the exchange
        with pytest.raises(P.PrismError):
            plan.build_finish(Qr, Kr, Vr)  # statistics first
        plan.build_stats(Vr, a)
        ranks.append((plan, Qr, Kr, Vr))
    slices = [p.stats_slice() for p, *_ in ranks]
    for r in range(2):  # the all-gather: every rank receives the other's slice
        for s in range(2):
            if s != r:
                lo = slices[s][1].data_ptr() - slices[s][0].data_ptr()
                slices[r][0][lo // 8: lo // 8 + slices[s][1].numel()].copy_(slices[s][1])
    for r, (plan, Qr, Kr, Vr) in enumerate(ranks):
        plan.build_finish(Qr, Kr, Vr)
        O_r, lse_r = plan.fwd()
        grads = plan.bwd(O_r, dO[:, :, r * hs:(r + 1) * hs].contiguous())
        torch.cuda.synchronize()
        plan.check()
        v = plan.view()
        check_shard_against_oracle(w, pl, bits, dOb, v, O_r, lse_r, grads, r * hs, hs, seed=70 + r)
        for key in ("zone_B", "zone_shape", "perm"):
            assert torch.equal(v[key], v_all[key]), key
        nb = int(v["n_blocks"][0])
        assert nb == int(v_all["n_blocks"][0])
        assert torch.equal(v["blk_off"][:, :nb + 1], v_all["blk_off"][:, :nb + 1])
        rp, rp_all = v["row_ptr"].cpu().numpy(), v_all["row_ptr"].cpu().numpy()
        col, col_all = v["col_idx"].cpu().numpy(), v_all["col_idx"].cpu().numpy()
        nbmax = v["nbmax"]
        for hh in range(hs):
            for i in range(nb):
                ra, rb = hh * nbmax + i, (r * hs + hh) * nbmax + i
                assert np.array_equal(col[rp[ra]:rp[ra + 1]], col_all[rp_all[rb]:rp_all[rb + 1]])
        assert torch.equal(O_r, O_all[:, :, r * hs:(r + 1) * hs])
        assert torch.equal(lse_r, lse_all[:, r * hs:(r + 1) * hs])
        plan.close()
    whole.close()


# ---------------------------------------------------------------------------
# Zeroth-order Taylor term for the key blocks outside S_i
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("name", ["tiny_8x16x16", "dynamic_16x32x32", "dynamic_small_d64", "batch2"])
def test_taylor_forward_parity(name):
    if name == "dynamic_small_d64":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=3, head_dim=64, planted=2)
    elif name == "batch2":  # two samples with their own block counts
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, batch=2)
    else:
        w = WORKLOADS[name]
    inp = make_inputs(w, 13)
    g = run_gpu(w, inp)
    out = g["plan"].fwd(taylor=True)
    for b in range(w.batch):
        pl, bits = oracle_plan(w, inp, b=b)
        compare_plan(w, pl, g, b=b)
        assert 0 < pl.cnt.min() and pl.cnt.max() < pl.nb  # blocks outside S_i exist
        mx, rel = check_forward_taylor(w, g["plan"], pl, bits, 4096 if w.N <= 4096 else 1024, b=b, out=out)
        # the acceptance bounds tell the Taylor output from the sparse one
        z, r = np.zeros(512, np.int32), np.arange(512, dtype=np.int32)
        O_s, _ = oracle.attn_fwd_rows(pl, *bits, z, r)
        mx_s, rel_s, _ = _err(out[0][b].float().cpu().numpy()[r, z], O_s)
        assert mx_s > ATOL or rel_s > RTOL_L2, (mx_s, rel_s)
        print(name, b, "taylor max-abs", mx, "rel-L2", rel)


def test_taylor_with_every_block_selected_is_the_sparse_forward():
    """No block outside S_i: every pooled column is masked, so the Taylor
    forward is the sparse forward bit for bit (two samples)."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=24, heads=2, top_k=10 ** 6, planted=1, batch=2)
    inp = make_inputs(w, 14)
    P = _lib()
    plan = P.PrismPlan(P.params_for(w))
    plan.build(*(x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a)))
    O_s, l_s = plan.fwd()
    O_t, l_t = plan.fwd(taylor=True)
    torch.cuda.synchronize()
    plan.check()
    assert torch.equal(O_s.view(torch.int16), O_t.view(torch.int16))
    assert torch.equal(l_s, l_t)


def test_taylor_leaves_the_backward_statistics_alone():
    """prism_attn_fwd_taylor does not touch what prism_attn_bwd reads: the
    gradients after fwd, fwd_taylor, bwd equal those after fwd, bwd (dK and
    dV bit for bit; dQ, whose fp32 partial sums land in any order, in at least
    nine elements of ten and within relative L2 2e-3 -- a Taylor LSE in place
    of the sparse one would move nearly every element)."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=16, heads=2, planted=1, backward=True)
    inp = make_inputs(w, 15)
    P = _lib()
    plan = P.PrismPlan(P.params_for(w))
    plan.build(*(x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a)))
    dO = inp.dO.cuda()
    O, _ = plan.fwd()
    ref = [t.clone() for t in plan.bwd(O, dO)]
    plan.fwd(taylor=True)
    got = plan.bwd(O, dO)
    torch.cuda.synchronize()
    plan.check()
    for a, b in zip(ref[1:], got[1:]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    same = (ref[0].view(torch.int16) == got[0].view(torch.int16)).double().mean().item()
    dq0, dq1 = ref[0].double(), got[0].double()
    rel = ((dq0 - dq1).norm() / dq0.norm()).item()
    assert same >= 0.9 and rel <= 2e-3, (same, rel)


# ---------------------------------------------------------------------------
# Hilbert-order fixed-block plans (the DFSAttn-style baseline)
# ---------------------------------------------------------------------------
def oracle_hilbert_plan(w, inp, bsize, b=0, heads=None):
    Qb, Kb, Vb = (bf16_bits(x[b]) for x in (inp.Q, inp.K, inp.V))
    sel = heads is None
    pl = oracle.plan_hilbert(Qb, Kb, Vb, w.T, w.H, w.W, w.heads, w.head_dim, bsize, w.top_k, _f32(w.top_p),
                             _f32(w.max_frac), with_select=sel)
    if not sel:
        cnt, cols, diag = oracle.select(pl.Qbar[heads], pl.Kbar[heads], w.top_k, _f32(w.top_p), _f32(w.max_frac))
        pl.cnt, pl.cols, pl.diag = cnt, cols, diag
    return pl, (Qb, Kb, Vb)


def compare_hilbert_plan(w, pl, view, b=0, heads=None):
    """Order and block table exact; selection exact up to counted near-ties."""
    assert np.all(view["zone_B"][b].cpu().numpy() == 0) and np.all(view["zone_shape"][b].cpu().numpy() == -1)
    np.testing.assert_array_equal(view["perm"][b].cpu().numpy(), pl.perm)
    assert view["n_blocks"][b] == pl.nb
    np.testing.assert_array_equal(view["blk_off"][b, : pl.nb + 1].cpu().numpy(), pl.blk_off())
    rp = view["row_ptr"].cpu().numpy()
    col = view["col_idx"].cpu().numpy()
    nbmax = view["nbmax"]
    ties = 0
    for hi, h in enumerate(range(w.heads) if heads is None else heads):
        for i in range(pl.nb):
            r = (b * w.heads + h) * nbmax + i
            g_set = col[rp[r]:rp[r + 1]]
            o_set = pl.cols[hi, i, : pl.cnt[hi, i]]
            if len(g_set) != len(o_set) or np.any(g_set != o_set):
                d = pl.diag[hi, i]
                assert d[0] < TIE or d[1] < TIE, f"head {h} row {i}: selection differs without a near-tie"
                ties += 1
    return ties


def run_gpu_hilbert(w, inp, bsize, backward=False, with_a=True):
    P = _lib()
    plan = P.PrismPlan(P.params_for(w, batch=inp.Q.shape[0], hilbert_block=bsize))
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    plan.build(Q, K, V, inp.a.cuda() if with_a else None)
    O, lse = plan.fwd()
    out = dict(O=O, lse=lse, plan=plan)
    if backward:
        out["dQ"], out["dK"], out["dV"] = plan.bwd(O, inp.dO.cuda())
    torch.cuda.synchronize()
    plan.check()
    out["view"] = plan.view()
    return out


@pytest.mark.parametrize("name,bsize", [("tiny_8x16x16", 64), ("dynamic_16x32x32", 128),
                                        ("dynamic_small_d64", 256), ("batch2", 128)])
def test_hilbert_plan_forward_backward_parity(name, bsize):
    if name == "dynamic_small_d64":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=40, heads=3, head_dim=64, planted=2)
    elif name == "batch2":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=24, W=32, heads=2, planted=2, batch=2)
    else:
        w = WORKLOADS[name]
    w = scaled(w, backward=True)
    inp = make_inputs(w, 17)
    g = run_gpu_hilbert(w, inp, bsize, backward=True, with_a=(name != "tiny_8x16x16"))
    for b in range(w.batch):
        pl, bits = oracle_hilbert_plan(w, inp, bsize, b=b)
        compare_hilbert_plan(w, pl, g["view"], b=b)
        assert 0 < pl.cnt.min() and pl.cnt.max() < pl.nb
        check_forward(w, inp, g, pl, bits, 1024, b=b)
        dOb = bf16_bits(inp.dO[b])
        rs = np.random.default_rng(8)
        req_h, req_t = sample_rows(rs, w, 256)
        dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h, req_t)
        assert_close("dQ", g["dQ"][b].float().cpu().numpy()[req_t, req_h], dQ_ref)
        req_h, req_t = pick_dkv_rows(pl, 0, 2, 8, rs)
        dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
        assert_close("dK", g["dK"][b].float().cpu().numpy()[req_t, req_h], dK_ref)
        assert_close("dV", g["dV"][b].float().cpu().numpy()[req_t, req_h], dV_ref)
        check_forward_taylor(w, g["plan"], pl, bits, 512, b=b)


def test_hilbert_plan_rejections():
    P = _lib()
    w = WORKLOADS["tiny_8x16x16"]
    with pytest.raises(P.PrismError):
        P.PrismPlan(P.Params(1, 8, 16, 16, 2, 64, 2, 0.9, hilbert_block=96))
    with pytest.raises(P.PrismError):
        P.PrismPlan(P.Params(1, 8, 16, 16, 2, 64, 2, 0.9, fixed_shape=(4, 4, 4), hilbert_block=64))
    plan = P.PrismPlan(P.params_for(w, hilbert_block=64))
    inp = make_inputs(w, 2)
    with pytest.raises(P.PrismError):  # no zone statistics in a Hilbert-order plan
        plan.build_stats(inp.V.cuda(), inp.a.cuda())


@pytest.mark.slow
def test_hilbert_plan_2k_full_size():
    """The 2K grid with 128-token Hilbert blocks: order exact, selection of one
    head exact up to near-ties, forward on sampled rows of that head."""
    w = WORKLOADS["latent2k_24x96x160"]
    inp = make_inputs(w, 0, device="cuda")
    g = run_gpu_hilbert(w, inp, 128)
    heads = [3]
    pl, bits = oracle_hilbert_plan(w, inp, 128, heads=heads)
    ties = compare_hilbert_plan(w, pl, g["view"], heads=heads)
    check_forward(w, inp, g, pl, bits, 128, heads=heads)
    print("2K Hilbert near-ties", ties, "blocks", pl.nb)


def test_head_sharded_hilbert_plan_builds_alone():
    """A Hilbert-order plan needs no zone statistics, so a shard of the heads
    is built with prism_plan_build alone; its order, blocks, selections and
    forward equal the whole layer's for those heads."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=4, planted=2)
    inp = make_inputs(w, 19)
    full = P.PrismPlan(P.params_for(w, hilbert_block=128))
    Q, K, V = (x.cuda() for x in (inp.Q, inp.K, inp.V))
    full.build(Q, K, V, None)
    O_full, _ = full.fwd()
    torch.cuda.synchronize()
    vf = full.view()
    hs = [2, 3]
    p = P.params_for(scaled(w, heads=2), hilbert_block=128)
    p.heads_total, p.head_offset = 4, 2
    shard = P.PrismPlan(p)
    Qs, Ks, Vs = (x[:, :, hs, :].contiguous().cuda() for x in (inp.Q, inp.K, inp.V))
    shard.build(Qs, Ks, Vs, None)
    O_sh, _ = shard.fwd()
    torch.cuda.synchronize()
    shard.check()
    vs = shard.view()
    assert vs["n_blocks"][0] == vf["n_blocks"][0]
    assert torch.equal(vs["perm"], vf["perm"])
    nbm = vf["nbmax"]
    rpf, cf = vf["row_ptr"].cpu().numpy(), vf["col_idx"].cpu().numpy()
    rps, cs = vs["row_ptr"].cpu().numpy(), vs["col_idx"].cpu().numpy()
    for hi, h in enumerate(hs):
        for i in range(vf["n_blocks"][0]):
            a = cf[rpf[h * nbm + i]:rpf[h * nbm + i + 1]]
            b = cs[rps[hi * nbm + i]:rps[hi * nbm + i + 1]]
            assert np.array_equal(a, b)
    assert torch.equal(O_sh.view(torch.int16), O_full[:, :, hs, :].contiguous().view(torch.int16))


def assert_close_scaled(name, gpu, ref):
    """The tolerance of the workloads (max-abs 2e-2, rel-L2 1e-2) is stated for
    their unit-scale data, whose gradients stay below ~4 in magnitude.  The
    kernels' error is relative (P and dS are rounded to bf16, 2^-9, before the
    tensor-core products), so for larger gradients the max-abs bound is scaled
    by max|ref| / 4; the rel-L2 bound is unchanged."""
    from conftest import record_error
    mx, rel, raw = _err(gpu, ref)
    record_error(name + " (Q x 6)", raw, mx, rel)
    bound = ATOL * max(1.0, float(np.abs(ref).max()) / 4.0)
    assert mx <= bound and rel <= RTOL_L2, f"{name}: max-abs {mx:.3e} (bound {bound:.3e}) rel-L2 {rel:.3e}"


def test_large_logits_forward_backward_and_taylor():
    """Q scaled by 6: logits of several tens, peaked softmax rows.  The online
    softmax's lazy rescaling (the running max may lag by up to 2^8 in P) and
    the exp2 ranges must still give the oracle's outputs (standard tolerance)
    and gradients (|dQ| up to ~9 here: scaled max-abs bound)."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2, backward=True)
    inp = make_inputs(w, 23, with_grad_output=True)
    inp.Q = (inp.Q.float() * 6.0).to(torch.bfloat16)
    g = run_gpu(w, inp, backward=True)
    pl, bits = oracle_plan(w, inp)
    compare_plan(w, pl, g)
    check_forward(w, inp, g, pl, bits, 1024)
    dOb = bf16_bits(inp.dO[0])
    rs = np.random.default_rng(6)
    req_h, req_t = sample_rows(rs, w, 256)
    dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, dOb, req_h, req_t)
    assert_close_scaled("dQ", g["dQ"][0].float().cpu().numpy()[req_t, req_h], dQ_ref)
    req_h, req_t = pick_dkv_rows(pl, 0, 2, 8, rs)
    dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, dOb, req_h, req_t)
    assert_close_scaled("dK", g["dK"][0].float().cpu().numpy()[req_t, req_h], dK_ref)
    assert_close_scaled("dV", g["dV"][0].float().cpu().numpy()[req_t, req_h], dV_ref)
    check_forward_taylor(w, g["plan"], pl, bits, 512)


# grids of odd aspect (one zone wide, long and thin), batch 3, head_dim 64,
# extreme k / p / cap, fixed shapes, Hilbert blocks: plan exactness, forward,
# Taylor forward and (some) gradients against the oracle
_ODD = [
    dict(T=8, H=8, W=64, heads=2, head_dim=64, top_k=1, top_p=0.5, max_frac=0.0, planted=1),
    dict(T=64, H=8, W=8, heads=1, head_dim=128, top_k=3, top_p=0.99, max_frac=0.25, planted=2, backward=True),
    dict(T=8, H=24, W=8, heads=3, head_dim=64, top_k=2, top_p=0.8, max_frac=0.5, batch=3, planted=1),
    dict(T=16, H=16, W=8, heads=2, head_dim=128, top_k=4, top_p=0.9, fixed_shape=(2, 4, 8), planted=1, backward=True),
    dict(T=8, H=8, W=8, heads=2, head_dim=64, top_k=1, top_p=1.0, planted=0),
    dict(T=16, H=8, W=24, heads=2, head_dim=128, top_k=2, top_p=0.95, max_frac=0.1, planted=2, hilbert=64),
]


@pytest.mark.parametrize("case", range(len(_ODD)))
def test_odd_grids_and_parameters(case):
    cfg = dict(_ODD[case])
    hb = cfg.pop("hilbert", 0)
    w = scaled(WORKLOADS["dynamic_16x32x32"], **cfg)
    inp = make_inputs(w, 100 + case, with_grad_output=True)
    P = _lib()
    plan = P.PrismPlan(P.params_for(w, hilbert_block=hb))
    Q, K, V, a = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a))
    plan.build(Q, K, V, a)
    O, lse = plan.fwd()
    out = dict(O=O, lse=lse, plan=plan)
    if w.backward:
        out["dQ"], out["dK"], out["dV"] = plan.bwd(O, inp.dO.cuda())
    torch.cuda.synchronize()
    plan.check()
    out["view"] = plan.view()
    taylor = plan.fwd(taylor=True)
    for b in range(w.batch):
        if hb:
            pl, bits = oracle_hilbert_plan(w, inp, hb, b=b)
            compare_hilbert_plan(w, pl, out["view"], b=b)
        else:
            pl, bits = oracle_plan(w, inp, b=b)
            compare_plan(w, pl, out["view"], b=b)
        check_forward(w, inp, out, pl, bits, min(w.N, 1024), b=b)
        check_forward_taylor(w, plan, pl, bits, 256, b=b, out=taylor)
        if w.backward:
            rs = np.random.default_rng(case)
            req_h, req_t = sample_rows(rs, w, 256)
            dQ_ref = oracle.attn_bwd_dq_rows(pl, *bits, bf16_bits(inp.dO[b]), req_h, req_t)
            assert_close("dQ", out["dQ"][b].float().cpu().numpy()[req_t, req_h], dQ_ref)
            req_h, req_t = pick_dkv_rows(pl, 0, 2, 8, rs)
            dK_ref, dV_ref = oracle.attn_bwd_dkv_rows(pl, *bits, bf16_bits(inp.dO[b]), req_h, req_t)
            assert_close("dK", out["dK"][b].float().cpu().numpy()[req_t, req_h], dK_ref)
            assert_close("dV", out["dV"][b].float().cpu().numpy()[req_t, req_h], dV_ref)


def test_hilbert_plan_update_and_host_step_without_audio():
    """A Hilbert-order plan reused for new Q, K, V (the gather reads the plan's
    permutation) attends like the oracle's plan of the first inputs applied to
    the second; a host-buffer step of that plan runs without a_norm and equals
    the device path bit for bit."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=1)
    first, second = make_inputs(w, 31), make_inputs(w, 32)
    plan = P.PrismPlan(P.params_for(w, hilbert_block=128))
    plan.build(*(x.cuda() for x in (first.Q, first.K, first.V)), None)
    plan.update_qkv(*(x.cuda() for x in (second.Q, second.K, second.V)))
    O, lse = plan.fwd()
    torch.cuda.synchronize()
    plan.check()
    pl, _ = oracle_hilbert_plan(w, first, 128)
    compare_hilbert_plan(w, pl, plan.view())
    bits2 = tuple(bf16_bits(x[0]) for x in (second.Q, second.K, second.V))
    rs = np.random.default_rng(2)
    req_h, req_t = sample_rows(rs, w, 512)
    O_ref, _ = oracle.attn_fwd_rows(pl, *bits2, req_h, req_t)
    assert_close("O", O[0].float().cpu().numpy()[req_t, req_h], O_ref)
    # host-buffer step, no audio norms
    plan.build(*(x.cuda() for x in (second.Q, second.K, second.V)), None)
    O_dev, _ = plan.fwd()
    torch.cuda.synchronize()
    pin = [x.pin_memory() for x in (second.Q, second.K, second.V)]
    Oh = torch.empty(second.Q.shape, dtype=torch.bfloat16).pin_memory()
    plan.step_wait(plan.step_host(*pin, None, Oh))
    assert torch.equal(Oh, O_dev.cpu())


def test_per_kernel_timers_count_launches_and_reset():
    """prism_plan_set_timing / prism_plan_read_timing: one record per launch of
    each timed kernel (the score / select pair once per head group), positive
    times, cleared by the read; nothing is recorded with timing off."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=16, heads=2, planted=1, backward=True)
    inp = make_inputs(w, 41, with_grad_output=True)
    plan = P.PrismPlan(P.params_for(w))
    Q, K, V, a, dO = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a, inp.dO))
    plan.set_timing(True)
    plan.read_timing()
    plan.build(Q, K, V, a)
    O, _ = plan.fwd()
    plan.bwd(O, dO)
    plan.fwd(taylor=True)
    t = plan.read_timing()
    for name in ("zone_stats_v", "zone_stats_a", "zone_decide", "permute_pool", "csr_csc", "attn_fwd",
                 "attn_bwd_pre", "attn_bwd", "dq_finalize", "taylor_pool", "attn_fwd_taylor"):
        assert t[name][1] == 1 and t[name][0] > 0, (name, t[name])
    assert t["select"][1] >= 2 and t["select"][1] % 2 == 0  # scores + select per head group
    assert all(n == 0 for _, n in plan.read_timing().values())
    plan.set_timing(False)
    plan.fwd()
    torch.cuda.synchronize()
    assert all(n == 0 for _, n in plan.read_timing().values())


def test_backward_is_deterministic():
    """dK and dV of repeated backward passes over the same plan and inputs are
    bit-identical: the two softmax groups of the backward kernel issue their dV
    and dK products in chunk order, so the fp32 sums are formed in one order.
    dQ is summed by reduce-adds from many key tiles in whatever order they land,
    so it agrees up to fp32 summation order (at most one bf16 ulp after
    rounding)."""
    P = _lib()
    w = scaled(WORKLOADS["dynamic_16x32x32"], backward=True)
    inp = make_inputs(w, 21)
    Q, K, V, a, dO = (x.cuda() for x in (inp.Q, inp.K, inp.V, inp.a, inp.dO))
    plan = P.PrismPlan(P.params_for(w))
    plan.build(Q, K, V, a)
    O, lse = plan.fwd()
    runs = [[t.clone() for t in plan.bwd(O, dO)] for _ in range(3)]
    torch.cuda.synchronize()
    plan.check()
    for r in runs[1:]:
        assert torch.equal(r[1], runs[0][1]), "dK differs between runs"
        assert torch.equal(r[2], runs[0][2]), "dV differs between runs"
        diff = (r[0].float() - runs[0][0].float()).abs()
        assert bool((diff <= 2.0 ** -7 * runs[0][0].float().abs() + 1e-6).all()), float(diff.max())
    plan.close()
