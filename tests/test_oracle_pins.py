"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks an oracle function against something other than itself:
hand-written fixtures, closed forms, a numeric minimisation, brute force, or a
library routine on a special case.  CPU only.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from dynamic_block_sparse_zone_b200.synth import WORKLOADS, bf16_bits, make_inputs, scaled

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bits of a float32 array (round to nearest even)."""
    return bf16_bits(torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16))


def golden_shapes():
    rows = []
    with open(os.path.join(GOLDEN, "candidate_shapes.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(x) for x in line.split()))
    return rows


# ---------------------------------------------------------------------------
# Candidate table, l*, nearest shape
# ---------------------------------------------------------------------------
def test_shape_table_matches_hand_written_list():
    table = [tuple(2 ** e for e in r) for r in oracle.shape_table()]
    assert table == golden_shapes()
    vols = [a * b * c for a, b, c in table]
    assert [vols.count(v) for v in (64, 128, 256)] == [7, 6, 3]
    assert all(e in (2, 4, 8) for s in table for e in s)
    # every shape with edges in {2,4,8} and volume in {64,128,256} is present
    brute = {s for s in itertools.product((2, 4, 8), repeat=3) if np.prod(s) in (64, 128, 256)}
    assert brute == set(table)


def test_lstar_identities():
    rs = np.random.default_rng(1)
    for _ in range(200):
        g = rs.uniform(1e-6, 3.0, size=3)
        S = int(rs.integers(6, 9))
        l = oracle.lstar(g, S)
        assert abs(l.sum() - S) < 1e-12
        for d, e in itertools.combinations(range(3), 2):
            assert abs((l[d] - l[e]) - (-0.5 * (math.log2(g[d]) - math.log2(g[e])))) < 1e-12


def test_lstar_is_the_constrained_minimum():
    """l* minimises sum_d g_d (b_d^2 - 1) subject to prod_d b_d = B."""
    from scipy.optimize import minimize

    rs = np.random.default_rng(2)
    for _ in range(20):
        g = rs.uniform(0.01, 2.0, size=3)
        S = int(rs.integers(6, 9))
        B = 2.0 ** S

        def loss(x):  # x = log2 b_T, log2 b_H; b_W closes the volume
            bt, bh = 2.0 ** x[0], 2.0 ** x[1]
            bw = B / (bt * bh)
            return g[0] * (bt * bt - 1) + g[1] * (bh * bh - 1) + g[2] * (bw * bw - 1)

        res = minimize(loss, x0=np.array([S / 3, S / 3]), method="Nelder-Mead",
                       options=dict(xatol=1e-10, fatol=1e-12, maxiter=20000))
        num = np.array([res.x[0], res.x[1], S - res.x[0] - res.x[1]])
        np.testing.assert_allclose(oracle.lstar(g, S), num, atol=1e-5)


def test_pick_shape_is_brute_force_nearest():
    shapes = golden_shapes()
    rs = np.random.default_rng(3)
    for _ in range(500):
        S = int(rs.integers(6, 9))
        l = rs.uniform(0.5, 3.5, size=3)
        l = l - l.mean() + S / 3.0
        best, bd = None, np.inf
        for idx, s in enumerate(shapes):
            e = np.log2(s)
            if e.sum() != S:
                continue
            d = float(((l - e) ** 2).sum())
            if d < bd:
                best, bd = idx, d
        idx, gap = oracle.pick_shape(l, S)
        assert idx == best
        assert gap >= 0.0


def test_pick_shape_isotropic_tie_breaks_to_lowest_index():
    # l* = (7/3,7/3,7/3): shapes 4x4x8, 4x8x4, 8x4x4 are equidistant -> 4x4x8
    idx, gap = oracle.pick_shape(np.array([7 / 3] * 3), 7)
    assert golden_shapes()[idx] == (4, 4, 8)
    assert gap < 1e-12
    idx, _ = oracle.pick_shape(np.array([2.0, 2.0, 2.0]), 6)
    assert golden_shapes()[idx] == (4, 4, 4)


# ---------------------------------------------------------------------------
# Zone statistics: separable fields have closed-form directional variances
# ---------------------------------------------------------------------------
def _separable(T, H, W, C, rs):
    """V[t,h,w,c] = al_c u_t + be_c v_h + ga_c w_w with small integers (exact in bf16)."""
    al, be, ga = (rs.integers(0, 4, size=C) for _ in range(3))
    u, v, w = rs.integers(-4, 5, size=T), rs.integers(-4, 5, size=H), rs.integers(-4, 5, size=W)
    V = (al[None, None, None, :] * u[:, None, None, None] + be[None, None, None, :] * v[None, :, None, None]
         + ga[None, None, None, :] * w[None, None, :, None]).astype(np.float32)
    return V, (al, be, ga), (u, v, w)


def test_zone_stats_closed_form():
    rs = np.random.default_rng(4)
    T, H, W, C = 16, 16, 24, 12
    V, (al, be, ga), (u, v, w) = _separable(T, H, W, C, rs)
    Vb = f32_bits(V)
    assert np.array_equal(torch.from_numpy(Vb.view(np.int16)).view(torch.bfloat16).float().numpy(), V)
    ua, va, wa = (rs.integers(0, 5, size=n).astype(np.float32) for n in (T, H, W))
    a = 1.0 + ua[:, None, None] + 2.0 * va[None, :, None] + 0.5 * wa[None, None, :]
    sv, sa, am, amax = oracle.zone_stats(Vb.reshape(-1, C), a, T, H, W)
    MH, MW = H // 8, W // 8
    for m in range(sv.shape[0]):
        zt, zh, zw = m // (MH * MW), (m // MW) % MH, m % MW
        zs = (slice(zt * 8, zt * 8 + 8), slice(zh * 8, zh * 8 + 8), slice(zw * 8, zw * 8 + 8))
        exp = [np.mean(al.astype(float) ** 2) * np.var(u[zs[0]]), np.mean(be.astype(float) ** 2) * np.var(v[zs[1]]),
               np.mean(ga.astype(float) ** 2) * np.var(w[zs[2]])]
        np.testing.assert_allclose(sv[m], exp, rtol=1e-12, atol=1e-12)
        exp_a = [np.var(ua[zs[0]]), 4.0 * np.var(va[zs[1]]), 0.25 * np.var(wa[zs[2]])]
        np.testing.assert_allclose(sa[m], exp_a, rtol=1e-12, atol=1e-12)
        assert am[m] == pytest.approx(1.0 + ua[zs[0]].mean() + 2 * va[zs[1]].mean() + 0.5 * wa[zs[2]].mean())
    assert amax == pytest.approx(a.max())


def test_zone_stats_single_axis_gives_unit_ratio():
    """A zone that varies along W only has r_W = 1, and g = (eps, eps, 1 + eps) with a = 0."""
    rs = np.random.default_rng(5)
    T, H, W, C = 8, 8, 8, 6
    V, _, _ = _separable(T, H, W, C, rs)
    Vw = np.broadcast_to(rs.integers(-4, 5, size=(1, 1, W, C)).astype(np.float32), (T, H, W, C)).copy()
    Vb = f32_bits(Vw)
    sv, sa, am, amax = oracle.zone_stats(Vb.reshape(-1, C), np.zeros((T, H, W), np.float32), T, H, W)
    assert sv[0, 0] == 0.0 and sv[0, 1] == 0.0 and sv[0, 2] > 0
    dec = oracle.zone_decide(sv, sa, am, amax, 1e-6)
    np.testing.assert_allclose(dec["g"][0], [1e-6, 1e-6, 1.0 + 1e-6], rtol=1e-12)
    # l*: the W edge is as short as the volume allows -> 8 x 8 x {1,2,4}
    shp = golden_shapes()[dec["zone_shape"][0]]
    assert shp[2] == min(s[2] for s in golden_shapes() if np.prod(s) == dec["zone_B"][0])


def test_audio_terms_are_scale_free_and_bounded():
    rs = np.random.default_rng(6)
    T, H, W, C = 16, 16, 16, 4
    V, _, _ = _separable(T, H, W, C, rs)
    Vb = f32_bits(V)
    a = rs.uniform(0, 1, size=(T, H, W)).astype(np.float32)
    sv, sa, am, amax = oracle.zone_stats(Vb.reshape(-1, C), a, T, H, W)
    sv2, sa2, am2, amax2 = oracle.zone_stats(Vb.reshape(-1, C), a * 4.0, T, H, W)
    d1 = oracle.zone_decide(sv, sa, am, amax, 1e-6)
    d2 = oracle.zone_decide(sv2, sa2, am2, amax2, 1e-6)
    np.testing.assert_allclose(d1["g"], d2["g"], rtol=1e-12)
    abar = am / amax
    assert np.all((abar >= 0) & (abar <= 1))


# ---------------------------------------------------------------------------
# Density and block volume on special cases (the density itself is a reading)
# ---------------------------------------------------------------------------
def _decide_with(sv_scale, a_mean, a_max=1.0):
    M = len(sv_scale)
    sv = np.array([[s, s, s] for s in sv_scale], float)
    sa = np.ones((M, 3))
    return oracle.zone_decide(sv, sa, np.asarray(a_mean, float), a_max, 1e-6)


def test_volume_special_cases():
    # identical variation everywhere, no audio: rho = 1 -> all 64
    d = _decide_with([1.0] * 6, [0.0] * 6)
    assert list(d["zone_B"]) == [64] * 6
    # one zone 5x the others: others rho = 0.2 < 0.25 -> 256; the peak zone 64
    d = _decide_with([5.0, 1.0, 1.0, 1.0], [0.0] * 4)
    assert list(d["zone_B"]) == [64, 256, 256, 256]
    # one zone 3x: others rho = 1/3 in [0.25, 0.5) -> 128
    d = _decide_with([3.0, 1.0, 1.0], [0.0] * 3)
    assert list(d["zone_B"]) == [64, 128, 128]
    # strong audio coupling overrides weak video change: abar = 1 -> 64
    d = _decide_with([5.0, 1.0, 1.0], [0.0, 1.0, 0.3])
    assert list(d["zone_B"]) == [64, 64, 128]
    # isotropic g -> equal l* ; the 64-volume shape is 4x4x4
    d = _decide_with([1.0], [0.0])
    assert golden_shapes()[d["zone_shape"][0]] == (4, 4, 4)


def test_constant_zone_is_isotropic():
    T = H = W = 8
    V = np.full((T, H, W, 2), 0.5, np.float32)
    sv, sa, am, amax = oracle.zone_stats(f32_bits(V).reshape(-1, 2),
                                         np.zeros((T, H, W), np.float32), T, H, W)
    assert np.all(sv == 0)
    d = oracle.zone_decide(sv, sa, am, amax, 1e-6)
    np.testing.assert_allclose(d["g"][0], [1 / 3 + 1e-6] * 3, rtol=1e-12)
    assert d["zone_B"][0] == 256  # no variation anywhere -> coarsest


# ---------------------------------------------------------------------------
# Blocks, permutation and pooling
# ---------------------------------------------------------------------------
def test_blocks_tile_each_zone_and_perm_is_block_contiguous():
    rs = np.random.default_rng(7)
    T, H, W = 16, 24, 16
    M = (T // 8) * (H // 8) * (W // 8)
    zs = rs.integers(0, 16, size=M).astype(np.int32)
    box = oracle.blocks(T, H, W, zs)
    shapes = golden_shapes()
    assert box.shape[0] == sum(512 // np.prod(shapes[s]) for s in zs)
    pm = oracle.perm(T, H, W, box)
    assert np.array_equal(np.sort(pm), np.arange(T * H * W))
    off = 0
    MH, MW = H // 8, W // 8
    zone_of_block = []
    for b in box:
        t0, h0, w0, bt, bh, bw = b
        toks = pm[off:off + bt * bh * bw]
        tt, hh, ww = toks // (H * W), (toks // W) % H, toks % W
        # contiguous range = exactly the box, raster order inside
        exp = [(t * H + h) * W + w for t in range(t0, t0 + bt) for h in range(h0, h0 + bh)
               for w in range(w0, w0 + bw)]
        assert list(toks) == exp
        z = {(t // 8, h // 8, w // 8) for t, h, w in zip(tt, hh, ww)}
        assert len(z) == 1
        zt, zh, zw = z.pop()
        zone_of_block.append((zt * MH + zh) * MW + zw)
        assert (bt, bh, bw) == shapes[zs[zone_of_block[-1]]]
        off += bt * bh * bw
    # zones appear in raster order, each as one run of blocks
    assert zone_of_block == sorted(zone_of_block)


def test_plan_with_given_zone_decisions_uses_them():
    """oracle.plan(zone_decisions=...) builds its blocks from the given shapes
    (checked against the hand-written candidate table), pools and selects on
    them, refuses a volume that differs from its shape's, and leaves the
    statistics it computes unchanged."""
    w = scaled(WORKLOADS["dynamic_16x32x32"], heads=2, head_dim=64)
    inp = make_inputs(w, 5)
    Qb, Kb, Vb = (bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V))
    a = inp.a[0].numpy()
    rs = np.random.default_rng(21)
    shapes = golden_shapes()
    M = w.N // 512
    zs = rs.integers(0, 16, size=M).astype(np.int32)
    zB = np.array([int(np.prod(shapes[c])) for c in zs], np.int32)
    args = (Qb, Kb, Vb, a, w.T, w.H, w.W, w.heads, w.head_dim, w.top_k, np.float32(w.top_p))
    ref = oracle.plan(*args)
    pl = oracle.plan(*args, zone_decisions=(zB, zs))
    assert np.array_equal(pl.zone_B, zB) and np.array_equal(pl.zone_shape, zs)
    assert np.array_equal(pl.box, oracle.blocks(w.T, w.H, w.W, zs))
    assert [tuple(b[3:]) for b in pl.box] == [shapes[c] for c in zs for _ in range(512 // int(np.prod(shapes[c])))]
    assert pl.nb == sum(512 // v for v in zB)
    np.testing.assert_array_equal(pl.sig_v, ref.sig_v)
    # the pooled means are block means of the given blocks
    j = pl.nb // 2
    t0, h0, w0, bt, bh, bw = pl.box[j]
    toks = [(t * w.H + h) * w.W + x for t in range(t0, t0 + bt) for h in range(h0, h0 + bh) for x in range(w0, w0 + bw)]
    q = (Qb.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    np.testing.assert_allclose(pl.Qbar[:, j, :], q[toks].mean(axis=0), rtol=0, atol=1e-12)
    # selection on the given blocks: every row holds at least top_k blocks and its own mass >= p
    assert np.all(pl.cnt >= min(w.top_k, pl.nb))
    bad = zB.copy()
    bad[0] = 128 if zB[0] != 128 else 64
    with pytest.raises(ValueError):
        oracle.plan(*args, zone_decisions=(bad, zs))


def test_pool_closed_form_on_linear_field():
    T, H, W, heads, D = 8, 16, 16, 2, 4
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    X = np.zeros((T, H, W, heads, D), np.float32)
    for c in range(D):
        X[..., 0, c] = t + 2 * h + 3 * w + c
        X[..., 1, c] = -(t + h) + c
    Xb = f32_bits(X).reshape(-1, heads, D)
    zs = np.array([0, 3, 9, 15], np.int32)
    box = oracle.blocks(T, H, W, zs)
    Xbar = oracle.pool(Xb, T, H, W, heads, D, box)
    for j, (t0, h0, w0, bt, bh, bw) in enumerate(box):
        ct, ch, cw = t0 + (bt - 1) / 2, h0 + (bh - 1) / 2, w0 + (bw - 1) / 2
        for c in range(D):
            assert Xbar[0, j, c] == ct + 2 * ch + 3 * cw + c
            assert Xbar[1, j, c] == -(ct + ch) + c


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------
def golden_select_rows():
    rows = []
    with open(os.path.join(GOLDEN, "select_rows.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            P, k, p, cap, exp = [s.strip() for s in line.split("|")]
            rows.append((np.array([float(x) for x in P.split()]), int(k), float(p), int(cap),
                         [int(x) for x in exp.split()]))
    return rows


@pytest.mark.parametrize("row", golden_select_rows())
def test_select_hand_worked(row):
    P, k, p, cap, exp = row
    sel, diag = oracle.select_row(np.log(P), k, p, cap)
    assert list(sel) == exp


def test_select_invariants_on_random_scores():
    rs = np.random.default_rng(8)
    for _ in range(300):
        nb = int(rs.integers(1, 60))
        z = rs.normal(0, rs.uniform(0.1, 3.0), size=nb)
        if rs.uniform() < 0.2:
            z = np.round(z, 1)  # force ties
        k = int(rs.integers(1, 10))
        p = float(rs.uniform(0.05, 1.0))
        frac = float(rs.choice([0.0, 0.1, 0.3]))
        cap = oracle.cap(nb, k, frac)
        sel, diag = oracle.select_row(z, k, p, cap)
        order = sorted(range(nb), key=lambda j: (-z[j], j))
        P = np.exp(z - z.max()); P /= P.sum()
        n = len(sel)
        assert list(sel) == sorted(order[:n])                 # a prefix of the order
        topk = set(order[:min(k, nb)])
        if diag[2] == 0:                                      # cap did not bind
            assert topk <= set(sel)
            mass = P[sel].sum()
            assert mass >= p - 1e-12 or n == nb
            if n > min(k, nb):                                # minimal prefix reaching p
                assert P[order[:n - 1]].sum() < p + 1e-12
        else:
            assert n == cap
    # k >= nb selects everything
    sel, _ = oracle.select_row(rs.normal(size=17), 17, 0.1, 17)
    assert list(sel) == list(range(17))


# ---------------------------------------------------------------------------
# Attention: dense reduction and masked dense, forward and backward
# ---------------------------------------------------------------------------
def _tiny_case(w, seed=0):
    inp = make_inputs(w, seed)
    Qb, Kb, Vb = (bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V))
    return inp, Qb, Kb, Vb


def _to64(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double()


def _token_mask(pl, h):
    N = pl.T * pl.H * pl.W
    tok_blk = np.zeros(N, np.int64)
    pm = pl.perm
    off = pl.blk_off()
    for j in range(pl.nb):
        tok_blk[pm[off[j]:off[j + 1]]] = j
    sel = np.zeros((pl.nb, pl.nb), bool)
    for i in range(pl.nb):
        sel[i, pl.cols[h, i, :pl.cnt[h, i]]] = True
    return torch.from_numpy(sel[tok_blk][:, tok_blk])


def test_attention_all_blocks_equals_dense_sdpa():
    w = scaled(WORKLOADS["tiny_8x16x16"], top_k=10 ** 6)
    inp, Qb, Kb, Vb = _tiny_case(w)
    a = inp.a[0].numpy()
    pl = oracle.plan(Qb, Kb, Vb, a, w.T, w.H, w.W, w.heads, w.head_dim, w.top_k, w.top_p,
                     fixed_shape=w.fixed_shape)
    assert np.all(pl.cnt == pl.nb)
    N = w.N
    req_h = np.repeat(np.arange(w.heads), N).astype(np.int32)
    req_t = np.tile(np.arange(N), w.heads).astype(np.int32)
    O, lse = oracle.attn_fwd_rows(pl, Qb, Kb, Vb, req_h, req_t)
    q, k, v = (_to64(x).permute(1, 0, 2) for x in (Qb, Kb, Vb))  # [h, N, D]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    np.testing.assert_allclose(O.reshape(w.heads, N, -1), ref.numpy(), atol=1e-12, rtol=1e-10)
    s = (q @ k.transpose(1, 2)) / math.sqrt(w.head_dim)
    np.testing.assert_allclose(lse.reshape(w.heads, N), torch.logsumexp(s, -1).numpy(), rtol=1e-12)


def _masked_dense(Qb, Kb, Vb, dOb, pl, h):
    q, k, v, do = (_to64(x)[:, h, :].clone().requires_grad_(True) for x in (Qb, Kb, Vb, dOb))
    mask = _token_mask(pl, h)
    o = torch.nn.functional.scaled_dot_product_attention(q[None], k[None], v[None], attn_mask=mask[None])[0]
    (o * do.detach()).sum().backward()
    return o.detach().numpy(), q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("name", ["tiny_8x16x16", "dynamic_small"])
def test_sparse_attention_equals_masked_dense_fwd_bwd(name):
    if name == "dynamic_small":
        w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=16, heads=2, head_dim=64, planted=1)
    else:
        w = WORKLOADS[name]
    inp = make_inputs(w, 0, with_grad_output=True)
    Qb, Kb, Vb, dOb = (bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V, inp.dO))
    pl = oracle.plan(Qb, Kb, Vb, inp.a[0].numpy(), w.T, w.H, w.W, w.heads, w.head_dim, w.top_k,
                     w.top_p, w.max_frac, fixed_shape=w.fixed_shape)
    assert 0 < pl.cnt.min() and pl.cnt.max() < pl.nb   # genuinely sparse rows
    N = w.N
    for h in range(w.heads):
        ref_o, ref_dq, ref_dk, ref_dv = _masked_dense(Qb, Kb, Vb, dOb, pl, h)
        rh = np.full(N, h, np.int32)
        rt = np.arange(N, dtype=np.int32)
        O, _ = oracle.attn_fwd_rows(pl, Qb, Kb, Vb, rh, rt)
        np.testing.assert_allclose(O, ref_o, atol=1e-12, rtol=1e-9)
        dQ = oracle.attn_bwd_dq_rows(pl, Qb, Kb, Vb, dOb, rh, rt)
        np.testing.assert_allclose(dQ, ref_dq, atol=1e-11, rtol=1e-8)
        sample = np.arange(0, N, 7, dtype=np.int32)
        dK, dV = oracle.attn_bwd_dkv_rows(pl, Qb, Kb, Vb, dOb, np.full(len(sample), h, np.int32), sample)
        np.testing.assert_allclose(dK, ref_dk[sample], atol=1e-11, rtol=1e-8)
        np.testing.assert_allclose(dV, ref_dv[sample], atol=1e-11, rtol=1e-8)


# ---------------------------------------------------------------------------
# Taylor term for the blocks outside S_i [In-Context Sparse Attention article,
# grouped computation]: block j outside S_i enters as |B_j| exp(q.kbar_j/sqrt D)
# with value vbar_j
# ---------------------------------------------------------------------------
def _mixed_blocks(T=8, H=16, W=16):
    """A block partition with volumes 64, 128 and 256 (one zone shape each,
    round robin over the zones) and its token -> block map."""
    table = oracle.shape_table()
    by_vol = {v: [i for i, e in enumerate(table) if int(e.sum()) == v] for v in (6, 7, 8)}
    M = (T // 8) * (H // 8) * (W // 8)
    zs = np.array([by_vol[(6, 7, 8)[m % 3]][m % len(by_vol[(6, 7, 8)[m % 3]])] for m in range(M)], np.int32)
    box = oracle.blocks(T, H, W, zs)
    tok_blk = np.zeros(T * H * W, np.int64)
    for j, b in enumerate(box):
        t, h, w_ = np.meshgrid(np.arange(b[0], b[0] + b[3]), np.arange(b[1], b[1] + b[4]),
                               np.arange(b[2], b[2] + b[5]), indexing="ij")
        tok_blk[((t * H + h) * W + w_).ravel()] = j
    return box, tok_blk


def _random_selection(rs, heads, nb):
    stride = nb
    cnt = np.zeros((heads, nb), np.int32)
    cols = np.full((heads, nb, stride), -1, np.int32)
    for h in range(heads):
        for i in range(nb):
            n = int(rs.integers(1, max(2, nb // 3)))
            sel = np.sort(rs.choice(nb, size=n, replace=False))
            cnt[h, i] = n
            cols[h, i, :n] = sel
    return cnt, cols


def _taylor_plan(T, H, W, heads, D, box, cnt, cols):
    from types import SimpleNamespace
    sizes = box[:, 3] * box[:, 4] * box[:, 5]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)
    return SimpleNamespace(T=T, H=H, W=W, heads=heads, D=D, nb=len(box), box=box, cnt=cnt, cols=cols,
                           perm=oracle.perm(T, H, W, box), blk_off=lambda: off)


def _dense(Qb, Kb, Vb, h):
    q, k, v = (_to64(x)[:, h, :].numpy() for x in (Qb, Kb, Vb))
    s = q @ k.T / math.sqrt(q.shape[1])
    mx = s.max(axis=1, keepdims=True)
    e = np.exp(s - mx)
    return (e @ v) / e.sum(axis=1, keepdims=True), (mx[:, 0] + np.log(e.sum(axis=1)))


def test_taylor_is_exact_for_blockwise_constant_keys_and_values():
    """With every key block's keys equal and its values equal, the zeroth-order
    term is the whole sum over the block: the output is dense attention over all
    tokens, whatever the selection (block volumes 64, 128 and 256 mixed)."""
    T, H, W, heads, D = 8, 16, 16, 2, 32
    rs = np.random.default_rng(5)
    box, tok_blk = _mixed_blocks(T, H, W)
    nb, N = len(box), T * H * W
    assert set((box[:, 3] * box[:, 4] * box[:, 5]).tolist()) == {64, 128, 256}
    kb = rs.normal(0, 1.0, (nb, heads, D)).astype(np.float32)
    vb = rs.normal(0, 1.0, (nb, heads, D)).astype(np.float32)
    Qb = f32_bits(rs.normal(0, 1.0, (N, heads, D)))
    Kb = f32_bits(kb[tok_blk])
    Vb = f32_bits(vb[tok_blk])
    cnt, cols = _random_selection(rs, heads, nb)
    pl = _taylor_plan(T, H, W, heads, D, box, cnt, cols)
    for h in range(heads):
        ref_o, ref_lse = _dense(Qb, Kb, Vb, h)
        O, lse = oracle.attn_fwd_taylor_rows(pl, Qb, Kb, Vb, np.full(N, h, np.int32), np.arange(N, dtype=np.int32))
        np.testing.assert_allclose(O, ref_o, atol=1e-12, rtol=1e-10)
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-12)
    # the sparse output alone misses the blocks outside S_i: the test can tell
    O_s, _ = oracle.attn_fwd_rows(pl, Qb, Kb, Vb, np.zeros(N, np.int32), np.arange(N, dtype=np.int32))
    assert np.max(np.abs(O_s - _dense(Qb, Kb, Vb, 0)[0])) > 1e-2


def test_taylor_with_zero_queries_is_the_mean_of_all_values():
    """q = 0 makes every score 0: exact and pooled terms alike weigh each token
    equally, so O is the mean of V over all N tokens and LSE = log N."""
    T, H, W, heads, D = 8, 16, 16, 2, 16
    rs = np.random.default_rng(6)
    box, _ = _mixed_blocks(T, H, W)
    nb, N = len(box), T * H * W
    Qb = f32_bits(np.zeros((N, heads, D)))
    Kb = f32_bits(rs.normal(0, 1.0, (N, heads, D)))
    Vb = f32_bits(rs.normal(0, 1.0, (N, heads, D)))
    cnt, cols = _random_selection(rs, heads, nb)
    pl = _taylor_plan(T, H, W, heads, D, box, cnt, cols)
    req_t = rs.integers(0, N, 64).astype(np.int32)
    for h in range(heads):
        O, lse = oracle.attn_fwd_taylor_rows(pl, Qb, Kb, Vb, np.full(64, h, np.int32), req_t)
        mean = _to64(Vb)[:, h, :].numpy().mean(axis=0)
        np.testing.assert_allclose(O, np.broadcast_to(mean, O.shape), atol=1e-13)
        np.testing.assert_allclose(lse, math.log(N), rtol=1e-14)


def test_taylor_error_is_second_order_around_the_block_mean():
    """Keys k_t = kbar_j + eps * delta_t with delta summing to zero over each
    block (tokens paired with opposite signs) and values constant per block:
    the first-order term of the expansion around the mean cancels, so the error
    against dense attention shrinks 4x when eps halves (2x would mean the
    expansion point is not the mean)."""
    T, H, W, heads, D = 8, 16, 16, 1, 16
    rs = np.random.default_rng(7)
    box, tok_blk = _mixed_blocks(T, H, W)
    nb, N = len(box), T * H * W
    base = rs.integers(-2, 3, (nb, heads, D)).astype(np.float32) * 0.5
    vb = rs.normal(0, 1.0, (nb, heads, D)).astype(np.float32)
    sign = rs.choice([-1.0, 1.0], (N, heads, D)).astype(np.float32)
    for j in range(nb):  # pair consecutive tokens of the block with opposite signs
        toks = np.nonzero(tok_blk == j)[0]
        sign[toks[1::2]] = -sign[toks[0::2]]
    Qb = f32_bits(rs.normal(0, 1.0, (N, heads, D)))
    Vb = f32_bits(vb[tok_blk])
    cnt, cols = _random_selection(rs, heads, nb)
    pl = _taylor_plan(T, H, W, heads, D, box, cnt, cols)
    req_t = np.arange(0, N, 5, dtype=np.int32)
    errs = []
    for k in (5, 6, 7):
        eps = 2.0 ** -k
        kk = base[tok_blk] + eps * sign
        Kb = f32_bits(kk)
        np.testing.assert_array_equal(_to64(Kb).numpy(), kk)  # exact in bf16
        O, _ = oracle.attn_fwd_taylor_rows(pl, Qb, Kb, Vb, np.zeros(len(req_t), np.int32), req_t)
        errs.append(np.max(np.abs(O - _dense(Qb, Kb, Vb, 0)[0][req_t])))
    assert errs[0] > 1e-6
    for a, b in zip(errs, errs[1:]):
        assert 3.8 < a / b < 4.2, errs


def test_taylor_with_every_block_selected_is_the_sparse_forward():
    """No block outside S_i: nothing to approximate."""
    w = WORKLOADS["tiny_8x16x16"]
    inp, Qb, Kb, Vb = _tiny_case(w, 2)
    pl = oracle.plan(Qb, Kb, Vb, inp.a[0].numpy(), w.T, w.H, w.W, w.heads, w.head_dim, 10 ** 6, 1.0)
    assert np.all(pl.cnt == pl.nb)
    rt = np.arange(0, w.N, 3, dtype=np.int32)
    rh = (rt % w.heads).astype(np.int32)
    O_t, l_t = oracle.attn_fwd_taylor_rows(pl, Qb, Kb, Vb, rh, rt)
    O_s, l_s = oracle.attn_fwd_rows(pl, Qb, Kb, Vb, rh, rt)
    np.testing.assert_array_equal(O_t, O_s)
    np.testing.assert_array_equal(l_t, l_s)


# ---------------------------------------------------------------------------
# Hilbert-order fixed blocks [DFSAttn page, first component]
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_hilbert_index_is_a_hilbert_curve(k):
    """On the 2^k cube the index is a bijection onto [0, 8^k), it starts at the
    origin, consecutive points are one unit step apart (a Hamiltonian path of
    the lattice), and every aligned 2^j sub-cube fills one interval of 8^j
    consecutive indices (the recursive structure of the Hilbert curve)."""
    S = 1 << k
    pts = np.stack(np.meshgrid(np.arange(S), np.arange(S), np.arange(S), indexing="ij"), -1).reshape(-1, 3)
    idx = oracle.hilbert_indices(pts, k).astype(np.int64)
    assert np.array_equal(np.sort(idx), np.arange(S ** 3))
    order = pts[np.argsort(idx)]
    assert np.array_equal(order[0], [0, 0, 0])
    steps = np.abs(np.diff(order, axis=0)).sum(axis=1)
    assert np.all(steps == 1)
    for j in range(1, k):
        cube = (pts >> j)
        cid = (cube[:, 0] * (S >> j) + cube[:, 1]) * (S >> j) + cube[:, 2]
        for c in np.unique(cid):
            sub = np.sort(idx[cid == c])
            assert sub[-1] - sub[0] == 8 ** j - 1 and sub[0] % 8 ** j == 0


def test_hilbert_perm_orders_the_grid_by_curve_index():
    """A non-cube grid takes the enclosing cube's curve: perm is a bijection of
    the tokens and their curve indices increase along it."""
    T, H, W = 8, 16, 24
    pm = oracle.hilbert_perm(T, H, W)
    assert np.array_equal(np.sort(pm), np.arange(T * H * W))
    t, h, w = pm // (H * W), (pm // W) % H, pm % W
    idx = oracle.hilbert_indices(np.stack([t, h, w], -1), 5).astype(np.int64)
    assert np.all(np.diff(idx) > 0)
    # within the cube's first 8x16x16 octant pair the grid is whole: unit steps there
    steps = np.abs(np.diff(np.stack([t, h, w], -1), axis=0)).sum(axis=1)
    assert np.mean(steps == 1) > 0.95


def test_pool_blocks_closed_forms():
    """Means over perm runs: a field constant on each block gives the constant;
    the field x = raster index gives the mean of the block's indices; on box
    blocks it equals the box pooling."""
    T, H, W, heads, D = 8, 16, 16, 2, 8
    N = T * H * W
    pm = oracle.hilbert_perm(T, H, W)
    off = np.arange(0, N + 1, 128)
    const = np.repeat(np.arange(N // 128, dtype=np.float32) * 0.5, 128)
    X = np.zeros((N, heads, D), np.float32)
    X[pm] = const[:, None, None]
    got = oracle.pool_blocks(f32_bits(X), heads, D, pm, off)
    np.testing.assert_array_equal(got, np.broadcast_to(const[::128][None, :, None], got.shape))
    Xi = np.broadcast_to(np.arange(N, dtype=np.float32)[:, None, None], (N, heads, D)).copy()
    Xi = Xi % 256  # exact in bf16
    got = oracle.pool_blocks(f32_bits(Xi), heads, D, pm, off)
    want = (pm % 256).reshape(-1, 128).mean(axis=1)
    np.testing.assert_allclose(got[0, :, 0], want, rtol=0, atol=1e-12)
    box, _ = _mixed_blocks(T, H, W)
    pb = oracle.perm(T, H, W, box)
    sizes = box[:, 3] * box[:, 4] * box[:, 5]
    offb = np.concatenate([[0], np.cumsum(sizes)])
    Xr = f32_bits(np.random.default_rng(3).normal(0, 1, (N, heads, D)))
    np.testing.assert_array_equal(oracle.pool_blocks(Xr, heads, D, pb, offb),
                                  oracle.pool(Xr, T, H, W, heads, D, box))


def test_hilbert_plan_attention_equals_masked_dense():
    """Selection and attention on Hilbert blocks: the sparse forward and its
    gradients equal dense SDPA under the plan's token mask (fp64)."""
    T, H, W, heads, D = 8, 16, 16, 2, 32
    w = scaled(WORKLOADS["tiny_8x16x16"], heads=heads, head_dim=D)
    inp = make_inputs(w, 4, with_grad_output=True)
    Qb, Kb, Vb, dOb = (bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V, inp.dO))
    pl = oracle.plan_hilbert(Qb, Kb, Vb, T, H, W, heads, D, 128, 2, 0.9)
    assert pl.nb == 16 and 0 < pl.cnt.min() and pl.cnt.max() < pl.nb
    N = T * H * W
    for h in range(heads):
        ref_o, ref_dq, ref_dk, ref_dv = _masked_dense(Qb, Kb, Vb, dOb, pl, h)
        rh, rt = np.full(N, h, np.int32), np.arange(N, dtype=np.int32)
        O, _ = oracle.attn_fwd_rows(pl, Qb, Kb, Vb, rh, rt)
        np.testing.assert_allclose(O, ref_o, atol=1e-12, rtol=1e-9)
        dQ = oracle.attn_bwd_dq_rows(pl, Qb, Kb, Vb, dOb, rh, rt)
        np.testing.assert_allclose(dQ, ref_dq, atol=1e-11, rtol=1e-8)
        sample = np.arange(0, N, 11, dtype=np.int32)
        dK, dV = oracle.attn_bwd_dkv_rows(pl, Qb, Kb, Vb, dOb, np.full(len(sample), h, np.int32), sample)
        np.testing.assert_allclose(dK, ref_dk[sample], atol=1e-11, rtol=1e-8)
        np.testing.assert_allclose(dV, ref_dv[sample], atol=1e-11, rtol=1e-8)


# ---------------------------------------------------------------------------
# Generator: planted zones stand out along their axis
# ---------------------------------------------------------------------------
def test_planted_zones_raise_directional_variation():
    w = WORKLOADS["dynamic_16x32x32"]
    inp = make_inputs(w, 0)
    Vb = bf16_bits(inp.V[0])
    sv, sa, am, amax = oracle.zone_stats(Vb.reshape(w.N, -1), inp.a[0].numpy(), w.T, w.H, w.W)
    planted = dict(inp.planted_zones[0])
    others = [m for m in range(w.zones) if m not in planted]
    for z, ax in planted.items():
        assert sv[z, ax] >= 4.0 * np.median(sv[others, ax])


def test_audio_norms_closed_forms_and_exact_sums():
    """a_{t,h,w} = ||h^_{t,h,w}||_2 [Prism guide, Method section 1]: closed forms
    (constant rows, one-hot rows, rows with integer norms) and, on random bf16
    rows, the exact rational sum of squares with a 50-digit square root."""
    from decimal import Decimal, getcontext
    from fractions import Fraction
    C = 3072
    rows = [np.full(C, 0.75, np.float32), np.full(C, -1.5, np.float32)]
    onehot = np.zeros(C, np.float32)
    onehot[1234] = -2.25
    rows.append(onehot)
    for trip, n in (((3, 4), 5), ((2, 3, 6), 7), ((1, 4, 8), 9), ((2, 6, 9), 11)):
        r = np.zeros(C, np.float32)
        r[[5, 700, 3000][:len(trip)]] = trip
        rows.append(r)
    h = f32_bits(np.stack(rows))
    a = oracle.audio_norms(h)
    assert a[0] == pytest.approx(0.75 * math.sqrt(C), rel=1e-15)
    assert a[1] == pytest.approx(1.5 * math.sqrt(C), rel=1e-15)
    assert a[2] == 2.25
    assert list(a[3:]) == [5.0, 7.0, 9.0, 11.0]

    getcontext().prec = 50
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((6, 257)) * rng.uniform(0.01, 30, (6, 1))).astype(np.float32)
    hb = f32_bits(x)
    a = oracle.audio_norms(hb)
    vals = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16).float().numpy().astype(np.float64)
    for r in range(vals.shape[0]):
        s = sum(Fraction(float(v)) ** 2 for v in vals[r])  # bf16 values are exact dyadic rationals
        exact = (Decimal(s.numerator) / Decimal(s.denominator)).sqrt()
        assert abs(Decimal(a[r]) - exact) / exact < Decimal("1e-14")
    # the batch and grid axes are kept
    assert oracle.audio_norms(hb.reshape(2, 3, 257)).shape == (2, 3)


def test_selection_validity_check_accepts_oracle_rows_and_rejects_planted_mistakes():
    """The check the GPU parity tests apply to a selection row that differs
    from the oracle's at a near-tie: every oracle row passes it, and a row with
    a planted mistake fails it (its best block dropped; one block too many)."""
    import copy
    from test_parity_gpu import valid_selection
    w = scaled(WORKLOADS["dynamic_16x32x32"], T=8, H=16, W=32, heads=2, planted=2)
    inp = make_inputs(w, 3)
    Qb, Kb, Vb = (bf16_bits(x[0]) for x in (inp.Q, inp.K, inp.V))
    pl = oracle.plan(Qb, Kb, Vb, inp.a[0].numpy(), w.T, w.H, w.W, w.heads, w.head_dim, w.top_k,
                     float(np.float32(w.top_p)), 0.0)
    dropped = extra = 0
    for h in range(w.heads):
        for i in range(pl.nb):
            row = pl.cols[h, i, :pl.cnt[h, i]]
            valid_selection(w, pl, h, i, row)
            z = pl.Qbar[h, i] @ pl.Kbar[h, :pl.nb].T / np.sqrt(w.head_dim)
            best = int(np.argmax(z))
            with pytest.raises(AssertionError):
                valid_selection(w, pl, h, i, np.sort(row[row != best]))
            dropped += 1
            if len(row) < pl.nb:
                out = np.setdiff1d(np.arange(pl.nb), row)
                nxt = out[np.argmax(z[out])]
                with pytest.raises(AssertionError):
                    valid_selection(w, pl, h, i, np.sort(np.append(row, nxt)))
                extra += 1
    assert dropped > 0 and extra > 0
