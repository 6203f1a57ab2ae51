"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test gets its expected values from a library routine (numpy/torch
matmul, torch's bf16 and e4m3 conversions), brute force over all subsets,
closed forms, hand-derived fixtures under tests/golden/, or central finite
differences of the pure fp64 forward -- never from the oracle function under
test.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f32_to_bf16_bits_torch(v):
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bits_to_f64(b):
    return (np.asarray(b, np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ scalars
def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(4000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 4000),
                        np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 2 ** -130, 3e38])])
    v = v.astype(np.float32)
    want = _bits_to_f64(_f32_to_bf16_bits_torch(v))
    got = np.array([oracle.round_bf16(float(a)) for a in v])
    assert np.array_equal(got, want)


def test_e4m3_codes_match_torch_and_golden():
    codes = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy().astype(np.float64)
    for c in range(256):
        ov = oracle.e4m3_value(c)
        if math.isnan(tv[c]):
            assert math.isnan(ov)
            continue
        assert ov == tv[c], c
        assert math.copysign(1, ov) == math.copysign(1, tv[c])
        assert oracle.e4m3_bits(ov) == c, c      # round trip
        assert oracle.round_e4m3(ov) == ov
    for line in open(os.path.join(GOLDEN, "e4m3_fn_values.txt")):
        if line.startswith("#") or not line.strip():
            continue
        code, val = line.split()
        assert oracle.e4m3_value(int(code, 16)) == float(val)
        assert oracle.e4m3_bits(float(val)) == int(code, 16)


def test_e4m3_rounding_matches_torch():
    rng = np.random.default_rng(2)
    v = rng.uniform(-448, 448, 20000) * 2.0 ** rng.integers(-14, 1, 20000)
    v = v.astype(np.float32).astype(np.float64)
    # add exact ties between neighbours (even / odd mantissa) and the subnormal range
    ties = [1.0625, 1.1875, 0.001953125 * 1.5, 0.001953125 * 2.5, 240.0 + 8.0, 416 + 16]
    v = np.concatenate([v, ties, [-t for t in ties]])
    want = torch.from_numpy(v.astype(np.float32)).to(torch.float8_e4m3fn).float().numpy()
    got = np.array([oracle.round_e4m3(a) for a in v])
    assert np.array_equal(got, want.astype(np.float64))
    # saturation to the largest finite value
    for a in (449.0, 463.9, 464.0, 500.0, 1e9):
        assert oracle.round_e4m3(a) == 448.0 and oracle.round_e4m3(-a) == -448.0


def test_mx_scale_golden():
    for line in open(os.path.join(GOLDEN, "mx_scale_cases.txt")):
        if line.startswith("#") or not line.strip():
            continue
        a, e = line.split()
        assert oracle.mx_scale_exp(float(a)) == int(e), a


def test_mx_quantize_blocks():
    # block 0: all zeros; block 1: amax exactly 448 * 2^-3; block 2: amax just above
    rows = np.zeros((1, 96), np.float32)
    rows[0, 32:64] = np.linspace(-56, 56, 32)
    rows[0, 64:96] = np.linspace(-1, 1, 32) * 57.0
    bits = _f32_to_bf16_bits_torch(rows)
    q, s = oracle.mx_quantize(bits)
    assert s[0, 0] == 0 and not q[0, :32].any()
    assert s[0, 1] == 127 - 3 and s[0, 2] == 127 - 2
    vals = _bits_to_f64(bits)[0]
    for b in range(3):
        e = int(s[0, b]) - 127
        deq = np.array([oracle.e4m3_value(c) for c in q[0, 32 * b:32 * b + 32]]) * 2.0 ** e
        ref = torch.from_numpy((vals[32 * b:32 * b + 32] / 2.0 ** e).astype(np.float32)).to(
            torch.float8_e4m3fn).float().numpy() * 2.0 ** e
        assert np.array_equal(deq, ref)
    fq = bits.copy()
    oracle.mx_fakequant_bf16(fq)
    assert np.array_equal(_bits_to_f64(fq)[0, 32:96],
                          np.concatenate([np.array([oracle.e4m3_value(c) for c in q[0, 32 * b:32 * b + 32]]) * 2.0 ** (int(s[0, b]) - 127) for b in (1, 2)]))


# ------------------------------------------------------------------ routing
def _tiny_router(T, H, E, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    x = _f32_to_bf16_bits_torch(rng.standard_normal((T, H)).astype(np.float32))
    Wr = (rng.standard_normal((E, H)) * scale).astype(np.float32)
    return x, Wr


def _logits_np(x, Wr, lbias=None):
    lg = _bits_to_f64(x) @ Wr.astype(np.float64).T
    return lg if lbias is None else lg + lbias.astype(np.float64)


@pytest.mark.parametrize("k", [1, 2, 3])
def test_softmax_topk_bruteforce(k):
    T, H, E = 40, 16, 8
    x, Wr = _tiny_router(T, H, E, seed=10 + k)
    L = oracle.Layer(T, H, E, k, 8, routed_scale=1.0).set(x=x, Wr=Wr)
    idx, w, gap = L.route()
    lg = _logits_np(x, Wr)
    for t in range(T):
        # the top-k set is the unique k-subset with the largest sum of logits
        best = max(itertools.combinations(range(E), k), key=lambda s: sum(lg[t, list(s)]))
        assert set(idx[t]) == set(best)
        # slots in descending score order
        assert list(idx[t]) == sorted(best, key=lambda e: -lg[t, e])
        sel = lg[t, idx[t]]
        ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-12, atol=0)


def test_sigmoid_group_limited_bruteforce():
    T, H, E, G, TG, k = 40, 16, 8, 4, 2, 3
    x, Wr = _tiny_router(T, H, E, seed=5)
    bias = (0.3 * np.random.default_rng(6).standard_normal(E)).astype(np.float32)
    lb = np.float32([0, -0.5, 0.2, 0, 0, 0.1, -1, 0])
    rs = 2.5
    L = oracle.Layer(T, H, E, k, 8, score_fn=1, n_group=G, topk_group=TG, routed_scale=rs)
    L.set(x=x, Wr=Wr, bias=bias, lbias=lb)
    idx, w, gap = L.route()
    lg = _logits_np(x, Wr, lb)
    s = 1 / (1 + np.exp(-lg))
    sc = s + bias
    gs = E // G
    for t in range(T):
        gscore = [max(sc[t, g * gs + a] + sc[t, g * gs + b] for a, b in itertools.combinations(range(gs), 2))
                  for g in range(G)]
        groups = max(itertools.combinations(range(G), TG), key=lambda c: sum(gscore[g] for g in c))
        cand = [g * gs + i for g in groups for i in range(gs)]
        best = max(itertools.combinations(cand, k), key=lambda c: sum(sc[t, list(c)]))
        assert set(idx[t]) == set(best), t
        assert list(idx[t]) == sorted(best, key=lambda e: -sc[t, e])
        ref = rs * s[t, idx[t]] / s[t, idx[t]].sum()      # unbiased scores, renormalised
        np.testing.assert_allclose(w[t], ref, rtol=1e-12, atol=0)


def test_ties_go_to_lower_index():
    T, H, E, k = 6, 16, 8, 3
    x, Wr = _tiny_router(T, H, E, seed=7)
    Wr[5] = Wr[2]          # experts 2 and 5 always tie
    Wr[6] = Wr[2]
    L = oracle.Layer(T, H, E, k, 8).set(x=x, Wr=Wr)
    idx, w, gap = L.route()
    lg = _logits_np(x, Wr)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-lg[t, e], e))
        assert list(idx[t]) == order[:k]
    # group ties: two identical groups, the lower group id wins
    Wr2 = Wr.copy()
    Wr2[4:6] = Wr2[0:2]
    L2 = oracle.Layer(T, H, E, 2, 8, score_fn=1, n_group=4, topk_group=1).set(x=x, Wr=Wr2)
    idx2, _, _ = L2.route()
    lg2 = _logits_np(x, Wr2)
    sc2 = 1 / (1 + np.exp(-lg2))
    for t in range(T):
        gsc = [sc2[t, 2 * g] + sc2[t, 2 * g + 1] for g in range(4)]
        gbest = sorted(range(4), key=lambda g: (-gsc[g], g))[0]
        assert set(idx2[t]) == {2 * gbest, 2 * gbest + 1}


def test_dispatch_invariants():
    T, H, E, k = 300, 16, 8, 3
    x, Wr = _tiny_router(T, H, E, seed=8)
    L = oracle.Layer(T, H, E, k, 8).set(x=x, Wr=Wr)
    idx, w, _ = L.route()
    counts, offsets, perm, inv = L.dispatch(idx)
    assert counts.sum() == T * k
    assert np.array_equal(np.bincount(idx.ravel(), minlength=E), counts)
    assert np.array_equal(perm[inv], np.arange(T * k))      # dispatch then inverse = identity
    assert np.array_equal(inv[perm], np.arange(T * k))
    for e in range(E):
        rows = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[rows] == e)
        toks = rows // k
        assert np.all(np.diff(toks) > 0)                     # ascending in token


# ------------------------------------------------------------------ expert math
def _mlp_np(xd, Wg, Wu, Wd):
    g = xd @ Wg.T
    u = xd @ Wu.T
    h = g / (1 + np.exp(-g)) * u
    return h @ Wd.T


def _rand_bf16(rng, shape, std):
    return _f32_to_bf16_bits_torch((rng.standard_normal(shape) * std).astype(np.float32))


@pytest.mark.parametrize("shared", [0, 1])
def test_single_expert_equals_dense_swiglu(shared):
    """E=1, top-1, weight 1 (softmax over one expert) is a dense SwiGLU MLP."""
    rng = np.random.default_rng(20 + shared)
    T, H, I, Is = 12, 64, 96, 32
    x = _rand_bf16(rng, (T, H), 1.0)
    Wr = rng.standard_normal((1, H)).astype(np.float32)
    Wgu = _rand_bf16(rng, (1, 2 * I, H), 0.1)
    Wdn = _rand_bf16(rng, (1, H, I), 0.1)
    Wgu_s = _rand_bf16(rng, (1, 2 * Is, H), 0.1) if shared else None
    Wdn_s = _rand_bf16(rng, (1, H, Is), 0.1) if shared else None
    L = oracle.Layer(T, H, 1, 1, I, S=shared, Is=Is if shared else 0, pure=True)
    L.set(x=x, Wr=Wr, Wgu=Wgu, Wdn=Wdn, Wgu_s=Wgu_s, Wdn_s=Wdn_s)
    idx, w, _ = L.route()
    assert np.all(idx == 0) and np.all(w == 1.0)
    y = L.fwd(idx, w)
    xd = _bits_to_f64(x)
    ref = _mlp_np(xd, _bits_to_f64(Wgu[0, :I]), _bits_to_f64(Wgu[0, I:]), _bits_to_f64(Wdn[0]))
    if shared:
        ref = ref + _mlp_np(xd, _bits_to_f64(Wgu_s[0, :Is]), _bits_to_f64(Wgu_s[0, Is:]), _bits_to_f64(Wdn_s[0]))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


def _assert_nearest_bf16(got, exact):
    """`got` holds bf16 values, each the nearest one to `exact`: exactly
    representable in bf16 (checked with torch's conversion, exact for such
    values) and within half a bf16 ulp (2^(e-8) for |exact| in [2^e, 2^(e+1)))."""
    got = np.asarray(got, np.float64)
    exact = np.asarray(exact, np.float64)
    f32 = got.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), got)
    assert np.array_equal(torch.from_numpy(f32).to(torch.bfloat16).float().numpy(), f32)
    nz = exact != 0
    assert np.all(got[~nz] == 0)
    half_ulp = 2.0 ** (np.floor(np.log2(np.abs(exact[nz]))) - 8)
    assert np.all(np.abs(got[nz] - exact[nz]) <= half_ulp)


def test_mirrors_sit_at_stored_tensors():
    """With mirrors on, the two-expert forward equals the weighted sum of per-expert
    MLPs with h and y rounded to the nearest bf16 (the layer stores them in bf16);
    the per-slot rows o are kept unrounded (they are stored in fp32)."""
    rng = np.random.default_rng(30)
    T, H, E, k, I = 16, 64, 4, 2, 64
    x = _rand_bf16(rng, (T, H), 1.0)
    Wr = rng.standard_normal((E, H)).astype(np.float32) / 8
    Wgu = _rand_bf16(rng, (E, 2 * I, H), 0.1)
    Wdn = _rand_bf16(rng, (E, H, I), 0.1)
    L = oracle.Layer(T, H, E, k, I).set(x=x, Wr=Wr, Wgu=Wgu, Wdn=Wdn)
    idx, w, _ = L.route()
    y, O, h = L.fwd(idx, w, want_slots=True)
    xd = _bits_to_f64(x)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            e = idx[t, j]
            g = xd[t] @ _bits_to_f64(Wgu[e, :I]).T
            u = xd[t] @ _bits_to_f64(Wgu[e, I:]).T
            _assert_nearest_bf16(h[t, j], g / (1 + np.exp(-g)) * u)
            o = h[t, j] @ _bits_to_f64(Wdn[e]).T
            np.testing.assert_allclose(O[t, j], o, rtol=1e-12, atol=1e-12)
            acc += w[t, j] * O[t, j]
        _assert_nearest_bf16(y[t], acc)


def test_mxfp8_single_expert_matches_fakequant_mlp():
    """MXFP8 mode: x and h quantised per 1x32 block (scale rule from the golden
    definition, e4m3 rounding by torch), weights fake-quantised by the caller."""
    rng = np.random.default_rng(40)
    T, H, I = 8, 64, 64
    x = _rand_bf16(rng, (T, H), 1.0)
    Wr = rng.standard_normal((1, H)).astype(np.float32)
    Wgu = _rand_bf16(rng, (1, 2 * I, H), 0.1)
    Wdn = _rand_bf16(rng, (1, H, I), 0.1)
    Wgu_q, Wdn_q = Wgu.copy(), Wdn.copy()
    oracle.mx_fakequant_bf16(Wgu_q)
    oracle.mx_fakequant_bf16(Wdn_q)
    L = oracle.Layer(T, H, 1, 1, I, mx=True, pure=True).set(x=x, Wr=Wr, Wgu=Wgu_q, Wdn=Wdn_q)
    idx, w, _ = L.route()
    y = L.fwd(idx, w)

    def fq(a):
        out = a.copy()
        for r in range(a.shape[0]):
            for b in range(0, a.shape[1], 32):
                blk = a[r, b:b + 32]
                amax = np.abs(blk).max()
                e = -127
                if amax > 0:
                    e = math.frexp(amax)[1] - 10
                    while amax > 448.0 * 2.0 ** e:
                        e += 1
                q = torch.from_numpy((blk / 2.0 ** e).astype(np.float32)).to(torch.float8_e4m3fn)
                out[r, b:b + 32] = q.float().numpy() * 2.0 ** e
        return out

    xd = fq(_bits_to_f64(x))
    g = xd @ _bits_to_f64(Wgu_q[0, :I]).T
    u = xd @ _bits_to_f64(Wgu_q[0, I:]).T
    hraw = g / (1 + np.exp(-g)) * u
    hq = fq(hraw)
    ref = hq @ _bits_to_f64(Wdn_q[0]).T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
    # the quantised h the down projection reads (h_mx): unrounded h, then per block
    # the scale byte of the golden rule and torch's e4m3 codes of h / 2^e
    oraw, ocodes, oscales = L.h_mx(idx, np.arange(T))
    np.testing.assert_allclose(oraw[:, 0], hraw, rtol=1e-12, atol=1e-15)
    for t in range(T):
        for b in range(I // 32):
            blk = oraw[t, 0, 32 * b:32 * b + 32]
            amax = np.abs(blk).max()
            e = -127
            if amax > 0:
                e = math.frexp(amax)[1] - 10
                while amax > 448.0 * 2.0 ** e:
                    e += 1
            assert oscales[t, 0, b] == e + 127
            codes = torch.from_numpy((blk / 2.0 ** e).astype(np.float32)).to(torch.float8_e4m3fn)
            assert np.array_equal(ocodes[t, 0, 32 * b:32 * b + 32], codes.view(torch.uint8).numpy())
    # the fake-quantised weights are exactly the dequantised MX codes
    q, s = oracle.mx_quantize(Wgu[0])
    deq = np.vectorize(oracle.e4m3_value)(q) * 2.0 ** (np.repeat(s.astype(np.int64), 32, axis=1) - 127)
    assert np.array_equal(deq, _bits_to_f64(Wgu_q[0]))


# ------------------------------------------------------------------ gradients
def _fd_layer(score_fn, seed):
    """A small pure-fp64 layer with inputs chosen so that routing has margins."""
    rng = np.random.default_rng(seed)
    T, H, E, k, I = 6, 32, 8, 2, 16
    S, Is = (1, 8) if score_fn else (0, 0)
    while True:
        x = rng.standard_normal((T, H))
        Wr = rng.standard_normal((E, H)) / math.sqrt(H)
        bias = 0.01 * rng.standard_normal(E) if score_fn else None
        L = oracle.Layer(T, H, E, k, I, S=S, Is=Is, score_fn=score_fn,
                         n_group=4 if score_fn else 1, topk_group=2 if score_fn else 1,
                         routed_scale=1.7 if score_fn else 1.0, pure=True)
        L.set(x=x, Wr=Wr, bias=bias, Wgu=rng.standard_normal((E, 2 * I, H)) * 0.3,
              Wdn=rng.standard_normal((E, H, I)) * 0.3,
              Wgu_s=rng.standard_normal((S, 2 * Is, H)) * 0.3 if S else None,
              Wdn_s=rng.standard_normal((S, H, Is)) * 0.3 if S else None,
              dy=rng.standard_normal((T, H)))
        idx, w, gap = L.route()
        if gap.min() > 1e-3:
            return L


def _loss(L):
    idx, w, _ = L.route()
    y = L.fwd(idx, w)
    return float((y * L.arrays["dy"]).sum())


@pytest.mark.parametrize("score_fn", [0, 1])
def test_gradients_match_finite_differences(score_fn):
    L = _fd_layer(score_fn, seed=50 + score_fn)
    c = L.cfg
    idx, w, _ = L.route()
    dx, dl, G = L.bwd(idx, w)
    eps = 1e-6
    rng = np.random.default_rng(3)

    def fd(name, pos):
        a = L.arrays[name]
        old = a[pos]
        a[pos] = old + eps
        L.set(**{name: a})
        lp = _loss(L)
        a[pos] = old - eps
        L.set(**{name: a})
        lm = _loss(L)
        a[pos] = old
        L.set(**{name: a})
        return (lp - lm) / (2 * eps)

    for _ in range(24):
        t, h = rng.integers(c.T), rng.integers(c.H)
        assert fd("x", (t, h)) == pytest.approx(dx[t, h], rel=1e-6, abs=1e-8)
    dWr = L.drouter(idx, w, np.arange(c.E))
    for _ in range(24):
        e, h = rng.integers(c.E), rng.integers(c.H)
        assert fd("Wr", (e, h)) == pytest.approx(dWr[e, h], rel=1e-6, abs=1e-8)
    groups = [(e, False) for e in range(c.E)] + [(s, True) for s in range(c.S)]
    for g, sh in groups:
        dgu, ddn = L.dw_full(idx, w, g, sh)
        wname_gu, wname_dn = ("Wgu_s", "Wdn_s") if sh else ("Wgu", "Wdn")
        for _ in range(4):
            n, h = rng.integers(dgu.shape[0]), rng.integers(c.H)
            assert fd(wname_gu, (g, n, h)) == pytest.approx(dgu[n, h], rel=1e-6, abs=1e-8)
            h2, i = rng.integers(c.H), rng.integers(ddn.shape[1])
            assert fd(wname_dn, (g, h2, i)) == pytest.approx(ddn[h2, i], rel=1e-6, abs=1e-8)


def test_dw_entries_agree_with_full():
    rng = np.random.default_rng(60)
    T, H, E, k, I = 24, 32, 4, 2, 32
    x = _rand_bf16(rng, (T, H), 1.0)
    L = oracle.Layer(T, H, E, k, I, S=1, Is=32).set(
        x=x, Wr=rng.standard_normal((E, H)).astype(np.float32) / 6,
        Wgu=_rand_bf16(rng, (E, 2 * I, H), 0.1), Wdn=_rand_bf16(rng, (E, H, I), 0.1),
        Wgu_s=_rand_bf16(rng, (1, 64, H), 0.1), Wdn_s=_rand_bf16(rng, (1, H, 32), 0.1),
        dy=_rand_bf16(rng, (T, H), 1.0))
    idx, w, _ = L.route()
    for g, sh in [(0, False), (3, False), (0, True)]:
        dgu, ddn = L.dw_full(idx, w, g, sh)
        r = rng.integers(0, dgu.shape[0], 20)
        cc = rng.integers(0, H, 20)
        assert np.array_equal(L.dw_entries(idx, w, g, sh, 0, r, cc), dgu[r, cc])
        r2 = rng.integers(0, H, 20)
        c2 = rng.integers(0, ddn.shape[1], 20)
        assert np.array_equal(L.dw_entries(idx, w, g, sh, 1, r2, c2), ddn[r2, c2])


# ------------------------------------------------------------------ top-k margins
def _sorted_desc(vals):
    """Indices by (value descending, index ascending), as the layer orders candidates."""
    return sorted(range(len(vals)), key=lambda e: (-vals[e], e))


def _gap_bruteforce(lg_t, k, score_fn, bias=None, n_group=1, topk_group=1):
    """Smallest adjacent gap among the top k+1 selection scores of one token and,
    with group-limited selection, among the top topk_group+1 group scores.  The
    group score is the best pair sum of the group (enumerated), the candidates
    are the experts of the kept groups."""
    E = len(lg_t)
    if score_fn == 0:
        p = np.exp(lg_t - lg_t.max())
        sc = p / p.sum()
    else:
        sc = 1 / (1 + np.exp(-lg_t)) + (0.0 if bias is None else bias.astype(np.float64))
    gap = math.inf
    cand = list(range(E))
    if n_group > 1 and topk_group < n_group:
        gs = E // n_group
        gsc = [max(sc[g * gs + a] + sc[g * gs + b] for a, b in itertools.combinations(range(gs), 2))
               if gs > 1 else sc[g * gs] for g in range(n_group)]
        go = _sorted_desc(gsc)
        for i in range(min(topk_group, n_group - 1)):
            gap = min(gap, gsc[go[i]] - gsc[go[i + 1]])
        cand = [g * gs + i for g in go[:topk_group] for i in range(gs)]
    order = sorted(cand, key=lambda e: (-sc[e], e))
    for j in range(min(k, len(order) - 1)):
        gap = min(gap, sc[order[j]] - sc[order[j + 1]])
    return gap


@pytest.mark.parametrize("k", [1, 3])
def test_margin_gap_softmax_bruteforce(k):
    """The gap that margin rejection reads is the smallest adjacent difference
    among the top k+1 softmax probabilities (not only the top k), ties giving 0."""
    T, H, E = 40, 16, 8
    x, Wr = _tiny_router(T, H, E, seed=70 + k)
    Wr[1] *= 3.0
    Wr[7] = Wr[1]                              # a tied pair, often on top: those tokens have gap 0
    L = oracle.Layer(T, H, E, k, 8).set(x=x, Wr=Wr)
    _, _, gap = L.route()
    lg = _logits_np(x, Wr)
    want = np.array([_gap_bruteforce(lg[t], k, 0) for t in range(T)])
    np.testing.assert_allclose(gap, want, rtol=1e-9, atol=1e-13)
    assert (want == 0).any() and (want > 0).any()


@pytest.mark.parametrize("k,TG", [(2, 2), (4, 3)])
def test_margin_gap_sigmoid_groups_bruteforce(k, TG):
    """Group-limited sigmoid routing: the gap covers the biased expert scores among
    the kept groups' experts and the group scores around the kept/dropped boundary,
    with the additive logit term in the logits."""
    T, H, E, G = 48, 16, 16, 4
    x, Wr = _tiny_router(T, H, E, seed=80 + k)
    bias = (0.2 * np.random.default_rng(81).standard_normal(E)).astype(np.float32)
    lb = (0.3 * np.random.default_rng(82).standard_normal(E)).astype(np.float32)
    L = oracle.Layer(T, H, E, k, 8, score_fn=1, n_group=G, topk_group=TG, routed_scale=1.3)
    L.set(x=x, Wr=Wr, bias=bias, lbias=lb)
    _, _, gap = L.route()
    lg = _logits_np(x, Wr, lb)
    want = np.array([_gap_bruteforce(lg[t], k, 1, bias, G, TG) for t in range(T)])
    np.testing.assert_allclose(gap, want, rtol=1e-9, atol=1e-13)
    # the group term decides the gap of some tokens and the expert term of others
    exp_only = np.array([_gap_bruteforce(lg[t], k, 1, bias) for t in range(T)])
    assert (want < exp_only).any()


def test_nan_scores_rank_last():
    """A NaN selection score ranks below every other score (as -inf), so the
    top-k stays k distinct experts with ties to the lower index: a token whose
    logits are all NaN takes experts 0..k-1; an expert whose logit term is NaN is
    never chosen while k other experts remain, and under softmax the other
    experts' weights stay the softmax over the selected logits.  (The GPU path
    follows the same rule; these inputs are not run there.)"""
    T, H, E, k = 12, 16, 8, 3
    x, Wr = _tiny_router(T, H, E, seed=90)
    x[4] = 0x7FC0                              # bf16 NaN: every logit of token 4 is NaN
    lb = np.zeros(E, np.float32)
    lb[2] = np.nan
    for score_fn, G, TG in [(0, 1, 1), (1, 4, 2)]:
        L = oracle.Layer(T, H, E, k, 8, score_fn=score_fn, n_group=G, topk_group=TG).set(x=x, Wr=Wr, lbias=lb)
        idx, w, _ = L.route()
        assert list(idx[4]) == [0, 1, 2]        # every score -inf: the lowest indices
        lg = _logits_np(x, Wr, lb)
        for t in range(T):
            if t == 4:
                continue
            assert 2 not in idx[t]
            sc = lg[t].copy() if score_fn == 0 else 1 / (1 + np.exp(-lg[t]))
            sc[2] = -np.inf
            if G > 1:
                gs = E // G
                gsc = [max(sc[g * gs + a] + sc[g * gs + b] for a, b in itertools.combinations(range(gs), 2))
                       for g in range(G)]
                gsc = [-np.inf if np.isnan(v) else v for v in gsc]
                keep = _sorted_desc(gsc)[:TG]
                sc = np.array([sc[e] if e // gs in keep else -np.inf for e in range(E)])
            assert list(idx[t]) == _sorted_desc(list(sc))[:k]
            if score_fn == 0:
                sel = lg[t, idx[t]]
                np.testing.assert_allclose(w[t], np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum(),
                                           rtol=1e-12)


# ------------------------------------------------------------------ backward rounding mirrors
def _rb(v):
    """Nearest bf16 value of fp64 values, ties to even (8 significant bits), by
    exact scaling: v = m 2^e with m in [0.5, 1) -> round m 2^8 to an integer."""
    v = np.asarray(v, np.float64)
    m, e = np.frexp(v)
    e = np.maximum(e, -125)                    # subnormal bf16 spacing 2^-133
    return np.ldexp(np.rint(np.ldexp(v, 8 - e)), e - 8)


def test_backward_mirrors_sit_at_stored_tensors():
    """With mirrors on, dx and the weight gradients equal a numpy restatement of
    the backward that rounds to the nearest bf16 exactly where the layer stores a
    bf16 tensor -- the saved g and u read by the SwiGLU backward, dGU, h, w*h, dx
    and dW -- and nowhere else: dh, the per-slot dx rows and the routing-gradient
    path stay unrounded.  Routing from the oracle (pinned above); softmax scoring
    and one shared expert."""
    rng = np.random.default_rng(95)
    T, H, E, k, I, Is = 16, 64, 4, 2, 32, 32
    x = _rand_bf16(rng, (T, H), 1.0)
    dy = _rand_bf16(rng, (T, H), 1.0)
    Wr = rng.standard_normal((E, H)).astype(np.float32) / 8
    Wgu = _rand_bf16(rng, (E, 2 * I, H), 0.1)
    Wdn = _rand_bf16(rng, (E, H, I), 0.1)
    Wgu_s = _rand_bf16(rng, (1, 2 * Is, H), 0.1)
    Wdn_s = _rand_bf16(rng, (1, H, Is), 0.1)
    L = oracle.Layer(T, H, E, k, I, S=1, Is=Is).set(x=x, Wr=Wr, Wgu=Wgu, Wdn=Wdn, Wgu_s=Wgu_s,
                                                     Wdn_s=Wdn_s, dy=dy)
    idx, w, _ = L.route()
    dx, _, _ = L.bwd(idx, w)
    xd, dyd = _bits_to_f64(x), _bits_to_f64(dy)
    Wr64 = Wr.astype(np.float64)

    def expert(shared, e):
        gu = _bits_to_f64(Wgu_s[e] if shared else Wgu[e])
        dn = _bits_to_f64(Wdn_s[e] if shared else Wdn[e])
        return gu[:len(gu) // 2], gu[len(gu) // 2:], dn

    def slot(t, shared, e, wj):
        Wg, Wu, Wd = expert(shared, e)
        g, u = Wg @ xd[t], Wu @ xd[t]                           # unrounded accumulators
        h = _rb(g / (1 + np.exp(-g)) * u)                        # stored h
        dh = Wd.T @ (wj * dyd[t])                                # dh: not stored, unrounded
        gb, ub = _rb(g), _rb(u)                                  # saved g, u
        sg = 1 / (1 + np.exp(-gb))
        dgu = np.concatenate([_rb(dh * ub * sg * (1 + gb * (1 - sg))), _rb(dh * gb * sg)])   # stored dGU
        return h, dgu, np.concatenate([Wg, Wu]).T @ dgu           # per-slot dx row: fp32, unrounded

    want_dx = np.zeros((T, H))
    rows = {g: [] for g in [(False, e) for e in range(E)] + [(True, 0)]}
    for t in range(T):
        G, acc = np.zeros(k), np.zeros(H)
        for j in range(k + 1):
            shared = j == k
            e = 0 if shared else idx[t, j]
            wj = 1.0 if shared else w[t, j]
            h, dgu, dxs = slot(t, shared, e, wj)
            acc += dxs
            if not shared:
                G[j] = dyd[t] @ (expert(False, e)[2] @ h)           # <dy, o_j>, o_j unrounded (fp32 slot row)
            rows[(shared, e)].append((t, wj, h, dgu))
        dl = w[t] * (G - (w[t] * G).sum())
        want_dx[t] = _rb(acc + dl @ Wr64[idx[t]])
    np.testing.assert_allclose(dx, want_dx, rtol=1e-9, atol=1e-12)
    for (shared, e), rs in rows.items():
        dgu_full, ddn_full = L.dw_full(idx, w, e, shared)
        toks = [r[0] for r in rs]
        DGU = np.array([r[3] for r in rs]).reshape(len(rs), -1)
        HW = _rb(np.array([r[1] * r[2] for r in rs]).reshape(len(rs), -1))     # stored w*h
        np.testing.assert_allclose(dgu_full, _rb(DGU.T @ xd[toks]), rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(ddn_full, _rb(dyd[toks].T @ HW), rtol=1e-9, atol=1e-12)


# ------------------------------------------------------------------ MXFP8 backward
def _fq_rows(a):
    """MXFP8 fake-quantisation of each row of `a` [..., K] in blocks of 32: scale
    exponent by the golden rule (smallest e with amax <= 448 * 2^e), codes by
    torch's e4m3 conversion of a / 2^e."""
    a = np.asarray(a, np.float64)
    out = np.empty_like(a)
    flat, res = a.reshape(-1, a.shape[-1]), out.reshape(-1, a.shape[-1])
    for r in range(flat.shape[0]):
        for b in range(0, flat.shape[1], 32):
            blk = flat[r, b:b + 32]
            amax = np.abs(blk).max()
            e = -127
            if amax > 0:
                e = math.frexp(amax)[1] - 10
                while amax > 448.0 * 2.0 ** e:
                    e += 1
            q = torch.from_numpy((blk / 2.0 ** e).astype(np.float32)).to(torch.float8_e4m3fn)
            res[r, b:b + 32] = q.float().numpy() * 2.0 ** e
    return out


def test_mx_fakequant_cols_is_rows_of_transpose():
    rng = np.random.default_rng(96)
    W = _rand_bf16(rng, (3, 64, 40), 0.3)
    got = W.copy()
    oracle.mx_fakequant_cols_bf16(got)
    want = np.stack([_fq_rows(_bits_to_f64(W[b]).T).T for b in range(3)])
    assert np.array_equal(_bits_to_f64(got), want)


def test_mxfp8_backward_restated():
    """MXFP8 backward: dx and the weight gradients equal a numpy restatement in
    which only the two data-gradient products take MXFP8 operands -- dy quantised
    along H times W_down quantised along H, and dGU (quantised from its unrounded
    value, blocks of 32 inside each half) times W_gate_up quantised along 2I --
    with the slot gradient read off the first product against the forward's
    quantised h; the weight gradients are bf16 products of the stored dGU and the
    quantised x, and of dy and bf16(w Q(h)).  Softmax scoring, one shared expert."""
    rng = np.random.default_rng(97)
    T, H, E, k, I, Is = 16, 64, 4, 2, 32, 32
    x = _rand_bf16(rng, (T, H), 1.0)
    dy = _rand_bf16(rng, (T, H), 1.0)
    Wr = rng.standard_normal((E, H)).astype(np.float32) / 8
    # rows of 2^0 .. 2^-19 magnitude: along a row an MX block holds values of one size, so it
    # keeps 4 significant bits; down a column it spans 19 binades, and the smallest values
    # fall below the e4m3 normal range of the block's scale -- the two copies differ there
    def graded(shape):
        a = rng.standard_normal(shape) * 0.1 * 2.0 ** -(np.arange(shape[1]) % 20)[None, :, None]
        return _f32_to_bf16_bits_torch(a.astype(np.float32))
    raw = {"Wgu": graded((E, 2 * I, H)), "Wdn": graded((E, H, I)), "Wgu_s": graded((1, 2 * Is, H)),
           "Wdn_s": graded((1, H, Is))}
    fwd, bwd = {}, {}
    for n, a in raw.items():                  # forward copies along the last axis, backward along the other
        fwd[n] = a.copy()
        oracle.mx_fakequant_bf16(fwd[n])
        bwd[n] = a.copy()
        oracle.mx_fakequant_cols_bf16(bwd[n])
        assert (fwd[n] != bwd[n]).mean() > 0.01
    L = oracle.Layer(T, H, E, k, I, S=1, Is=Is, mx=True).set(
        x=x, Wr=Wr, dy=dy, Wgu=fwd["Wgu"], Wdn=fwd["Wdn"], Wgu_s=fwd["Wgu_s"], Wdn_s=fwd["Wdn_s"],
        Wgu_b=bwd["Wgu"], Wdn_b=bwd["Wdn"], Wgu_sb=bwd["Wgu_s"], Wdn_sb=bwd["Wdn_s"])
    idx, w, _ = L.route()
    dx, _, G = L.bwd(idx, w)
    xq, dyd = _fq_rows(_bits_to_f64(x)), _bits_to_f64(dy)
    dyq = _fq_rows(dyd)
    Wr64 = Wr.astype(np.float64)

    def mats(shared, e):
        f = lambda n: _bits_to_f64(fwd[n + ("_s" if shared else "")][e])
        b = lambda n: _bits_to_f64(bwd[n + ("_s" if shared else "")][e])
        gu, dn, gub, dnb = f("Wgu"), f("Wdn"), b("Wgu"), b("Wdn")
        n2 = len(gu) // 2
        return gu[:n2], gu[n2:], dn, gub, dnb

    def slot(t, shared, e, wj):
        Wg, Wu, Wd, Wgub, Wdnb = mats(shared, e)
        g, u = Wg @ xq[t], Wu @ xq[t]
        hq = _fq_rows(g / (1 + np.exp(-g)) * u)                 # the forward's quantised h
        a = Wdnb.T @ dyq[t]                                      # Q(dy) W_down (copy along H)
        dh = wj * a
        gb, ub = _rb(g), _rb(u)
        sg = 1 / (1 + np.exp(-gb))
        dgu_raw = np.concatenate([dh * ub * sg * (1 + gb * (1 - sg)), dh * gb * sg])
        dxs = Wgub.T @ _fq_rows(dgu_raw)                          # Q(dGU) W_gate_up (copy along 2I)
        return a @ hq, hq, _rb(dgu_raw), dxs

    want_dx, want_G = np.zeros((T, H)), np.zeros((T, k))
    rows = {g: [] for g in [(False, e) for e in range(E)] + [(True, 0)]}
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k + 1):
            shared = j == k
            e = 0 if shared else idx[t, j]
            wj = 1.0 if shared else w[t, j]
            Gj, hq, dgu, dxs = slot(t, shared, e, wj)
            acc += dxs
            if not shared:
                want_G[t, j] = Gj
            rows[(shared, e)].append((t, wj, hq, dgu))
        dl = w[t] * (want_G[t] - (w[t] * want_G[t]).sum())
        want_dx[t] = _rb(acc + dl @ Wr64[idx[t]])
    np.testing.assert_allclose(G, want_G, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(dx, want_dx, rtol=1e-9, atol=1e-12)
    for (shared, e), rs in rows.items():
        dgu_full, ddn_full = L.dw_full(idx, w, e, shared)
        toks = [r[0] for r in rs]
        DGU = np.array([r[3] for r in rs]).reshape(len(rs), -1)
        HW = _rb(np.array([r[1] * r[2] for r in rs]).reshape(len(rs), -1))
        want_gu, want_dn = _rb(DGU.T @ xq[toks]), _rb(dyd[toks].T @ HW)
        np.testing.assert_allclose(dgu_full, want_gu, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(ddn_full, want_dn, rtol=1e-9, atol=1e-12)
        r_, c_ = np.array([0, 5, 2 * (Is if shared else I) - 1]), np.array([3, H - 1, 17])
        np.testing.assert_allclose(L.dw_entries(idx, w, e, shared, 0, r_, c_), want_gu[r_, c_], rtol=1e-9,
                                   atol=1e-12)
        r_, c_ = np.array([0, H - 1, 9]), np.array([0, 31, 20])
        np.testing.assert_allclose(L.dw_entries(idx, w, e, shared, 1, r_, c_), want_dn[r_, c_], rtol=1e-9,
                                   atol=1e-12)
