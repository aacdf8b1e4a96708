"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: closed forms, brute
force over all subsets of tiny inputs, library routines (numpy matmul, scipy softmax),
and the invariants the method statement fixes (p=1 and W>=N give full causal attention,
minimality of the selected set, pre-RoPE index scores, planted needles are selected).
"""
import itertools
import math

import numpy as np
import pytest
from scipy.special import softmax

import oracle
import synth
from synth import bf16_bits_to_f32, f32_to_bf16_bits

D = 128


# ------------------------------------------------------------------ independent references


def _rope_complex(x, pos, base=1.0e6):
    """Rotate-half RoPE written as a complex rotation of (x_c + i x_{c+D/2})."""
    half = x.shape[-1] // 2
    theta = base ** (-2.0 * np.arange(half) / x.shape[-1])
    z = (x[..., :half] + 1j * x[..., half:]) * np.exp(1j * np.multiply.outer(pos, theta))
    return np.concatenate([z.real, z.imag], axis=-1)


def _brute_attention(q, k, v, i, keys):
    """softmax(q_i . k_j / sqrt(D)) v over the listed key positions (fp64, numpy/scipy)."""
    qr = _rope_complex(q, np.float64(i))
    kr = _rope_complex(k[keys], np.asarray(keys, dtype=np.float64))
    w = softmax(kr @ qr / math.sqrt(q.shape[-1]))
    return w @ v[keys]


def _rand_bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


# ------------------------------------------------------------------ RoPE


def test_rope_closed_forms():
    # pair c turns by pos * base^(-2c/D): c=0 turns by pos radians; c=32 with base 1e6 by pos/1000.
    e0 = np.zeros(D)
    e0[0] = 1.0
    y = oracle.rope(e0, 1.0)
    assert y[0] == pytest.approx(math.cos(1.0), abs=1e-15)
    assert y[64] == pytest.approx(math.sin(1.0), abs=1e-15)
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2
    e32 = np.zeros(D)
    e32[32] = 1.0
    y = oracle.rope(e32, 1000.0)
    assert y[32] == pytest.approx(math.cos(1.0), abs=1e-13)
    assert y[96] == pytest.approx(math.sin(1.0), abs=1e-13)
    # second-half basis vector rotates the other way round the pair
    e64 = np.zeros(D)
    e64[64] = 1.0
    y = oracle.rope(e64, 2.0)
    assert y[0] == pytest.approx(-math.sin(2.0), abs=1e-15)
    assert y[64] == pytest.approx(math.cos(2.0), abs=1e-15)
    # position 0 is the identity
    x = np.random.default_rng(0).standard_normal(D)
    assert np.array_equal(oracle.rope(x, 0.0), x)


def test_rope_is_norm_preserving_and_relative():
    rng = np.random.default_rng(1)
    for _ in range(20):
        q, k = rng.standard_normal(D), rng.standard_normal(D)
        i, j, dl = rng.integers(0, 1 << 20, size=3)
        qi, kj = oracle.rope(q, i), oracle.rope(k, j)
        assert np.linalg.norm(qi) == pytest.approx(np.linalg.norm(q), rel=1e-13)
        a = qi @ kj
        b = oracle.rope(q, i + dl) @ oracle.rope(k, j + dl)
        assert a == pytest.approx(b, abs=1e-8)
        # matches the complex-rotation form
        assert np.allclose(qi, _rope_complex(q, float(i)), atol=1e-9)


# ------------------------------------------------------------------ index scores


def test_index_scores_match_matmul():
    rng = np.random.default_rng(2)
    N, Hkv, r = 300, 3, 16
    k = _rand_bf16(rng, (N, Hkv, D))
    q = _rand_bf16(rng, (D,))
    wq = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    wk = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    for g in range(Hkv):
        s = oracle.index_scores(k, g, q, wq, wk)
        kf = bf16_bits_to_f32(k[:, g]).astype(np.float64)
        qf = bf16_bits_to_f32(q).astype(np.float64)
        ref = (kf @ wk.astype(np.float64)) @ (wq.astype(np.float64).T @ qf)
        assert np.allclose(s, ref, rtol=1e-12, atol=1e-12)


def test_index_softmax_inside_head_rows_matches_scipy():
    rng = np.random.default_rng(3)
    N, Hkv, r = 200, 2, 16
    k = _rand_bf16(rng, (N, Hkv, D))
    v = _rand_bf16(rng, (N, Hkv, D))
    q = _rand_bf16(rng, (3, D))
    wq = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    wk = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    pos = [50, 120, 199]
    res = oracle.head_rows(k, v, q, pos, g=1, retrieval=True, wq=wq, wk=wk, top_p=0.9, want_pi=True)
    kf = bf16_bits_to_f32(k[:, 1]).astype(np.float64)
    for t, i in enumerate(pos):
        qf = bf16_bits_to_f32(q[t]).astype(np.float64)
        s = (kf[: i + 1] @ wk.astype(np.float64)) @ (wq.astype(np.float64).T @ qf)
        assert np.allclose(res.pi[t, : i + 1], softmax(s), rtol=1e-11, atol=1e-15)


def test_indexer_is_pre_rope():
    # Two keys with the same pre-RoPE content at different positions get the same index score.
    rng = np.random.default_rng(4)
    N, r = 64, 16
    k = _rand_bf16(rng, (N, 1, D))
    v = _rand_bf16(rng, (N, 1, D))
    k[40] = k[7]
    q = _rand_bf16(rng, (1, D))
    wq = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    wk = (rng.standard_normal((D, r)) / math.sqrt(D)).astype(np.float32)
    res = oracle.head_rows(k, v, q, [N - 1], g=0, retrieval=True, wq=wq, wk=wk, want_pi=True)
    assert res.pi[0, 7] == res.pi[0, 40]


def test_index_scores_invariant_to_common_position_shift():
    s = synth.spec("toy_decode_4k", prefix=1023)
    x = synth.generate(s)
    for h in (0, 5):
        a = oracle.layer_rows(x, 0, h, [0], want_pi=True)
        b = oracle.layer_rows(x, 0, h, [0], want_pi=True, pos_offset=123457)
        assert np.array_equal(a.pi, b.pi)
        assert np.array_equal(a.sel[0], b.sel[0])
        assert np.allclose(a.out, b.out, atol=1e-8)
    # the attention output of local heads is shift-invariant too (RoPE is relative)
    a = oracle.layer_rows(x, 0, 1, [0])
    b = oracle.layer_rows(x, 0, 1, [0], pos_offset=999_999)
    assert np.allclose(a.out, b.out, atol=1e-8)


# ------------------------------------------------------------------ top-p


def _subset_mass(pi, idx):
    return float(sum(pi[list(idx)]))


@pytest.mark.parametrize("seed", range(40))
def test_topp_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(1, 11))
    # coarse grid -> frequent exact ties
    s = np.round(rng.standard_normal(n) * 2.0 * 2) / 2 if seed % 2 else rng.standard_normal(n) * 3.0
    p = float(rng.uniform(0.05, 0.99))
    res = oracle.topp(s, p)
    pi = softmax(s)
    sel = res.selected
    # valid: reaches p; minimal: no subset with one member fewer does
    assert _subset_mass(pi, sel) >= p - 1e-12
    m = res.count
    for sub in itertools.combinations(range(n), m - 1):
        assert _subset_mass(pi, sub) < p + 1e-12
    # maximal mass among subsets of size m, and lowest indices among equal-mass ones
    best = max(_subset_mass(pi, sub) for sub in itertools.combinations(range(n), m))
    assert _subset_mass(pi, sel) == pytest.approx(best, rel=1e-12)
    ties = [sub for sub in itertools.combinations(range(n), m)
            if abs(_subset_mass(pi, sub) - best) <= 1e-12 * best]
    assert tuple(sel) == min(ties)


def test_topp_dropping_last_member_falls_below_p():
    rng = np.random.default_rng(5)
    for _ in range(50):
        n = int(rng.integers(2, 5000))
        s = rng.standard_normal(n) * rng.uniform(0.1, 6)
        p = float(rng.uniform(0.01, 0.999))
        res = oracle.topp(s, p)
        assert res.mass >= p
        assert res.cum_prev < p
        pi = softmax(s)
        sel = res.selected
        assert _subset_mass(pi, sel) == pytest.approx(res.mass, rel=1e-10)
        # the dropped member is the lowest-ranked one: its score is the minimum over J
        last = res.order[res.count - 1]
        assert s[last] == s[sel].min()


def test_topp_all_equal_scores():
    for n, p in [(10, 0.55), (7, 0.5), (1000, 0.9001), (3, 0.1), (64, 0.999)]:
        res = oracle.topp(np.zeros(n), p)
        assert res.count == math.ceil(p * n)
        assert np.array_equal(res.selected, np.arange(res.count))


def test_topp_mass_exactly_p_stops_there():
    # "mass >= p": with n equal scores each key holds exactly 1/n (a power of two here, so
    # the fp64 sums are exact) and the set stops as soon as the running mass equals p.
    for n, p, K in [(4, 0.5, 2), (8, 0.25, 2), (2, 0.5, 1), (16, 0.75, 12)]:
        res = oracle.topp(np.full(n, -3.5), p)
        assert res.count == K
        assert res.mass == p


def test_topp_limits():
    s = np.array([0.3, 2.0, -1.0, 2.0, 1.9])
    res = oracle.topp(s, 1e-300)
    assert res.count == 1 and res.selected.tolist() == [1]  # argmax, lower index of the tie
    res = oracle.topp(s, 1.0)
    assert res.count == 5
    res = oracle.topp(np.array([5.0]), 0.5)
    assert res.count == 1 and res.mass == 1.0


# ------------------------------------------------------------------ layer rows


def _small_layer(rng, N=300, Hkv=2):
    k = _rand_bf16(rng, (N, Hkv, D))
    v = _rand_bf16(rng, (N, Hkv, D))
    wq = (rng.standard_normal((D, 16)) / math.sqrt(D)).astype(np.float32)
    wk = (rng.standard_normal((D, 16)) / math.sqrt(D)).astype(np.float32)
    return k, v, wq, wk


def test_p1_and_full_window_equal_full_causal_attention():
    rng = np.random.default_rng(6)
    k, v, wq, wk = _small_layer(rng)
    N = k.shape[0]
    q = _rand_bf16(rng, (4, D))
    pos = [0, 17, 150, N - 1]
    kf = bf16_bits_to_f32(k).astype(np.float64)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    ret = oracle.head_rows(k, v, q, pos, g=1, retrieval=True, wq=wq, wk=wk, top_p=1.0)
    loc = oracle.head_rows(k, v, q, pos, g=1, retrieval=False, window=N, n_sink=0)
    for t, i in enumerate(pos):
        ref = _brute_attention(qf[t], kf[:, 1], vf[:, 1], i, list(range(i + 1)))
        assert np.allclose(ret.out[t], ref, atol=1e-10)
        assert np.allclose(loc.out[t], ref, atol=1e-10)
        assert ret.count[t] == i + 1 and loc.count[t] == i + 1


@pytest.mark.parametrize("W,S", [(1, 0), (5, 0), (5, 3), (64, 4), (1, 7)])
def test_local_mask_matches_explicit_mask(W, S):
    rng = np.random.default_rng(7 + W + S)
    k, v, _, _ = _small_layer(rng, N=120)
    q = _rand_bf16(rng, (5, D))
    pos = [0, 3, 9, 64, 119]
    kf = bf16_bits_to_f32(k).astype(np.float64)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    res = oracle.head_rows(k, v, q, pos, g=0, retrieval=False, window=W, n_sink=S)
    for t, i in enumerate(pos):
        keys = [j for j in range(i + 1) if (i - j < W) or (j < S)]
        assert res.sel[t].tolist() == keys
        ref = _brute_attention(qf[t], kf[:, 0], vf[:, 0], i, keys)
        assert np.allclose(res.out[t], ref, atol=1e-10)
    if W == 1 and S == 0:  # attends to itself only: o = v_i exactly
        for t, i in enumerate(pos):
            assert np.array_equal(res.out[t], vf[i, 0])


def test_sinks_covering_the_prefix_give_full_causal():
    rng = np.random.default_rng(8)
    k, v, _, _ = _small_layer(rng, N=50)
    q = _rand_bf16(rng, (1, D))
    a = oracle.head_rows(k, v, q, [30], g=0, retrieval=False, window=2, n_sink=31)
    b = oracle.head_rows(k, v, q, [30], g=0, retrieval=False, window=1000, n_sink=0)
    assert a.sel[0].tolist() == list(range(31))
    assert np.allclose(a.out, b.out, atol=1e-12)


def test_sparse_attention_equals_attention_over_the_selected_set():
    rng = np.random.default_rng(9)
    k, v, wq, wk = _small_layer(rng, N=400)
    q = _rand_bf16(rng, (3, D))
    pos = [10, 200, 399]
    res = oracle.head_rows(k, v, q, pos, g=0, retrieval=True, wq=wq, wk=wk, top_p=0.7)
    kf = bf16_bits_to_f32(k).astype(np.float64)
    vf = bf16_bits_to_f32(v).astype(np.float64)
    qf = bf16_bits_to_f32(q).astype(np.float64)
    for t, i in enumerate(pos):
        # selection from library-routine scores
        s = (kf[: i + 1, 0] @ wk.astype(np.float64)) @ (wq.astype(np.float64).T @ qf[t])
        order = np.lexsort((np.arange(i + 1), -s))
        cum = np.cumsum(softmax(s)[order])
        K = int(np.searchsorted(cum, 0.7, side="left")) + 1
        assert res.count[t] == K
        assert res.sel[t].tolist() == sorted(order[:K].tolist())
        ref = _brute_attention(qf[t], kf[:, 0], vf[:, 0], i, sorted(order[:K].tolist()))
        assert np.allclose(res.out[t], ref, atol=1e-10)


def test_attend_set_single_key_and_arbitrary_sets():
    # one key: the softmax weight is 1, so the output is that key's value row exactly
    s = synth.spec("prefill_32k", chunk=64, prefix=100, window=32, needles=())
    x = synth.generate(s)
    vf = bf16_bits_to_f32(x.v[0]).astype(np.float64)
    for h, row, j in [(0, 0, 0), (9, 5, 77), (31, 63, 163)]:
        out = oracle.attend_set(x, 0, h, row, [j])
        assert np.array_equal(out, vf[j, s.kv_head(h)])
    # an arbitrary set: brute-force attention over exactly those keys
    kf = bf16_bits_to_f32(x.k[0]).astype(np.float64)
    qf = bf16_bits_to_f32(x.q[0]).astype(np.float64)
    rng = np.random.default_rng(3)
    for h, row in [(2, 10), (26, 60)]:
        i = s.prefix + row
        J = sorted(rng.choice(i + 1, size=37, replace=False).tolist())
        ref = _brute_attention(qf[row, h], kf[:, s.kv_head(h)], vf[:, s.kv_head(h)], i, J)
        assert np.allclose(oracle.attend_set(x, 0, h, row, J), ref, atol=1e-10)
    with pytest.raises(ValueError):
        oracle.attend_set(x, 0, 0, 0, [s.prefix + 1])  # a key after the row


def test_gqa_maps_heads_to_their_kv_head():
    s = synth.spec("toy_decode_4k", n_kv_heads=8, retrieval_heads=(0, 5), prefix=255, window=64,
                   needles=())
    x = synth.generate(s)
    kf = bf16_bits_to_f32(x.k[0]).astype(np.float64)
    vf = bf16_bits_to_f32(x.v[0]).astype(np.float64)
    qf = bf16_bits_to_f32(x.q[0, 0]).astype(np.float64)
    i = s.prefix
    for h in (1, 6):  # MHA: head h reads KV head h
        res = oracle.layer_rows(x, 0, h, [0])
        keys = [j for j in range(i + 1) if i - j < s.window or j < s.n_sink]
        ref = _brute_attention(qf[h], kf[:, h], vf[:, h], i, keys)
        assert np.allclose(res.out[0], ref, atol=1e-10)


def test_decode_row_equals_prefill_row():
    # A prefill row at position i sees exactly what a decode step with N = i + 1 sees.
    s = synth.spec("prefill_32k", chunk=256, prefix=0, window=64, needles=(16,))
    x = synth.generate(s)
    rows = [0, 100, 255]
    for h in (0, 1, 7):
        full = oracle.layer_rows(x, 0, h, rows)
        for t, i in enumerate(rows):
            retrieval = h in s.retrieval_heads
            slot = s.retrieval_heads.index(h) if retrieval else 0
            one = oracle.head_rows(x.k[0, : i + 1], x.v[0, : i + 1], x.q[0, [i], h], [i],
                                   g=s.kv_head(h), retrieval=retrieval,
                                   wq=x.wq[slot] if retrieval else None,
                                   wk=x.wk[slot] if retrieval else None, window=s.window,
                                   n_sink=s.n_sink)
            assert np.array_equal(one.out[0], full.out[t])
            assert np.array_equal(one.sel[0], full.sel[t])


# ------------------------------------------------------------------ planted needles


def test_toy_needles_margin_and_selection():
    s = synth.spec("toy_decode_4k")
    x = synth.generate(s)
    for (b, h), npos in x.needle_pos.items():
        slot = s.retrieval_heads.index(h)
        sc = oracle.index_scores(x.k[b], s.kv_head(h), x.q[b, 0, h], x.wq[slot], x.wk[slot])
        others = np.delete(sc, npos)
        assert sc[npos].min() - others.max() >= 8.0
        res = oracle.layer_rows(x, b, h, [0])
        assert set(npos.tolist()) <= set(res.sel[0].tolist())


def test_many_needles_form_the_top_of_the_order():
    # With more needles than the mass target needs, the selection is a subset of the needles;
    # otherwise it contains them all.
    s = synth.spec("decode_128k", batch=3, prefix=16383, needles=(1, 16, 400))
    x = synth.generate(s)
    checked = 0
    for (b, h), npos in x.needle_pos.items():
        slot = s.retrieval_heads.index(h)
        sc = oracle.index_scores(x.k[b], s.kv_head(h), x.q[b, 0, h], x.wq[slot], x.wk[slot])
        assert sc[npos].min() - np.delete(sc, npos).max() >= 8.0
        res = oracle.layer_rows(x, b, h, [0])
        sel = set(res.sel[0].tolist())
        nset = set(npos.tolist())
        assert sel <= nset or nset <= sel
        checked += 1
    assert checked >= 5


# ---------------------------------------------------------------- bf16 index-key storage


def _bf16_nearest_by_enumeration(x: float) -> float:
    """The bf16 value nearest to x, ties to the even significand: the bf16 neighbours of x
    (from its float32 bits) compared in exact rational arithmetic."""
    from fractions import Fraction

    u = int(np.array([np.float32(x)]).view(np.uint32)[0]) & 0xFFFF0000
    cands = []
    for d in range(-2, 3):
        v = (u + (d << 16)) & 0xFFFFFFFF
        c = float(np.array([v], dtype=np.uint32).view(np.float32)[0])
        if np.isfinite(c):
            cands.append((c, v >> 16))
    X = Fraction(x)
    return min(cands, key=lambda cv: (abs(Fraction(cv[0]) - X), cv[1] & 1))[0]


def test_round_bf16_matches_exact_nearest_even():
    rng = np.random.default_rng(3)
    xs = list(rng.standard_normal(3000) * 4.0) + list(rng.standard_normal(500) * 1e-3)
    # exact halfway cases: 1 + 2^-8 lies between 1 and 1 + 2^-7 (even: 1); 1 + 3 * 2^-8 between
    # 1 + 2^-7 and 1 + 2^-6 (even: 1 + 2^-6)
    xs += [1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, 2.0, -0.5, 1 + 2 ** -9]
    for x in xs:
        assert oracle.round_bf16(x) == _bf16_nearest_by_enumeration(x), x
    assert oracle.round_bf16(1 + 2 ** -8) == 1.0 and oracle.round_bf16(1 + 3 * 2 ** -8) == 1 + 2 ** -6


def test_bf16_index_keys_change_scores_only_by_key_rounding():
    # keys whose projections are exact in bf16 (weights and keys small dyadic numbers) give the
    # same scores with fp32 and bf16 storage; a weight with more significant bits moves them
    rng = np.random.default_rng(4)
    D, r, n = 128, 16, 40
    k = rng.integers(-4, 5, size=(n, 1, D)).astype(np.float32)
    q = rng.integers(-4, 5, size=D).astype(np.float32)
    wq = np.zeros((D, r), np.float32)
    wk = np.zeros((D, r), np.float32)
    for c in range(r):  # each index dim reads one key dim with weight 1/4: exact in bf16
        wq[c, c] = wk[c, c] = 0.25
    kb = synth.f32_to_bf16_bits(k)
    qb = synth.f32_to_bf16_bits(q)
    s32 = oracle.index_scores(kb, 0, qb, wq, wk)
    s16 = oracle.index_scores(kb, 0, qb, wq, wk, index_bf16=True)
    assert np.array_equal(s32, s16)
    wk2 = wk.copy()
    wk2[0, 0] = 0.25 + 2 ** -12  # 11 significant bits: bf16 storage rounds the key component
    s32 = oracle.index_scores(kb, 0, qb, wq, wk2)
    s16 = oracle.index_scores(kb, 0, qb, wq, wk2, index_bf16=True)
    kt = k[:, 0].astype(np.float64) @ wk2.astype(np.float64)
    qt = q.astype(np.float64) @ wq.astype(np.float64)
    want = np.array([[oracle.round_bf16(v) for v in row] for row in kt]) @ qt
    assert np.allclose(s16, want, rtol=0, atol=1e-12)
    assert not np.array_equal(s32, s16)


# ---------------------------------------------------------------- fixed top-k (ablation mode)


def test_topk_equals_topp_at_the_mass_of_its_set():
    # with distinct scores, the k highest keys are exactly the top-p set for p = their mass
    # (the already pinned top-p rule), for every k
    rng = np.random.default_rng(8)
    s = rng.standard_normal(300) * 3.0
    for k in (1, 2, 7, 50, 299):
        tk = oracle.topk(s, k)
        tp = oracle.topp(s, tk.mass * (1 - 1e-12))
        assert tk.count == k and np.array_equal(tk.selected, tp.selected)
        assert tk.mass == pytest.approx(float(np.sort(softmax(s))[::-1][:k].sum()), rel=1e-12)


def test_topk_ties_and_limits():
    s = np.zeros(40)
    tk = oracle.topk(s, 9)
    assert tk.count == 9 and np.array_equal(tk.selected, np.arange(9))  # all equal: lowest positions
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    assert np.array_equal(oracle.topk(s, 2).selected, [1, 2])  # the tie at 3 goes to the lower positions
    assert np.array_equal(oracle.topk(s, 4).selected, [1, 2, 3, 4])
    assert oracle.topk(s, 99).count == 5  # k >= n keeps every key


# ------------------------------------------------------------------ K-cache clustering


def _bf16_keys(n, r=16, seed=0, blobs=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, r))
    if blobs is not None:
        x = x * 0.05 + blobs[rng.integers(0, len(blobs), n)]
    return np.array([[oracle.round_bf16(v) for v in row] for row in x])


def _quantised(kt):
    return np.rint(kt * 2.0**27) / 2.0**27


def test_kmeans_assigns_every_key_to_a_nearest_centre():
    kt = _bf16_keys(600, seed=1)
    for K, iters in [(5, 0), (9, 2), (16, 4)]:
        cent, counts, assign = oracle.kmeans(kt, K, iters)
        d = ((_quantised(kt)[:, None, :] - cent[None, :, :]) ** 2).sum(-1)
        best = d.min(1)
        assert np.all(np.abs(d[np.arange(len(kt)), assign] - best) <= 1e-12 * (1 + best))
        # ties go to the lower centre: no strictly-lower-index centre is as near
        for j in range(len(kt)):
            near = np.flatnonzero(np.abs(d[j] - best[j]) <= 1e-12 * (1 + best[j]))
            assert assign[j] == near.min()
        assert counts.sum() == len(kt) and np.array_equal(np.bincount(assign, minlength=K), counts)


def test_kmeans_objective_never_increases_over_passes():
    kt = _bf16_keys(800, seed=2)
    xq = _quantised(kt)
    prev = None
    for iters in range(6):
        cent, counts, assign = oracle.kmeans(kt, 12, iters)
        obj = ((xq - cent[assign]) ** 2).sum()
        if prev is not None:
            assert obj <= prev * (1 + 1e-12)
        prev = obj


def test_kmeans_closed_forms():
    kt = _bf16_keys(300, seed=3)
    xq = _quantised(kt)
    # one cluster: its centre is the mean of every key (exact on the 2^-27 grid)
    cent, counts, assign = oracle.kmeans(kt, 1, 3)
    assert counts.tolist() == [300] and np.all(assign == 0)
    assert np.allclose(cent[0], xq.mean(0), rtol=0, atol=1e-15)
    # as many clusters as keys: every key starts as its own centre and stays there
    cent, counts, assign = oracle.kmeans(kt, 300, 2)
    assert np.array_equal(assign, np.arange(300)) and np.all(counts == 1)
    assert np.array_equal(cent, xq)
    # one pass from the evenly spaced start: the centres are the means of the first assignment
    cent0, _, assign0 = oracle.kmeans(kt, 7, 0)
    assert np.array_equal(cent0, xq[[(2 * k + 1) * 300 // 14 for k in range(7)]])
    cent1, _, _ = oracle.kmeans(kt, 7, 1)
    for k in range(7):
        m = assign0 == k
        assert np.allclose(cent1[k], xq[m].mean(0), rtol=0, atol=1e-15)


def test_kmeans_separates_far_blobs():
    blobs = np.zeros((3, 16))
    blobs[0, 0], blobs[1, 1], blobs[2, 2] = 40.0, 40.0, 40.0
    kt = _bf16_keys(450, seed=4, blobs=blobs)
    cent, counts, assign = oracle.kmeans(kt, 3, 5)
    near = np.argmax(np.abs(kt[:, :3]), axis=1)  # the blob each key came from
    # a one-to-one map between clusters and blobs
    pairs = {(int(a), int(b)) for a, b in zip(assign, near)}
    assert len(pairs) == 3 and len({a for a, _ in pairs}) == 3


def _brute_cluster_hit(qt, cent, counts, p):
    """Smallest set of clusters, closed upward in centre score (with ties to the lower index),
    whose weight reaches p of the total: by enumeration of every subset."""
    import itertools

    K = len(counts)
    c = cent @ qt
    live = [k for k in range(K) if counts[k] > 0]
    cmax = max(c[k] for k in live)
    wt = {k: counts[k] * np.exp(c[k] - cmax) for k in live}
    tot = sum(wt.values())
    best = None
    for m in range(1, len(live) + 1):
        for S in itertools.combinations(live, m):
            Ss = set(S)
            closed = all(((c[o], -o) <= (c[k], -k)) or (o in Ss) for k in Ss for o in live
                         if (c[o], -o) > (c[k], -k))
            if closed and sum(wt[k] for k in S) >= p * tot * (1 - 1e-12):
                best = Ss
                break
        if best is not None:
            break
    return best


def test_cluster_select_matches_enumeration():
    rng = np.random.default_rng(5)
    for trial in range(30):
        K = int(rng.integers(2, 8))
        cent = rng.standard_normal((K, 16))
        counts = rng.integers(0, 50, K).astype(np.int64)
        counts[rng.integers(0, K)] = 7  # at least one non-empty cluster
        qt = rng.standard_normal(16)
        p = float(rng.choice([0.3, 0.5, 0.8, 0.9, 0.99]))
        hit, w, wt = oracle.cluster_select(qt, cent, counts, p)
        assert set(np.flatnonzero(hit).tolist()) == _brute_cluster_hit(qt, cent, counts, p)
        assert np.all(~hit[counts == 0])
        assert abs(w.sum() - 1.0) < 1e-12 and w[hit].sum() >= p * (1 - 1e-12)


def test_cluster_select_limits():
    cent = np.eye(4, 16)
    counts = np.array([5, 0, 3, 2], dtype=np.int64)
    hit, w, _ = oracle.cluster_select(np.zeros(16), cent, counts, 1.0)
    assert hit.tolist() == [True, False, True, True]  # p = 1: every non-empty cluster
    # equal centre scores: weights are the sizes, taken in index order
    hit, w, _ = oracle.cluster_select(np.zeros(16), cent, counts, 0.5)
    assert hit.tolist() == [True, False, False, False] and np.allclose(w, counts / 10.0)
    hit, _, _ = oracle.cluster_select(np.zeros(16), cent, counts, 0.6)
    assert hit.tolist() == [True, False, True, False]


def test_cluster_row_single_cluster_is_dense_attention():
    # one cluster holds every key: the clustered row attends to all of them, as p = 1 does
    s = synth.spec("toy_decode_4k", prefix=511, index_bf16=True)
    x = synth.generate(s)
    n = 512
    r = oracle.cluster_row(x, 0, 0, n, 1, 2, 0.9)
    assert np.array_equal(r.sel, np.arange(n))
    ref = oracle.layer_rows(x, 0, 0, [0], top_p=1.0)
    assert np.allclose(r.out, ref.out[0], rtol=0, atol=1e-12)
    # keys cached after the clustering are always kept
    r2 = oracle.cluster_row(x, 0, 0, n, 16, 2, 0.5, n_clustered=400)
    assert np.all(np.isin(np.arange(400, n), r2.sel)) and np.all(np.diff(r2.sel) > 0)
    assert set(r2.sel[r2.sel < 400].tolist()) == set(np.flatnonzero(r2.hit[r2.assign]).tolist())
