"""K-cache clustering (RTPurboV2, aitntnews page, finding 3): the CUDA k-means against the oracle's
(centres, sizes and assignments bit for bit), and the clustered decode selection and attention
against the oracle's cluster rows.

Tolerances: the cluster hit set is identical to the oracle's except for a cluster whose oracle
weight fraction before it (in the (c desc, k asc) order) lies within 1e-6 of p, since the GPU
scores centres from the fp32 index query and sums the weights in another order; the reported hit
weight fraction and last-cluster fraction within 1e-5; outputs under the attention tolerances,
against the oracle's attention over the GPU's set where the sets legitimately differ.
"""
import numpy as np
import pytest

import oracle
import synth
from parity import build_cache, check_outputs, p32, torch_bf16

pytestmark = pytest.mark.gpu

W_TOL = 1e-5
CUT_TOL = 1e-6


def _layer(x, K, max_seq=None):
    from long_context_sparse_idx16_b200 import Layer

    s = x.spec
    return Layer.from_spec(s, x, max_seq=max_seq or s.n_total, max_chunk=1, n_clusters=K)


def _gpu_clusters(layer):
    cl = layer.clusters()
    return (cl["centres"].cpu().numpy(), cl["counts"].cpu().numpy(), cl["assign"].cpu().numpy(), cl["ready"])


def _oracle_kmeans(x, b, slot, n, K, iters):
    s = x.spec
    kt = oracle.index_keys_bf16(x.k[b], s.kv_head(s.retrieval_heads[slot]), x.wk[slot], n)
    return kt, oracle.kmeans(kt, K, iters)


def _check_build(x, layer, K, iters, lens, problems=None):
    s = x.spec
    cent, counts, assign, ready = _gpu_clusters(layer)
    assert ready
    view = layer.cache()
    import torch

    from long_context_sparse_idx16_b200 import _DeviceArray

    keys = torch.as_tensor(_DeviceArray(view.idx_bf16, (s.batch, len(s.retrieval_heads), view.max_seq, 16), "<i2"),
                           device="cuda")
    problems = problems or [(b, slot) for b in range(s.batch) for slot in range(len(s.retrieval_heads))]
    for b, slot in problems:
        n = lens[b]
        kt, (oc, on, oa) = _oracle_kmeans(x, b, slot, n, K, iters)
        # the stored bf16 index keys are the oracle's keys, bit for bit
        stored = keys[b, slot, :n].cpu().numpy().view(np.uint16)
        assert np.array_equal(synth.bf16_bits_to_f32(stored).astype(np.float64), kt), f"b={b} slot={slot}: keys"
        assert np.array_equal(assign[b, slot, :n], oa), (
            f"b={b} slot={slot}: {int(np.count_nonzero(assign[b, slot, :n] != oa))} assignments differ")
        assert np.array_equal(counts[b, slot], on), f"b={b} slot={slot}: cluster sizes"
        assert np.array_equal(cent[b, slot].view(np.uint64), oc.view(np.uint64)), f"b={b} slot={slot}: centres"


@pytest.mark.parametrize("K,iters", [(1, 2), (16, 0), (64, 4), (130, 3)])
def test_kmeans_bit_exact(K, iters):
    x = synth.generate(synth.spec("decode_128k", batch=2, prefix=6143, index_bf16=True))
    layer = _layer(x, K)
    build_cache(layer, x, x.spec.n_total)
    layer.cluster_build(iters)
    assert layer.check() == 0
    assert [layer.cluster_len(b) for b in range(2)] == [6144, 6144]
    _check_build(x, layer, K, iters, [6144, 6144])
    layer.close()


def test_kmeans_bit_exact_ragged_and_max_clusters():
    # per-sequence lengths, K = 1024 (the largest, 128 KB of centres per CTA), a ragged tail
    x = synth.generate(synth.spec("toy_decode_4k", batch=3, prefix=4095, index_bf16=True))
    lens = [4096, 1500, 2777]
    layer = _layer(x, 1024)
    build_cache(layer, x, 4096)
    for b, n in enumerate(lens):
        layer.truncate_seq(b, n)
    layer.cluster_build(2)
    assert layer.check() == 0
    assert [layer.cluster_len(b) for b in range(3)] == lens
    _check_build(x, layer, 1024, 2, lens)
    layer.close()


def _order_before(r, qt):
    """Oracle weight fraction before each cluster in the (c desc, k asc) order."""
    c = r.cent @ qt
    live = np.flatnonzero(r.counts > 0)
    order = sorted(live, key=lambda k: (-c[k], k))
    before = np.full(len(r.counts), np.nan)
    acc = 0.0
    for k in order:
        before[k] = acc
        acc += r.w[k]
    return before


def _check_clustered_decode(x, layer, K, iters, lens, ncl, p, heads=None, row=0):
    s = x.spec
    layer.set_top_p(p)
    out, st = layer.decode(torch_bf16(x.q[:, row]), stats=True, sel_cap=max(lens))
    assert layer.check() == 0
    out = out.cpu().numpy()
    cnt, mass, thr, idx = (t.cpu().numpy() for t in (st[0], st[1], st[2], st[3]))
    _, _, assign, _ = _gpu_clusters(layer)
    gpus, refs = [], []
    n_moved = 0
    for b in range(s.batch):
        n = lens[b]
        for h in (heads or range(s.n_q_heads)):
            if h not in s.retrieval_heads:
                r = oracle.head_rows(x.k[b, :n], x.v[b, :n], x.q[b, row, h], [n - 1], g=s.kv_head(h), retrieval=False,
                                     wq=None, wk=None, top_p=1.0, top_k=0, window=s.window, n_sink=s.n_sink,
                                     rope_base=s.rope_base, index_bf16=True)
                gpus.append(out[b, h])
                refs.append(r.out[0])
                continue
            slot = s.retrieval_heads.index(h)
            r = oracle.cluster_row(x, b, h, n, K, iters, p32(p), n_clustered=ncl[b], row=row)
            k = int(cnt[b, slot])
            sel = idx[b, slot, :k].astype(np.int64)
            assert np.all(np.diff(sel) > 0), "selected positions must be strictly ascending"
            # the set is whole clusters plus every key cached after the clustering
            hit_gpu = np.zeros(K, dtype=bool)
            hit_gpu[np.unique(assign[b, slot, sel[sel < ncl[b]]])] = True
            want = np.concatenate([np.flatnonzero(hit_gpu[r.assign]), np.arange(ncl[b], n)])
            assert np.array_equal(sel, want), f"b={b} h={h}: the set is not a union of whole clusters"
            diff = np.flatnonzero(hit_gpu != r.hit)
            if len(diff):
                qt = oracle.index_query(x.q[b, row, h], x.wq[slot])
                before = _order_before(r, qt)
                bad = [int(c) for c in diff if not abs(before[c] - p32(p)) <= CUT_TOL]
                assert not bad, f"b={b} h={h}: clusters {bad} differ beyond the cut tolerance"
                n_moved += len(diff)
                ref = oracle.attend_set(x, b, h, row, sel, pos=n - 1)
            else:
                assert abs(float(mass[b, slot]) - float(r.w[r.hit].sum())) <= W_TOL
                assert abs(float(thr[b, slot]) - r.w_t) <= W_TOL
                ref = r.out
            assert float(mass[b, slot]) >= p32(p) - W_TOL or p >= 1.0
            gpus.append(out[b, h])
            refs.append(ref)
    check_outputs(np.stack(gpus), np.stack(refs), f"clustered decode K={K} p={p}")
    return n_moved


@pytest.mark.parametrize("K,p", [(64, 0.9), (128, 0.5), (16, 0.99)])
def test_clustered_decode_matches_oracle(K, p):
    # cluster 7800 keys, then append 392 more (the decode query's own key last): those are kept
    x = synth.generate(synth.spec("decode_128k", batch=2, prefix=8191, index_bf16=True))
    N = x.spec.n_total
    layer = _layer(x, K)
    build_cache(layer, x, 7800)
    layer.cluster_build(4)
    build_cache(layer, x, N)
    assert layer.check() == 0
    _check_clustered_decode(x, layer, K, 4, [N, N], [7800, 7800], p)
    layer.close()


def test_clustered_decode_ragged():
    x = synth.generate(synth.spec("decode_128k", batch=3, prefix=6143, index_bf16=True))
    lens0, lens = [3000, 6144, 4500], [3200, 6144, 5000]
    layer = _layer(x, 48)
    build_cache(layer, x, 6144)
    for b, n in enumerate(lens0):
        layer.truncate_seq(b, n)
    layer.cluster_build(3)
    for b in range(3):  # each sequence grows on its own after the clustering
        if lens[b] > lens0[b]:
            layer.append_kv_seq(b, torch_bf16(x.k[b, lens0[b]:lens[b]]), torch_bf16(x.v[b, lens0[b]:lens[b]]))
    assert [layer.cluster_len(b) for b in range(3)] == lens0
    _check_clustered_decode(x, layer, 48, 3, lens, lens0, 0.8)
    layer.close()


def test_one_cluster_is_dense_and_truncation_ends_clustering():
    from parity import run_decode

    x = synth.generate(synth.spec("decode_128k", batch=1, prefix=4095, index_bf16=True))
    N = x.spec.n_total
    layer = _layer(x, 1)
    build_cache(layer, x, N)
    layer.cluster_build(1)
    # one cluster holds every key: the selection is every causal key, as at p = 1
    layer.set_top_p(0.5)
    out, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=N)
    assert layer.check() == 0
    assert np.all(st[0].cpu().numpy() == N)
    dense = layer.decode(torch_bf16(x.q[:, 0])).cpu().numpy()  # same again
    assert np.array_equal(out.cpu().numpy(), dense)
    # truncating below the clustered length ends the clustered selection: per-key top-p again
    layer.truncate(N - 1)
    assert layer.cluster_len(0) == 0 and not layer.clusters()["ready"]
    build_cache(layer, x, N)
    run_decode(x, layer=layer)
    layer.close()


@pytest.mark.slow
def test_clustered_decode_full_128k_sampled():
    # the 128K layer shape (B=8, five retrieval heads) with K = 128 (the page's example): k-means
    # bit-exact and the clustered decode on two sampled sequences
    x = synth.generate(synth.spec("decode_128k", index_bf16=True))
    N = x.spec.n_total
    K, iters = 128, 4
    layer = _layer(x, K)
    build_cache(layer, x, N)
    layer.cluster_build(iters)
    assert layer.check() == 0
    _check_build(x, layer, K, iters, [N] * 8, problems=[(0, 0), (5, 3)])
    layer.close()


def test_cluster_build_errors():
    from long_context_sparse_idx16_b200 import RTPError

    x = synth.generate(synth.spec("toy_decode_4k", prefix=99, index_bf16=True))
    layer = _layer(x, 64)
    build_cache(layer, x, 40)
    with pytest.raises(RTPError):  # fewer keys than clusters
        layer.cluster_build(2)
    build_cache(layer, x, 100)
    with pytest.raises(RTPError):
        layer.cluster_build(-1)
    layer.cluster_build(0)
    assert layer.cluster_len(0) == 100
    layer.cluster_drop()
    assert layer.cluster_len(0) == 0
    layer.close()
    from long_context_sparse_idx16_b200 import Layer

    plain = Layer.from_spec(x.spec, x, max_chunk=1)
    build_cache(plain, x, 100)
    with pytest.raises(RTPError):  # created without n_clusters
        plain.cluster_build(1)
    plain.close()


def test_clustered_decode_overflow_and_dense_override():
    from long_context_sparse_idx16_b200 import RTP_EOVERFLOW

    x = synth.generate(synth.spec("decode_128k", batch=1, prefix=4095, index_bf16=True))
    N = x.spec.n_total
    K, cap = 32, 200
    from long_context_sparse_idx16_b200 import Layer

    layer = Layer.from_spec(x.spec, x, max_seq=N, max_chunk=1, n_clusters=K, max_select=cap)
    build_cache(layer, x, N)
    layer.cluster_build(3)
    layer.set_top_p(0.99)  # most clusters: far more than 200 keys
    _, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=cap)
    assert layer.check() == RTP_EOVERFLOW
    cnt, idx = st[0].cpu().numpy(), st[3].cpu().numpy()
    slot = 0
    r = oracle.cluster_row(x, 0, x.spec.retrieval_heads[slot], N, K, 3, p32(0.99))
    assert int(cnt[0, slot]) == cap and len(r.sel) > cap
    assert np.array_equal(idx[0, slot, :cap], r.sel[:cap])  # the truncated list is the set's prefix
    # p = 1 keeps every causal key whatever the clustering
    layer.set_top_p(1.0)
    _, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=cap)
    assert layer.check() == 0 and np.all(st[0].cpu().numpy() == N)
    layer.close()


def test_every_key_its_own_cluster():
    # K = n: every centre is its key, so the clusters taken are single keys ordered by score
    x = synth.generate(synth.spec("toy_decode_4k", prefix=511, index_bf16=True))
    N = x.spec.n_total
    layer = _layer(x, N)
    build_cache(layer, x, N)
    layer.cluster_build(2)
    assert layer.check() == 0
    _check_build(x, layer, N, 2, [N])
    _check_clustered_decode(x, layer, N, 2, [N], [N], 0.9)
    layer.close()


def test_index_key_outside_the_clustering_range_is_reported():
    from long_context_sparse_idx16_b200 import RTP_ERANGE, Layer

    s = synth.spec("toy_decode_4k", prefix=255, index_bf16=True)
    x = synth.generate(s)
    big = (x.wk * 40000.0).astype(np.float32)  # many index keys of magnitude above 2^15
    layer = Layer(batch=s.batch, n_q_heads=s.n_q_heads, n_kv_heads=s.n_kv_heads, head_class=s.head_class,
                  wq=x.wq, wk=big, top_p=s.top_p, window=s.window, n_sink=s.n_sink, max_seq=s.n_total,
                  rope_base=s.rope_base, index_bf16=True, max_chunk=1, n_clusters=8)
    build_cache(layer, x, s.n_total)
    layer.cluster_build(1)
    assert layer.check() == RTP_ERANGE
    layer.close()


def test_dense_prefill_then_clustered_decode():
    # the page's own pipeline (aitntnews page, experiments): retrieval heads attend densely in
    # prefill, the prefill's K cache is clustered, decode selects by clusters
    from long_context_sparse_idx16_b200 import Layer

    C, K = 2048, 64
    s = synth.spec("prefill_32k", prefix=0, chunk=C + 1, window=512, index_bf16=True, prefill_dense=True)
    x = synth.generate(s)
    layer = Layer.from_spec(s, x, max_seq=C + 1, max_chunk=C, n_clusters=K)
    build_cache(layer, x, C)
    out = layer.prefill_chunk(torch_bf16(x.q[:, :C])).cpu().numpy()
    assert layer.check() == 0
    rows = [0, 1, 700, C - 1]
    local = [h for h in range(s.n_q_heads) if h not in s.retrieval_heads][0]
    for h in (s.retrieval_heads[0], s.retrieval_heads[-1], local):
        r = oracle.layer_rows(x, 0, h, rows)  # dense prefill: p = 1 for the retrieval heads
        check_outputs(out[0, rows, h], r.out, f"dense prefill h={h}")
    layer.cluster_build(3)
    build_cache(layer, x, C + 1)  # the decode token's key, cached after the clustering
    assert layer.cluster_len(0) == C
    _check_clustered_decode(x, layer, K, 3, [C + 1], [C], 0.9, row=C)
    layer.close()
