"""GPU chunked-prefill parity: every row of the chunk runs its own top-p selection (retrieval
heads) or its own window (local heads); the CUDA path through the C ABI against the fp64 oracle."""
import numpy as np
import pytest

import synth
from parity import build_cache, run_prefill, torch_bf16

pytestmark = pytest.mark.gpu


def small(name="prefill_32k", **kw):
    base = dict(prefix=0, chunk=300, window=96, n_clusters=8, needles=(64,))
    base.update(kw)
    return synth.generate(synth.spec(name, **base))


def test_prefill_small_from_empty():
    # 300 rows = two full 128-row tiles and a ragged tail of 44; keys 0..299
    run_prefill(small())


def test_prefill_small_with_prefix():
    # rows at positions 1000..1199 over a 1200-key cache; rows of one tile need different cuts
    run_prefill(small(prefix=1000, chunk=200, window=128))


@pytest.mark.parametrize("p", [0.05, 0.5, 0.95, 0.999, 1.0])
def test_prefill_p_sweep(p):
    run_prefill(small(prefix=700, chunk=130, needles=()), top_p=p)


def test_prefill_all_ties():
    # every index score is exactly 0: each row keeps the lowest ceil(p (pos+1)) positions
    x = small(prefix=500, chunk=150, zero_index_weights=True, needles=())
    res = run_prefill(x, exact_sets=True)
    p = float(np.float32(0.9))  # p as the ABI carries it
    for (b, h), (cnt, cnt_ref, nd) in res["summary"].items():
        pos = x.spec.prefix + np.arange(x.spec.chunk)
        assert np.array_equal(cnt, np.ceil(p * (pos + 1)).astype(np.int64)) and nd == 0


@pytest.mark.parametrize("W,S", [(1, 0), (1, 4), (7, 0), (100000, 4), (64, 70)])
def test_prefill_window_shapes(W, S):
    run_prefill(small(prefix=400, chunk=140, window=W, n_sink=S))


def test_prefill_single_row_and_gqa_shapes():
    run_prefill(small(prefix=999, chunk=1))
    run_prefill(small(prefix=300, chunk=100, n_kv_heads=8))  # MHA
    run_prefill(small(prefix=300, chunk=100, n_q_heads=16, n_kv_heads=1, retrieval_heads=(3, 9, 15)))


def test_prefill_two_chunks_in_sequence():
    # the second chunk's rows see the first chunk's keys through the cache
    from long_context_sparse_idx16_b200 import Layer

    x = small(prefix=0, chunk=512)
    s = x.spec
    layer = Layer.from_spec(s, x, max_seq=s.n_total, max_chunk=256)
    build_cache(layer, x, 256)
    first = layer.prefill_chunk(torch_bf16(x.q[:, :256]))
    build_cache(layer, x, 512)
    second = layer.prefill_chunk(torch_bf16(x.q[:, 256:]))
    assert layer.check() == 0
    import torch

    whole = torch.cat([first, second], dim=1).cpu().numpy()
    import oracle
    from parity import check_outputs

    for h in range(s.n_q_heads):
        rows = np.arange(0, 512, 37)
        ref = oracle.layer_rows(x, 0, h, rows).out
        check_outputs(whole[0, rows, h], ref, f"two chunks h={h}")
    layer.close()


def test_prefill_multi_tile_keys_batch2():
    # keys span many 64-key tiles; B=2 with needles planted in different heads
    run_prefill(small(batch=2, prefix=1800, chunk=260, window=512, needles=(1, 16)))


def test_prefill_deterministic():
    x = small(prefix=600, chunk=128)
    a = run_prefill(x)["out"]
    b = run_prefill(x)["out"]
    assert np.array_equal(a, b)


def _spread_rows(C: int, n: int, seed: int, tile: int = 128) -> np.ndarray:
    """n distinct chunk rows: the first and last two, pairs across row-tile boundaries spread
    over the chunk, and seeded random rows (even and odd rows alike)."""
    rows = {0, 1, C - 2, C - 1}
    n_tiles = (C + tile - 1) // tile
    for k in np.linspace(1, n_tiles - 1, min(n_tiles - 1, n // 4)).astype(np.int64):
        rows.update((int(k) * tile - 1, int(k) * tile))
    rng = np.random.default_rng(seed)
    while len(rows) < n:
        rows.add(int(rng.integers(0, C)))
    return np.array(sorted(r for r in rows if 0 <= r < C), dtype=np.int64)


def test_prefill_row_lists_match_bitmap():
    # the row-subset position lists give the same sets as the full bitmap (ragged tail included)
    x = small(prefix=900, chunk=260, window=128)
    rows = [0, 1, 63, 64, 65, 127, 128, 200, 255, 256, 259]
    run_prefill(x, rows=rows, sets="rows")
    run_prefill(x, rows=rows, sets="bitmap")


@pytest.mark.slow
def test_prefill_32k_full_every_retrieval_row():
    # the full 32K chunk (B=1, C=32768 from an empty cache): every row of every retrieval head
    # (sets through the bitmap, outputs), and 512 rows of every local head
    x = synth.generate(synth.spec("prefill_32k"))
    run_prefill(x, rows=None, local_rows=_spread_rows(x.spec.chunk, 512, seed=5), sets="bitmap")


@pytest.mark.slow
def test_prefill_1m_full_sampled_rows():
    # a 16384-row chunk on a 1032192-key prefix: 256 rows of each retrieval head with their sets
    # (row lists), both query types, tile-boundary pairs and the first and last rows; 64 rows of
    # each local head
    x = synth.generate(synth.spec("prefill_1m"))
    C = x.spec.chunk
    rows = _spread_rows(C, 256, seed=6)
    assert len(rows) >= 256 and {0, C - 1} <= set(rows.tolist())
    assert (rows % 2 == 0).any() and (rows % 2 == 1).any()  # needle-aimed and N(0, 1) queries
    run_prefill(x, rows=rows, local_rows=_spread_rows(C, 64, seed=7), sets="rows", row_block=64)


def test_prefill_bitmap_needs_words():
    # a bitmap pointer with no room is an argument error, caught before any launch
    import torch

    from long_context_sparse_idx16_b200 import Layer, RTPError, rtp_prefill_chunk, rtp_prefill_stats

    x = small(prefix=100, chunk=64)
    s = x.spec
    layer = Layer.from_spec(s, x, max_seq=s.n_total, max_chunk=s.chunk)
    build_cache(layer, x, s.n_total)
    q = torch_bf16(x.q)
    out = torch.empty((s.batch, s.chunk, s.n_q_heads, 128), dtype=torch.float32, device="cuda")
    bm = torch.zeros(16, dtype=torch.int32, device="cuda")
    st = rtp_prefill_stats(None, None, bm.data_ptr(), 0, None, 0, None, 0)
    with pytest.raises(RTPError):
        rtp_prefill_chunk(layer.handle, q.data_ptr(), s.chunk, out.data_ptr(), st, 0)
    assert layer.check() == 0
    layer.close()


def test_prefill_chunk_larger_than_cache_is_rejected():
    import torch

    from long_context_sparse_idx16_b200 import Layer, RTPError

    x = small(prefix=0, chunk=128)
    s = x.spec
    layer = Layer.from_spec(s, x, max_seq=s.n_total, max_chunk=s.chunk)
    build_cache(layer, x, 64)  # only half the chunk's keys appended
    with pytest.raises(RTPError):
        layer.prefill_chunk(torch_bf16(x.q))
    layer.close()


def test_prefill_bf16_index_keys():
    # bf16 index-key storage feeds the same tensor-core scoring (its hi/lo split is exact)
    run_prefill(small(prefix=700, chunk=200, window=128, index_bf16=True))
    run_prefill(small(prefix=0, chunk=260, index_bf16=True), top_p=0.5)


def test_prefill_fixed_top_k():
    run_prefill(small(prefix=600, chunk=200, window=128, top_k=40))
    # all ties: each row keeps its lowest min(k, pos + 1) positions
    x = small(prefix=0, chunk=150, zero_index_weights=True, needles=(), top_k=25)
    res = run_prefill(x, exact_sets=True)
    for (b, h), (cnt, cnt_ref, nd) in res["summary"].items():
        assert np.array_equal(cnt, np.minimum(25, np.arange(150) + 1)) and nd == 0


def test_prefill_dense_retrieval_heads():
    # the pages' own prefill: retrieval heads attend to every causal key; decode still selects
    from long_context_sparse_idx16_b200 import Layer
    from parity import run_decode

    x = small(prefix=500, chunk=180, window=64, prefill_dense=True)
    run_prefill(x, sets=None)
    xd = synth.generate(synth.spec("toy_decode_4k", prefill_dense=True))
    run_decode(xd)


def test_prefill_long_rows_split_over_attention_ctas():
    # 300K cached keys: each row tile's keys are split over two attention CTAs whose partial
    # softmax states the last one merges; sets through the bitmap, outputs against the oracle
    x = synth.generate(synth.spec("prefill_1m", prefix=300000, chunk=200))
    run_prefill(x, rows=np.arange(0, 200, 3), local_rows=np.arange(0, 200, 25), heads=[0, 1, 13, 26], sets="bitmap")
