"""GPU decode parity: the CUDA path (through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest

import synth
from parity import run_decode

pytestmark = pytest.mark.gpu


def test_decode_toy_4k():
    x = synth.generate(synth.spec("toy_decode_4k"))
    res = run_decode(x)
    # the three planted needles are selected by their heads
    for (b, h), npos in x.needle_pos.items():
        assert res["summary"][(b, h)][0] >= len(npos)


@pytest.mark.parametrize("p", [0.05, 0.5, 0.8, 0.95, 0.999, 1.0])
def test_decode_toy_no_needles_p_sweep(p):
    # without needles the index softmax is diffuse: hundreds to thousands of keys selected
    x = synth.generate(synth.spec("toy_decode_4k", needles=()))
    run_decode(x, top_p=p)


@pytest.mark.parametrize("prefix", [0, 1, 2, 3, 16, 511, 1000])
def test_decode_short_contexts(prefix):
    x = synth.generate(synth.spec("toy_decode_4k", prefix=prefix, needles=()))
    run_decode(x)


def test_decode_all_ties():
    # zero index weights: every index score is exactly 0, the cut falls inside one tie group
    # and the lowest positions must be taken
    x = synth.generate(synth.spec("toy_decode_4k", zero_index_weights=True, needles=()))
    res = run_decode(x)
    N = x.spec.n_total
    for (b, h), (k, k_ref, nd) in res["summary"].items():
        assert k == int(np.ceil(0.9 * N)) and nd == 0


@pytest.mark.parametrize("W,S", [(1, 0), (1, 4), (7, 0), (4096, 0), (100000, 4), (512, 600)])
def test_decode_window_shapes(W, S):
    x = synth.generate(synth.spec("toy_decode_4k", window=W, n_sink=S, prefix=2047))
    run_decode(x)


def test_decode_gqa_mha_and_wide_groups():
    x = synth.generate(synth.spec("toy_decode_4k", n_kv_heads=8, prefix=1023))  # MHA
    run_decode(x)
    x = synth.generate(synth.spec("toy_decode_4k", n_q_heads=16, n_kv_heads=1, retrieval_heads=(3, 9, 15),
                                  prefix=1023))  # 16 query heads on one KV head
    run_decode(x)


@pytest.mark.parametrize("p", [0.999, 1.0])
def test_decode_long_selections_span_many_ctas(p):
    # ~16K selected keys per problem: more than 64 gather chunks, so the gather's work items
    # run over several chunks each (p = 1 through the dense path; p = 0.999 with all index
    # scores tied, through the selected lists: the lowest ceil(0.999 N) positions)
    x = synth.generate(synth.spec("decode_128k", batch=2, prefix=16383, needles=(), query_mode="gauss",
                                  zero_index_weights=p < 1.0))
    res = run_decode(x, top_p=p)
    assert min(k for k, _, _ in res["summary"].values()) > 64 * 128


def test_decode_128k_layer_short():
    # the 128K layer shape (B=8, 32/4 heads, 5 retrieval heads, W=8192) at 16K context
    x = synth.generate(synth.spec("decode_128k", prefix=16383,
                                  needles=(1, 16, 1024, 1, 16, 1024, 1, 16)))
    run_decode(x)


def test_decode_deterministic():
    import torch

    from long_context_sparse_idx16_b200 import Layer
    from parity import build_cache, torch_bf16

    x = synth.generate(synth.spec("toy_decode_4k", needles=()))
    s = x.spec
    layer = Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, s.n_total)
    q = torch_bf16(x.q[:, 0])
    o1, st1 = layer.decode(q, stats=True, sel_cap=s.n_total)
    o2, st2 = layer.decode(q, stats=True, sel_cap=s.n_total)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    for a, b in zip(st1, st2):
        assert torch.equal(a, b)
    layer.close()


@pytest.mark.parametrize("p", [0.8, 0.9, 0.95])
def test_decode_1m_full_size(p):
    # Full 1M-context decode workload (B=1, N=2^20); every retrieval head and four local heads
    # checked against the oracle.  The layer is built once and reused across p.
    from long_context_sparse_idx16_b200 import Layer
    from parity import build_cache

    key = "decode_1m"
    st = _state.get(key)
    if st is None:
        x = synth.generate(synth.spec("decode_1m"))
        layer = Layer.from_spec(x.spec, x, max_chunk=1)
        build_cache(layer, x, x.spec.n_total)
        st = _state[key] = (x, layer)
    x, layer = st
    heads = list(x.spec.retrieval_heads) + [1, 8, 17, 31]
    res = run_decode(x, top_p=p, heads=heads, layer=layer)
    counts = [v[0] for v in res["summary"].values()]
    assert max(counts) >= 100 and min(counts) <= 64  # budgets span orders of magnitude
    span = _state.setdefault("decode_1m_counts", {})
    span[p] = counts
    if len(span) == 3:
        # over the p sweep the set sizes span about 10 to 10^4 (needle-aimed queries keep a
        # dozen keys, the Gaussian query about eight thousand at p = 0.95)
        allc = [c for v in span.values() for c in v]
        assert min(allc) <= 16 and max(allc) >= 8000, (min(allc), max(allc))


def test_decode_128k_full_size():
    # Full 128K decode workload (B=8), decoded twice on one layer: the selection scratch is
    # cleaned by each launch for the next, and the exact selection makes both launches give
    # the same bits.  The layer is then checked against the oracle.
    import torch

    from long_context_sparse_idx16_b200 import Layer
    from parity import build_cache, torch_bf16

    x = synth.generate(synth.spec("decode_128k"))
    s = x.spec
    layer = Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, s.n_total)
    q = torch_bf16(x.q[:, 0])
    o1, st1 = layer.decode(q, stats=True, sel_cap=s.n_total)
    o2, st2 = layer.decode(q, stats=True, sel_cap=s.n_total)
    torch.cuda.synchronize()
    assert layer.check() == 0
    assert torch.equal(o1, o2)
    for a, b in zip(st1, st2):
        assert torch.equal(a, b)
    heads = list(s.retrieval_heads) + [2, 12, 20, 31]
    run_decode(x, heads=heads, layer=layer)
    layer.close()


_state = {}


def test_decode_bf16_index_keys():
    # bf16 index-key storage: the oracle rounds its fp64 index keys to bf16 the same way
    run_decode(synth.generate(synth.spec("toy_decode_4k", index_bf16=True)))
    run_decode(synth.generate(synth.spec("decode_128k", prefix=16383, index_bf16=True,
                                         needles=(1, 16, 1024, 1, 16, 1024, 1, 16))))


def test_decode_1m_bf16_index_keys():
    # the full 1M workload with bf16 index keys (half the index stream), p = 0.9
    x = synth.generate(synth.spec("decode_1m", index_bf16=True))
    res = run_decode(x, top_p=0.9, heads=list(x.spec.retrieval_heads) + [1, 31])
    counts = [v[0] for v in res["summary"].values()]
    assert max(counts) >= 1000 and min(counts) <= 16


@pytest.mark.parametrize("k", [1, 64, 700, 5000])
def test_decode_fixed_top_k(k):
    # the pages' fixed-budget ablation: each retrieval head keeps its k highest-scoring keys
    # (5000 > N = 4096 keeps every key)
    run_decode(synth.generate(synth.spec("toy_decode_4k", top_k=k)))


def test_decode_fixed_top_k_ties_and_128k_layer():
    # all index scores equal: the budget takes the lowest positions
    x = synth.generate(synth.spec("toy_decode_4k", top_k=300, zero_index_weights=True, needles=()))
    res = run_decode(x)
    assert all(v[0] == 300 and v[2] == 0 for v in res["summary"].values())
    run_decode(synth.generate(synth.spec("decode_128k", prefix=16383, top_k=4096,
                                         needles=(1, 16, 1024, 1, 16, 1024, 1, 16))))


@pytest.mark.parametrize("k", [4096, 16384])
def test_decode_1m_fixed_top_k(k):
    # the pages' budgets (4096 and 16384 tokens) at 1M keys
    x = synth.generate(synth.spec("decode_1m", top_k=k))
    res = run_decode(x, heads=list(x.spec.retrieval_heads) + [2])
    assert all(v[0] == k for (b, h), v in res["summary"].items())
