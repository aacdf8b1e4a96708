"""Ragged batches: the sequences of one layer at different lengths, in decode and in chunked
prefill.  Each sequence's rows are checked against the oracle over that sequence's own keys."""
import numpy as np
import pytest

import oracle
import synth
from parity import bitmap_positions, build_cache, check_outputs, check_selection, p32, torch_bf16

pytestmark = pytest.mark.gpu


def _oracle_rows(x, b, h, n, q_rows, positions, p):
    s = x.spec
    ret = h in s.retrieval_heads
    slot = s.retrieval_heads.index(h) if ret else 0
    return oracle.head_rows(x.k[b, :n], x.v[b, :n], q_rows, positions, g=s.kv_head(h), retrieval=ret,
                            wq=x.wq[slot] if ret else None, wk=x.wk[slot] if ret else None, top_p=p,
                            top_k=s.top_k, window=s.window, n_sink=s.n_sink, rope_base=s.rope_base,
                            want_pi=ret, index_bf16=s.index_bf16)


def _ragged_decode(x, lens, *, top_p=None, via_seq=False):
    from long_context_sparse_idx16_b200 import Layer

    s = x.spec
    N = s.n_total
    p = s.top_p if top_p is None else top_p
    layer = Layer.from_spec(s, x, max_seq=N, max_chunk=1)
    if via_seq:  # every sequence appended on its own, in two pieces
        for b, n in enumerate(lens):
            for t0, t1 in ((0, n // 2), (n // 2, n)):
                if t1 > t0:
                    layer.append_kv_seq(b, torch_bf16(x.k[b, t0:t1]), torch_bf16(x.v[b, t0:t1]))
    else:  # the whole batch to N, then every sequence rolled back to its length
        build_cache(layer, x, N)
        for b, n in enumerate(lens):
            layer.truncate_seq(b, n)
    assert [layer.seq_len_of(b) for b in range(s.batch)] == list(lens) and layer.seq_len == max(lens)
    layer.set_top_p(p)
    out, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=N)
    assert layer.check() == 0, "kernel error word set"
    out = out.cpu().numpy()
    cnt, idx = st[0].cpu().numpy(), st[3].cpu().numpy()
    refs, gpus = [], []
    for b, n in enumerate(lens):
        for h in range(s.n_q_heads):
            r = _oracle_rows(x, b, h, n, x.q[b, 0, h], [n - 1], p32(p))
            ref = r.out[0]
            if h in s.retrieval_heads:
                slot = s.retrieval_heads.index(h)
                k = int(cnt[b, slot])
                sel = idx[b, slot, :k].astype(np.int64)
                assert np.all(np.diff(sel) > 0) and (k == 0 or sel[-1] <= n - 1), f"b={b}: positions past its length"
                nd = check_selection(sel, r, 0, p32(p), f"b={b} n={n} h={h}", top_k=s.top_k)
                if nd:
                    ref = oracle.attend_set(x, b, h, 0, sel, pos=n - 1)
            refs.append(ref)
            gpus.append(out[b, h])
    check_outputs(np.stack(gpus), np.stack(refs), f"ragged decode {lens}")
    layer.close()


def _toy(B, **kw):
    return synth.spec("toy_decode_4k", batch=B, needles=(3,) * B, **kw)


@pytest.mark.parametrize("p", [0.9, 1.0])
def test_decode_ragged_lengths(p):
    # a full-length sequence, one inside the window, one of a single key, one past the window;
    # p = 1 takes the dense path (every key of the sequence's own length)
    x = synth.generate(_toy(4))
    _ragged_decode(x, (4096, 300, 1, 2049), top_p=p)


def test_decode_ragged_lengths_appended_per_sequence():
    x = synth.generate(_toy(3, seed=5))
    _ragged_decode(x, (1500, 4096, 777), via_seq=True)


def test_decode_ragged_fixed_top_k_and_bf16_keys():
    # the fixed budget larger than a short sequence keeps all of it
    x = synth.generate(_toy(3, top_k=600, index_bf16=True, seed=6))
    _ragged_decode(x, (4096, 500, 2000))


@pytest.mark.parametrize("p", [0.9, 1.0])
def test_decode_ragged_128k_layer_shape(p):
    # the 128K layer's shape (B=8, 32/4 heads, 5 retrieval heads) with eight different lengths;
    # at p = 1 the longer sequences span more than 64 gather chunks
    s = synth.spec("decode_128k", prefix=16383, needles=(1, 16, 1024, 1, 16, 1024, 1, 16))
    x = synth.generate(s)
    _ragged_decode(x, (16384, 9000, 12345, 1, 16000, 8193, 4097, 300), top_p=p)


def test_prefill_ragged_lengths():
    from long_context_sparse_idx16_b200 import Layer

    C = 200
    s = synth.spec("prefill_32k", batch=3, prefix=2800, chunk=C, needles=(64, 64, 64), window=512)
    x = synth.generate(s)
    N = s.n_total
    lens = (3000, 1700, C)  # the shortest sequence is the chunk alone
    layer = Layer.from_spec(s, x, max_seq=N, max_chunk=C)
    build_cache(layer, x, N)
    for b, n in enumerate(lens):
        layer.truncate_seq(b, n)
    # row i of sequence b sits at position lens[b] - C + i: its keys are that sequence's own
    words = (N + 31) // 32
    out, st = layer.prefill_chunk(torch_bf16(x.q[:, :C]), stats=True, bitmap_words=words)
    assert layer.check() == 0, "kernel error word set"
    out = out.cpu().numpy()
    cnt, bm = st[0].cpu().numpy(), st[2].cpu().numpy()
    p = s.top_p
    refs, gpus = [], []
    rows = np.arange(0, C, 7)
    for b, n in enumerate(lens):
        for h in range(s.n_q_heads):
            r = _oracle_rows(x, b, h, n, x.q[b, rows, h], n - C + rows, p32(p))
            for t, i in enumerate(rows):
                ref = r.out[t]
                if h in s.retrieval_heads:
                    slot = s.retrieval_heads.index(h)
                    pos = n - C + int(i)
                    sel = bitmap_positions(bm[b, i, slot], pos + 1)
                    assert len(sel) == int(cnt[b, i, slot])
                    nd = check_selection(sel, r, t, p32(p), f"b={b} n={n} h={h} row={i}")
                    if nd:
                        ref = oracle.attend_set(x, b, h, int(i), sel, pos=pos)
                refs.append(ref)
                gpus.append(out[b, i, h])
    check_outputs(np.stack(gpus), np.stack(refs), f"ragged prefill {lens}")
    layer.close()


def test_ragged_length_errors():
    import torch

    from long_context_sparse_idx16_b200 import Layer, RTPError

    s = _toy(2)
    x = synth.generate(s)
    layer = Layer.from_spec(s, x, max_seq=100, max_chunk=8)
    k = torch_bf16(x.k[0, :60])
    layer.append_kv_seq(1, k, torch_bf16(x.v[0, :60]))
    assert layer.seq_len_of(0) == 0 and layer.seq_len_of(1) == 60 and layer.seq_len == 60
    with pytest.raises(RTPError):  # sequence 0 is empty
        layer.decode(torch_bf16(x.q[:, 0]))
    with pytest.raises(RTPError):  # 60 + 60 > max_seq for sequence 1
        layer.append_kv_seq(1, k, torch_bf16(x.v[0, :60]))
    with pytest.raises(RTPError):
        layer.append_kv_seq(2, k, torch_bf16(x.v[0, :60]))
    with pytest.raises(RTPError):
        layer.truncate_seq(0, 1)
    layer.truncate(30)  # every sequence longer than 30 rolls back to 30
    assert layer.seq_len_of(1) == 30 and layer.seq_len_of(0) == 0 and layer.seq_len == 30
    layer.close()
    assert torch.cuda.is_available()
