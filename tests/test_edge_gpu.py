"""Edge cases of the layer on the GPU: an empty cache, a full cache, a selection larger than
max_select, and a truncated cache appended again."""
import numpy as np
import pytest

import synth
from parity import build_cache, torch_bf16

pytestmark = pytest.mark.gpu


def test_decode_on_empty_cache_is_rejected():
    from long_context_sparse_idx16_b200 import RTP_EINVAL, Layer, RTPError

    x = synth.generate(synth.spec("toy_decode_4k", prefix=63))
    layer = Layer.from_spec(x.spec, x, max_chunk=1)
    with pytest.raises(RTPError) as e:
        layer.decode(torch_bf16(x.q[:, 0]))
    assert e.value.status == RTP_EINVAL
    assert layer.check() == 0
    layer.close()


def test_append_beyond_capacity_is_rejected_without_writing():
    from long_context_sparse_idx16_b200 import RTP_ECAPACITY, Layer, RTPError

    x = synth.generate(synth.spec("toy_decode_4k", prefix=63))
    s = x.spec
    layer = Layer.from_spec(s, x, max_seq=s.n_total, max_chunk=1)
    build_cache(layer, x, s.n_total - 8)
    with pytest.raises(RTPError) as e:  # 16 more tokens than the 8 slots left
        layer.append_kv(torch_bf16(x.k[:, :16]), torch_bf16(x.v[:, :16]))
    assert e.value.status == RTP_ECAPACITY
    assert layer.seq_len == s.n_total - 8
    build_cache(layer, x, s.n_total)  # the cache still fills up to max_seq
    assert layer.seq_len == s.n_total
    assert layer.check() == 0
    layer.close()


def test_selection_larger_than_max_select_is_reported():
    # p = 0.999 without needles selects about a thousand keys per head; the lists hold 64
    import torch

    from long_context_sparse_idx16_b200 import RTP_EOVERFLOW, Layer

    s = synth.spec("toy_decode_4k", needles=(), top_p=0.999)
    x = synth.generate(s)
    cap = 64
    layer = Layer.from_spec(s, x, max_chunk=1, max_select=cap)
    build_cache(layer, x, s.n_total)
    out, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=cap)
    assert layer.check() == RTP_EOVERFLOW
    assert layer.check() == 0  # reported once, then cleared
    cnt = st[0].cpu().numpy()
    assert (cnt == cap).all()
    idx = st[3].cpu().numpy()
    assert (np.diff(idx, axis=-1) > 0).all()  # the kept prefix of each list is ascending
    assert torch.isfinite(out).all()
    layer.close()


def test_truncate_and_append_again_gives_the_same_decode():
    import torch

    from long_context_sparse_idx16_b200 import Layer

    x = synth.generate(synth.spec("toy_decode_4k", prefix=1023))
    s = x.spec
    layer = Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, s.n_total)
    q = torch_bf16(x.q[:, 0])
    o1 = layer.decode(q)
    layer.truncate(s.n_total - 100)
    build_cache(layer, x, s.n_total)
    o2 = layer.decode(q)
    torch.cuda.synchronize()
    assert layer.check() == 0
    assert torch.equal(o1, o2)
    layer.close()


def test_decode_barrier_timeout_is_reported_and_recovers():
    """A grid-barrier wait limit of one clock cycle makes the decode selection give up at its
    first barrier: rtp_check reports RTP_ETIMEOUT once and resets the selection scratch, and
    with the default limit restored the next decode on the same layer matches the oracle."""
    from long_context_sparse_idx16_b200 import RTP_ETIMEOUT, Layer
    from parity import run_decode

    # 32K keys x 2 retrieval heads: a cooperative grid of 16 CTAs, so the first CTA to reach a
    # barrier has to wait for the others
    x = synth.generate(synth.spec("toy_decode_4k", prefix=32767))
    s = x.spec
    layer = Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, s.n_total)
    run_decode(x, layer=layer)  # a clean decode first
    layer.set_wait_limit(1)
    q = torch_bf16(x.q[:, 0])
    seen = None
    for _ in range(5):
        layer.decode(q)
        seen = layer.check()
        if seen == RTP_ETIMEOUT:
            break
    assert seen == RTP_ETIMEOUT
    assert layer.check() == 0  # reported once, then cleared
    layer.set_wait_limit(0)
    for _ in range(2):  # two clean decodes after the reset: the scratch starts from zero
        run_decode(x, layer=layer)
    layer.close()


def test_value_outside_fp16_range_is_reported():
    """A value beyond the fp16 cache range (|x| > 65504, representable in the bf16 input) makes
    the append record RTP_ERANGE; rolling the token back and appending a good one leaves a
    layer whose decode matches the oracle."""
    from long_context_sparse_idx16_b200 import RTP_ERANGE, Layer
    from parity import run_decode

    x = synth.generate(synth.spec("toy_decode_4k", prefix=1023))
    s = x.spec
    N = s.n_total
    layer = Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, N - 1)
    bad_v = x.v[:, N - 1:N].copy()
    bad_v[0, 0, 1, 5] = 0x47C3  # bf16 bits of 99840.0
    layer.append_kv(torch_bf16(x.k[:, N - 1:N]), torch_bf16(bad_v))
    assert layer.check() == RTP_ERANGE
    assert layer.check() == 0
    layer.truncate(N - 1)
    build_cache(layer, x, N)
    run_decode(x, layer=layer)
    layer.close()
