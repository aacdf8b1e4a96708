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
