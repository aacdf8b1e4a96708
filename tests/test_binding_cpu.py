"""Argument checks of the Python binding's Layer methods (no GPU needed).

The library reads and writes raw device pointers sized from the layer's configuration, so
the binding refuses tensors of the wrong shape, dtype, device or memory layout before any
library call.  These tests build a Layer object without a device (a null library handle):
whatever passes the checks reaches the library, whose null-layer check answers RTP_EINVAL.
"""
import pytest

torch = pytest.importorskip("torch")

from long_context_sparse_idx16_b200 import Layer, RTPError  # noqa: E402


class _Stream:
    cuda_stream = 0


S = _Stream()


def _layer(device="cpu"):
    lay = Layer.__new__(Layer)
    lay.batch, lay.n_q_heads, lay.n_kv_heads, lay.n_retrieval = 2, 4, 2, 1
    lay.device = torch.device(device)
    lay.handle = None
    return lay


def _kv(T=3, B=2, H=2, dtype=torch.bfloat16):
    return torch.zeros((B, T, H, 128), dtype=dtype), torch.zeros((B, T, H, 128), dtype=dtype)


def test_append_kv_checks():
    lay = _layer()
    k, v = _kv()
    with pytest.raises(RTPError):  # valid tensors reach the library (null layer)
        lay.append_kv(k, v, stream=S)
    with pytest.raises(ValueError, match="dtype"):
        lay.append_kv(*_kv(dtype=torch.float32), stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.append_kv(*_kv(B=1), stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.append_kv(*_kv(H=4), stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.append_kv(k, torch.zeros((2, 2, 2, 128), dtype=torch.bfloat16), stream=S)
    with pytest.raises(ValueError, match="4-dimensional"):
        lay.append_kv(k[0], v[0], stream=S)
    kt = torch.zeros((2, 2, 3, 128), dtype=torch.bfloat16).transpose(1, 2)  # right shape, strided
    with pytest.raises(ValueError, match="contiguous"):
        lay.append_kv(kt, v, stream=S)
    with pytest.raises(ValueError, match="tensor on cuda"):
        _layer("cuda").append_kv(k, v, stream=S)


def test_decode_checks():
    lay = _layer()
    q = torch.zeros((2, 4, 128), dtype=torch.bfloat16)
    out = torch.zeros((2, 4, 128), dtype=torch.float32)
    with pytest.raises(RTPError):
        lay.decode(q, out, stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.decode(torch.zeros((2, 8, 128), dtype=torch.bfloat16), out, stream=S)
    with pytest.raises(ValueError, match="dtype"):
        lay.decode(q.float(), out, stream=S)
    with pytest.raises(ValueError, match="dtype"):
        lay.decode(q, out.to(torch.bfloat16), stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.decode(q, torch.zeros((2, 4, 64), dtype=torch.float32), stream=S)
    with pytest.raises(ValueError, match="sel_cap"):
        lay.decode(q, out, stats=True, sel_cap=-1, stream=S)


def test_prefill_chunk_checks():
    lay = _layer()
    q = torch.zeros((2, 5, 4, 128), dtype=torch.bfloat16)
    out = torch.zeros((2, 5, 4, 128), dtype=torch.float32)
    with pytest.raises(RTPError):
        lay.prefill_chunk(q, out, stream=S)
    with pytest.raises(ValueError, match="4-dimensional"):
        lay.prefill_chunk(q[0], stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.prefill_chunk(q, torch.zeros((2, 6, 4, 128), dtype=torch.float32), stream=S)
    with pytest.raises(ValueError, match="shape"):
        lay.prefill_chunk(torch.zeros((3, 5, 4, 128), dtype=torch.bfloat16), stream=S)
    with pytest.raises(ValueError, match="bitmap_words"):
        lay.prefill_chunk(q, out, stats=True, bitmap_words=-2, stream=S)
    with pytest.raises(TypeError):
        lay.prefill_chunk(q, out.numpy(), stream=S)
