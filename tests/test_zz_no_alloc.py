"""The no-allocation attention entry point (rtp_gather_attn_noalloc) gives the same outputs as
the layer's own decode for the retrieval heads, on two calls in a row.

It exists for callers that cannot allocate device memory (graph capture, engines owning all
device memory, fully committed devices).  This file is collected last so that a run stopping
at the first failure has already run every other test; it also passes alone in a fresh process
(its first call looks up the built-in scratch array's address).
"""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import ABS_TOL, REL_L2_TOL, build_cache, torch_bf16

pytestmark = pytest.mark.gpu


def test_noalloc_gather_matches_layer_decode_twice():
    import torch

    import long_context_sparse_idx16_b200 as rtp

    # no needles and p = 0.999: about a thousand selected keys per head, several 128-key chunks
    s = synth.spec("toy_decode_4k", needles=(), top_p=0.999)
    x = synth.generate(s)
    layer = rtp.Layer.from_spec(s, x, max_chunk=1)
    build_cache(layer, x, s.n_total)
    N = s.n_total
    out, st = layer.decode(torch_bf16(x.q[:, 0]), stats=True, sel_cap=N)
    torch.cuda.synchronize()
    cnt = st[0].contiguous()  # [B][Hr]
    idx = st[3].contiguous()  # [B][Hr][N]
    assert int(cnt.min()) > 128  # several 128-key chunks per problem: the merge path runs
    view = layer.cache()
    B, Hr = s.batch, len(s.retrieval_heads)
    # RoPE'd fp32 queries of the retrieval heads at position N-1, and their KV blocks
    qr = np.zeros((B * Hr, 128), dtype=np.float32)
    blk = np.zeros(B * Hr, dtype=np.int32)
    for b in range(B):
        for i, h in enumerate(s.retrieval_heads):
            qv = synth.bf16_bits_to_f32(x.q[b, 0, h]).astype(np.float64)
            qr[b * Hr + i] = oracle.rope(qv, N - 1, s.rope_base).astype(np.float32)
            blk[b * Hr + i] = b * s.n_kv_heads + s.kv_head(h)
    q_d = torch.from_numpy(qr).cuda()
    blk_d = torch.from_numpy(blk).cuda()
    ref = torch.stack([out[b, h] for b in range(B) for h in s.retrieval_heads]).cpu().numpy()
    stream = torch.cuda.current_stream().cuda_stream
    results = []
    for _ in range(2):
        o = torch.full((B * Hr, 128), float("nan"), dtype=torch.float32, device="cuda")
        rtp.rtp_gather_attn_noalloc(view.k, view.v, blk_d.data_ptr(), view.max_seq * 128, q_d.data_ptr(),
                                    idx.data_ptr(), N, cnt.data_ptr(), B * Hr, N, 1.0 / math.sqrt(128),
                                    o.data_ptr(), stream)
        torch.cuda.synchronize()
        results.append(o.cpu().numpy())
    for r in results:
        assert np.all(np.isfinite(r))
        err = np.abs(r - ref).max()
        rel = np.linalg.norm(r - ref) / np.linalg.norm(ref)
        assert err <= ABS_TOL and rel <= REL_L2_TOL, (err, rel)
    assert np.array_equal(results[0], results[1])
    # sizes beyond the built-in scratch are rejected before any launch
    with pytest.raises(rtp.RTPError) as ei:
        rtp.rtp_gather_attn_noalloc(view.k, view.v, None, view.max_seq * 128, q_d.data_ptr(), idx.data_ptr(),
                                    1 << 20, cnt.data_ptr(), 40, 1 << 20, 0.088, o.data_ptr(), stream)
    assert ei.value.status == rtp.RTP_EINVAL
    layer.close()
