"""The no-allocation attention entry point (rtp_gather_attn_noalloc) against the fp64 oracle.

The entry point exists for callers that cannot allocate device memory: code running while a
CUDA graph is captured (allocation cannot be captured), engines that own all device memory
through their own pool, processes whose device memory is fully committed.  Its outputs are
compared with the oracle's exact attention over the same key lists, and with the layer's own
decode, on two calls in a row.  This file is collected last so that a run stopping at the first
failure has already run every other test; it also passes alone in a fresh process (its first
call looks up the built-in scratch array's address).
"""
import math

import numpy as np
import pytest

import oracle
import synth
from parity import ABS_TOL, REL_L2_TOL, build_cache, check_outputs, torch_bf16

pytestmark = pytest.mark.gpu


def test_noalloc_gather_matches_oracle_and_layer_twice():
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
    layer_out = torch.stack([out[b, h] for b in range(B) for h in s.retrieval_heads]).cpu().numpy()
    cnt_h, idx_h = cnt.cpu().numpy().ravel(), idx.cpu().numpy().reshape(B * Hr, N)
    ref = np.stack([oracle.attend_set(x, b, h, 0, idx_h[b * Hr + i, :cnt_h[b * Hr + i]])
                    for b in range(B) for i, h in enumerate(s.retrieval_heads)])
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
        check_outputs(r, ref, "no-alloc vs oracle")
        err = np.abs(r - layer_out).max()
        rel = np.linalg.norm(r - layer_out) / np.linalg.norm(layer_out)
        assert err <= ABS_TOL and rel <= REL_L2_TOL, (err, rel)
    assert np.array_equal(results[0], results[1])
    # sizes beyond the built-in scratch are rejected before any launch
    with pytest.raises(rtp.RTPError) as ei:
        rtp.rtp_gather_attn_noalloc(view.k, view.v, None, view.max_seq * 128, q_d.data_ptr(), idx.data_ptr(),
                                    1 << 20, cnt.data_ptr(), 40, 1 << 20, 0.088, o.data_ptr(), stream)
    assert ei.value.status == rtp.RTP_EINVAL
    layer.close()


def _h2f(bits: np.ndarray) -> np.ndarray:
    return bits.view(np.float16).astype(np.float64)


def test_noalloc_gather_edge_problems():
    """kv_block = NULL (one KV block per problem), an empty list (output zeros), a count above
    max_count (clamped), a single-chunk problem beside multi-chunk ones in the same call, and
    repeated positions; compared with a plain fp64 softmax over the listed fp16 rows."""
    import torch

    import long_context_sparse_idx16_b200 as rtp

    rng = np.random.default_rng(11)
    P, L, D = 6, 1500, 128
    max_count = 700
    kv = rng.standard_normal((2, P, L, D)).astype(np.float16)
    q = rng.standard_normal((P, D)).astype(np.float32)
    counts = np.array([0, 90, 700, 1400, 129, 300], dtype=np.int32)  # 1400 > max_count: clamped to 700
    idx = np.zeros((P, max_count), dtype=np.int32)
    for p in range(P):
        n = min(int(counts[p]), max_count)
        if p == 5:  # positions may repeat and come in any order
            idx[p, :n] = rng.integers(0, 40, n)
        else:
            idx[p, :n] = rng.choice(L, n, replace=False)
    scale = 1.0 / math.sqrt(D)
    ref = np.zeros((P, D))
    for p in range(P):
        n = min(int(counts[p]), max_count)
        if n == 0:
            continue
        K = kv[0, p, idx[p, :n]].astype(np.float64)
        V = kv[1, p, idx[p, :n]].astype(np.float64)
        z = (K @ q[p].astype(np.float64)) * scale
        w = np.exp(z - z.max())
        ref[p] = (w / w.sum()) @ V
    k_d = torch.from_numpy(kv[0].copy()).cuda()
    v_d = torch.from_numpy(kv[1].copy()).cuda()
    q_d = torch.from_numpy(q).cuda()
    idx_d = torch.from_numpy(idx).cuda()
    cnt_d = torch.from_numpy(counts).cuda()
    stream = torch.cuda.current_stream().cuda_stream
    results = []
    for _ in range(2):
        o = torch.full((P, D), float("nan"), dtype=torch.float32, device="cuda")
        rtp.rtp_gather_attn_noalloc(k_d.data_ptr(), v_d.data_ptr(), None, L * D, q_d.data_ptr(), idx_d.data_ptr(),
                                    max_count, cnt_d.data_ptr(), P, max_count, scale, o.data_ptr(), stream)
        torch.cuda.synchronize()
        results.append(o.cpu().numpy())
    for r in results:
        assert np.all(r[0] == 0.0)  # the empty problem's row is zeros
        check_outputs(r[1:], ref[1:], "no-alloc edge problems")
    assert np.array_equal(results[0], results[1])
