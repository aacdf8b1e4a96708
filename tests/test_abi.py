"""The C-ABI library loads, exports every entry point include/*.h declares, lays out its
structs as a C compiler does, and rejects bad arguments on the host (no GPU needed)."""
import ctypes as C
import glob
import os
import re
import subprocess
import tempfile

import pytest

import long_context_sparse_idx16_b200 as rtp
from long_context_sparse_idx16_b200 import build as rtp_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    rtp_build.build()
    return rtp.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(rtp_\w+)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "rtp_create" in names and "rtp_prefill_chunk" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", rtp.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\b(rtp_\w+)\b", out))
    assert set(names) <= exported


def test_struct_layout_matches_c():
    src = r'''
#include <stddef.h>
#include <stdio.h>
#include "rtp.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(rtp_config), offsetof(rtp_config, max_seq),
         offsetof(rtp_config, rope_base), offsetof(rtp_config, wq_index),
         offsetof(rtp_config, max_select), offsetof(rtp_config, max_chunk),
         offsetof(rtp_config, index_bf16), offsetof(rtp_config, top_k));
  printf("%zu %zu %zu %zu %zu %zu\n", offsetof(rtp_config, n_clusters), sizeof(rtp_cluster_view),
         offsetof(rtp_cluster_view, n_clusters), offsetof(rtp_cluster_view, ready),
         offsetof(rtp_cluster_view, max_seq), offsetof(rtp_cluster_view, assign_stride));
  printf("%zu %zu %zu %zu %zu %zu\n", sizeof(rtp_decode_stats), offsetof(rtp_decode_stats, sel_index_cap),
         sizeof(rtp_cache_view), offsetof(rtp_cache_view, idx_bf16), sizeof(rtp_prefill_stats),
         offsetof(rtp_prefill_stats, row_sel_cap));
  return 0;
}
'''
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        open(c, "w").write(src)
        exe = os.path.join(d, "p")
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), "-I", "/usr/local/cuda/include", c, "-o", exe])
        a, c3, b = subprocess.check_output([exe], text=True).splitlines()
    cfg = rtp.rtp_config
    assert [int(t) for t in a.split()] == [C.sizeof(cfg), cfg.max_seq.offset, cfg.rope_base.offset,
                                          cfg.wq_index.offset, cfg.max_select.offset, cfg.max_chunk.offset,
                                          cfg.index_bf16.offset, cfg.top_k.offset]
    cv = rtp.rtp_cluster_view
    assert [int(t) for t in c3.split()] == [cfg.n_clusters.offset, C.sizeof(cv), cv.n_clusters.offset,
                                           cv.ready.offset, cv.max_seq.offset, cv.assign_stride.offset]
    st = rtp.rtp_decode_stats
    ps = rtp.rtp_prefill_stats
    assert [int(t) for t in b.split()] == [C.sizeof(st), st.sel_index_cap.offset, C.sizeof(rtp.rtp_cache_view),
                                          rtp.rtp_cache_view.idx_bf16.offset, C.sizeof(ps),
                                          ps.row_sel_cap.offset]


def _cfg(**kw):
    import numpy as np

    hc = np.array([1, 0, 0, 0], dtype=np.uint8)
    w = np.zeros((1, 128, 16), dtype=np.float32)
    base = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, index_dim=16, max_seq=64,
                head_class=hc.ctypes.data, top_p=0.9, window=8, n_sink=2, rope_base=1e6, sm_scale=0.0,
                wq_index=w.ctypes.data, wk_index=w.ctypes.data, max_select=0, max_chunk=0)
    base.update(kw)
    return rtp.rtp_config(**base), (hc, w)


@pytest.mark.parametrize("bad", [dict(head_dim=64), dict(index_dim=8), dict(top_p=0.0), dict(top_p=1.5),
                                 dict(n_kv_heads=3), dict(window=0), dict(n_sink=-1), dict(max_seq=0),
                                 dict(max_select=65), dict(batch=0), dict(head_class=None),
                                 dict(n_q_heads=64, n_kv_heads=2), dict(rope_base=1.0), dict(sm_scale=-1.0),
                                 dict(max_chunk=-1), dict(max_seq=1 << 31), dict(wq_index=None), dict(index_bf16=2), dict(top_k=-1), dict(prefill_dense=3),
                                 dict(wk_index=None), dict(top_p=float("nan")), dict(max_select=-1),
                                 dict(n_clusters=-1), dict(n_clusters=1025), dict(n_clusters=8),
                                 dict(n_clusters=8, index_bf16=1, top_k=16)])
def test_create_rejects_bad_config_on_host(lib, bad):
    cfg, keep = _cfg(**bad)
    h = C.c_void_p()
    st = lib.rtp_create(C.byref(cfg), C.byref(h))
    assert st == rtp.RTP_EINVAL
    assert h.value is None
    assert rtp.rtp_last_error(None).startswith("rtp_create")


def test_calls_on_null_layer_are_rejected(lib):
    assert lib.rtp_append_kv(None, None, None, 1, None) == rtp.RTP_EINVAL
    assert lib.rtp_decode(None, None, None, None, None) == rtp.RTP_EINVAL
    assert lib.rtp_prefill_chunk(None, None, 1, None, None, None) == rtp.RTP_EINVAL
    assert lib.rtp_set_top_p(None, 0.5) == rtp.RTP_EINVAL
    assert lib.rtp_seq_len(None) == -1
    assert lib.rtp_destroy(None) == rtp.RTP_OK
    assert lib.rtp_create(None, None) == rtp.RTP_EINVAL
    assert lib.rtp_cluster_build(None, 4, None) == rtp.RTP_EINVAL
    assert lib.rtp_cluster_drop(None) == rtp.RTP_EINVAL
    assert lib.rtp_cluster_len(None, 0) == -1
    assert lib.rtp_get_clusters(None, None) == rtp.RTP_EINVAL


def test_create_rejects_bad_head_maps_on_host(lib):
    import numpy as np

    # a class entry other than 0 (local) or 1 (retrieval)
    hc = np.array([1, 2, 0, 0], dtype=np.uint8)
    cfg, keep = _cfg(head_class=hc.ctypes.data)
    h = C.c_void_p()
    assert lib.rtp_create(C.byref(cfg), C.byref(h)) == rtp.RTP_EINVAL
    assert h.value is None
    # more (sequence, retrieval head) problems than the selection scratch is laid out for
    hc = np.ones(16, dtype=np.uint8)
    cfg, keep = _cfg(batch=129, n_q_heads=16, n_kv_heads=1, head_class=hc.ctypes.data)
    assert lib.rtp_create(C.byref(cfg), C.byref(h)) == rtp.RTP_EINVAL
    assert h.value is None
    assert "2048" in rtp.rtp_last_error(None)


def test_noalloc_gather_rejects_misaligned_arguments_on_host(lib):
    """The allocation-free attention reads K/V rows and queries as 16-byte vectors: a stride that
    is not a multiple of 8 fp16 elements, or a K, V or q pointer off a 16-byte boundary, is
    refused before any CUDA call (the pointers here are never dereferenced)."""
    base = 1 << 20
    args = dict(k=base, v=base + 4096, kv_block=None, kv_stride=128, q=base + 8192, idx=base + 12288,
                idx_stride=16, cnt=base + 16384, P=1, max_count=16, sm_scale=0.088, out=base + 20480,
                stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return lib.rtp_gather_attn_noalloc(a["k"], a["v"], a["kv_block"], a["kv_stride"], a["q"], a["idx"],
                                           a["idx_stride"], a["cnt"], a["P"], a["max_count"], a["sm_scale"],
                                           a["out"], a["stream"])

    assert call(kv_stride=130) == rtp.RTP_EINVAL
    assert "16-byte" in rtp.rtp_last_error(None)
    assert call(kv_stride=1028) == rtp.RTP_EINVAL
    assert call(k=base + 8) == rtp.RTP_EINVAL
    assert call(v=base + 4100) == rtp.RTP_EINVAL
    assert call(q=base + 8196) == rtp.RTP_EINVAL
    assert call(P=0) == rtp.RTP_EINVAL
    assert call(idx_stride=8) == rtp.RTP_EINVAL
