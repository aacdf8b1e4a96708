"""Python binding of librtp (include/rtp.h): the head-wise sparse attention layer on B200.

Argument marshalling only.  Every step of the layer runs in the CUDA kernels of
librtp.so; PyTorch provides device memory and the current stream.  Importing the
package does not need a GPU, but every call does, and the library must have been built
(``python -m long_context_sparse_idx16_b200.build``): there is no fallback of any kind.

The module-level functions carry the C names (rtp_create, rtp_append_kv, rtp_decode,
rtp_prefill_chunk, rtp_destroy, ...); ``Layer`` wraps them for torch tensors.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Sequence

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librtp.so")

RTP_OK, RTP_EINVAL, RTP_ENOMEM, RTP_ECAPACITY, RTP_EOVERFLOW = 0, 1, 2, 3, 4
RTP_ECUDA, RTP_ETIMEOUT, RTP_EINTERNAL, RTP_ERANGE = 5, 6, 7, 8
STATUS_NAMES = {0: "RTP_OK", 1: "RTP_EINVAL", 2: "RTP_ENOMEM", 3: "RTP_ECAPACITY", 4: "RTP_EOVERFLOW",
                5: "RTP_ECUDA", 6: "RTP_ETIMEOUT", 7: "RTP_EINTERNAL", 8: "RTP_ERANGE"}


class rtp_config(C.Structure):
    _fields_ = [
        ("batch", C.c_int32), ("n_q_heads", C.c_int32), ("n_kv_heads", C.c_int32),
        ("head_dim", C.c_int32), ("index_dim", C.c_int32), ("max_seq", C.c_int64),
        ("head_class", C.c_void_p), ("top_p", C.c_float), ("window", C.c_int32),
        ("n_sink", C.c_int32), ("rope_base", C.c_double), ("sm_scale", C.c_float),
        ("wq_index", C.c_void_p), ("wk_index", C.c_void_p), ("max_select", C.c_int64),
        ("max_chunk", C.c_int32), ("index_bf16", C.c_int32), ("prefill_dense", C.c_int32),
        ("top_k", C.c_int64), ("n_clusters", C.c_int32),
    ]


class rtp_decode_stats(C.Structure):
    _fields_ = [("sel_count", C.c_void_p), ("sel_mass", C.c_void_p), ("threshold", C.c_void_p),
                ("sel_index", C.c_void_p), ("sel_index_cap", C.c_int64)]


class rtp_prefill_stats(C.Structure):
    _fields_ = [("sel_count", C.c_void_p), ("sel_mass", C.c_void_p), ("sel_bitmap", C.c_void_p),
                ("bitmap_words", C.c_int64), ("rows", C.c_void_p), ("n_rows", C.c_int32),
                ("row_sel", C.c_void_p), ("row_sel_cap", C.c_int64)]


class rtp_cache_view(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("idx", C.c_void_p), ("max_seq", C.c_int64),
                ("n_retrieval", C.c_int32), ("idx_bf16", C.c_void_p)]


class rtp_cluster_view(C.Structure):
    _fields_ = [("centres", C.c_void_p), ("counts", C.c_void_p), ("assign", C.c_void_p),
                ("n_clusters", C.c_int32), ("ready", C.c_int32), ("max_seq", C.c_int64),
                ("assign_stride", C.c_int64)]


class _DeviceArray:
    """A borrowed device array described by __cuda_array_interface__ (viewed by torch, no copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(int(d) for d in shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 2, "strides": None}


class RTPError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None


def lib() -> C.CDLL:
    """The loaded librtp.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"librtp.so is missing at {LIB_PATH}; build it with "
                              "`python -m long_context_sparse_idx16_b200.build`")
        L = C.CDLL(LIB_PATH)
        P, i32, i64, f32 = C.c_void_p, C.c_int32, C.c_int64, C.c_float
        sigs = {
            "rtp_create": ([C.POINTER(rtp_config), C.POINTER(C.c_void_p)], C.c_int),
            "rtp_destroy": ([P], C.c_int),
            "rtp_append_kv": ([P, P, P, i32, P], C.c_int),
            "rtp_append_kv_seq": ([P, i32, P, P, i32, P], C.c_int),
            "rtp_seq_len_of": ([P, i32], i64),
            "rtp_truncate_seq": ([P, i32, i64], C.c_int),
            "rtp_decode": ([P, P, P, C.POINTER(rtp_decode_stats), P], C.c_int),
            "rtp_prefill_chunk": ([P, P, i32, P, C.POINTER(rtp_prefill_stats), P], C.c_int),
            "rtp_set_top_p": ([P, f32], C.c_int),
            "rtp_set_wait_limit": ([P, i64], C.c_int),
            "rtp_seq_len": ([P], i64),
            "rtp_reset": ([P], C.c_int),
            "rtp_check": ([P, P], C.c_int),
            "rtp_get_cache": ([P, C.POINTER(rtp_cache_view)], C.c_int),
            "rtp_truncate": ([P, i64], C.c_int),
            "rtp_gather_attn_noalloc": ([P, P, P, i64, P, P, i64, P, i32, i64, f32, P, P], C.c_int),
            "rtp_profile_enable": ([P, C.c_int], C.c_int),
            "rtp_profile_read": ([P, C.c_char_p, C.POINTER(C.c_double), C.POINTER(C.c_int64)], C.c_int),
            "rtp_last_error": ([P], C.c_char_p),
            "rtp_probe_ex2": ([i32, i32, P, C.POINTER(C.c_int64), P], C.c_int),
            "rtp_cluster_build": ([P, i32, P], C.c_int),
            "rtp_cluster_drop": ([P], C.c_int),
            "rtp_cluster_len": ([P, i32], i64),
            "rtp_get_clusters": ([P, C.POINTER(rtp_cluster_view)], C.c_int),
        }
        for name, (args, res) in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def _check(st: int, layer=None) -> None:
    if st != RTP_OK:
        msg = lib().rtp_last_error(layer)
        raise RTPError(st, msg.decode() if msg else "")


# ---------------------------------------------------------------- C names


def rtp_create(cfg: rtp_config) -> C.c_void_p:
    h = C.c_void_p()
    _check(lib().rtp_create(C.byref(cfg), C.byref(h)))
    return h


def rtp_destroy(layer) -> None:
    _check(lib().rtp_destroy(layer))


def rtp_append_kv(layer, k_ptr: int, v_ptr: int, T: int, stream: int) -> None:
    _check(lib().rtp_append_kv(layer, k_ptr, v_ptr, T, stream), layer)


def rtp_append_kv_seq(layer, b: int, k_ptr: int, v_ptr: int, T: int, stream: int) -> None:
    _check(lib().rtp_append_kv_seq(layer, b, k_ptr, v_ptr, T, stream), layer)


def rtp_decode(layer, q_ptr: int, out_ptr: int, stats: Optional[rtp_decode_stats], stream: int) -> None:
    _check(lib().rtp_decode(layer, q_ptr, out_ptr, C.byref(stats) if stats is not None else None, stream), layer)


def rtp_prefill_chunk(layer, q_ptr: int, C_rows: int, out_ptr: int, stats: Optional[rtp_prefill_stats],
                      stream: int) -> None:
    _check(lib().rtp_prefill_chunk(layer, q_ptr, C_rows, out_ptr,
                                   C.byref(stats) if stats is not None else None, stream), layer)


def rtp_set_top_p(layer, p: float) -> None:
    _check(lib().rtp_set_top_p(layer, p), layer)


def rtp_set_wait_limit(layer, cycles: int) -> None:
    """Test knob: clock-cycle limit of the decode selection's grid-barrier waits (0: default)."""
    _check(lib().rtp_set_wait_limit(layer, int(cycles)), layer)


def rtp_seq_len(layer) -> int:
    return int(lib().rtp_seq_len(layer))


def rtp_seq_len_of(layer, b: int) -> int:
    return int(lib().rtp_seq_len_of(layer, b))


def rtp_truncate_seq(layer, b: int, new_len: int) -> None:
    _check(lib().rtp_truncate_seq(layer, b, new_len), layer)


def rtp_reset(layer) -> None:
    _check(lib().rtp_reset(layer), layer)


def rtp_truncate(layer, new_len: int) -> None:
    _check(lib().rtp_truncate(layer, new_len), layer)


def rtp_profile_enable(layer, on: bool) -> None:
    _check(lib().rtp_profile_enable(layer, 1 if on else 0), layer)


def rtp_profile_read(layer, kernel: Optional[str]):
    """(total device ms, launches) of the named kernel since the last read (clears it)."""
    ms = C.c_double()
    n = C.c_int64()
    _check(lib().rtp_profile_read(layer, kernel.encode() if kernel else None, C.byref(ms), C.byref(n)), layer)
    return ms.value, n.value


def rtp_gather_attn_noalloc(k_ptr: int, v_ptr: int, kv_block_ptr: Optional[int], kv_stride: int, q_ptr: int,
                            idx_ptr: int, idx_stride: int, cnt_ptr: int, P: int, max_count: int,
                            sm_scale: float, out_ptr: int, stream: int) -> None:
    """Attention over caller-given key lists without any device allocation (see rtp.h)."""
    _check(lib().rtp_gather_attn_noalloc(k_ptr, v_ptr, kv_block_ptr, kv_stride, q_ptr, idx_ptr, idx_stride,
                                         cnt_ptr, P, max_count, sm_scale, out_ptr, stream))


def rtp_probe_ex2(blocks: int, iters: int, out_ptr: int, stream: int) -> int:
    """Launch the exponential-rate probe; returns the number of exponentials it evaluates."""
    n = C.c_int64()
    _check(lib().rtp_probe_ex2(blocks, iters, out_ptr, C.byref(n), stream))
    return n.value


def rtp_check(layer, stream: int) -> int:
    """Synchronise the stream; return the status of errors recorded by kernels."""
    return int(lib().rtp_check(layer, stream))


def rtp_get_cache(layer) -> rtp_cache_view:
    v = rtp_cache_view()
    _check(lib().rtp_get_cache(layer, C.byref(v)), layer)
    return v


def rtp_cluster_build(layer, iters: int, stream: int) -> None:
    _check(lib().rtp_cluster_build(layer, iters, stream), layer)


def rtp_cluster_drop(layer) -> None:
    _check(lib().rtp_cluster_drop(layer), layer)


def rtp_cluster_len(layer, b: int) -> int:
    return int(lib().rtp_cluster_len(layer, b))


def rtp_get_clusters(layer) -> rtp_cluster_view:
    v = rtp_cluster_view()
    _check(lib().rtp_get_clusters(layer, C.byref(v)), layer)
    return v


def rtp_last_error(layer=None) -> str:
    m = lib().rtp_last_error(layer)
    return m.decode() if m else ""


# ---------------------------------------------------------------- torch convenience


def _stream_handle(stream=None) -> int:
    import torch

    s = stream if stream is not None else torch.cuda.current_stream()
    return int(s.cuda_stream)


def _need(t, name: str, shape, dtype, device) -> None:
    """Raise unless t is a contiguous tensor of exactly this shape, dtype and device: the
    library reads and writes raw device pointers sized from the layer's configuration."""
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if t.device != device:
        raise ValueError(f"{name}: expected a tensor on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name}: expected dtype {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")


def _dim(t, name: str, ndim: int, axis: int) -> int:
    """Size of one axis of a tensor that must have ndim dimensions."""
    if getattr(t, "dim", None) is None or t.dim() != ndim:
        raise ValueError(f"{name}: expected a {ndim}-dimensional tensor")
    return int(t.shape[axis])


class Layer:
    """One sparse attention layer: owns a librtp layer on the current CUDA device."""

    def __init__(self, *, batch: int, n_q_heads: int, n_kv_heads: int, head_class: Sequence[int],
                 wq: Optional[np.ndarray], wk: Optional[np.ndarray], top_p: float, window: int,
                 n_sink: int, max_seq: int, rope_base: float = 1.0e6, sm_scale: float = 0.0,
                 max_select: int = 0, max_chunk: int = 0, index_bf16: bool = False,
                 prefill_dense: bool = False, top_k: int = 0, n_clusters: int = 0):
        self._hc = np.ascontiguousarray(np.asarray(head_class, dtype=np.uint8))
        self.n_retrieval = int(self._hc.sum())
        self._wq = None if wq is None else np.ascontiguousarray(wq, dtype=np.float32)
        self._wk = None if wk is None else np.ascontiguousarray(wk, dtype=np.float32)
        cfg = rtp_config(
            batch=batch, n_q_heads=n_q_heads, n_kv_heads=n_kv_heads, head_dim=128, index_dim=16,
            max_seq=max_seq, head_class=self._hc.ctypes.data, top_p=top_p, window=window,
            n_sink=n_sink, rope_base=rope_base, sm_scale=sm_scale,
            wq_index=self._wq.ctypes.data if self._wq is not None else None,
            wk_index=self._wk.ctypes.data if self._wk is not None else None,
            max_select=max_select, max_chunk=max_chunk, index_bf16=1 if index_bf16 else 0,
            prefill_dense=1 if prefill_dense else 0, top_k=int(top_k), n_clusters=int(n_clusters))
        self.batch, self.n_q_heads, self.n_kv_heads = batch, n_q_heads, n_kv_heads
        self.handle = rtp_create(cfg)
        import torch

        self.device = torch.device("cuda", torch.cuda.current_device())  # where rtp_create put it

    @classmethod
    def from_spec(cls, spec, inputs=None, *, max_seq: Optional[int] = None, **kw):
        """A layer shaped like a synthetic workload spec (weights from `inputs`)."""
        wq = inputs.wq if inputs is not None else None
        wk = inputs.wk if inputs is not None else None
        return cls(batch=spec.batch, n_q_heads=spec.n_q_heads, n_kv_heads=spec.n_kv_heads,
                   head_class=spec.head_class, wq=wq, wk=wk, top_p=spec.top_p, window=spec.window,
                   n_sink=spec.n_sink, max_seq=max_seq or spec.n_total, rope_base=spec.rope_base,
                   index_bf16=getattr(spec, "index_bf16", False),
                   prefill_dense=getattr(spec, "prefill_dense", False), top_k=getattr(spec, "top_k", 0), **kw)

    def close(self) -> None:
        if getattr(self, "handle", None):
            rtp_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def seq_len(self) -> int:
        return rtp_seq_len(self.handle)

    def set_top_p(self, p: float) -> None:
        rtp_set_top_p(self.handle, p)

    def set_wait_limit(self, cycles: int) -> None:
        rtp_set_wait_limit(self.handle, cycles)

    def reset(self) -> None:
        rtp_reset(self.handle)

    def truncate(self, new_len: int) -> None:
        rtp_truncate(self.handle, new_len)

    def seq_len_of(self, b: int) -> int:
        return rtp_seq_len_of(self.handle, b)

    def truncate_seq(self, b: int, new_len: int) -> None:
        rtp_truncate_seq(self.handle, b, new_len)

    def append_kv_seq(self, b: int, k, v, stream=None) -> None:
        """Append to sequence b alone: k, v torch bf16 CUDA tensors [T][Hkv][128] (k pre-RoPE)."""
        import torch

        T = _dim(k, "k", 3, 0)
        _need(k, "k", (T, self.n_kv_heads, 128), torch.bfloat16, self.device)
        _need(v, "v", (T, self.n_kv_heads, 128), torch.bfloat16, self.device)
        rtp_append_kv_seq(self.handle, b, k.data_ptr(), v.data_ptr(), T, _stream_handle(stream))

    def profile(self, on: bool) -> None:
        rtp_profile_enable(self.handle, on)

    def profile_read(self, kernel: Optional[str] = None):
        return rtp_profile_read(self.handle, kernel)

    def append_kv(self, k, v, stream=None) -> None:
        """k, v: torch bf16 CUDA tensors [B][T][Hkv][128] (k pre-RoPE)."""
        import torch

        T = _dim(k, "k", 4, 1)
        _need(k, "k", (self.batch, T, self.n_kv_heads, 128), torch.bfloat16, self.device)
        _need(v, "v", (self.batch, T, self.n_kv_heads, 128), torch.bfloat16, self.device)
        rtp_append_kv(self.handle, k.data_ptr(), v.data_ptr(), T, _stream_handle(stream))

    def decode(self, q, out=None, stats: bool = False, sel_cap: int = 0, stream=None):
        """q: torch bf16 CUDA tensor [B][Hq][128] at position len-1.  Returns out (fp32) and,
        with stats=True, (sel_count, sel_mass, threshold, sel_index) per (b, retrieval head);
        sel_index holds the first sel_cap selected positions (None when sel_cap == 0)."""
        import torch

        _need(q, "q", (self.batch, self.n_q_heads, 128), torch.bfloat16, self.device)
        if out is None:
            out = torch.empty((self.batch, self.n_q_heads, 128), dtype=torch.float32, device=q.device)
        _need(out, "out", (self.batch, self.n_q_heads, 128), torch.float32, self.device)
        if sel_cap < 0:
            raise ValueError("sel_cap must be >= 0")
        st = None
        tensors = None
        if stats and self.n_retrieval:
            shp = (self.batch, self.n_retrieval)
            idx = (torch.full((self.batch, self.n_retrieval, sel_cap), -1, dtype=torch.int32, device=q.device)
                   if sel_cap > 0 else None)
            tensors = (torch.empty(shp, dtype=torch.int32, device=q.device),
                       torch.empty(shp, dtype=torch.float32, device=q.device),
                       torch.empty(shp, dtype=torch.float32, device=q.device), idx)
            st = rtp_decode_stats(tensors[0].data_ptr(), tensors[1].data_ptr(), tensors[2].data_ptr(),
                                  idx.data_ptr() if idx is not None else None, sel_cap)
        rtp_decode(self.handle, q.data_ptr(), out.data_ptr(), st, _stream_handle(stream))
        return (out, tensors) if stats else out

    def prefill_chunk(self, q, out=None, stats: bool = False, bitmap_words: int = 0, rows=None,
                      row_sel_cap: int = 0, stream=None):
        """q: torch bf16 CUDA tensor [B][C][Hq][128]; row i at position len-C+i.

        With stats, also returns (sel_count [B][C][Hr] int32, sel_mass [B][C][Hr] fp32,
        sel_bitmap [B][C][Hr][bitmap_words] int32 or None, row_sel [B][len(rows)][Hr][row_sel_cap]
        int32 or None).  `rows` (distinct chunk rows) asks for those rows' selected positions,
        ascending, the first row_sel_cap of each (unused entries stay -1)."""
        import torch

        Cr = _dim(q, "q", 4, 1)
        _need(q, "q", (self.batch, Cr, self.n_q_heads, 128), torch.bfloat16, self.device)
        if out is None:
            out = torch.empty((self.batch, Cr, self.n_q_heads, 128), dtype=torch.float32, device=q.device)
        _need(out, "out", (self.batch, Cr, self.n_q_heads, 128), torch.float32, self.device)
        if bitmap_words < 0:
            raise ValueError("bitmap_words must be >= 0")
        if rows is not None and (not stats or row_sel_cap < 1):
            raise ValueError("rows needs stats=True and row_sel_cap >= 1")
        st = None
        tensors = None
        if stats and self.n_retrieval:
            shp = (self.batch, Cr, self.n_retrieval)
            bm = (torch.zeros(shp + (bitmap_words,), dtype=torch.int32, device=q.device)
                  if bitmap_words > 0 else None)
            rl = rs = None
            if rows is not None:
                rl = torch.as_tensor(list(rows), dtype=torch.int32).to(q.device)
                if rl.numel() < 1 or int(rl.min()) < 0 or int(rl.max()) >= Cr:
                    raise ValueError("rows must be chunk rows in [0, C)")
                rs = torch.full((self.batch, rl.numel(), self.n_retrieval, row_sel_cap), -1, dtype=torch.int32,
                                device=q.device)
            tensors = (torch.empty(shp, dtype=torch.int32, device=q.device),
                       torch.empty(shp, dtype=torch.float32, device=q.device), bm, rs)
            st = rtp_prefill_stats(tensors[0].data_ptr(), tensors[1].data_ptr(),
                                   bm.data_ptr() if bm is not None else None, bitmap_words,
                                   rl.data_ptr() if rl is not None else None, rl.numel() if rl is not None else 0,
                                   rs.data_ptr() if rs is not None else None, row_sel_cap)
            self._keep = rl  # the row list must outlive the asynchronous call
        rtp_prefill_chunk(self.handle, q.data_ptr(), Cr, out.data_ptr(), st, _stream_handle(stream))
        return (out, tensors) if stats else out

    def check(self, stream=None) -> int:
        return rtp_check(self.handle, _stream_handle(stream))

    def cache(self) -> rtp_cache_view:
        return rtp_get_cache(self.handle)

    def cluster_build(self, iters: int, stream=None) -> None:
        """K-means of every sequence's index keys (rtp_cluster_build); decode then selects by clusters."""
        rtp_cluster_build(self.handle, iters, _stream_handle(stream))

    def cluster_drop(self) -> None:
        rtp_cluster_drop(self.handle)

    def cluster_len(self, b: int) -> int:
        return rtp_cluster_len(self.handle, b)

    def clusters(self):
        """Device views of the clustering: centres fp64 [B][Hr][K][16], counts int32 [B][Hr][K] and
        assign [B][Hr][max_seq] (uint16 cluster ids, returned widened to int32)."""
        import torch

        v = rtp_get_clusters(self.handle)
        B, Hr, K = self.batch, self.n_retrieval, v.n_clusters
        if K < 1 or Hr < 1:
            raise RTPError(RTP_EINVAL, "the layer has no clustering")
        cent = torch.as_tensor(_DeviceArray(v.centres, (B, Hr, K, 16), "<f8"), device=self.device)
        counts = torch.as_tensor(_DeviceArray(v.counts, (B, Hr, K), "<i4"), device=self.device)
        asg = torch.as_tensor(_DeviceArray(v.assign, (B, Hr, v.assign_stride), "<i2"), device=self.device)
        asg = asg[:, :, :v.max_seq].to(torch.int32) & 0xFFFF
        return {"centres": cent, "counts": counts, "assign": asg, "ready": bool(v.ready)}
