"""fp64 CPU oracle of the head-wise sparse attention layer (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import this
package.  It wraps oracle/rtp_oracle.c (plain C, fp64) through ctypes and shares no code
with the CUDA library.  What each function computes, and which passage of the pages it
follows, is written in rtp_oracle.c.

Parity pins: every function here is pinned by tests/test_oracle_pins.py (closed forms,
brute force on tiny inputs, library routines, invariants); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i64, i32, f64 = C.c_int64, C.c_int, C.c_double
        L.orc_head_rows.restype = C.c_int
        L.orc_head_rows.argtypes = [P, P, i64, i64, i32, i32, i32, P, i64, P, i64, i32, P, P, f64,
                                    i64, i64, f64, f64, i64, P, P, P, P, P, P, i64, P, i64, i32, i32, i64]
        L.orc_topk.restype = i64
        L.orc_topk.argtypes = [P, i64, i64, P, P, P, P, P]
        L.orc_topp.restype = i64
        L.orc_topp.argtypes = [P, i64, f64, P, P, P, P, P]
        L.orc_rope.restype = None
        L.orc_rope.argtypes = [P, f64, i32, f64, P]
        L.orc_index_scores.restype = None
        L.orc_index_scores.argtypes = [P, i64, i64, i32, i32, i32, P, P, P, P, i32]
        L.orc_round_bf16.restype = f64
        L.orc_round_bf16.argtypes = [f64]
        L.orc_attend_set.restype = None
        L.orc_attend_set.argtypes = [P, P, i64, i32, i32, P, i64, f64, f64, i64, P, i64, P]
        L.orc_max_threads.restype = C.c_int
        L.orc_max_threads.argtypes = []
        L.orc_index_keys_bf16.restype = None
        L.orc_index_keys_bf16.argtypes = [P, i64, i64, i32, i32, i32, P, P]
        L.orc_index_query.restype = None
        L.orc_index_query.argtypes = [P, i32, i32, P, P]
        L.orc_kmeans.restype = None
        L.orc_kmeans.argtypes = [P, i64, i32, i32, i32, P, P, P]
        L.orc_cluster_select.restype = C.c_int
        L.orc_cluster_select.argtypes = [P, P, P, i32, i32, f64, P, P, P]
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def max_threads() -> int:
    return int(lib().orc_max_threads())


def rope(x: np.ndarray, pos: float, base: float = 1.0e6) -> np.ndarray:
    """Rotate-half RoPE of one fp64 vector at position ``pos``."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    y = np.empty_like(x)
    lib().orc_rope(_p(x), float(pos), int(x.shape[0]), float(base), _p(y))
    return y


@dataclass
class TopP:
    count: int
    order: np.ndarray  # key order (s desc, j asc); order[:count] is the selected set
    pi: np.ndarray  # softmax mass per key
    mass: float  # cumulative mass of the selected set
    pi_t: float  # mass of the last member
    cum_prev: float  # cumulative mass of the first count-1 members

    @property
    def selected(self) -> np.ndarray:
        return np.sort(self.order[: self.count])


def topp(scores: np.ndarray, p: float) -> TopP:
    """Top-p selection over a score vector (the retrieval-head selection rule)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.empty(max(n, 1), dtype=np.int64)
    pi = np.empty(max(n, 1), dtype=np.float64)
    mass = C.c_double()
    pt = C.c_double()
    cp = C.c_double()
    K = lib().orc_topp(_p(s), n, float(p), _p(order), _p(pi), C.byref(mass), C.byref(pt), C.byref(cp))
    return TopP(int(K), order[:n], pi[:n], mass.value, pt.value, cp.value)


def round_bf16(x: float) -> float:
    """x rounded to the nearest bf16 value, ties to even (the bf16 index-key storage)."""
    return float(lib().orc_round_bf16(float(x)))


def topk(scores: np.ndarray, k: int) -> TopP:
    """Fixed top-k selection over a score vector (the pages' fixed-budget ablation)."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.empty(max(n, 1), dtype=np.int64)
    pi = np.empty(max(n, 1), dtype=np.float64)
    mass = C.c_double()
    pt = C.c_double()
    cp = C.c_double()
    K = lib().orc_topk(_p(s), n, int(k), _p(order), _p(pi), C.byref(mass), C.byref(pt), C.byref(cp))
    return TopP(int(K), order[:n], pi[:n], mass.value, pt.value, cp.value)


def index_scores(k_seq: np.ndarray, g: int, q_vec: np.ndarray, wq: np.ndarray, wk: np.ndarray,
                 n: Optional[int] = None, index_bf16: bool = False) -> np.ndarray:
    """Pre-RoPE index scores of one query against keys 0..n-1 of KV head g.

    k_seq: bf16 bits [N][Hkv][D] of one sequence; q_vec: bf16 bits [D]; wq/wk: fp32 [D][r].
    index_bf16: the index keys are stored in bf16 (each component rounded, ties to even).
    """
    k_seq = np.ascontiguousarray(k_seq, dtype=np.uint16)
    N, Hkv, D = k_seq.shape
    n = N if n is None else n
    r = wq.shape[1]
    q_vec = np.ascontiguousarray(q_vec, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.float32)
    wk = np.ascontiguousarray(wk, dtype=np.float32)
    s = np.empty(n, dtype=np.float64)
    lib().orc_index_scores(_p(k_seq), n, Hkv * D, g, D, r, _p(q_vec), _p(wq), _p(wk), _p(s), 1 if index_bf16 else 0)
    return s


@dataclass
class Rows:
    out: np.ndarray  # [nrows][D]
    count: np.ndarray  # [nrows]
    mass: np.ndarray
    pi_t: np.ndarray
    cum_prev: np.ndarray
    sel: Optional[list]  # per row: ascending selected positions (None if not requested)
    pi: Optional[np.ndarray]  # [nrows][max_pos+1] index-softmax masses (retrieval, optional)


def head_rows(k_seq: np.ndarray, v_seq: np.ndarray, q_rows: np.ndarray, positions: Sequence[int], *,
              g: int, retrieval: bool, wq: Optional[np.ndarray] = None, wk: Optional[np.ndarray] = None,
              top_p: float = 0.9, window: int = 8192, n_sink: int = 4, rope_base: float = 1.0e6,
              sm_scale: Optional[float] = None, pos_offset: int = 0, want_sel: bool = True,
              want_pi: bool = False, threads: Optional[int] = None, index_bf16: bool = False,
              top_k: int = 0) -> Rows:
    """Oracle output of one query head for several query rows of one sequence.

    k_seq, v_seq: bf16 bits [N][Hkv][D] (pre-RoPE keys); q_rows: bf16 bits [nrows][D];
    positions: absolute position of each row (its own key is at that position).
    """
    k_seq = np.ascontiguousarray(k_seq, dtype=np.uint16)
    v_seq = np.ascontiguousarray(v_seq, dtype=np.uint16)
    N, Hkv, D = k_seq.shape
    q_rows = np.ascontiguousarray(np.atleast_2d(q_rows), dtype=np.uint16)
    pos = np.ascontiguousarray(np.asarray(positions, dtype=np.int64))
    nrows = pos.shape[0]
    r = 16 if wq is None else wq.shape[1]
    if retrieval:
        wq = np.ascontiguousarray(wq, dtype=np.float32)
        wk = np.ascontiguousarray(wk, dtype=np.float32)
    scale = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    out = np.zeros((nrows, D), dtype=np.float64)
    cnt = np.zeros(nrows, dtype=np.int64)
    mass = np.zeros(nrows)
    pit = np.zeros(nrows)
    cpv = np.zeros(nrows)
    maxpos = int(pos.max()) if nrows else 0
    cap = (maxpos + 1) if retrieval else (window + n_sink + 1)
    sel = np.zeros((nrows, cap), dtype=np.int64) if want_sel else None
    pi = np.zeros((nrows, maxpos + 1), dtype=np.float64) if (want_pi and retrieval) else None
    th = max_threads() if threads is None else threads
    rc = lib().orc_head_rows(
        _p(k_seq), _p(v_seq), N, Hkv * D, g, D, r, _p(q_rows), q_rows.shape[1], _p(pos), nrows,
        1 if retrieval else 0, _p(wq) if retrieval else None, _p(wk) if retrieval else None,
        float(top_p), int(window), int(n_sink), float(rope_base), float(scale), int(pos_offset),
        _p(out), _p(cnt), _p(mass), _p(pit), _p(cpv), _p(sel), cap if want_sel else 0,
        _p(pi), (maxpos + 1) if pi is not None else 0, int(th), 1 if index_bf16 else 0, int(top_k))
    if rc != 0:
        raise ValueError("oracle: a row position lies outside the key range")
    sels = [sel[t, : min(int(cnt[t]), cap)].copy() for t in range(nrows)] if want_sel else None
    return Rows(out, cnt, mass, pit, cpv, sels, pi)


def layer_rows(inputs, b: int, h: int, rows: Sequence[int], *, top_p: Optional[float] = None,
               want_sel: bool = True, want_pi: bool = False, threads: Optional[int] = None,
               pos_offset: int = 0) -> Rows:
    """Oracle output of query head h of sequence b for chunk rows ``rows`` of a generated workload
    (synth.LayerInputs): row i sits at position prefix + i."""
    s = inputs.spec
    rows = np.asarray(rows, dtype=np.int64)
    retrieval = h in s.retrieval_heads
    slot = s.retrieval_heads.index(h) if retrieval else 0
    p = s.top_p if top_p is None else top_p
    top_k = s.top_k
    if s.prefill_dense and s.chunk > 1:  # the pages' own prefill: retrieval heads see every causal key
        p, top_k = 1.0, 0
    return head_rows(
        inputs.k[b], inputs.v[b], inputs.q[b, rows, h], s.prefix + rows, g=s.kv_head(h),
        retrieval=retrieval, wq=inputs.wq[slot] if retrieval else None,
        wk=inputs.wk[slot] if retrieval else None, top_p=p, top_k=top_k,
        window=s.window, n_sink=s.n_sink, rope_base=s.rope_base, want_sel=want_sel,
        want_pi=want_pi, threads=threads, pos_offset=pos_offset, index_bf16=s.index_bf16)


def attend_set(inputs, b: int, h: int, row: int, sel: Sequence[int], *, pos_offset: int = 0,
               pos: Optional[int] = None) -> np.ndarray:
    """Exact attention of chunk row ``row`` of query head h (sequence b) over the key set ``sel``
    (no selection step): for checking an output whose set legitimately differs from the
    oracle's own.  pos: the row's position when it is not prefix + row (a sequence of a ragged
    batch)."""
    s = inputs.spec
    k_seq = np.ascontiguousarray(inputs.k[b], dtype=np.uint16)
    v_seq = np.ascontiguousarray(inputs.v[b], dtype=np.uint16)
    N, Hkv, D = k_seq.shape
    q = np.ascontiguousarray(inputs.q[b, row, h], dtype=np.uint16)
    J = np.ascontiguousarray(np.asarray(sel, dtype=np.int64))
    pos = s.prefix + int(row) if pos is None else int(pos)
    if J.size and (J.min() < 0 or J.max() > pos):
        raise ValueError("attend_set: a key lies outside the row's causal range")
    out = np.zeros(D, dtype=np.float64)
    lib().orc_attend_set(_p(k_seq), _p(v_seq), Hkv * D, s.kv_head(h), D, _p(q), pos, float(s.rope_base),
                         1.0 / np.sqrt(D), int(pos_offset), _p(J), int(J.size), _p(out))
    return out


# ------------------------------------------------------------------ K-cache clustering


def index_keys_bf16(k_seq: np.ndarray, g: int, wk: np.ndarray, n: Optional[int] = None) -> np.ndarray:
    """Stored bf16 index keys kt_j = bf16(Wk^T k_j) of KV head g for j < n, fp64 [n][r]."""
    k_seq = np.ascontiguousarray(k_seq, dtype=np.uint16)
    N, Hkv, D = k_seq.shape
    n = N if n is None else n
    wk = np.ascontiguousarray(wk, dtype=np.float32)
    r = wk.shape[1]
    kt = np.empty((n, r), dtype=np.float64)
    lib().orc_index_keys_bf16(_p(k_seq), n, Hkv * D, g, D, r, _p(wk), _p(kt))
    return kt


def index_query(q_vec: np.ndarray, wq: np.ndarray) -> np.ndarray:
    """Index query Wq^T q of one bf16 query vector, fp64 [r]."""
    q_vec = np.ascontiguousarray(q_vec, dtype=np.uint16)
    wq = np.ascontiguousarray(wq, dtype=np.float32)
    qt = np.empty(wq.shape[1], dtype=np.float64)
    lib().orc_index_query(_p(q_vec), q_vec.shape[0], wq.shape[1], _p(wq), _p(qt))
    return qt


def kmeans(kt: np.ndarray, K: int, iters: int):
    """Lloyd's k-means of the index keys kt [n][r] (readings in rtp_oracle.c): (centres [K][r],
    cluster sizes [K], assignment [n])."""
    kt = np.ascontiguousarray(kt, dtype=np.float64)
    n, r = kt.shape
    cent = np.empty((K, r), dtype=np.float64)
    counts = np.empty(K, dtype=np.int64)
    assign = np.empty(n, dtype=np.int32)
    lib().orc_kmeans(_p(kt), n, r, K, iters, _p(cent), _p(counts), _p(assign))
    return cent, counts, assign


def cluster_select(qt: np.ndarray, cent: np.ndarray, counts: np.ndarray, p: float):
    """Coarse match of an index query against the centres: (hit [K] bool, weight fractions [K],
    weight fraction of the last cluster taken)."""
    qt = np.ascontiguousarray(qt, dtype=np.float64)
    cent = np.ascontiguousarray(cent, dtype=np.float64)
    counts = np.ascontiguousarray(counts, dtype=np.int64)
    K, r = cent.shape
    hit = np.empty(K, dtype=np.int32)
    w = np.empty(K, dtype=np.float64)
    wt = np.zeros(1, dtype=np.float64)
    lib().orc_cluster_select(_p(qt), _p(cent), _p(counts), K, r, float(p), _p(hit), _p(w), _p(wt))
    return hit.astype(bool), w, float(wt[0])


@dataclass
class ClusterRow:
    out: np.ndarray      # [D]
    sel: np.ndarray      # ascending selected positions
    hit: np.ndarray      # [K] clusters hit
    w: np.ndarray        # [K] cluster weight fractions
    w_t: float           # weight fraction of the last cluster taken
    cent: np.ndarray
    counts: np.ndarray
    assign: np.ndarray


def cluster_row(inputs, b: int, h: int, n: int, K: int, iters: int, p: float,
                n_clustered: Optional[int] = None, row: int = 0) -> ClusterRow:
    """The clustered selection and attention of query row ``row`` of retrieval head h, sequence
    b, at position n - 1: keys 0 .. n_clustered - 1 clustered, the later ones always kept."""
    s = inputs.spec
    slot = s.retrieval_heads.index(h)
    g = s.kv_head(h)
    nc = n if n_clustered is None else n_clustered
    kt = index_keys_bf16(inputs.k[b], g, inputs.wk[slot], nc)
    cent, counts, assign = kmeans(kt, K, iters)
    qt = index_query(inputs.q[b, row, h], inputs.wq[slot])
    hit, w, wt = cluster_select(qt, cent, counts, p)
    sel = np.concatenate([np.flatnonzero(hit[assign]), np.arange(nc, n)]).astype(np.int64)
    out = attend_set(inputs, b, h, row, sel, pos=n - 1)
    return ClusterRow(out, sel, hit, w, wt, cent, counts, assign)
