"""Seeded synthetic inputs for the head-wise sparse attention layer.

This module draws random numbers and shapes them into the workloads the RTPurbo
pages describe (Full Attention Strikes Back, arXiv:2605.16928): Gaussian or
clustered pre-RoPE keys, a diffuse topic, planted needle keys, and queries aimed
at a needle, a cluster centre, the diffuse centre or nothing at all.

It holds none of the layer's arithmetic: no RoPE, no scoring of the cache, no
softmax, no top-p selection, no attention.  The only linear algebra on the
indexer weights is what aiming a key or a query along a chosen index-space
direction needs (a least-squares solve and a projection).  Everything is
returned as bf16 bit patterns (uint16) for q/k/v and fp32 for the indexer
weights, so the GPU path and the oracle read identical values.

Needle margin: a needle key is k = beta * u + xi_perp, with u the unit key-space
direction whose index score grows fastest for the aimed query, and xi_perp a
Gaussian draw with its u-component removed.  beta is set from a Gaussian
high-probability bound on the largest u-component of the ordinary keys plus an
8-unit score margin, so needles score at least 8 above every other key without
this module ever scoring the cache (the tests check the margin with the oracle).
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import numpy as np

# --------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even from fp32)
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (RNE) and return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).copy()
    u += ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    u >>= 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# Workload specifications
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class LayerSpec:
    """One attention layer plus the synthetic workload that drives it.

    The cache holds ``prefix`` tokens before the measured call; the measured
    call appends ``chunk`` tokens and runs their queries (chunk == 1: decode,
    query at position prefix; chunk > 1: chunked prefill, query row i at
    position prefix + i).
    """

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    retrieval_heads: Tuple[int, ...]
    window: int
    n_sink: int
    top_p: float
    prefix: int
    chunk: int
    seed: int
    head_dim: int = 128
    index_dim: int = 16
    rope_base: float = 1.0e6
    # key mixture
    n_clusters: int = 0  # 0: pre-RoPE keys ~ N(0, I)
    cluster_sigma: float = 0.5
    diffuse_frac: float = 0.0
    diffuse_sigma: float = 1.0
    needles: Tuple[int, ...] = ()  # needles per sequence
    # query recipe: "gauss", "decode_mix", "self_similar", "needle_half"
    query_mode: str = "gauss"
    # retrieval-head query types cycled over heads ("needle", "cluster", "diffuse", "gauss")
    query_cycle: Tuple[str, ...] = ("needle",)
    # degenerate variants used by edge-case tests
    zero_index_weights: bool = False  # every index score is exactly 0 (all ties)
    p_sweep: Tuple[float, ...] = ()
    # layer options the workload runs with (no effect on the generated numbers)
    index_bf16: bool = False  # index keys stored in bf16 instead of fp32
    top_k: int = 0  # > 0: retrieval heads keep a fixed budget of k keys instead of top-p
    prefill_dense: bool = False  # retrieval heads attend to every causal key in prefill

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_total(self) -> int:
        return self.prefix + self.chunk

    @property
    def head_class(self) -> np.ndarray:
        hc = np.zeros(self.n_q_heads, dtype=np.uint8)
        hc[list(self.retrieval_heads)] = 1
        return hc

    def kv_head(self, h: int) -> int:
        return h // self.group


_LAYER_32_4 = dict(n_q_heads=32, n_kv_heads=4, retrieval_heads=(0, 7, 13, 19, 26), window=8192, n_sink=4)

SPECS: Dict[str, LayerSpec] = {
    # Decode correctness toy: B=1, N=4096, 8/2 heads, heads {0,5} retrieval, W=512, S=4, p=0.9,
    # q/k ~ N(0,1), 3 needles aimed at the decode query, seed 0.
    "toy_decode_4k": LayerSpec(
        name="toy_decode_4k", batch=1, n_q_heads=8, n_kv_heads=2, retrieval_heads=(0, 5),
        window=512, n_sink=4, top_p=0.9, prefix=4095, chunk=1, seed=0,
        needles=(3,), query_mode="gauss"),
    # Decode at 128K: B=8, 32/4 heads, 5 retrieval heads, 64 clusters, needles {1,16,4096} per sequence.
    "decode_128k": LayerSpec(
        name="decode_128k", batch=8, prefix=131071, chunk=1, top_p=0.9, seed=1,
        n_clusters=64, needles=(1, 16, 4096, 1, 16, 4096, 1, 16), query_mode="decode_mix",
        **_LAYER_32_4),
    # Chunked prefill at 32K: B=1, P=0, C=32768, same mixture as the 128K decode workload.
    "prefill_32k": LayerSpec(
        name="prefill_32k", batch=1, prefix=0, chunk=32768, top_p=0.9, seed=2,
        n_clusters=64, needles=(4096,), query_mode="self_similar", **_LAYER_32_4),
    # Decode at 1M: B=1, N=2^20, 256 clusters + 10% diffuse topic + 32 needles; p swept.
    "decode_1m": LayerSpec(
        name="decode_1m", batch=1, prefix=1048575, chunk=1, top_p=0.9, seed=3,
        n_clusters=256, diffuse_frac=0.1, needles=(32,), query_mode="decode_mix",
        query_cycle=("needle", "cluster", "diffuse", "gauss"), p_sweep=(0.8, 0.9, 0.95),
        **_LAYER_32_4),
    # Chunked prefill near 1M: 16384-token chunk on a 1032192-token cache; half the chunk's
    # retrieval-head queries aimed at the needles, half N(0,1).
    "prefill_1m": LayerSpec(
        name="prefill_1m", batch=1, prefix=1032192, chunk=16384, top_p=0.9, seed=4,
        n_clusters=256, diffuse_frac=0.1, needles=(32,), query_mode="needle_half",
        **_LAYER_32_4),
}


def spec(name: str, **overrides) -> LayerSpec:
    """A named workload, optionally with fields overridden (smaller sizes for tests)."""
    s = SPECS[name]
    return replace(s, **overrides) if overrides else s


# --------------------------------------------------------------------------
# Generated inputs
# --------------------------------------------------------------------------


@dataclass
class LayerInputs:
    spec: LayerSpec
    wq: np.ndarray  # fp32 [Hr][D][r]
    wk: np.ndarray  # fp32 [Hr][D][r]
    k: np.ndarray  # bf16 bits [B][N][Hkv][D], pre-RoPE, positions 0..N-1
    v: np.ndarray  # bf16 bits [B][N][Hkv][D]
    q: np.ndarray  # bf16 bits [B][C][Hq][D], pre-RoPE, row i at position prefix + i
    needle_pos: Dict[Tuple[int, int], np.ndarray] = field(default_factory=dict)  # (b, h) -> positions
    query_type: Dict[Tuple[int, int], str] = field(default_factory=dict)  # (b, h) -> decode query type

    @property
    def n_total(self) -> int:
        return self.k.shape[1]


_CHUNK = 1 << 16  # positions per independently seeded key/value block


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _block_rng(seed: int, tag: int, b: int, blk: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, tag, b, blk]))


def _unit(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x)


def _aim_query(wq: np.ndarray, z: np.ndarray, xi: np.ndarray) -> np.ndarray:
    """A pre-RoPE query whose index-space image is z: least-squares part along the
    columns of wq (D x r) plus xi with its component in that column space removed."""
    wq64 = wq.astype(np.float64)
    g = wq64.T @ wq64
    along = wq64 @ np.linalg.solve(g, z)
    xi2 = np.atleast_2d(xi)
    perp = xi2 - (wq64 @ np.linalg.solve(g, wq64.T @ xi2.T)).T
    out = along[None, :] + perp
    return out if xi.ndim == 2 else out[0]


def _needle_key(u: np.ndarray, beta: float, xi: np.ndarray) -> np.ndarray:
    return beta * u + (xi - (u @ xi) * u)


def generate(s: LayerSpec, *, with_values: bool = True) -> LayerInputs:
    """Draw all inputs of workload ``s`` from its seed (deterministic)."""
    B, Hq, Hkv, D, r = s.batch, s.n_q_heads, s.n_kv_heads, s.head_dim, s.index_dim
    N, C, P = s.n_total, s.chunk, s.prefix
    R = list(s.retrieval_heads)
    Hr = len(R)
    ss = s.seed

    # Indexer weights Wq_h, Wk_h ~ N(0, 1/D), fp32, one pair per retrieval head.
    rw = np.random.default_rng(np.random.SeedSequence([ss, 1]))
    wq = (rw.standard_normal((Hr, D, r)) / math.sqrt(D)).astype(np.float32)
    wk = (rw.standard_normal((Hr, D, r)) / math.sqrt(D)).astype(np.float32)
    if s.zero_index_weights:
        wk[:] = 0.0

    # Cluster centres (per KV head), diffuse centre, per-position assignments.
    rc = np.random.default_rng(np.random.SeedSequence([ss, 2]))
    centres = rc.standard_normal((max(s.n_clusters, 1), Hkv, D)) if s.n_clusters else None
    diffuse_c = rc.standard_normal((Hkv, D))
    # assignment per (b, position): -1 diffuse, else cluster id
    assign = None
    if s.n_clusters:
        assign = rc.integers(0, s.n_clusters, size=(B, N), dtype=np.int32)
        if s.diffuse_frac > 0:
            for b in range(B):
                nd = int(round(s.diffuse_frac * N))
                idx = rc.choice(N, size=nd, replace=False)
                assign[b, idx] = -1

    # ------------------------------------------------------------------ keys / values
    k = np.empty((B, N, Hkv, D), dtype=np.uint16)
    v = np.empty((B, N, Hkv, D), dtype=np.uint16) if with_values else np.zeros((B, 0, Hkv, D), np.uint16)

    def fill_block(args):
        b, blk = args
        lo, hi = blk * _CHUNK, min(N, (blk + 1) * _CHUNK)
        g = _block_rng(ss, 10, b, blk)
        n = hi - lo
        x = g.standard_normal((n, Hkv, D), dtype=np.float32)
        if s.n_clusters:
            a = assign[b, lo:hi]
            cl = a >= 0
            x[cl] *= np.float32(s.cluster_sigma)
            x[cl] += centres[a[cl]].astype(np.float32)
            if s.diffuse_frac > 0:
                df = ~cl
                x[df] *= np.float32(s.diffuse_sigma)
                x[df] += diffuse_c.astype(np.float32)
        k[b, lo:hi] = f32_to_bf16_bits(x)
        if with_values:
            gv = _block_rng(ss, 11, b, blk)
            v[b, lo:hi] = f32_to_bf16_bits(gv.standard_normal((n, Hkv, D), dtype=np.float32))

    jobs = [(b, blk) for b in range(B) for blk in range((N + _CHUNK - 1) // _CHUNK)]
    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(fill_block, jobs))

    # Per-component standard deviation of ordinary keys (for the needle margin bound).
    key_sd = 1.0
    if s.n_clusters:
        key_sd = math.sqrt(1.0 + s.cluster_sigma ** 2)
        if s.diffuse_frac > 0:
            key_sd = max(key_sd, math.sqrt(1.0 + s.diffuse_sigma ** 2))
    tail = math.sqrt(2.0 * math.log(max(N, 2))) + 3.0

    # ------------------------------------------------------------------ queries
    rq = np.random.default_rng(np.random.SeedSequence([ss, 3]))
    q64 = rq.standard_normal((B, C, Hq, D))  # N(0, I) base draw for every head and row
    query_type: Dict[Tuple[int, int], str] = {}
    # index-space aim per (b, retrieval slot): unit direction and score scale lam
    aim_dir: Dict[Tuple[int, int], np.ndarray] = {}
    aim_lam: Dict[Tuple[int, int], float] = {}
    lam_default = math.sqrt(r)  # |Wq^T q| of a N(0, I) query is about sqrt(r)

    needles_per_b = list(s.needles) + [0] * max(0, B - len(s.needles)) if s.needles else [0] * B
    needles_per_b = needles_per_b[:B]

    if s.query_mode == "self_similar":
        # Queries drawn like the keys of their KV head (cluster mixture) plus N(0, 1) noise.
        for b in range(B):
            qa = rq.integers(0, max(s.n_clusters, 1), size=(C,))
            for h in range(Hq):
                g = s.kv_head(h)
                base = np.zeros((C, D)) if centres is None else centres[qa, g]
                q64[b, :, h] = base + s.cluster_sigma * rq.standard_normal((C, D)) + q64[b, :, h]
        for b in range(B):
            for i, h in enumerate(R):
                aim_dir[(b, i)] = _unit(rq.standard_normal(r))
                aim_lam[(b, i)] = lam_default
    elif s.query_mode == "needle_half":
        for b in range(B):
            for i, h in enumerate(R):
                z = _unit(rq.standard_normal(r))
                aim_dir[(b, i)] = z
                aim_lam[(b, i)] = lam_default
                # even rows aimed at the needles, odd rows N(0, I)
                q64[b, 0::2, h] = _aim_query(wq[i], lam_default * z, q64[b, 0::2, h])
    elif s.query_mode in ("gauss", "decode_mix"):
        for b in range(B):
            # which retrieval slots own needles in this sequence (round robin)
            nn = needles_per_b[b]
            owners = {i % Hr for i in range(nn)} if Hr else set()
            for i, h in enumerate(R):
                if s.query_mode == "gauss":
                    qz = wq[i].astype(np.float64).T @ q64[b, C - 1, h]
                    aim_dir[(b, i)] = _unit(qz)
                    aim_lam[(b, i)] = float(np.linalg.norm(qz))
                    query_type[(b, h)] = "gauss"
                    continue
                if len(s.query_cycle) > 1:
                    kind = s.query_cycle[i % len(s.query_cycle)]
                else:
                    kind = "needle" if i in owners else "cluster"
                query_type[(b, h)] = kind
                g = s.kv_head(h)
                if kind == "needle":
                    z = _unit(rq.standard_normal(r))
                elif kind == "cluster":
                    m = int(rq.integers(0, s.n_clusters))
                    z = _unit(wk[i].astype(np.float64).T @ centres[m, g])
                elif kind == "diffuse":
                    z = _unit(wk[i].astype(np.float64).T @ diffuse_c[g])
                else:
                    z = None
                if z is None:
                    qz = wq[i].astype(np.float64).T @ q64[b, C - 1, h]
                    aim_dir[(b, i)] = _unit(qz)
                    aim_lam[(b, i)] = float(np.linalg.norm(qz))
                else:
                    aim_dir[(b, i)] = z
                    aim_lam[(b, i)] = lam_default
                    q64[b, :, h] = _aim_query(wq[i], lam_default * z, q64[b, C - 1, h])[None, :]
    else:
        raise ValueError(f"unknown query_mode {s.query_mode}")

    q = f32_to_bf16_bits(q64.astype(np.float32))

    # ------------------------------------------------------------------ needles
    rn = np.random.default_rng(np.random.SeedSequence([ss, 4]))
    needle_pos: Dict[Tuple[int, int], np.ndarray] = {}
    hi_pos = max(P + C - 1, s.n_sink + 1)  # needles sit before the last query position
    for b in range(B):
        nn = needles_per_b[b]
        if nn == 0 or Hr == 0:
            continue
        avail = hi_pos - s.n_sink
        nn = min(nn, avail)
        pos = np.sort(rn.choice(avail, size=nn, replace=False) + s.n_sink)
        for n_i, pos_n in enumerate(pos):
            i = n_i % Hr
            h = R[i]
            if s.query_mode == "decode_mix" and query_type.get((b, h)) not in (None, "needle"):
                # needles go to needle-type heads only
                owners = [j for j, hh in enumerate(R) if query_type.get((b, hh)) == "needle"]
                if not owners:
                    continue
                i = owners[n_i % len(owners)]
                h = R[i]
            g = s.kv_head(h)
            z = aim_dir[(b, i)]
            wz = wk[i].astype(np.float64) @ z  # key-space direction raising this head's index score
            sig = float(np.linalg.norm(wz))
            if sig == 0.0:
                continue
            u = wz / sig
            beta = key_sd * tail + 8.0 / (aim_lam[(b, i)] * sig)
            xi = rn.standard_normal(D)
            k[b, pos_n, g] = f32_to_bf16_bits(_needle_key(u, beta, xi).astype(np.float32))
            needle_pos.setdefault((b, h), []).append(int(pos_n))
    needle_pos = {key: np.asarray(val, dtype=np.int64) for key, val in needle_pos.items()}

    return LayerInputs(spec=s, wq=wq, wk=wk, k=k, v=v, q=q, needle_pos=needle_pos, query_type=query_type)
