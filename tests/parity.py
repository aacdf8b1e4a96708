"""Helpers shared by the GPU parity tests: drive the CUDA layer through the C ABI on a
seeded workload and compare with the fp64 oracle under the stated tolerances.

Tolerances (from the method statement):
  * selected index sets identical except for keys whose oracle probability lies within
    1e-6 of the threshold probability (the mass of the last member);  keys at the mass
    boundary may also move when the oracle's cumulative mass before or after the last
    member lies within 1e-6 of p (fp summation may legitimately move the cut there);
  * selected mass (oracle probabilities over the GPU's set) >= p - 1e-5;
  * attention outputs within 1e-2 max-abs and 1e-3 relative L2 -- against the oracle's output,
    or, for a row whose set legitimately differs from the oracle's, against the oracle's exact
    attention over the GPU's set.

p crosses the C ABI as fp32, so the oracle is given the same fp32 value.
"""
from __future__ import annotations

import numpy as np

import oracle

SET_TOL = 1e-6
MASS_TOL = 1e-5
ABS_TOL = 1e-2
REL_L2_TOL = 1e-3


def p32(p: float) -> float:
    """The value p takes after crossing the ABI as a C float."""
    return float(np.float32(p))


def torch_bf16(bits: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def build_cache(layer, x, upto: int, chunk: int = 1 << 16):
    """Append positions [layer.seq_len, upto) of workload x to the layer."""
    start = layer.seq_len
    for t0 in range(start, upto, chunk):
        t1 = min(upto, t0 + chunk)
        layer.append_kv(torch_bf16(x.k[:, t0:t1]), torch_bf16(x.v[:, t0:t1]))


def check_selection(gpu_sel: np.ndarray, ref: "oracle.Rows", t: int, p: float, what: str, top_k: int = 0):
    """Compare a GPU selected set (ascending positions) with oracle row t (needs ref.pi).

    Returns the number of differing keys.  Besides the per-key rule, the count of differing keys
    may not exceed the number of oracle keys within 1e-6 of the threshold probability plus one
    (a cut moved at a mass boundary), so a gross cut error cannot hide in a wide band."""
    o_sel = ref.sel[t]
    pi = ref.pi[t]
    diff = np.setxor1d(gpu_sel, o_sel)
    pt = ref.pi_t[t]
    boundary = abs(ref.cum_prev[t] - p) <= SET_TOL or abs(ref.mass[t] - p) <= SET_TOL
    bad = [j for j in diff if abs(pi[j] - pt) > SET_TOL]
    if bad and boundary:
        # at a mass boundary the cut may move by one key: the first key outside the oracle set
        rest = np.ones(pi.shape[0], dtype=bool)
        rest[o_sel] = False
        p_next = float(pi[rest].max()) if rest.any() else pt
        bad = [j for j in bad if abs(pi[j] - p_next) > SET_TOL]
    assert not bad, (f"{what}: {len(bad)} selected keys differ beyond tolerance, e.g. {bad[:5]} "
                     f"pi={[float(pi[j]) for j in bad[:5]]} pi_t={pt} |gpu|={len(gpu_sel)} |ref|={len(o_sel)}")
    if len(diff):
        n_band = int(np.count_nonzero(np.abs(pi - pt) <= SET_TOL))
        assert len(diff) <= n_band + 1, (f"{what}: {len(diff)} keys differ, more than the {n_band} keys "
                                         f"within 1e-6 of the threshold probability plus one")
    if top_k > 0:  # a fixed budget: exactly min(k, n) keys, no mass target
        assert len(gpu_sel) == len(o_sel), f"{what}: {len(gpu_sel)} keys selected, the budget gives {len(o_sel)}"
        return len(diff)
    mass = float(pi[gpu_sel].sum()) if len(gpu_sel) else 0.0
    assert mass >= p - MASS_TOL, f"{what}: selected mass {mass} < p - 1e-5 (p={p})"
    return len(diff)


def check_outputs(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite outputs"
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err.max() <= ABS_TOL, f"{what}: max-abs error {err.max():.3e} > {ABS_TOL}"
    assert rel <= REL_L2_TOL, f"{what}: relative L2 error {rel:.3e} > {REL_L2_TOL}"
    return float(err.max()), float(rel)


def run_decode(x, *, top_p=None, heads=None, batches=None, max_select=0, sel_cap=None, layer=None):
    """Decode the workload's query row on the GPU and check it against the oracle.

    Returns a dict of GPU outputs and the per-(b, h) comparison summaries.
    """
    import torch

    from long_context_sparse_idx16_b200 import Layer

    s = x.spec
    N = s.n_total
    p = s.top_p if top_p is None else top_p
    own = layer is None
    if own:
        layer = Layer.from_spec(s, x, max_seq=N, max_chunk=1, max_select=max_select)
        build_cache(layer, x, N)
    else:
        layer.set_top_p(p)
    layer.set_top_p(p)
    q = torch_bf16(x.q[:, 0])
    cap = N if sel_cap is None else sel_cap
    out, st = layer.decode(q, stats=True, sel_cap=cap)
    assert layer.check() == 0, "kernel error word set"
    out = out.cpu().numpy()
    cnt = st[0].cpu().numpy() if st else None
    mass = st[1].cpu().numpy() if st else None
    idx = st[3].cpu().numpy() if st else None
    heads = range(s.n_q_heads) if heads is None else heads
    batches = range(s.batch) if batches is None else batches
    refs, gpus, gpus2 = [], [], []
    summary = {}
    for b in batches:
        for h in heads:
            r = oracle.layer_rows(x, b, h, [0], top_p=p32(p), want_pi=h in s.retrieval_heads)
            ref_out = r.out[0]
            gpus.append(out[b, h])
            if h in s.retrieval_heads:
                slot = s.retrieval_heads.index(h)
                k = int(cnt[b, slot])
                sel = idx[b, slot, :k].astype(np.int64)
                assert np.all(np.diff(sel) > 0), "selected positions must be strictly ascending"
                nd = check_selection(sel, r, 0, p32(p), f"b={b} h={h}", top_k=s.top_k)
                if s.top_k == 0:
                    assert abs(float(mass[b, slot]) - float(r.pi[0][sel].sum())) <= 1e-5
                if nd:
                    ref_out = oracle.attend_set(x, b, h, 0, sel)
                summary[(b, h)] = (k, int(r.count[0]), nd)
            refs.append(ref_out)
    err = check_outputs(np.stack(gpus), np.stack(refs), f"{s.name} p={p}")
    if own:
        layer.close()
    return {"out": out, "count": cnt, "summary": summary, "err": err}


def bitmap_positions(words: np.ndarray, n: int) -> np.ndarray:
    """Ascending positions j < n whose bit is set in a little-endian 32-bit word bitmap."""
    bits = np.unpackbits(np.ascontiguousarray(words).view(np.uint8), bitorder="little")[:n]
    return np.flatnonzero(bits).astype(np.int64)


def run_prefill(x, *, top_p=None, rows=None, heads=None, batches=None, sets="bitmap", layer=None,
                exact_sets=False, row_block=2048, local_rows=None):
    """Prefill the workload's chunk on the GPU (one call, C = chunk) and check the given rows
    (default: all) of the given heads against the oracle.

    sets: "bitmap" compares each checked row's selected set through the full selection bitmap;
    "rows" through the row-subset position lists (a second, identical call that must reproduce
    the first call's outputs bit for bit), which stays cheap at 1M keys; None checks counts,
    masses and outputs only.  exact_sets: the GPU's sets must equal the oracle's (for exact
    ties, where the order rule alone decides).  local_rows: the rows checked for local heads
    (default: the same rows).  The oracle runs row_block rows at a time."""
    import torch

    from long_context_sparse_idx16_b200 import Layer

    s = x.spec
    N, C = s.n_total, s.chunk
    p = s.top_p if top_p is None else top_p
    own = layer is None
    if own:
        layer = Layer.from_spec(s, x, max_seq=N, max_chunk=C)
        build_cache(layer, x, N)
    layer.set_top_p(p)
    words = (N + 31) // 32 if sets == "bitmap" else 0
    q = torch_bf16(x.q)
    out, st = layer.prefill_chunk(q, stats=True, bitmap_words=words)
    assert layer.check() == 0, "kernel error word set"
    rows = np.arange(C) if rows is None else np.asarray(rows, dtype=np.int64)
    local_rows = rows if local_rows is None else np.asarray(local_rows, dtype=np.int64)
    row_lists = None
    if sets == "rows" and st is not None:
        cap = int(st[0][:, torch.as_tensor(rows, device=out.device)].max()) + 1
        out2, st2 = layer.prefill_chunk(q, stats=True, rows=rows.tolist(), row_sel_cap=cap)
        assert layer.check() == 0, "kernel error word set"
        # the same selection; a chunk whose long rows split their keys over several attention
        # CTAs (not done when rows are listed) differs from the listed call only in rounding, so
        # both calls' outputs are compared with the oracle below
        assert torch.equal(st[0], st2[0]), "a repeated prefill call selects differently"
        row_lists = st2[3].cpu().numpy()  # [B][len(rows)][Hr][cap]
    heads = range(s.n_q_heads) if heads is None else heads
    batches = range(s.batch) if batches is None else batches
    summary = {}
    refs, gpus, gpus2 = [], [], []
    for b in batches:
        for h in heads:
            ret = h in s.retrieval_heads
            hrows = rows if ret else local_rows
            rows_t = torch.as_tensor(hrows, device=out.device)
            out_h = out[b, rows_t, h].cpu().numpy()
            if row_lists is not None:
                gpus2.append(out2[b, rows_t, h].cpu().numpy())
            if not ret:
                for b0 in range(0, len(hrows), row_block):
                    r = oracle.layer_rows(x, b, h, hrows[b0:b0 + row_block])
                    refs.append(r.out)
                gpus.append(out_h)
                continue
            slot = s.retrieval_heads.index(h)
            cnt = st[0][b, rows_t, slot].cpu().numpy()
            mass = st[1][b, rows_t, slot].cpu().numpy()
            ndiff = 0
            counts_ref = []
            for b0 in range(0, len(hrows), row_block):
                blk = hrows[b0:b0 + row_block]
                r = oracle.layer_rows(x, b, h, blk, top_p=p32(p), want_pi=sets is not None)
                ref_out = r.out.copy()
                bm = (st[2][b, torch.as_tensor(blk, device=out.device), slot].cpu().numpy()
                      if sets == "bitmap" else None)
                counts_ref.append(r.count)
                for t, i in enumerate(blk):
                    k = int(cnt[b0 + t])
                    pos = s.prefix + int(i)
                    if sets is None:
                        if s.prefill_dense:
                            assert k == pos + 1, f"b={b} h={h} row={i}: dense prefill counts {k} keys"
                        elif s.top_k == 0:
                            assert float(mass[b0 + t]) >= p - MASS_TOL
                        continue
                    if sets == "bitmap":
                        sel = bitmap_positions(bm[t], pos + 1)
                        assert len(sel) == k, f"b={b} h={h} row={i}: bitmap has {len(sel)} keys, count {k}"
                    else:
                        sel = row_lists[b, b0 + t, slot, :k].astype(np.int64)
                        assert np.all(np.diff(sel) > 0) and (k == 0 or (sel[0] >= 0 and sel[-1] <= pos)), \
                            f"b={b} h={h} row={i}: listed positions not ascending inside the causal range"
                    if exact_sets:
                        assert np.array_equal(sel, r.sel[t]), f"b={b} h={h} row={i}: set differs"
                    nd = check_selection(sel, r, t, p32(p), f"b={b} h={h} row={i}", top_k=s.top_k)
                    if s.top_k == 0:
                        assert abs(float(mass[b0 + t]) - float(r.pi[t][sel].sum())) <= MASS_TOL, \
                            f"b={b} h={h} row={i}: mass {mass[b0 + t]} vs {r.pi[t][sel].sum()}"
                    if nd:
                        ref_out[t] = oracle.attend_set(x, b, h, int(i), sel)
                    ndiff += nd
                refs.append(ref_out)
                del r
            gpus.append(out_h)
            summary[(b, h)] = (cnt.copy(), np.concatenate(counts_ref), ndiff)
    err = check_outputs(np.concatenate(gpus), np.concatenate(refs), f"{s.name} prefill p={p}")
    if gpus2:
        check_outputs(np.concatenate(gpus2), np.concatenate(refs), f"{s.name} prefill p={p}, listed rows")
    if own:
        layer.close()
    return {"out": out[:, torch.as_tensor(rows, device=out.device)].cpu().numpy(), "summary": summary, "err": err}
