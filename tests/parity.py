"""Parity of the CUDA path against the fp64 oracle (test infrastructure).

Selection rule: where the oracle's score gap at rank K (sigma_(K) - sigma_(K+1)) exceeds 1e-3,
the GPU must select exactly the oracle's chunks (compared as sets).  Elsewhere several
selections are correct: the GPU's must then be a valid top-K within 1e-3 (every chunk it keeps
scores, in fp64, at least sigma_(K) - 1e-3), with unique eligible ids, min(K, n) of them.  On
every row the list must be in (sigma desc, c asc) order: descending in the fp64 sigma up to
1e-3, and exactly equal sigmas in ascending chunk order.
Outputs are always compared with the oracle run on the GPU's own selection.

Tolerances: fp32 inputs, max_row |O - O_ref|_inf / |O_ref|_inf <= 1e-5 and |lse - lse_ref| <=
1e-5 * max(1, |lse_ref|); bf16 inputs, |x - ref| <= 2e-3 + 1e-2 |ref| elementwise for O and lse.
"""
import numpy as np
import torch

import oracle

GAP = 1e-3


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def eligible(pos, S, W):
    first = pos - W + 1
    return 0 if first <= 0 else first // S


def check_selection(gidx, oidx, gap, sig_gpu, sig_ora, n):
    """gidx/oidx [R,K] int; gap [R]; sig_gpu [R,K] fp64 sigma of the GPU's chunks; sig_ora [R,K]
    the oracle's sorted sigmas; n [R] eligible counts.  Returns (exact_rows, tie_rows)."""
    R, K = gidx.shape
    exact = ties = 0
    if K == 0:
        return R, 0
    for r in range(R):
        k = min(K, int(n[r]))
        g = gidx[r]
        assert (g[k:] == -1).all(), ("padding", r, g, k)
        sel = g[:k]
        assert (sel >= 0).all() and (sel < n[r]).all(), ("range", r, sel, n[r])
        assert len(set(sel.tolist())) == k, ("duplicate", r, sel)
        # the list is ordered by (sigma desc, c asc): descending in the oracle's fp64 sigma up to
        # rounding, and chunks whose sigma is exactly equal in lower-index-first order
        for j in range(k - 1):
            a, b_ = sig_gpu[r, j], sig_gpu[r, j + 1]
            assert a >= b_ - GAP, ("order", r, sel, sig_gpu[r, :k])
            if a == b_:
                assert sel[j] < sel[j + 1], ("tie order", r, sel, sig_gpu[r, :k])
        if not (gap[r] > GAP):
            ties += 1
            if k > 0:
                floor = sig_ora[r, k - 1] - GAP
                assert (sig_gpu[r, :k] >= floor).all(), ("near-tie invalid", r, sel, sig_gpu[r],
                                                         floor)
        else:
            exact += 1
            assert set(sel.tolist()) == set(oidx[r, :k].tolist()), (
                "selection", r, sorted(sel.tolist()), sorted(oidx[r, :k].tolist()), gap[r])
    return exact, ties


def compare_outputs(out, ref, lse, lse_ref, dtype):
    """out/ref [..., d]; lse/lse_ref [...].  Returns error summary; raises on violation."""
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    lse = np.asarray(lse, np.float64)
    lse_ref = np.asarray(lse_ref, np.float64)
    assert np.isfinite(out).all() and np.isfinite(lse).all()
    if dtype == torch.float32:
        row_err = np.abs(out - ref).max(-1) / np.maximum(np.abs(ref).max(-1), 1e-30)
        lse_err = np.abs(lse - lse_ref) / np.maximum(1.0, np.abs(lse_ref))
        worst = float(row_err.max(initial=0.0))
        assert worst <= 1e-5, ("fp32 out rel err", worst)
        assert float(lse_err.max(initial=0.0)) <= 1e-5, ("fp32 lse err", float(lse_err.max()))
        return {"out_rel_row_max": worst, "lse_rel_max": float(lse_err.max(initial=0.0))}
    viol = np.abs(out - ref) - (2e-3 + 1e-2 * np.abs(ref))
    lviol = np.abs(lse - lse_ref) - (2e-3 + 1e-2 * np.abs(lse_ref))
    assert viol.max(initial=-1) <= 0, ("bf16 out", float(np.abs(out - ref).max()))
    assert lviol.max(initial=-1) <= 0, ("bf16 lse", float(np.abs(lse - lse_ref).max()))
    return {"out_abs_max": float(np.abs(out - ref).max(initial=0.0)),
            "lse_abs_max": float(np.abs(lse - lse_ref).max(initial=0.0))}


def full_check(wl, out, lse, idx, threads=0):
    """Every query of a (small) workload."""
    arrs = [f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    kw = dict(S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0, threads=threads)
    own = oracle.forward(*arrs, **kw)
    gidx = idx.cpu().numpy()
    forced = oracle.forward(*arrs, idx_in=gidx, **kw)
    B, Hkv, Nq, K = gidx.shape
    n = np.array([eligible(wl.q_pos0 + i, wl.S, wl.W) for i in range(Nq)])
    R = B * Hkv * Nq
    exact, ties = check_selection(gidx.reshape(R, K), own["idx"].reshape(R, K),
                                  own["gap"].reshape(R), forced["sigma"].reshape(R, K),
                                  own["sigma"].reshape(R, K), np.tile(n, B * Hkv))
    errs = compare_outputs(f64(out), forced["out"], f64(lse), forced["lse"], wl.q.dtype)
    errs.update(exact_rows=exact, tie_rows=ties)
    return errs


def sample_rows(wl, n_rows, seed=0):
    """(b, g, i) rows spread over positions: the last query without a distant chunk, the first
    with one, the first and last query of several chunk phases, the last query, and random."""
    B, Hkv, Nq = wl.q.shape[0], wl.K.shape[1], wl.q.shape[2]
    rng = np.random.default_rng(seed)
    S, W = wl.S, wl.W
    special = {Nq - 1, 0}
    first = S + W - 1 - wl.q_pos0
    for i in (first - 1, first):
        if 0 <= i < Nq:
            special.add(i)
    for t in rng.integers(0, max(1, Nq // S), size=8):
        for off in (0, S - 1):
            i = int(t) * S + off
            if 0 <= i < Nq:
                special.add(i)
    rows = [(int(rng.integers(B)), int(rng.integers(Hkv)), i) for i in sorted(special)]
    while len(rows) < n_rows:
        rows.append((int(rng.integers(B)), int(rng.integers(Hkv)), int(rng.integers(Nq))))
    return rows[:max(n_rows, len(special))]


def sampled_check(wl, out, lse, idx, rows, threads=0):
    """Rows (b, g, i) of a large workload; only the data those rows need is copied."""
    Hq, d = wl.q.shape[1], wl.q.shape[3]
    Hkv = wl.K.shape[1]
    G = Hq // Hkv
    S, W, K = wl.S, wl.W, wl.K_top
    gidx_all = idx
    sel_q, frc_q, meta = [], [], []
    klm_cache = {}
    empty = np.zeros((0, d))
    no_rows = np.zeros(0, np.int64)
    # rows of the same (b, g) share one gathered set of K/V rows and one token -> row map, in
    # batches (a map covers the whole sequence: 32 MB at 4M tokens)
    order = sorted(range(len(rows)), key=lambda j: (rows[j][0], rows[j][1]))
    batches, cur = [], []
    for j in order:
        if cur and (rows[cur[0]][:2] != rows[j][:2] or len(cur) == 32):
            batches.append(cur)
            cur = []
        cur.append(j)
    if cur:
        batches.append(cur)
    slots = [None] * len(rows)
    for bt in batches:
        b, g = rows[bt[0]][:2]
        if (b, g) not in klm_cache:
            klm_cache[(b, g)] = (f64(wl.k_lm[b, g]), f64(wl.b_lm[b, g]))
        klm, blm = klm_cache[(b, g)]
        toks = set()
        sels = {}
        for j in bt:
            i = rows[j][2]
            pos = wl.q_pos0 + i
            n = eligible(pos, S, W)
            gsel = gidx_all[b, g, i].cpu().numpy()
            sels[j] = (pos, n, gsel)
            toks |= set(range(S * n, pos + 1))
            for c in gsel:
                if c >= 0:
                    toks |= set(range(int(c) * S, int(c) * S + S))
        toks = np.array(sorted(toks), np.int64)
        tt = torch.from_numpy(toks).to(wl.K.device)
        Kr = f64(wl.K[b, g].index_select(0, tt))
        Vr = f64(wl.V[b, g].index_select(0, tt))
        row_map = -np.ones(wl.K.shape[2], np.int64)
        row_map[toks] = np.arange(len(toks))
        for j in bt:
            i = rows[j][2]
            pos, n, gsel = sels[j]
            qh = f64(wl.q[b, g * G:(g + 1) * G, i])
            qch = f64(wl.q_cal[b, g * G:(g + 1) * G, i])
            slots[j] = (oracle.Query(pos, qh, qch, klm, blm, empty, empty, row_map=no_rows),
                        oracle.Query(pos, qh, qch, klm, blm, Kr, Vr, row_map=row_map,
                                     idx_in=gsel),
                        (b, g, i, n, gsel))
    for sq, fq, m in slots:
        sel_q.append(sq)
        frc_q.append(fq)
        meta.append(m)
    kw = dict(d=d, G=G, S=S, K_top=K, W=W, threads=threads)
    own = oracle.run_queries(sel_q, select_only=True, **kw)
    forced = oracle.run_queries(frc_q, **kw)
    gidx = np.stack([m[4] for m in meta])
    exact, ties = check_selection(gidx, np.stack([r["idx"] for r in own]),
                                  np.array([r["gap"] for r in own]),
                                  np.stack([r["sigma"] for r in forced]),
                                  np.stack([r["sigma"] for r in own]),
                                  np.array([m[3] for m in meta]))
    outs = np.stack([f64(out[b, g * G:(g + 1) * G, i]) for (b, g, i, _, _) in meta])
    lses = np.stack([f64(lse[b, g * G:(g + 1) * G, i]) for (b, g, i, _, _) in meta])
    errs = compare_outputs(outs, np.stack([r["out"] for r in forced]), lses,
                           np.stack([r["lse"] for r in forced]), wl.q.dtype)
    errs.update(exact_rows=exact, tie_rows=ties, rows=len(rows))
    return errs
