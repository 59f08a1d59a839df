"""fp64 CPU oracle of the HiLS attention forward pass -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  The CUDA product path never imports, links or calls it.

The arithmetic lives in ``hils_oracle.c`` (plain C, fp64); its header lists the steps, the
sources on the pages and the readings R1-R11.  This module only marshals numpy arrays.
"""
import ctypes
import math

import numpy as np

from . import build as _build

_lib = None


class Cfg(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("G", ctypes.c_int32), ("S", ctypes.c_int32),
                ("K_top", ctypes.c_int32), ("W", ctypes.c_int32), ("n_chunks", ctypes.c_int64),
                ("scale", ctypes.c_double)]


class Rows(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("row_map", ctypes.c_void_p),
                ("n_tokens", ctypes.c_int64)]


class Job(ctypes.Structure):
    _fields_ = [("pos", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("q_hs", ctypes.c_int64),
                ("qc", ctypes.c_void_p), ("qc_hs", ctypes.c_int64),
                ("klm", ctypes.c_void_p), ("blm", ctypes.c_void_p),
                ("K", Rows), ("V", Rows),
                ("idx_in", ctypes.c_void_p), ("idx_out", ctypes.c_void_p),
                ("sigma_out", ctypes.c_void_p), ("gap_out", ctypes.c_void_p),
                ("s_sel_out", ctypes.c_void_p), ("s_sel_hs", ctypes.c_int64),
                ("out", ctypes.c_void_p), ("out_hs", ctypes.c_int64),
                ("lse_out", ctypes.c_void_p), ("lse_hs", ctypes.c_int64),
                ("unit_o_out", ctypes.c_void_p), ("unit_o_hs", ctypes.c_int64),
                ("unit_lse_out", ctypes.c_void_p), ("unit_lse_hs", ctypes.c_int64),
                ("status", ctypes.c_int32)]


class Problem(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("N_q", ctypes.c_int64), ("N_kv", ctypes.c_int64), ("d", ctypes.c_int64),
                ("q_pos0", ctypes.c_int64), ("S", ctypes.c_int32), ("K_top", ctypes.c_int32),
                ("W", ctypes.c_int32), ("scale", ctypes.c_double)]


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        l = ctypes.CDLL(path)
        l.hils_oracle_run.restype = ctypes.c_int
        l.hils_oracle_run.argtypes = [ctypes.POINTER(Cfg), ctypes.c_int64, ctypes.POINTER(Job),
                                      ctypes.c_int]
        l.hils_oracle_forward.restype = ctypes.c_int
        l.hils_oracle_forward.argtypes = [ctypes.POINTER(Problem)] + [ctypes.c_void_p] * 15 + [
            ctypes.c_int]
        l.hils_oracle_landmarks.restype = ctypes.c_int
        l.hils_oracle_landmarks.argtypes = [ctypes.c_int64] * 4 + [ctypes.c_int32,
                                                                   ctypes.c_double] + [
            ctypes.c_void_p] * 4
        l.hils_oracle_backward.restype = ctypes.c_int
        l.hils_oracle_backward.argtypes = [ctypes.POINTER(Problem)] + [ctypes.c_void_p] * 15 + [
            ctypes.c_int]
        l.hils_oracle_hope_rotates.restype = ctypes.c_int
        l.hils_oracle_hope_rotates.argtypes = [ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                               ctypes.c_double]
        l.hils_oracle_hope_rotate.restype = ctypes.c_int
        l.hils_oracle_hope_rotate.argtypes = [ctypes.c_int64] * 5 + [ctypes.c_double] * 2 + [
            ctypes.c_void_p] * 2
        l.hils_oracle_qcal_hope.restype = ctypes.c_int
        l.hils_oracle_qcal_hope.argtypes = [ctypes.c_int64] * 7 + [ctypes.c_double] * 2 + [
            ctypes.c_void_p] * 6
        l.hils_oracle_n_eligible.restype = ctypes.c_int64
        l.hils_oracle_n_eligible.argtypes = [ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]
        l.hils_oracle_default_threads.restype = ctypes.c_int
        _lib = l
    return _lib


def default_threads() -> int:
    return int(lib().hils_oracle_default_threads())


def n_eligible(pos: int, S: int, W: int) -> int:
    """Rule R1: eligible distant chunks of the query at position ``pos``."""
    return int(lib().hils_oracle_n_eligible(pos, S, W))


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data


def forward(q, qc, K, V, klm, blm, *, S, K_top, W, q_pos0=0, scale=0.0, idx_in=None,
            units=False, threads=0):
    """Whole problem. q, qc [B,Hq,N_q,d]; K, V [B,Hkv,N_kv,d]; klm [B,Hkv,C,d]; blm [B,Hkv,C].

    Returns a dict with out, lse, idx, sigma, gap, s_sel (and unit_o, unit_lse if ``units``).
    """
    q, qc, K, V, klm, blm = (_f64(x) for x in (q, qc, K, V, klm, blm))
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = K.shape
    C = Nkv // S
    assert klm.shape == (B, Hkv, C, d), (klm.shape, (B, Hkv, C, d))
    assert blm.shape == (B, Hkv, C)
    pr = Problem(B, Hq, Hkv, Nq, Nkv, d, q_pos0, S, K_top, W, float(scale))
    r = {
        "idx": np.empty((B, Hkv, Nq, K_top), np.int32),
        "sigma": np.empty((B, Hkv, Nq, K_top)),
        "gap": np.empty((B, Hkv, Nq)),
        "s_sel": np.empty((B, Hq, Nq, K_top)),
        "out": np.empty((B, Hq, Nq, d)),
        "lse": np.empty((B, Hq, Nq)),
    }
    if units:
        r["unit_o"] = np.empty((B, Hq, Nq, K_top + 1, d))
        r["unit_lse"] = np.empty((B, Hq, Nq, K_top + 1))
    idx_arr = None
    if idx_in is not None:
        idx_arr = np.ascontiguousarray(np.asarray(idx_in, dtype=np.int32))
        assert idx_arr.shape == (B, Hkv, Nq, K_top)
    rc = lib().hils_oracle_forward(
        ctypes.byref(pr), _ptr(q), _ptr(qc), _ptr(K), _ptr(V), _ptr(klm), _ptr(blm),
        _ptr(idx_arr), _ptr(r["idx"]), _ptr(r["sigma"]), _ptr(r["gap"]), _ptr(r["s_sel"]),
        _ptr(r["out"]), _ptr(r["lse"]), _ptr(r.get("unit_o")), _ptr(r.get("unit_lse")),
        int(threads))
    if rc != 0:
        raise RuntimeError("hils_oracle_forward failed with status %d" % rc)
    return r


def landmarks(qlm, K, *, S, scale=0.0):
    """Landmark construction (R15): qlm [B,Hkv,C,d] landmark queries, K [B,Hkv,N_kv,d] keys,
    C = N_kv // S.  Returns (klm [B,Hkv,C,d], blm [B,Hkv,C])."""
    qlm, K = _f64(qlm), _f64(K)
    B, Hkv, Nkv, d = K.shape
    C = Nkv // S if S > 0 else 0   # (S <= 0 is rejected by the C side)
    assert qlm.shape == (B, Hkv, C, d), (qlm.shape, (B, Hkv, C, d))
    klm = np.empty((B, Hkv, C, d))
    blm = np.empty((B, Hkv, C))
    rc = lib().hils_oracle_landmarks(B, Hkv, Nkv, d, S, float(scale), _ptr(qlm), _ptr(K),
                                     _ptr(klm), _ptr(blm))
    if rc != 0:
        raise RuntimeError("hils_oracle_landmarks failed with status %d" % rc)
    return klm, blm


def backward(q, qc, K, V, klm, blm, idx, dO, dlse=None, *, S, K_top, W, q_pos0=0, scale=0.0,
             threads=0):
    """Gradients of sum(dO * out) + sum(dlse * lse) with the selection ``idx`` [B,Hkv,N_q,K_top]
    held fixed.  Returns a dict with dq, dqc, dK, dV, dklm, dblm (fp64, shaped like q, qc, K, V,
    klm, blm)."""
    q, qc, K, V, klm, blm, dO = (_f64(x) for x in (q, qc, K, V, klm, blm, dO))
    dlse = None if dlse is None else _f64(dlse)
    B, Hq, Nq, d = q.shape
    _, Hkv, Nkv, _ = K.shape
    C = Nkv // S
    assert klm.shape == (B, Hkv, C, d) and blm.shape == (B, Hkv, C) and dO.shape == q.shape
    assert dlse is None or dlse.shape == (B, Hq, Nq)
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32))
    assert idx.shape == (B, Hkv, Nq, K_top)
    pr = Problem(B, Hq, Hkv, Nq, Nkv, d, q_pos0, S, K_top, W, float(scale))
    r = {"dq": np.empty_like(q), "dqc": np.empty_like(q), "dK": np.empty_like(K),
         "dV": np.empty_like(K), "dklm": np.empty_like(klm), "dblm": np.empty_like(blm)}
    rc = lib().hils_oracle_backward(
        ctypes.byref(pr), _ptr(q), _ptr(qc), _ptr(K), _ptr(V), _ptr(klm), _ptr(blm), _ptr(idx),
        _ptr(dO), _ptr(dlse), _ptr(r["dq"]), _ptr(r["dqc"]), _ptr(r["dK"]), _ptr(r["dV"]),
        _ptr(r["dklm"]), _ptr(r["dblm"]), int(threads))
    if rc != 0:
        raise RuntimeError("hils_oracle_backward failed with status %d" % rc)
    return r


def hope_rotates(m, d, base, train_len):
    """HoPE (R17): whether dimension pair (m, m + d/2) rotates."""
    return bool(lib().hils_oracle_hope_rotates(m, d, float(base), float(train_len)))


def hope_rotate(x, *, base, train_len, pos0=0):
    """HoPE (R17) of x [B, H, N, d], token n at position pos0 + n."""
    x = _f64(x)
    B, H, N, d = x.shape
    out = np.empty_like(x)
    rc = lib().hils_oracle_hope_rotate(B, H, N, d, pos0, float(base), float(train_len),
                                       _ptr(x), _ptr(out))
    if rc != 0:
        raise RuntimeError("hils_oracle_hope_rotate failed with status %d" % rc)
    return out


def qcal_hope(q, hidden, W_down, W_up, *, base, train_len, pos0=0):
    """Q-Cal and HoPE: q [B,Hq,N_q,d], hidden [B,N_q,d_model], W_down [Hq,r,d_model], W_up
    [Hq,d,r].  Returns (HoPE(q), HoPE(q + W_up W_down hidden)) at positions pos0 + i."""
    q, hidden, W_down, W_up = (_f64(x) for x in (q, hidden, W_down, W_up))
    B, Hq, Nq, d = q.shape
    dm = hidden.shape[2]
    r = W_down.shape[1]
    assert hidden.shape == (B, Nq, dm) and W_down.shape == (Hq, r, dm) and W_up.shape == (Hq, d, r)
    q_out, qc_out = np.empty_like(q), np.empty_like(q)
    rc = lib().hils_oracle_qcal_hope(B, Hq, Nq, d, dm, r, pos0, float(base), float(train_len),
                                     _ptr(q), _ptr(hidden), _ptr(W_down), _ptr(W_up),
                                     _ptr(q_out), _ptr(qc_out))
    if rc != 0:
        raise RuntimeError("hils_oracle_qcal_hope failed with status %d" % rc)
    return q_out, qc_out


class Query:
    """One (query token, KV head) problem for :func:`run_queries`.

    q, qc: [G, d] the group's token / calibrated queries; klm [C, d]; blm [C];
    K_rows, V_rows: [R, d] the token rows provided; row_map: int64 [N_kv] token -> row (-1 =
    not provided), or None when K_rows / V_rows hold every token 0..N_kv-1.
    """

    def __init__(self, pos, q, qc, klm, blm, K_rows, V_rows, row_map=None, idx_in=None):
        self.pos = int(pos)
        self.q, self.qc, self.klm, self.blm = _f64(q), _f64(qc), _f64(klm), _f64(blm)
        self.K_rows, self.V_rows = _f64(K_rows), _f64(V_rows)
        self.row_map = None if row_map is None else np.ascontiguousarray(row_map, np.int64)
        self.idx_in = None if idx_in is None else np.ascontiguousarray(idx_in, np.int32)


def run_queries(queries, *, d, G, S, K_top, W, scale=0.0, units=False, threads=0,
                select_only=False):
    """Runs independent (query, KV head) problems; returns one result dict per query with
    idx [K], sigma [K], gap, s_sel [G,K], out [G,d], lse [G] (+ unit_o, unit_lse).
    select_only: steps 1-2 only (out / lse are not computed and no K/V rows are read)."""
    n = len(queries)
    jobs = (Job * max(n, 1))()
    results = []
    for j, qu in enumerate(queries):
        n_tok = qu.K_rows.shape[0] if qu.row_map is None else qu.row_map.shape[0]
        r = {"idx": np.empty(K_top, np.int32), "sigma": np.empty(K_top), "gap": np.empty(1),
             "s_sel": np.empty((G, K_top)), "out": np.empty((G, d)), "lse": np.empty(G)}
        if units:
            r["unit_o"] = np.empty((G, K_top + 1, d))
            r["unit_lse"] = np.empty((G, K_top + 1))
        jb = jobs[j]
        jb.pos = qu.pos
        jb.q, jb.q_hs = _ptr(qu.q), d
        jb.qc, jb.qc_hs = _ptr(qu.qc), d
        jb.klm, jb.blm = _ptr(qu.klm), _ptr(qu.blm)
        jb.K = Rows(_ptr(qu.K_rows), _ptr(qu.row_map), n_tok)
        jb.V = Rows(_ptr(qu.V_rows), _ptr(qu.row_map), n_tok)
        jb.idx_in = _ptr(qu.idx_in)
        jb.idx_out, jb.sigma_out, jb.gap_out = _ptr(r["idx"]), _ptr(r["sigma"]), _ptr(r["gap"])
        jb.s_sel_out, jb.s_sel_hs = _ptr(r["s_sel"]), K_top
        if select_only:
            r.pop("out")
            r.pop("lse")
        jb.out, jb.out_hs = _ptr(r.get("out")), d
        jb.lse_out, jb.lse_hs = _ptr(r.get("lse")), 1
        jb.unit_o_out, jb.unit_o_hs = _ptr(r.get("unit_o")), (K_top + 1) * d
        jb.unit_lse_out, jb.unit_lse_hs = _ptr(r.get("unit_lse")), K_top + 1
        results.append(r)
    n_chunks = min(qu.klm.shape[0] for qu in queries) if queries else 0
    cfg = Cfg(d, G, S, K_top, W, n_chunks, float(scale))
    rc = lib().hils_oracle_run(ctypes.byref(cfg), n, jobs, int(threads))
    for j in range(n):
        results[j]["status"] = int(jobs[j].status)
        results[j]["gap"] = float(results[j]["gap"][0])
    if rc != 0:
        raise RuntimeError("hils_oracle_run failed with status %d" % rc)
    return results


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
