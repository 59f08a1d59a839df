"""Backward pass (hils_backward) against the fp64 oracle's backward, through the C ABI.

Both sides differentiate sum(dout * out) + sum(dlse * lse) with the same selection, the one the
oracle's own forward makes (the top-K passes no gradient).  Every gradient element is compared:
dq, dq_cal, dK, dV, dk_lm, db_lm.

Tolerance, per gradient tensor and (b, head or kv-group) plane, on the largest absolute
difference relative to the plane's largest reference magnitude.
* fp32 inputs: every product and sum is fp32, so the only differences from the fp64 oracle are
  fp32 rounding (logits, exponentials, sums of up to ~10^4 terms): 3e-5 (about 250 fp32 ulps).
* bf16 inputs: the logits and dout . V products take the inputs exactly, but the fused weights
  a and the logit gradients dx enter the dq, dK and dV products rounded to bf16 (relative error
  up to 2^-9 per term, independent between terms), so an output's error is a sum of n terms
  each off by up to 2^-9 of itself: about 2^-9 / sqrt(3) * ||terms||_2, far below the plane's
  maximum for the row counts here; 1e-2 of the plane's maximum bounds it with room.

At the full 7B-like size (N = 131072) the oracle runs one query at a time: the sampled queries'
dq and dq_cal rows (which depend on that query alone) are compared under the same rule, and two
identities that hold at any size check the key-side gradients of every row at once: the V
gradient summed over the tokens equals the output gradient summed over the rows (each row's
fused weights sum to one), and sum q . dq = sum K . dK, sum q_cal . dq_cal = sum k_lm . dk_lm
(the logits and the chunk scores depend on those pairs only through their dot products).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from hierarchical_chunk_sparse_scoring_b200 import binding as hb
from hierarchical_chunk_sparse_scoring_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = 3e-5
GRADS = [("dq", "dq"), ("dq_cal", "dqc"), ("dK", "dK"), ("dV", "dV"), ("dk_lm", "dklm"),
         ("db_lm", "dblm")]


def _upstream(wl, seed, with_dlse=True):
    g = torch.Generator(device="cuda").manual_seed(seed)
    dout = (torch.randn(wl.q.shape, generator=g, device="cuda")).to(wl.q.dtype).contiguous()
    dlse = torch.randn(wl.q.shape[:3], generator=g, device="cuda") if with_dlse else None
    return dout, dlse


def _arrays(wl):
    return [parity.f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]


def _tol(dtype):
    return 3e-5 if dtype == torch.float32 else 1e-2


def _compare(got, want, name, tol=TOL):
    got = got.detach().cpu().double().numpy()
    assert np.isfinite(got).all(), name
    assert got.shape == want.shape, (name, got.shape, want.shape)
    worst = 0.0
    # planes: (b, kv group) for K-side tensors, (b, head) for the rest; db_lm one plane per (b, g)
    planes = got.reshape(got.shape[0] * got.shape[1], -1)
    wplanes = want.reshape(planes.shape)
    for p in range(planes.shape[0]):
        scale = float(np.abs(wplanes[p]).max(initial=0.0))
        err = float(np.abs(planes[p] - wplanes[p]).max(initial=0.0))
        if scale == 0.0:
            assert err == 0.0, (name, p, err)
            continue
        worst = max(worst, err / scale)
        assert err <= tol * scale, (name, p, err, scale)
    return worst


def _check_all(wl, dout, dlse):
    arrs = _arrays(wl)
    kw = dict(S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0)
    idx = oracle.forward(*arrs, **kw)["idx"]
    ref = oracle.backward(*arrs, idx, parity.f64(dout), None if dlse is None else parity.f64(dlse),
                          **kw)
    got = hb.backward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm,
                      torch.from_numpy(idx).cuda(), dout, dlse, **kw)
    torch.cuda.synchronize()
    return {name: _compare(got[name], ref[oname], name, _tol(wl.q.dtype))
            for name, oname in GRADS}


def _suffix(wl, n_q):
    """The workload's last n_q queries over all of its keys."""
    N = wl.q.shape[2]
    return W.Workload(wl.name + "_suffix", wl.q[:, :, N - n_q:].contiguous(),
                      wl.q_cal[:, :, N - n_q:].contiguous(), wl.K, wl.V, wl.k_lm, wl.b_lm, wl.S,
                      wl.K_top, wl.W, wl.q_pos0 + N - n_q)


CASES = [
    ("tiny_fp32", {}, None),                                        # fp32, G=1, d=64, K=4
    ("small_mha_bf16", dict(B=2, Hq=2, Hkv=2, N=1500), None),       # bf16 MHA, ragged tail
    ("gqa7b_prefill", dict(N=2048), None),                          # bf16, G=4, d=128, K=16
    ("gqa7b_prefill", dict(N=1800, dtype=torch.float32), None),     # fp32 GQA, ragged
    ("extreme", dict(N=6000), 400),                                 # G=8, S=128, W=2048, K=16
]


@pytest.mark.parametrize("name,kw,n_q", CASES, ids=lambda x: x if isinstance(x, str) else (
    ",".join("%s=%s" % (k, v) for k, v in x.items()) if isinstance(x, dict) else str(x)))
def test_backward_matches_oracle(name, kw, n_q):
    wl = W.make(name, "cuda", **kw)
    if n_q is not None:   # (the oracle's cost grows with W + K S per row)
        wl = _suffix(wl, n_q)
    dout, dlse = _upstream(wl, seed=len(name) + wl.q.shape[2])
    print("worst |diff| / plane max:", name, kw, _check_all(wl, dout, dlse))


def _random(B, Hq, Hkv, N, d, S, K, W_, dtype, seed, q_pos0=0, N_q=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    N_q = N - q_pos0 if N_q is None else N_q
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    return W.Workload("bwd_random", r(B, Hq, N_q, d), r(B, Hq, N_q, d), r(B, Hkv, N, d),
                      r(B, Hkv, N, d), r(B, Hkv, N // S, d),
                      torch.rand((B, Hkv, N // S), generator=g, device="cuda") * 2 - 1, S, K, W_,
                      q_pos0)


EDGE = {
    "s16_k32_g2": dict(B=1, Hq=4, Hkv=2, N=1500, d=128, S=16, K=32, W_=64,
                       dtype=torch.float32),                # smallest tiles, largest K
    "s32_g16_d64": dict(B=2, Hq=16, Hkv=1, N=1200, d=64, S=32, K=4, W_=100,
                        dtype=torch.bfloat16),               # 16 heads per KV head
    "k0_window_only": dict(B=1, Hq=2, Hkv=1, N=700, d=64, S=64, K=0, W_=96,
                           dtype=torch.float32),             # windowed attention only
    "suffix_queries": dict(B=1, Hq=4, Hkv=1, N=3000, d=128, S=64, K=8, W_=128, q_pos0=2000,
                           dtype=torch.bfloat16),            # queries 2000..2999 only
    "few_queries_mid": dict(B=1, Hq=2, Hkv=2, N=2600, d=64, S=128, K=6, W_=256, q_pos0=1000,
                            N_q=300, dtype=torch.float32),   # keys past the last query unread
    "w1_s64": dict(B=1, Hq=2, Hkv=2, N=1000, d=128, S=64, K=8, W_=1,
                   dtype=torch.bfloat16),                    # window of a single token
}


@pytest.mark.parametrize("case", sorted(EDGE))
def test_backward_edge_cases(case):
    kw = dict(EDGE[case])
    wl = _random(**kw, seed=len(case) * 7)
    dout, dlse = _upstream(wl, seed=3, with_dlse=case != "k0_window_only")
    print("worst |diff| / plane max:", case, _check_all(wl, dout, dlse))


def spread_selection(B, Hkv, N_q, K, S, W, q_pos0, seed):
    """A valid selection that does not come from either side: per query min(K, n) distinct
    eligible chunks, spread evenly over [0, n) from a seeded random offset, -1 padded."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    pos = torch.arange(N_q, device="cuda") + q_pos0
    n = torch.clamp(pos - W + 1, min=0) // S                       # eligible chunks (R1)
    u = torch.rand((B, Hkv, N_q, 1), generator=g, device="cuda")
    k = torch.arange(K, device="cuda").view(1, 1, 1, K)
    nn = n.view(1, 1, N_q, 1).expand(B, Hkv, N_q, K)
    spread = torch.floor((k + u) * nn / K).long()
    few = k.expand(B, Hkv, N_q, K)
    idx = torch.where(nn > K, spread, torch.where(few < nn, few, torch.full_like(few, -1)))
    return idx.to(torch.int32).contiguous()


def test_backward_full_size_sampled():
    wl = W.make("gqa7b_prefill", "cuda")   # N = 131072, 32/8 heads, d = 128, K = 16
    kw = wl.kwargs()
    B0, Hkv0, N0 = wl.q.shape[0], wl.K.shape[1], wl.q.shape[2]
    idx = spread_selection(B0, Hkv0, N0, wl.K_top, wl.S, wl.W, wl.q_pos0, seed=17)
    dout, dlse = _upstream(wl, seed=99)
    got = hb.backward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, idx, dout, dlse, **kw)
    torch.cuda.synchronize()
    B, Hq, N, d = wl.q.shape
    Hkv = wl.K.shape[1]
    G = Hq // Hkv
    # identities over every row
    for b in range(B):
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)
            sv = got["dV"][b, g].double().sum(0)
            so = dout[b, hs].double().sum((0, 1))
            assert float((sv - so).abs().max()) <= 1e-4 * float(so.abs().max()) + 1e-3
            for (x, dx, y, dy) in (("q", "dq", "K", "dK"), ("q_cal", "dq_cal", "k_lm", "dk_lm")):
                xs = getattr(wl, x)[b, hs].double()
                ys = getattr(wl, y)[b, g].double()
                lhs = (xs * got[dx][b, hs].double())
                rhs = (ys * got[dy][b, g].double())
                mag = float(lhs.abs().sum()) + float(rhs.abs().sum())
                assert abs(float(lhs.sum()) - float(rhs.sum())) <= 1e-5 * mag, (x, y)
    # sampled rows: the oracle per query, one KV group at a time
    rng = np.random.default_rng(5)
    qs = sorted(set(rng.integers(0, N, 6).tolist()) | {0, 1100, N - 1})
    for g in (0, Hkv - 1):
        hs = slice(g * G, (g + 1) * G)
        Kf, Vf = parity.f64(wl.K[:, g:g + 1]), parity.f64(wl.V[:, g:g + 1])
        klm, blm = parity.f64(wl.k_lm[:, g:g + 1]), parity.f64(wl.b_lm[:, g:g + 1])
        for i in qs:
            sl = slice(i, i + 1)
            ref = oracle.backward(parity.f64(wl.q[:, hs, sl]), parity.f64(wl.q_cal[:, hs, sl]),
                                  Kf, Vf, klm, blm, idx[:, g:g + 1, sl].cpu().numpy(),
                                  parity.f64(dout[:, hs, sl]), parity.f64(dlse[:, hs, sl]),
                                  S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=i)
            _compare(got["dq"][:, hs, sl], ref["dq"], "dq", _tol(wl.q.dtype))
            _compare(got["dq_cal"][:, hs, sl], ref["dqc"], "dq_cal", _tol(wl.q.dtype))
