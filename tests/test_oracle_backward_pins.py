"""Pins of the oracle's backward pass (CPU only).

The backward is pinned against things it shares no arithmetic with:
* central finite differences of the oracle's forward (itself pinned in test_oracle_pins.py):
  every input tensor, with the selection held fixed; a dropped term, a wrong sign or a swapped
  operand anywhere in the chain rule moves some entry far outside the O(h^2) error;
* K_top = 0 reduces the method to windowed softmax attention, whose gradient torch's autograd
  gives for a plain masked-softmax implementation (a library routine, fp64 on the CPU);
* invariants that hold for any input: every row's attention weights sum to one, so the V
  gradient summed over the tokens equals the summed output gradient; the chunk scores depend on
  qc and klm only through qc . klm and the token logits on q and K only through q . K, so the
  gradients satisfy sum qc . dqc = sum klm . dklm and sum q . dq = sum K . dK (Euler's relation
  for a function of a bilinear form);
* tokens after the last query and chunks no query selected receive exactly zero.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _problem(seed, B=1, Hq=4, Hkv=2, d=8, N=48, S=4, K_top=3, W=6, q_pos0=0, N_q=None,
             bias_spread=1.0):
    rng = np.random.default_rng(seed)
    N_q = N - q_pos0 if N_q is None else N_q
    C = N // S
    r = lambda *s: rng.standard_normal(s)
    x = dict(q=r(B, Hq, N_q, d), qc=r(B, Hq, N_q, d), K=r(B, Hkv, N, d), V=r(B, Hkv, N, d),
             klm=r(B, Hkv, C, d), blm=bias_spread * rng.uniform(-1, 1, (B, Hkv, C)))
    kw = dict(S=S, K_top=K_top, W=W, q_pos0=q_pos0)
    fwd = oracle.forward(*(x[k] for k in ("q", "qc", "K", "V", "klm", "blm")), **kw)
    dO = r(B, Hq, N_q, d)
    dlse = r(B, Hq, N_q)
    return x, kw, fwd["idx"], dO, dlse


def _loss(x, kw, idx, dO, dlse):
    f = oracle.forward(*(x[k] for k in ("q", "qc", "K", "V", "klm", "blm")), idx_in=idx, **kw)
    return float((f["out"] * dO).sum() + (f["lse"] * dlse).sum())


NAMES = [("q", "dq"), ("qc", "dqc"), ("K", "dK"), ("V", "dV"), ("klm", "dklm"), ("blm", "dblm")]


@pytest.mark.parametrize("case", [
    dict(seed=1),
    dict(seed=2, Hq=2, Hkv=2, W=5, S=3, N=40, K_top=2),            # G = 1, odd S and W
    dict(seed=3, Hq=6, Hkv=2, K_top=5, N=60, S=5, W=7),            # G = 3, some n <= K
    dict(seed=4, B=2, Hq=2, Hkv=1, N=50, q_pos0=30, N_q=20),       # queries from position 30
])
def test_backward_matches_finite_differences(case):
    x, kw, idx, dO, dlse = _problem(**case)
    g = oracle.backward(*(x[k] for k in ("q", "qc", "K", "V", "klm", "blm")), idx, dO, dlse,
                        **kw)
    rng = np.random.default_rng(100 + case["seed"])
    h = 1e-5
    for name, gname in NAMES:
        a = x[name]
        flat = a.reshape(-1)
        picks = rng.choice(flat.size, size=min(flat.size, 24), replace=False)
        # also every entry with a non-zero gradient among the biases (few of them)
        if name == "blm":
            picks = np.arange(flat.size)
        for e in picks:
            old = flat[e]
            flat[e] = old + h
            lp = _loss(x, kw, idx, dO, dlse)
            flat[e] = old - h
            lm = _loss(x, kw, idx, dO, dlse)
            flat[e] = old
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[e]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, int(e), fd, an)


def test_zero_for_unreached_tokens_and_unselected_chunks():
    # queries 0..29 of a 48-token sequence: tokens 30.. are attended by nobody
    x, kw, idx, dO, dlse = _problem(seed=5, N=48, q_pos0=0, N_q=30)
    g = oracle.backward(*(x[k] for k in ("q", "qc", "K", "V", "klm", "blm")), idx, dO, dlse,
                        **kw)
    assert (g["dK"][:, :, 30:] == 0).all() and (g["dV"][:, :, 30:] == 0).all()
    C = x["klm"].shape[2]
    for bg in range(idx.shape[0] * idx.shape[1]):
        b, gi = divmod(bg, idx.shape[1])
        chosen = set(int(c) for c in idx[b, gi].reshape(-1) if c >= 0)
        for c in range(C):
            if c not in chosen:
                assert (g["dklm"][b, gi, c] == 0).all() and g["dblm"][b, gi, c] == 0
    assert len(chosen) > 0


def test_k0_equals_autograd_windowed_attention():
    # K_top = 0: every query attends its window [S n, p] only (R1, R7); out = softmax attention
    B, H, N, d, S, W = 1, 3, 37, 8, 4, 6
    rng = np.random.default_rng(7)
    q, K, V = (rng.standard_normal(s) for s in ((B, H, N, d), (B, H, N, d), (B, H, N, d)))
    qc = rng.standard_normal((B, H, N, d))
    klm = rng.standard_normal((B, H, N // S, d))
    blm = rng.uniform(-1, 1, (B, H, N // S))
    dO, dlse = rng.standard_normal((B, H, N, d)), rng.standard_normal((B, H, N))
    idx = np.full((B, H, N, 0), -1, np.int32)
    g = oracle.backward(q, qc, K, V, klm, blm, idx, dO, dlse, S=S, K_top=0, W=W)
    # autograd of masked softmax attention
    tq, tK, tV = (torch.tensor(a, requires_grad=True) for a in (q, K, V))
    pos = torch.arange(N)
    n = torch.clamp(pos - W + 1, min=0) // S
    mask = (pos[None, :] <= pos[:, None]) & (pos[None, :] >= S * n[:, None])
    logits = torch.einsum("bhid,bhjd->bhij", tq, tK) / math.sqrt(d)
    logits = logits.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(logits, -1)
    out = torch.einsum("bhij,bhjd->bhid", torch.softmax(logits, -1), tV)
    ((out * torch.tensor(dO)).sum() + (lse * torch.tensor(dlse)).sum()).backward()
    for got, want in ((g["dq"], tq.grad), (g["dK"], tK.grad), (g["dV"], tV.grad)):
        assert np.allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)
    assert (g["dqc"] == 0).all() and (g["dklm"] == 0).all() and (g["dblm"] == 0).all()


@pytest.mark.parametrize("seed", [11, 12])
def test_backward_invariants(seed):
    x, kw, idx, dO, dlse = _problem(seed=seed, B=2, Hq=6, Hkv=2, N=64, S=4, K_top=4, W=8,
                                    bias_spread=2.0)
    g = oracle.backward(*(x[k] for k in ("q", "qc", "K", "V", "klm", "blm")), idx, dO, dlse,
                        **kw)
    B, Hq = x["q"].shape[:2]
    Hkv = x["K"].shape[1]
    G = Hq // Hkv
    for b in range(B):
        for gi in range(Hkv):
            hs = slice(gi * G, (gi + 1) * G)
            # sum over tokens of dV = sum over the group's rows of dO
            assert np.allclose(g["dV"][b, gi].sum(0), dO[b, hs].sum((0, 1)), atol=1e-10)
            # Euler relations of the two bilinear forms
            lhs = (x["qc"][b, hs] * g["dqc"][b, hs]).sum()
            rhs = (x["klm"][b, gi] * g["dklm"][b, gi]).sum()
            assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), (lhs, rhs)
            lhs = (x["q"][b, hs] * g["dq"][b, hs]).sum()
            rhs = (x["K"][b, gi] * g["dK"][b, gi]).sum()
            assert abs(lhs - rhs) <= 1e-10 * max(1.0, abs(lhs)), (lhs, rhs)
