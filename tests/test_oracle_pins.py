"""Pins of the fp64 CPU oracle to things other than itself.

Each test ties one oracle function to a value printed on the pages, a closed form, a textbook
routine (torch's scaled_dot_product_attention in fp64) or brute force, chosen so that a dropped
term, a wrong sign, scale or index, or a swapped operand fails at least one of them.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _golden(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _sdpa(q, K, V, mask, scale):
    """Textbook softmax attention in fp64 (library routine). q [B,Hq,Nq,d], K/V [B,Hkv,N,d]
    with query head h reading KV head h // (Hq/Hkv); mask [Nq, N] bool (True = attend)."""
    G = q.shape[1] // K.shape[1]
    Kt = torch.from_numpy(K).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(V).repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), Kt, Vt, attn_mask=torch.from_numpy(mask), scale=scale).numpy()


# ---------------------------------------------------------------- P1: value printed on the page
def test_qcal_worked_example_score(golden_dir):
    g = _golden(golden_dir, "qcal_score_example.json")
    d = g["d"]
    qc = np.array(g["q_cal"]).reshape(1, 1, 1, d)
    q = np.array(g["q"]).reshape(1, 1, 1, d)
    np.testing.assert_allclose(np.array(g["q"]) + np.array(g["delta_q"]), g["q_cal"], atol=1e-15)
    klm = np.zeros((1, 1, 2, d))
    klm[0, 0, 0] = g["k_landmark"]
    blm = np.array([[[g["b_landmark"], 0.0]]])
    K = np.zeros((1, 1, 2, d))
    V = np.zeros((1, 1, 2, d))
    # S=1, W=1, query at position 1: chunk 0 is the only eligible distant chunk (rule R1)
    r = oracle.forward(q, qc, K, V, klm, blm, S=1, K_top=1, W=1, q_pos0=1)
    assert r["idx"][0, 0, 0, 0] == 0
    assert abs(r["s_sel"][0, 0, 0, 0] - g["score"]) < 1e-15
    assert abs(r["sigma"][0, 0, 0, 0] - g["score"]) < 1e-15
    r1 = oracle.forward(q, qc, K, V, klm, blm, S=1, K_top=1, W=1, q_pos0=1, scale=1.0)
    assert abs(r1["s_sel"][0, 0, 0, 0] - g["dot_unscaled"]) < 1e-15


# ---------------------------------------------------------------- rule R1 table (hand-worked)
def test_eligibility_table(golden_dir):
    g = _golden(golden_dir, "eligibility_r1.json")
    for pos, S, W, n, ws, wl in g["rows"]:
        assert oracle.n_eligible(pos, S, W) == n, (pos, S, W)
        assert S * n == ws and pos - ws + 1 == wl


@pytest.mark.parametrize("seed", range(5))
def test_eligibility_covers_prefix_once(seed):
    rng = np.random.default_rng(seed)
    for _ in range(200):
        S = int(rng.integers(1, 70))
        W = int(rng.integers(1, 300))
        p = int(rng.integers(0, 3000))
        n = oracle.n_eligible(p, S, W)
        start = S * n
        covered = np.zeros(p + 1, np.int32)
        for c in range(n):
            covered[c * S:(c + 1) * S] += 1
        covered[start:p + 1] += 1
        assert (covered == 1).all()
        assert p - start + 1 >= min(W, p + 1)
        assert p - start + 1 <= W + S - 1 or n == 0
        # the window never reaches back past a chunk that is still eligible
        assert start == S * n


# ---------------------------------------------------------------- P2: brute-force top-K
@pytest.mark.parametrize("seed", range(30))
def test_topk_matches_bruteforce(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 9))
    K_top = int(rng.integers(0, 7))
    d = 3
    N = n + 1                      # S=1, W=1: the query at position n sees n distant chunks
    blm = rng.integers(-2, 3, size=(1, 1, N)).astype(np.float64)   # many exact ties
    klm = np.zeros((1, 1, N, d))   # sigma_c = b_c exactly
    q = rng.standard_normal((1, 1, 1, d))
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    r = oracle.forward(q, q, K, V, klm, blm, S=1, K_top=K_top, W=1, q_pos0=n)
    idx = r["idx"][0, 0, 0]
    sigma = blm[0, 0, :n]
    k = min(K_top, n)
    valid = []
    for T in itertools.combinations(range(n), k):
        ok = all(sigma[c] > sigma[o] or (sigma[c] == sigma[o] and c < o)
                 for c in T for o in range(n) if o not in T)
        if ok:
            valid.append(set(T))
    assert len(valid) == 1
    assert set(int(c) for c in idx[:k]) == valid[0]
    assert (idx[k:] == -1).all()
    chosen = [int(c) for c in idx[:k]]
    assert chosen == sorted(chosen, key=lambda c: (-sigma[c], c))
    if n > K_top and K_top > 0:
        srt = sorted(range(n), key=lambda c: (-sigma[c], c))
        assert r["gap"][0, 0, 0] == sigma[srt[K_top - 1]] - sigma[srt[K_top]]


def test_group_selection_uses_max_over_heads():
    """GQA rule: a chunk that one head rates highly is kept even if another head dislikes it
    (max), which a mean or sum over heads would not do."""
    d, X = 2, 4.0
    s = math.sqrt(d)
    qc = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, d) * s
    klm = np.zeros((1, 1, 3, d))
    klm[0, 0, 0] = [X, -X]          # head scores (X, -X): max X, mean 0
    klm[0, 0, 1] = [0.6 * X, 0.6 * X]  # head scores (0.6X, 0.6X): max 0.6X, mean 0.6X
    blm = np.zeros((1, 1, 3))
    K = np.zeros((1, 1, 3, d))
    V = np.zeros((1, 1, 3, d))
    r = oracle.forward(qc, qc, K, V, klm, blm, S=1, K_top=1, W=1, q_pos0=2)
    assert r["idx"][0, 0, 0, 0] == 0
    np.testing.assert_allclose(r["sigma"][0, 0, 0, 0], X, rtol=1e-15)
    # each head fuses with its own score (rule R4)
    np.testing.assert_allclose(r["s_sel"][0, :, 0, 0], [X, -X], rtol=1e-15)


# ---------------------------------------------------------------- P3: Gibbs identity
@pytest.mark.parametrize("W", [1, 3, 7])
def test_full_attention_when_every_chunk_is_a_token(W):
    """S=1, klm = the token key, b = 0, qc = q, K_top >= n: the surrogate score of each chunk is
    its exact log-mass, so HiLS is full causal softmax attention (GQA included)."""
    rng = np.random.default_rng(11 + W)
    B, Hq, Hkv, N, d = 2, 4, 2, 40, 8
    q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    r = oracle.forward(q, q, K, V, K, np.zeros((B, Hkv, N)), S=1, K_top=N, W=W)
    mask = np.tril(np.ones((N, N), dtype=bool))
    ref = _sdpa(q, K, V, mask, 1 / math.sqrt(d))
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)


def _exact_landmarks(q_vec, K, S, C, scale):
    """Landmark of each chunk built for one query: p = softmax of its logits in the chunk,
    k' = sum_j p_j K_j and b' = -sum_j p_j log p_j (the page's landmark summary)."""
    klm = np.zeros((C, K.shape[1]))
    blm = np.zeros(C)
    for c in range(C):
        x = K[c * S:(c + 1) * S] @ q_vec * scale
        p = np.exp(x - x.max())
        p /= p.sum()
        klm[c] = p @ K[c * S:(c + 1) * S]
        blm[c] = -(p * np.log(p)).sum()
    return klm, blm


@pytest.mark.parametrize("S,W,N", [(4, 5, 37), (8, 8, 64), (3, 1, 20)])
def test_full_attention_with_exact_entropy_landmarks(S, W, N):
    rng = np.random.default_rng(S * 100 + W)
    d = 6
    scale = 1 / math.sqrt(d)
    q = rng.standard_normal((1, 1, 1, d)) * 2
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    C = N // S
    klm, blm = _exact_landmarks(q[0, 0, 0], K[0, 0], S, C, scale)
    r = oracle.forward(q, q, K, V, klm[None, None], blm[None, None], S=S, K_top=C, W=W,
                       q_pos0=N - 1)
    mask = np.ones((1, N), dtype=bool)
    ref = _sdpa(q, K, V, mask, scale)
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)
    x = K[0, 0] @ q[0, 0, 0] * scale
    assert abs(r["lse"][0, 0, 0] - (x.max() + np.log(np.exp(x - x.max()).sum()))) < 1e-12


def test_exact_surrogates_select_like_block_sparse_attention():
    """With exact landmarks the surrogate ranking is the exact chunk-mass ranking of naive BSA."""
    rng = np.random.default_rng(5)
    S, W, N, d, Kt = 8, 8, 160, 4, 5
    scale = 1 / math.sqrt(d)
    q = rng.standard_normal((1, 1, 1, d)) * 3
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    C = N // S
    klm, blm = _exact_landmarks(q[0, 0, 0], K[0, 0], S, C, scale)
    r = oracle.forward(q, q, K, V, klm[None, None], blm[None, None], S=S, K_top=Kt, W=W,
                       q_pos0=N - 1)
    n = oracle.n_eligible(N - 1, S, W)
    x = K[0, 0] @ q[0, 0, 0] * scale
    mass = np.array([np.exp(x[c * S:(c + 1) * S]).sum() for c in range(n)])
    bsa = sorted(range(n), key=lambda c: (-mass[c], c))[:Kt]
    assert [int(c) for c in r["idx"][0, 0, 0]] == bsa


# ---------------------------------------------------------------- landmark construction (R15)
def _lse(x):
    m = x.max()
    return m + math.log(np.exp(x - m).sum())


@pytest.mark.parametrize("scale", [0.0, 0.37])
def test_landmark_surrogate_is_exact_at_its_expansion_point(scale):
    """Gibbs identity: at the landmark query itself, scale * q'.k' + H(p) is the chunk's exact
    log-mass log sum_j exp(scale * q'.K_j) (a wrong chunk offset, scale, weight or entropy sign
    breaks it)."""
    rng = np.random.default_rng(11)
    B, Hkv, S, d = 2, 3, 16, 8
    N = 5 * S + 7                                   # a partial last chunk gets no landmark
    K = rng.standard_normal((B, Hkv, N, d))
    C = N // S
    qlm = rng.standard_normal((B, Hkv, C, d)) * 2
    klm, blm = oracle.landmarks(qlm, K, S=S, scale=scale)
    assert klm.shape == (B, Hkv, C, d) and blm.shape == (B, Hkv, C)
    sc = scale if scale > 0 else 1 / math.sqrt(d)
    for b, g, c in itertools.product(range(B), range(Hkv), range(C)):
        ref = _lse(K[b, g, c * S:(c + 1) * S] @ qlm[b, g, c] * sc)
        s_hat = sc * qlm[b, g, c] @ klm[b, g, c] + blm[b, g, c]
        assert abs(s_hat - ref) < 1e-12 * max(1.0, abs(ref))


def test_landmark_surrogate_is_a_tangent_of_the_chunk_log_mass():
    """First-order Taylor expansion of the chunk log-mass at the landmark query ([Reader] "Paper
    Primer"): moving the query by t leaves an error that shrinks as t^2, and the tangent plane
    of the convex log-mass never lies above it."""
    rng = np.random.default_rng(12)
    d, S = 8, 32
    K = rng.standard_normal((1, 1, S, d))
    q0 = rng.standard_normal((1, 1, 1, d))
    klm, blm = oracle.landmarks(q0, K, S=S)
    sc = 1 / math.sqrt(d)
    delta = rng.standard_normal(d)
    errs = []
    for t in (0.04, 0.02, 0.01):
        q = q0[0, 0, 0] + t * delta
        true = _lse(K[0, 0] @ q * sc)
        s_hat = sc * q @ klm[0, 0, 0] + blm[0, 0, 0]
        assert s_hat <= true + 1e-14
        errs.append(true - s_hat)
    assert 3.6 < errs[0] / errs[1] < 4.4 and 3.6 < errs[1] / errs[2] < 4.4


def test_landmark_of_a_flat_chunk_is_the_mean_key_with_maximal_entropy():
    """Uniform attention inside the chunk (a zero landmark query, or identical keys): the summary
    is the mean-pooled key and the bias is log S, the largest entropy possible."""
    rng = np.random.default_rng(13)
    d, S, C = 4, 8, 3
    K = rng.standard_normal((1, 2, C * S, d))
    K[0, 1] = np.repeat(rng.standard_normal((C, 1, d)), S, axis=1).reshape(C * S, d)
    qlm = np.zeros((1, 2, C, d))
    qlm[0, 1] = rng.standard_normal((C, d)) * 5
    klm, blm = oracle.landmarks(qlm, K, S=S)
    np.testing.assert_allclose(blm, math.log(S), rtol=0, atol=1e-13)
    for g in range(2):
        np.testing.assert_allclose(klm[0, g], K[0, g].reshape(C, S, d).mean(axis=1),
                                   rtol=0, atol=1e-13)
    # any other chunk has a smaller entropy
    qr = rng.standard_normal((1, 2, C, d)) * 3
    _, b2 = oracle.landmarks(qr, rng.standard_normal((1, 2, C * S, d)), S=S)
    assert (b2 > 0).all() and (b2 < math.log(S)).all()


def test_landmark_of_a_concentrated_chunk_is_its_dominant_key():
    """One key dominating the chunk's softmax: the summary is that key and the entropy bias
    vanishes; a one-token chunk is exactly its key with bias 0."""
    rng = np.random.default_rng(14)
    d, S = 6, 16
    K = rng.standard_normal((1, 1, S, d)) * 0.1
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    K[0, 0, 5] = 40.0 * math.sqrt(d) * u     # logit about 40 above the rest
    klm, blm = oracle.landmarks(u[None, None, None], K, S=S)
    np.testing.assert_allclose(klm[0, 0, 0], K[0, 0, 5], rtol=0, atol=1e-12)
    assert 0.0 <= blm[0, 0, 0] < 1e-14
    K1 = rng.standard_normal((1, 1, 5, d))
    k1, b1 = oracle.landmarks(rng.standard_normal((1, 1, 5, d)), K1, S=1)
    np.testing.assert_array_equal(k1, K1)
    np.testing.assert_array_equal(b1, np.zeros((1, 1, 5)))


@pytest.mark.parametrize("S,W,N", [(4, 5, 37), (8, 8, 64)])
def test_oracle_landmarks_give_full_attention(S, W, N):
    """Landmarks built for the query itself (every chunk's landmark query = q) make every
    surrogate exact, so with K covering all chunks HiLS is full causal attention."""
    rng = np.random.default_rng(S + N)
    d = 6
    q = rng.standard_normal((1, 1, 1, d)) * 2
    K = rng.standard_normal((1, 1, N, d))
    V = rng.standard_normal((1, 1, N, d))
    C = N // S
    klm, blm = oracle.landmarks(np.broadcast_to(q, (1, 1, C, d)), K, S=S)
    r = oracle.forward(q, q, K, V, klm, blm, S=S, K_top=C, W=W, q_pos0=N - 1)
    ref = _sdpa(q, K, V, np.ones((1, N), dtype=bool), 1 / math.sqrt(d))
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)


def test_landmarks_reject_bad_sizes():
    with pytest.raises(RuntimeError):
        oracle.landmarks(np.zeros((1, 1, 0, 4)), np.zeros((1, 1, 8, 4)), S=0)


# ---------------------------------------------------------------- P4: K=0 is windowed attention
def test_k0_is_sliding_window_attention():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, N, d, S, W = 1, 2, 1, 96, 8, 16, 20
    q = rng.standard_normal((B, Hq, N, d))
    K = rng.standard_normal((B, Hkv, N, d))
    V = rng.standard_normal((B, Hkv, N, d))
    klm = rng.standard_normal((B, Hkv, N // S, d))
    blm = rng.uniform(-1, 1, (B, Hkv, N // S))
    r = oracle.forward(q, q, K, V, klm, blm, S=S, K_top=0, W=W)
    mask = np.zeros((N, N), dtype=bool)
    for p in range(N):
        mask[p, S * oracle.n_eligible(p, S, W):p + 1] = True
    ref = _sdpa(q, K, V, mask, 1 / math.sqrt(d))
    np.testing.assert_allclose(r["out"], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- P5: hand-worked example
def _hand_problem(g, exp_klm=None, exp_blm=None):
    N, d = g["N"], g["d"]
    q = np.array(g["q"], float).reshape(1, 1, N, d)
    qc = np.array(g["q_cal"], float).reshape(1, 1, N, d)
    K = np.log(np.array(g["exp_logit_K"], float)).reshape(1, 1, N, d)
    V = np.array(g["V"], float).reshape(1, 1, N, d)
    klm = np.log(np.array(exp_klm or g["exp_klm"], float)).reshape(1, 1, -1, d)
    blm = np.log(np.array(exp_blm or g["exp_blm"], float)).reshape(1, 1, -1)
    return q, qc, K, V, klm, blm


def test_hand_worked_two_chunk_example(golden_dir):
    g = _golden(golden_dir, "two_chunk_hand_example.json")
    args = _hand_problem(g)
    kw = dict(S=g["S"], W=g["W"], scale=g["scale"])
    r1 = oracle.forward(*args, K_top=1, **kw)
    for p in range(6):
        assert abs(r1["out"][0, 0, p, 0] - float(Fraction(g["expected_K1"]["O"][p]))) < 1e-14
        assert abs(r1["lse"][0, 0, p] - math.log(g["expected_K1"]["exp_LSE"][p])) < 1e-14
    assert list(r1["idx"][0, 0, 5]) == g["expected_K1"]["idx_p5"]
    assert abs(r1["gap"][0, 0, 5] - math.log(g["expected_K1"]["gap_p5_exp"])) < 1e-14
    r2 = oracle.forward(*args, K_top=2, **kw)
    assert abs(r2["out"][0, 0, 5, 0] - float(Fraction(g["expected_K2_p5"]["O"]))) < 1e-14
    assert abs(r2["lse"][0, 0, 5] - math.log(g["expected_K2_p5"]["exp_LSE"])) < 1e-14
    assert list(r2["idx"][0, 0, 5]) == g["expected_K2_p5"]["idx"]
    r0 = oracle.forward(*args, K_top=0, **kw)
    for p in range(6):
        assert abs(r0["out"][0, 0, p, 0] - float(Fraction(g["expected_K0"]["O"][p]))) < 1e-14
        assert abs(r0["lse"][0, 0, p] - math.log(g["expected_K0"]["exp_LSE"][p])) < 1e-14
    t = g["tie_case"]
    rt = oracle.forward(*_hand_problem(g, t["exp_klm"], t["exp_blm"]), K_top=t["K_top"], **kw)
    assert list(rt["idx"][0, 0, 5]) == t["idx_p5"]
    assert abs(rt["out"][0, 0, 5, 0] - float(Fraction(t["O_p5"]))) < 1e-14
    assert abs(rt["lse"][0, 0, 5] - math.log(t["exp_LSE_p5"])) < 1e-14


# ---------------------------------------------------------------- P6: invariants
def _random_problem(seed, B=1, Hq=4, Hkv=2, N=160, d=8, S=8, scale_v=1.0):
    rng = np.random.default_rng(seed)
    C = N // S
    return dict(
        q=rng.standard_normal((B, Hq, N, d)),
        qc=rng.standard_normal((B, Hq, N, d)),
        K=rng.standard_normal((B, Hkv, N, d)),
        V=rng.standard_normal((B, Hkv, N, d)) * scale_v,
        klm=rng.standard_normal((B, Hkv, C, d)),
        blm=rng.uniform(-1, 1, (B, Hkv, C)),
    )


def test_invariants():
    S, W, Kt = 8, 12, 3
    P = _random_problem(1)
    r = oracle.forward(**P, S=S, K_top=Kt, W=W, units=True)
    B, Hq, N, d = P["q"].shape
    Hkv = P["K"].shape[1]
    G = Hq // Hkv
    for i in range(N):
        n = oracle.n_eligible(i, S, W)
        for g in range(Hkv):
            idx = r["idx"][0, g, i]
            k = min(Kt, n)
            sel = [int(c) for c in idx[:k]]
            assert len(set(sel)) == k and all(0 <= c < n for c in sel)
            assert (idx[k:] == -1).all()
            for h in range(g * G, (g + 1) * G):
                scores = np.append(r["s_sel"][0, h, i], r["unit_lse"][0, h, i, Kt])
                w = np.exp(scores - r["lse"][0, h, i])
                assert abs(w.sum() - 1) < 1e-12
                np.testing.assert_allclose(w @ r["unit_o"][0, h, i], r["out"][0, h, i],
                                           atol=1e-12)
                rows = list(range(S * n, i + 1))
                for c in sel:
                    rows += list(range(c * S, c * S + S))
                Vr = P["V"][0, g, rows]
                assert (r["out"][0, h, i] <= Vr.max(0) + 1e-12).all()
                assert (r["out"][0, h, i] >= Vr.min(0) - 1e-12).all()


def test_constant_and_linear_in_v():
    S, W, Kt = 8, 12, 3
    P = _random_problem(2)
    const = np.broadcast_to(np.arange(P["V"].shape[-1], dtype=float), P["V"].shape).copy()
    rc = oracle.forward(**{**P, "V": const}, S=S, K_top=Kt, W=W)
    expect = np.broadcast_to(np.arange(P["V"].shape[-1], dtype=float), rc["out"].shape)
    np.testing.assert_allclose(rc["out"], expect, atol=1e-12)
    V2 = np.random.default_rng(9).standard_normal(P["V"].shape)
    ra = oracle.forward(**P, S=S, K_top=Kt, W=W)
    rb = oracle.forward(**{**P, "V": V2}, S=S, K_top=Kt, W=W)
    rab = oracle.forward(**{**P, "V": 2 * P["V"] - 3 * V2}, S=S, K_top=Kt, W=W)
    np.testing.assert_allclose(rab["out"], 2 * ra["out"] - 3 * rb["out"], atol=1e-11)


def test_minus_inf_bias_gets_zero_weight():
    S, W, Kt = 8, 12, 19
    P = _random_problem(4, Hq=2, Hkv=1)
    P["blm"][..., 3] = -np.inf
    r = oracle.forward(**P, S=S, K_top=Kt, W=W, units=True)
    i = P["q"].shape[2] - 1
    idx = list(r["idx"][0, 0, i])
    assert 3 in idx and idx.index(3) == oracle.n_eligible(i, S, W) - 1
    P2 = {k: v.copy() for k, v in P.items()}
    P2["V"][0, 0, 24:32] = 1e6          # chunk 3's values cannot leak into the output
    r2 = oracle.forward(**P2, S=S, K_top=Kt, W=W)
    np.testing.assert_allclose(r2["out"][0, :, i], r["out"][0, :, i], atol=1e-12)


# ---------------------------------------------------------------- P7: GQA structure
def test_replicated_heads_equal_single_head():
    S, W, Kt = 8, 12, 3
    P = _random_problem(6, Hq=1, Hkv=1)
    rep = {**P, "q": np.repeat(P["q"], 3, 1), "qc": np.repeat(P["qc"], 3, 1)}
    r1 = oracle.forward(**P, S=S, K_top=Kt, W=W)
    r3 = oracle.forward(**rep, S=S, K_top=Kt, W=W)
    assert (r3["idx"] == r1["idx"]).all()
    for h in range(3):
        np.testing.assert_array_equal(r3["out"][:, h], r1["out"][:, 0])


def test_groups_are_independent():
    S, W, Kt = 8, 12, 3
    P = _random_problem(7, Hq=4, Hkv=2)
    r = oracle.forward(**P, S=S, K_top=Kt, W=W)
    for g in range(2):
        sub = dict(q=P["q"][:, 2 * g:2 * g + 2], qc=P["qc"][:, 2 * g:2 * g + 2],
                   K=P["K"][:, g:g + 1], V=P["V"][:, g:g + 1], klm=P["klm"][:, g:g + 1],
                   blm=P["blm"][:, g:g + 1])
        rs = oracle.forward(**sub, S=S, K_top=Kt, W=W)
        np.testing.assert_array_equal(rs["idx"][:, 0], r["idx"][:, g])
        np.testing.assert_array_equal(rs["out"], r["out"][:, 2 * g:2 * g + 2])


# ---------------------------------------------------------------- oracle API plumbing
def test_forced_selection_and_sampled_jobs_agree():
    S, W, Kt = 8, 12, 3
    P = _random_problem(8, B=2)
    r = oracle.forward(**P, S=S, K_top=Kt, W=W, units=True)
    rf = oracle.forward(**P, S=S, K_top=Kt, W=W, idx_in=r["idx"])
    np.testing.assert_array_equal(rf["out"], r["out"])
    # the same rows through the per-query job API with a partial row map
    b, g, i = 1, 1, 150
    G = 2
    n = oracle.n_eligible(i, S, W)
    need = set(range(S * n, i + 1))
    for c in r["idx"][b, g, i]:
        if c >= 0:
            need |= set(range(c * S, c * S + S))
    need = sorted(need)
    row_map = -np.ones(P["K"].shape[2], np.int64)
    row_map[need] = np.arange(len(need))
    qu = oracle.Query(i, P["q"][b, g * G:(g + 1) * G, i], P["qc"][b, g * G:(g + 1) * G, i],
                      P["klm"][b, g], P["blm"][b, g], P["K"][b, g, need], P["V"][b, g, need],
                      row_map=row_map)
    (rq,) = oracle.run_queries([qu], d=8, G=G, S=S, K_top=Kt, W=W, units=True)
    np.testing.assert_array_equal(rq["idx"], r["idx"][b, g, i])
    np.testing.assert_array_equal(rq["out"], r["out"][b, g * G:(g + 1) * G, i])
    # a missing row is reported, not read
    row_map[need[0]] = -1
    qu2 = oracle.Query(i, qu.q, qu.qc, qu.klm, qu.blm, qu.K_rows, qu.V_rows, row_map=row_map)
    with pytest.raises(RuntimeError):
        oracle.run_queries([qu2], d=8, G=G, S=S, K_top=Kt, W=W)


def test_rejects_bad_arguments():
    P = _random_problem(9)
    with pytest.raises(RuntimeError):
        oracle.forward(**P, S=8, K_top=3, W=12, idx_in=np.full((1, 2, 160, 3), 999, np.int32))
