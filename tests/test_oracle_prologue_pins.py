"""Pins of the oracle's query prologue, Q-Cal and HoPE (CPU only).

* The pages' Q-Cal worked example ([Reader] "Implementation and Training Recipes"): with
  W_down hidden = (1, 0) and W_up's first column (0.1, 0.2, 0.1, 0.2) the correction is that
  column and the calibrated query is (0.6, -0.3, 0.6, -0.3) (tests/golden/qcal_score_example.json).
* Hand-derived closed forms of the rotation for d = 4, base = 4 (pair frequencies 1 and 1/2):
  both pairs turning, and only the first (training length between the two periods, 2 pi and
  4 pi).
* The number of rotating pairs against its closed form
  min(d/2, floor((d/2) ln(L / 2 pi) / ln(base)) + 1) for L >= 2 pi.
* Relative position: R_p x . R_s y = x . R_{s-p} y, and rotations keep norms.
* The low-rank correction against numpy's matmul, with and without rotation (the correction
  is rotated like the query: q_cal - q = R(W_up W_down hidden)).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "qcal_score_example.json")


def test_qcal_worked_example():
    g = json.load(open(GOLDEN))
    d = g["d"]
    q = np.array(g["q"], dtype=np.float64).reshape(1, 1, 1, d)
    hidden = np.array([1.0, 0.0]).reshape(1, 1, 2)
    W_down = np.eye(2).reshape(1, 2, 2)
    W_up = np.zeros((1, d, 2))
    W_up[0, :, 0] = g["delta_q"]
    W_up[0, :, 1] = [3.0, -1.0, 2.0, 5.0]   # multiplies the zero component of W_down hidden
    q_out, qc = oracle.qcal_hope(q, hidden, W_down, W_up, base=10000.0, train_len=0.0)
    assert np.allclose(qc.reshape(d), g["q_cal"], rtol=0, atol=1e-15)
    assert np.array_equal(q_out, q)
    # and its surrogate score with the example's landmark (step 1): 0.06
    k = np.array(g["k_landmark"])
    assert abs(float(qc.reshape(d) @ k) / math.sqrt(d) + g["b_landmark"] - g["score"]) < 1e-15


@pytest.mark.parametrize("p", [0, 1, 7, 1000, 123457])
def test_rotation_closed_form_d4(p):
    x = np.array([0.3, -1.2, 0.8, 0.5])
    got = oracle.hope_rotate(x.reshape(1, 1, 1, 4), base=4.0, train_len=1e9, pos0=p)[0, 0, 0]
    want = [x[0] * math.cos(p) - x[2] * math.sin(p),
            x[1] * math.cos(p / 2) - x[3] * math.sin(p / 2),
            x[0] * math.sin(p) + x[2] * math.cos(p),
            x[1] * math.sin(p / 2) + x[3] * math.cos(p / 2)]
    assert np.allclose(got, want, rtol=0, atol=1e-12)
    # training length 10: period 2 pi fits, 4 pi does not -> only the first pair turns
    got = oracle.hope_rotate(x.reshape(1, 1, 1, 4), base=4.0, train_len=10.0, pos0=p)[0, 0, 0]
    want = [x[0] * math.cos(p) - x[2] * math.sin(p), x[1],
            x[0] * math.sin(p) + x[2] * math.cos(p), x[3]]
    assert np.allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d,base,L", [(128, 10000.0, 4000.0), (128, 10000.0, 8000.0),
                                      (64, 500000.0, 33000.0), (128, 10000.0, 1e12),
                                      (128, 10000.0, 3.0)])
def test_rotating_pair_count(d, base, L):
    n = sum(oracle.hope_rotates(m, d, base, L) for m in range(d // 2))
    want = 0 if L < 2 * math.pi else min(d // 2, math.floor(
        (d / 2) * math.log(L / (2 * math.pi)) / math.log(base)) + 1)
    assert n == want
    # a prefix of the pairs: the highest frequencies
    flags = [oracle.hope_rotates(m, d, base, L) for m in range(d // 2)]
    assert flags == sorted(flags, reverse=True)


def test_relative_position_and_norm():
    rng = np.random.default_rng(3)
    d = 64
    x, y = rng.standard_normal(d), rng.standard_normal(d)
    for p, s in [(0, 5), (17, 17), (100, 4096), (70000, 70003)]:
        rx = oracle.hope_rotate(x.reshape(1, 1, 1, d), base=10000.0, train_len=2000.0, pos0=p)
        ry = oracle.hope_rotate(y.reshape(1, 1, 1, d), base=10000.0, train_len=2000.0, pos0=s)
        ryd = oracle.hope_rotate(y.reshape(1, 1, 1, d), base=10000.0, train_len=2000.0,
                                 pos0=s - p)
        assert abs(float(rx.ravel() @ ry.ravel()) - float(x @ ryd.ravel())) < 1e-11
        assert abs(np.linalg.norm(rx) - np.linalg.norm(x)) < 1e-12


def test_low_rank_against_matmul():
    rng = np.random.default_rng(4)
    B, Hq, N, d, dm, r = 2, 3, 5, 8, 16, 4
    q = rng.standard_normal((B, Hq, N, d))
    hidden = rng.standard_normal((B, N, dm))
    W_down = rng.standard_normal((Hq, r, dm))
    W_up = rng.standard_normal((Hq, d, r))
    corr = np.einsum("hdr,hrm,bnm->bhnd", W_up, W_down, hidden)
    q_out, qc = oracle.qcal_hope(q, hidden, W_down, W_up, base=10000.0, train_len=0.0)
    assert np.allclose(qc, q + corr, rtol=1e-13, atol=1e-12) and np.array_equal(q_out, q)
    q_out, qc = oracle.qcal_hope(q, hidden, W_down, W_up, base=100.0, train_len=60.0, pos0=9)
    assert np.allclose(q_out, oracle.hope_rotate(q, base=100.0, train_len=60.0, pos0=9),
                       rtol=0, atol=1e-13)
    assert np.allclose(qc - q_out, oracle.hope_rotate(corr, base=100.0, train_len=60.0, pos0=9),
                       rtol=1e-12, atol=1e-12)
