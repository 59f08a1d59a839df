"""Landmark construction on the GPU (hils_landmarks) against the fp64 oracle, through the C ABI.

k_lm[c] = sum_j p_j K_j and b_lm[c] = H(p) with p = softmax(scale q_lm[c] . K_j) over the chunk's
keys ([Reader] "The HiLS-Attention Mechanism": chunk summary and entropy bias).

Tolerances.  fp32 inputs: k_lm within 1e-5 of its row's largest entry (relative, per row, as for
the forward's outputs); b_lm within 1e-5 * max(1, |x|max) where |x|max is the chunk's largest
logit magnitude (the entropy is computed as ln Z - sum_j p_j x_j, whose rounding grows with the
logits; for a concentrated chunk both terms are close to the largest logit).  bf16 inputs:
|x - ref| <= 2e-3 + 1e-2 |ref| elementwise for k_lm (rounded to bf16 on output) and b_lm.

End to end (the exact-surrogate pin, now on the device): landmarks built on the GPU from a
decode query itself, with one head per KV group (q_cal = q) and K covering every eligible chunk,
make hils_forward equal full causal softmax attention of that query.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from hierarchical_chunk_sparse_scoring_b200 import binding as hb

pytestmark = pytest.mark.gpu


def _inputs(B, Hkv, N, d, S, dtype, seed, concentrated=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    C = N // S
    K = torch.randn((B, Hkv, N, d), generator=g, device="cuda") / math.sqrt(d)
    q_lm = torch.randn((B, Hkv, C, d), generator=g, device="cuda") / math.sqrt(d)
    if concentrated and C > 0:
        # each landmark query points hard at one key of its chunk (logit ~ 40): p is close to
        # one-hot and the entropy close to 0
        j = torch.randint(0, S, (B, Hkv, C), generator=g, device="cuda")
        rows = torch.arange(C, device="cuda") * S
        key = torch.gather(K, 2, (rows + j).unsqueeze(-1).expand(B, Hkv, C, d))
        q_lm = 40.0 * math.sqrt(d) * key / (key.norm(dim=-1, keepdim=True) ** 2)
    return q_lm.to(dtype), K.to(dtype)


CASES = [
    dict(B=2, Hkv=3, N=1000, d=64, S=64),      # partial last chunk
    dict(B=1, Hkv=2, N=4096, d=128, S=128),
    dict(B=1, Hkv=1, N=777, d=32, S=16),
    dict(B=2, Hkv=1, N=100, d=16, S=1),        # one key per chunk: k_lm = K, b_lm = 0
    dict(B=1, Hkv=2, N=2000, d=128, S=64, concentrated=True),
    dict(B=1, Hkv=1, N=3000, d=64, S=100),     # chunk size not a multiple of the key batches
]


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("case", range(len(CASES)))
def test_landmarks_match_oracle(case, dtype):
    kw = dict(CASES[case])
    conc = kw.pop("concentrated", False)
    q_lm, K = _inputs(**kw, dtype=dtype, seed=100 + case, concentrated=conc)
    S = kw["S"]
    k_lm, b_lm = hb.landmarks(q_lm, K, S=S)
    torch.cuda.synchronize()
    ref_k, ref_b = oracle.landmarks(parity.f64(q_lm), parity.f64(K), S=S)
    got_k, got_b = parity.f64(k_lm), parity.f64(b_lm)
    assert np.isfinite(got_k).all() and np.isfinite(got_b).all()
    if dtype == torch.float32:
        row = np.abs(got_k - ref_k).max(-1) / np.maximum(np.abs(ref_k).max(-1), 1e-30)
        assert float(row.max(initial=0)) <= 1e-5, float(row.max())
        d = kw["d"]
        Kc = parity.f64(K)[:, :, :ref_k.shape[2] * S].reshape(*ref_k.shape[:3], S, d)
        xmax = np.abs(np.einsum("bgcd,bgcjd->bgcj", parity.f64(q_lm), Kc)).max(-1) / math.sqrt(d)
        assert (np.abs(got_b - ref_b) <= 1e-5 * np.maximum(1.0, xmax)).all(), float(
            np.abs(got_b - ref_b).max())
    else:
        assert (np.abs(got_k - ref_k) <= 2e-3 + 1e-2 * np.abs(ref_k)).all()
        assert (np.abs(got_b - ref_b) <= 2e-3 + 1e-2 * np.abs(ref_b)).all()
    if S == 1:
        assert np.array_equal(got_k, parity.f64(K)) and (got_b == 0).all()


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
def test_gpu_landmarks_make_hils_full_attention(dtype):
    # decode query at p = N - 1, S = 64, W = 64: n = floor((N - 64) / 64) = 32 eligible chunks,
    # all selected with K = 32; each chunk's landmark query is the decode query itself
    B, H, N, d, S, W = 3, 2, 64 * 33 + 17, 64, 64, 64
    g = torch.Generator(device="cuda").manual_seed(7)
    q = (torch.randn((B, H, 1, d), generator=g, device="cuda") * 2 / math.sqrt(d)).to(dtype)
    K = (torch.randn((B, H, N, d), generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    V = (torch.randn((B, H, N, d), generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    C = N // S
    q_lm = q.expand(B, H, C, d).contiguous()
    k_lm, b_lm = hb.landmarks(q_lm, K, S=S)
    out, lse, idx = hb.forward(q, q, K, V, k_lm, b_lm, S=S, K_top=32, W=W, q_pos0=N - 1)
    torch.cuda.synchronize()
    n = parity.eligible(N - 1, S, W)
    assert n == 32 and bool((idx >= 0).all())
    # full causal attention of the query over tokens 0..N-1, fp64
    qf, Kf, Vf = parity.f64(q)[:, :, 0], parity.f64(K), parity.f64(V)
    x = np.einsum("bhd,bhnd->bhn", qf, Kf) / math.sqrt(d)
    ref_lse = np.log(np.exp(x - x.max(-1, keepdims=True)).sum(-1)) + x.max(-1)
    ref = np.einsum("bhn,bhnd->bhd", np.exp(x - ref_lse[..., None]), Vf)
    got = parity.f64(out)[:, :, 0]
    got_l = parity.f64(lse)[:, :, 0]
    if dtype == torch.float32:
        err = np.abs(got - ref).max(-1) / np.abs(ref).max(-1)
        assert float(err.max()) <= 1e-5, float(err.max())
        assert float(np.abs(got_l - ref_lse).max()) <= 1e-5 * max(1.0, float(np.abs(ref_lse).max()))
    else:
        assert (np.abs(got - ref) <= 2e-3 + 1e-2 * np.abs(ref)).all()
        assert (np.abs(got_l - ref_lse) <= 2e-3 + 1e-2 * np.abs(ref_lse)).all()
