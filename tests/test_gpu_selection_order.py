"""The selection's tie rule and order on the GPU, on every selection kernel.

The top-K keeps the K largest group scores sigma with ties to the lower chunk index, and lists
them by (sigma descending, chunk ascending) ([Reader] "Limitations of Naive Sparse Attention":
top-K distant chunks; the lower-index tie-break is the reading this build fixes for ties).
Random inputs almost never tie, so the ties are built in, in two ways that make the scores
equal in every precision:

* int_bias: landmark keys 0 and integer biases.  Every score is exactly its bias (q_cal . 0 = 0
  in fp32 and fp64), so hundreds of chunks share each value and only the index rule decides.
  The GPU's ordered idx must equal the oracle's exactly, on every row (the decode cases also
  have far more than 64 tied survivors per row).
* dup_rows: pairs of chunks (2j, 2j+1) with identical landmark rows and biases.  The two scores
  of a pair are computed by identical arithmetic, so wherever the odd chunk is selected the even
  one must be too, and listed just before it.

Each case runs through the entry point whose kernels it names (forward, hils_select, and the
allocation-free hils_select_noalloc for decode).
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

# name -> (shape, dtype, kernels exercised)
CASES = {
    "tc_g1_d64_k8": (dict(B=1, Hq=2, Hkv=2, N=5000, d=64, S=64, K=8, W_=128),
                     torch.bfloat16, "score_topk_tc, two CTAs per SM"),
    "tc_g1_d128_k16": (dict(B=1, Hq=2, Hkv=2, N=5000, d=128, S=64, K=16, W_=256),
                       torch.bfloat16, "score_topk_tc"),
    "tc_g2_d64_k32": (dict(B=1, Hq=4, Hkv=2, N=4000, d=64, S=32, K=32, W_=128),
                      torch.bfloat16, "score_topk_tc, 32-slot lists"),
    "tc_g4_d128": (dict(B=1, Hq=8, Hkv=2, N=20000, d=128, S=64, K=16, W_=128),
                   torch.bfloat16, "score_topk_t_tc (two merge warps) with per-head scores "
                   "for the two-CTA attention"),
    "tc_g4_d64": (dict(B=1, Hq=8, Hkv=2, N=20000, d=64, S=64, K=16, W_=128),
                  torch.bfloat16, "score_topk_tc, four heads over fewer than 8192 chunks"),
    "tc_g8_d128_s128": (dict(B=1, Hq=8, Hkv=1, N=40000, d=128, S=128, K=16, W_=256),
                        torch.bfloat16, "score_topk_t_tc (landmark-major), eight heads"),
    "tc_g8_d64_k32": (dict(B=1, Hq=8, Hkv=1, N=20000, d=64, S=32, K=32, W_=128),
                      torch.bfloat16, "score_topk_t_tc, 32-slot lists, d = 64"),
    "rows_fp32": (dict(B=1, Hq=4, Hkv=2, N=3000, d=64, S=32, K=8, W_=96),
                  torch.float32, "select_rows"),
    "rows_g16": (dict(B=1, Hq=16, Hkv=1, N=2000, d=64, S=32, K=8, W_=64),
                 torch.bfloat16, "select_rows"),
    "decode_tc_d128": (dict(B=3, Hq=8, Hkv=2, N=70000, d=128, S=64, K=16, W_=512, q_pos0=69999,
                            N_q=1), torch.bfloat16, "select_stream_tc, select_topk"),
    "decode_d64_g16": (dict(B=2, Hq=16, Hkv=1, N=30000, d=64, S=64, K=32, W_=256, q_pos0=29999,
                            N_q=1), torch.bfloat16, "select_stream_tc, select_topk"),
    "decode_fp32": (dict(B=2, Hq=4, Hkv=2, N=50000, d=128, S=64, K=16, W_=512, q_pos0=49999,
                         N_q=1), torch.float32, "select_stream, select_topk"),
    # one row over 4,680 chunks (one top-K CTA for the whole row)
    "decode_one_row": (dict(B=1, Hq=8, Hkv=1, N=300000, d=128, S=64, K=16, W_=512,
                            q_pos0=299999, N_q=1), torch.bfloat16, "select_stream_tc, select_topk"),
    # one row over 18,734 chunks: the two-level top-K over the streaming scorer's group maxima
    "decode_long_row": (dict(B=1, Hq=8, Hkv=1, N=600000, d=64, S=32, K=16, W_=512,
                             q_pos0=599999, N_q=1), torch.bfloat16,
                        "select_stream_tc with group maxima, two-level select_topk"),
    "decode_multi_query": (dict(B=2, Hq=4, Hkv=2, N=9000, d=128, S=64, K=8, W_=256,
                                q_pos0=8996, N_q=4), torch.bfloat16,
                           "select_stream_tc, select_topk"),
}


def _case(B, Hq, Hkv, N, d, S, K, W_, dtype, seed, mode, q_pos0=0, N_q=None):
    g = torch.Generator(device="cuda").manual_seed(seed)
    N_q = N - q_pos0 if N_q is None else N_q
    C = N // S
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    q, q_cal = r(B, Hq, N_q, d), r(B, Hq, N_q, d)
    if mode == "int_bias":
        k_lm = torch.zeros((B, Hkv, C, d), dtype=dtype, device="cuda")
        b_lm = torch.randint(-1, 2, (B, Hkv, C), generator=g, device="cuda").float()
    else:
        k_lm = r(B, Hkv, C, d)
        b_lm = torch.rand((B, Hkv, C), generator=g, device="cuda") * 2 - 1
        even = torch.arange(0, C - C % 2, 2, device="cuda")
        k_lm[:, :, even + 1] = k_lm[:, :, even]
        b_lm[:, :, even + 1] = b_lm[:, :, even]
    return W.Workload("ties_" + mode, q, q_cal, r(B, Hkv, N, d), r(B, Hkv, N, d), k_lm, b_lm,
                      S, K, W_, q_pos0)


def _selections(wl, decode):
    d = wl.dims
    out, lse, idx_f = hb.forward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, **wl.kwargs())
    idx_s, s_sel = hb.select(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"], Hkv=d["Hkv"],
                             **wl.kwargs())
    sels = {"forward": idx_f, "select": idx_s}
    if decode:
        sels["select_noalloc"] = hb.select_noalloc(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"],
                                                   Hkv=d["Hkv"], **wl.kwargs())[0]
    torch.cuda.synchronize()
    return out, lse, sels


@pytest.mark.parametrize("mode", ["int_bias", "dup_rows"])
@pytest.mark.parametrize("case", sorted(CASES))
def test_tie_rule_and_order(case, mode):
    shape, dtype, _ = CASES[case]
    wl = _case(**shape, dtype=dtype, seed=len(case) * 31 + (mode == "dup_rows"), mode=mode)
    decode = "N_q" in shape
    out, lse, sels = _selections(wl, decode)
    arrs = [parity.f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    kw = dict(S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0)
    own = oracle.forward(*arrs, **kw)
    K = wl.K_top
    want = own["idx"].reshape(-1, K)
    Nq = wl.q.shape[2]
    n = np.tile(np.array([parity.eligible(wl.q_pos0 + i, wl.S, wl.W) for i in range(Nq)]),
                wl.q.shape[0] * wl.K.shape[1])
    for name, idx in sels.items():
        got = idx.cpu().numpy().reshape(-1, K)
        if mode == "int_bias":
            bad = [r for r in range(got.shape[0]) if not np.array_equal(got[r], want[r])]
            assert not bad, (name, bad[:3], got[bad[0]], want[bad[0]])
        else:
            for r in range(got.shape[0]):
                row = got[r].tolist()
                for k, c in enumerate(row):
                    if c >= 0 and c % 2 == 1:
                        assert c - 1 in row, (name, r, "odd chunk kept without its twin", row)
                        assert row.index(c - 1) == k - 1, (name, r, "twins not adjacent", row)
            forced = oracle.forward(*arrs, idx_in=idx.cpu().numpy(), **kw)
            parity.check_selection(got, want, own["gap"].reshape(-1),
                                   forced["sigma"].reshape(-1, K), own["sigma"].reshape(-1, K), n)
    # the forward's outputs on its own selection
    forced = oracle.forward(*arrs, idx_in=sels["forward"].cpu().numpy(), **kw)
    parity.compare_outputs(parity.f64(out), forced["out"], parity.f64(lse), forced["lse"],
                           wl.q.dtype)
