"""Incremental decode (hils_decode_step) against the fp64 oracle, through the C ABI.

A cache of fixed capacity is filled one token per call: each call appends the token's key and
value, builds the landmark of the chunk the token completes ([Reader] "The HiLS-Attention
Mechanism": chunk summary and entropy bias from the chunk's landmark query) and runs the forward
for the token's query over the prefix ([Reader] Fig. 6 caption: per-token decode).  Checked
along the way: the cache rows are the appended tokens bit for bit, every emitted landmark matches
the oracle's landmark construction, and every checked step's selection and outputs match the
oracle's forward on the prefix (same rules and tolerances as the other parity tests).  A step is
also captured in a CUDA graph and replayed.
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


def _tokens(B, Hq, Hkv, d, S, T, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    return dict(k=r(B, Hkv, T, d), v=r(B, Hkv, T, d), q=r(B, Hq, T, d), qc=r(B, Hq, T, d),
                qlm=r(B, Hkv, T // S + 1, d))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_incremental_decode_matches_oracle(dtype, d):
    B, Hq, Hkv, S, Wn, Kt, cap, T = 2, 4, 2, 16, 48, 4, 512, 300
    tk = _tokens(B, Hq, Hkv, d, S, T, dtype, seed=11 + d)
    Kc = torch.zeros((B, Hkv, cap, d), dtype=dtype, device="cuda")
    Vc = torch.zeros_like(Kc)
    k_lm = torch.zeros((B, Hkv, cap // S, d), dtype=dtype, device="cuda")
    b_lm = torch.zeros((B, Hkv, cap // S), dtype=torch.float32, device="cuda")
    checked = 0
    for pos in range(T):
        completes = (pos + 1) % S == 0
        q = tk["q"][:, :, pos:pos + 1].contiguous()
        qc = tk["qc"][:, :, pos:pos + 1].contiguous()
        out, lse, idx = hb.decode_step(
            q, qc, tk["k"][:, :, pos].contiguous(), tk["v"][:, :, pos].contiguous(),
            tk["qlm"][:, :, pos // S].contiguous() if completes else None, Kc, Vc, k_lm, b_lm,
            pos=pos, S=S, K_top=Kt, W=Wn)
        if not (completes or pos % 5 == 0 or pos == T - 1):
            continue
        torch.cuda.synchronize()
        checked += 1
        L = pos + 1
        assert torch.equal(Kc[:, :, :L], tk["k"][:, :, :L])
        assert torch.equal(Vc[:, :, :L], tk["v"][:, :, :L])
        C = L // S
        if C > 0:
            ref_k, ref_b = oracle.landmarks(parity.f64(tk["qlm"][:, :, :C]),
                                            parity.f64(tk["k"][:, :, :C * S]), S=S)
            got_k, got_b = parity.f64(k_lm[:, :, :C]), parity.f64(b_lm[:, :, :C])
            if dtype == torch.float32:
                row = np.abs(got_k - ref_k).max(-1) / np.abs(ref_k).max(-1)
                assert float(row.max()) <= 1e-5
                assert (np.abs(got_b - ref_b) <= 1e-5 * np.maximum(1.0, np.abs(ref_b))).all()
            else:
                assert (np.abs(got_k - ref_k) <= 2e-3 + 1e-2 * np.abs(ref_k)).all()
                assert (np.abs(got_b - ref_b) <= 2e-3 + 1e-2 * np.abs(ref_b)).all()
        # the forward over the prefix, with the landmarks the steps built
        wl = W.Workload("decode_step", q, qc, Kc[:, :, :L], Vc[:, :, :L], k_lm[:, :, :C],
                        b_lm[:, :, :C], S, Kt, Wn, pos)
        parity.full_check(wl, out, lse, idx)
    assert checked >= 60


def test_decode_step_in_a_cuda_graph():
    B, Hq, Hkv, d, S, Wn, Kt, cap = 2, 8, 2, 128, 64, 256, 8, 8192
    pos = 64 * 100 - 1   # completes chunk 99
    g = torch.Generator(device="cuda").manual_seed(5)
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(torch.bfloat16)
    Kc, Vc = r(B, Hkv, cap, d), r(B, Hkv, cap, d)
    k_lm = r(B, Hkv, cap // S, d)
    b_lm = torch.rand((B, Hkv, cap // S), generator=g, device="cuda") * 2 - 1
    q, qc = r(B, Hq, 1, d), r(B, Hq, 1, d)
    kn, vn, qlm = r(B, Hkv, d), r(B, Hkv, d), r(B, Hkv, d)
    p = hb.make_params(B, Hq, Hkv, 1, cap, d, S=S, K_top=Kt, W=Wn, q_pos0=pos)
    ws = hb.workspace(p, q.device)
    out0, lse0, idx0 = hb.decode_step(q, qc, kn, vn, qlm, Kc, Vc, k_lm, b_lm, pos=pos, S=S,
                                      K_top=Kt, W=Wn, ws=ws)
    torch.cuda.synchronize()
    ref = (out0.clone(), lse0.clone(), idx0.clone(), k_lm.clone(), b_lm.clone())
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    out, lse, idx = torch.empty_like(out0), torch.empty_like(lse0), torch.empty_like(idx0)
    with torch.cuda.stream(s):
        wsg = hb.workspace(p, q.device, stream=s)
        hb.decode_step(q, qc, kn, vn, qlm, Kc, Vc, k_lm, b_lm, pos=pos, S=S, K_top=Kt, W=Wn,
                       out=out, lse=lse, idx=idx, ws=wsg, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        hb.decode_step(q, qc, kn, vn, qlm, Kc, Vc, k_lm, b_lm, pos=pos, S=S, K_top=Kt, W=Wn,
                       out=out, lse=lse, idx=idx, ws=wsg, stream=s)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(idx, ref[2])
        assert torch.equal(out, ref[0]) and torch.equal(lse, ref[1])
        assert torch.equal(k_lm, ref[3]) and torch.equal(b_lm, ref[4])
    del graph
