"""hils_select_noalloc: the allocation-free variant of steps 1-2.

Some callers cannot give the library a workspace (a plugin host that passes only input and
output tensors, or a serving loop whose device memory is planned ahead so cudaMalloc is off the
request path).  This entry point uses a fixed scratch array inside the library instead; these
tests call it through the C ABI and compare it with hils_select on the same inputs, twice in a
row (the scratch keeps the previous call's contents, so the second call checks that nothing
stale leaks through), read its status word, and check the decode path's split lists on the
cases where their padding matters (fewer eligible chunks than K, -inf biases, exact ties).
The file is collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from hierarchical_chunk_sparse_scoring_b200 import binding as hb
from hierarchical_chunk_sparse_scoring_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _noalloc(wl):
    B, Hq, N_q, d = wl.q_cal.shape
    Hkv, N_kv = wl.K.shape[1], wl.K.shape[2]
    p = hb.make_params(B, Hq, Hkv, N_q, N_kv, d, dtype=wl.q_cal.dtype, **wl.kwargs())
    idx = torch.full((B, Hkv, N_q, wl.K_top), -7, dtype=torch.int32, device="cuda")
    s_sel = torch.full((B, Hq, N_q, wl.K_top), 123.0, dtype=torch.float32, device="cuda")
    st = hb.lib().hils_select_noalloc(ctypes.byref(p), hb._ptr(wl.q_cal), hb._ptr(wl.k_lm),
                                      hb._ptr(wl.b_lm), hb._ptr(idx), hb._ptr(s_sel),
                                      hb._stream(None))
    torch.cuda.synchronize()
    return st, idx, s_sel


def _compare(wl, ref_idx, ref_s):
    for _ in range(2):
        st, idx, s_sel = _noalloc(wl)
        assert st == 0, hb.STATUS.get(st)
        assert hb.select_noalloc_status() == 0
        assert torch.equal(idx, ref_idx)
        fin = torch.isfinite(ref_s)
        assert torch.equal(torch.isfinite(s_sel), fin)
        tol = 1e-5 if wl.q.dtype == torch.float32 else 1e-4
        if bool(fin.any()):
            assert float((s_sel[fin] - ref_s[fin]).abs().max()) <= tol * max(
                1.0, float(ref_s[fin].abs().max()))


@pytest.mark.parametrize("name,kw", [("long_decode", dict(B=4, N=65536)),      # split lists
                                     ("gqa7b_prefill", dict(N=2048)),           # tensor cores
                                     ("tiny_fp32", {})])                        # CUDA cores
def test_noalloc_select_matches_select(name, kw):
    wl = W.make(name, "cuda", **kw)
    d = wl.dims
    ref_idx, ref_s = hb.select(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"], Hkv=d["Hkv"],
                               **wl.kwargs())
    torch.cuda.synchronize()
    _compare(wl, ref_idx, ref_s)


def _decode_case(B, Hq, Hkv, N, d, S, K, W_, dtype, seed, mode):
    g = torch.Generator(device="cuda").manual_seed(seed)
    C = N // S
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    k_lm = r(B, Hkv, C, d)
    b_lm = torch.rand((B, Hkv, C), generator=g, device="cuda") * 2 - 1
    if mode == "neg_inf":
        b_lm[..., ::3] = -math.inf
    elif mode == "ties":
        # landmark keys 0 and integer biases: every score is exactly its bias in any precision,
        # so hundreds of chunks tie and only the lower-index rule decides
        k_lm = torch.zeros_like(k_lm)
        b_lm = torch.randint(0, 2, (B, Hkv, C), generator=g, device="cuda").float()
    q_cal = r(B, Hq, 1, d)
    return W.Workload("decode_" + mode, q_cal, q_cal, r(B, Hkv, N, d), r(B, Hkv, N, d), k_lm,
                      b_lm, S, K, W_, N - 1)


@pytest.mark.parametrize("mode,N,K", [("fewer_than_k", 64 * 20 + 300, 32),
                                      ("neg_inf", 40000, 16), ("ties", 70000, 16)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_noalloc_decode_split_lists(mode, N, K, dtype):
    wl = _decode_case(B=3, Hq=8, Hkv=2, N=N, d=128, S=64, K=K, W_=256, dtype=dtype,
                      seed=17 + N, mode=mode)
    d = wl.dims
    ref_idx, ref_s = hb.select(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"], Hkv=d["Hkv"],
                               **wl.kwargs())
    torch.cuda.synchronize()
    _compare(wl, ref_idx, ref_s)
    # and the oracle's own ordered selection, exactly, wherever the rank-K gap is clear or the
    # scores tie exactly by construction
    arrs = [parity.f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    own = oracle.forward(*arrs, S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0)
    got = ref_idx.cpu().numpy().reshape(-1, K)
    want = own["idx"].reshape(-1, K)
    gap = own["gap"].reshape(-1)
    for r in range(got.shape[0]):
        if mode == "ties" or gap[r] > parity.GAP:
            assert np.array_equal(got[r], want[r]), (r, got[r], want[r])


def test_noalloc_rejects_oversize_scratch():
    # 4096 decode rows x 1024 splits x 32 ids x 8 bytes is far beyond the fixed scratch; the
    # pointers are real (small) device buffers, so a check that ran after a launch could only
    # misreport, never touch memory it does not own
    p = hb.make_params(64, 64, 64, 1, 1 << 25, 64, S=64, K_top=32, W=64, q_pos0=(1 << 25) - 1)
    buf = torch.zeros(1024, dtype=torch.float32, device="cuda")
    idx = torch.zeros(1024, dtype=torch.int32, device="cuda")
    assert hb.lib().hils_select_noalloc(ctypes.byref(p), hb._ptr(buf), hb._ptr(buf),
                                        hb._ptr(buf), hb._ptr(idx), None, None) == 3
    assert hb.lib().hils_select_noalloc_max_bytes() == 8 << 20
    torch.cuda.synchronize()
    assert bool((buf == 0).all()) and bool((idx == 0).all())
