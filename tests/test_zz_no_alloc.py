"""hils_select_noalloc: the allocation-free variant of steps 1-2.

Some callers cannot give the library a workspace (a plugin host that passes only input and
output tensors, or a serving loop whose device memory is planned ahead so cudaMalloc is off the
request path).  This entry point uses a fixed scratch array inside the library instead; these
tests call it through the C ABI and compare it with hils_select on the same inputs, twice in a
row (the scratch keeps the previous call's contents, so the second call checks that nothing
stale leaks through).  The file is collected last on purpose.
"""
import ctypes

import pytest
import torch

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


@pytest.mark.parametrize("name,kw", [("long_decode", dict(B=4, N=65536)),      # split lists
                                     ("gqa7b_prefill", dict(N=2048)),           # tensor cores
                                     ("tiny_fp32", {})])                        # CUDA cores
def test_noalloc_select_matches_select(name, kw):
    wl = W.make(name, "cuda", **kw)
    d = wl.dims
    ref_idx, ref_s = hb.select(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"], Hkv=d["Hkv"],
                               **wl.kwargs())
    torch.cuda.synchronize()
    for _ in range(2):
        st, idx, s_sel = _noalloc(wl)
        assert st == 0, hb.STATUS.get(st)
        assert torch.equal(idx, ref_idx)
        fin = torch.isfinite(ref_s)
        assert torch.equal(torch.isfinite(s_sel), fin)
        tol = 1e-5 if wl.q.dtype == torch.float32 else 1e-4
        assert float((s_sel[fin] - ref_s[fin]).abs().max()) <= tol * max(
            1.0, float(ref_s[fin].abs().max()))


def test_noalloc_rejects_oversize_scratch():
    # 4096 decode rows x 1024 splits x 32 ids x 8 bytes is far beyond the fixed scratch
    p = hb.make_params(64, 64, 64, 1, 1 << 25, 64, S=64, K_top=32, W=64, q_pos0=(1 << 25) - 1)
    dummy = ctypes.c_void_p(4096)
    assert hb.lib().hils_select_noalloc(ctypes.byref(p), dummy, dummy, dummy, dummy, None,
                                        None) == 3
    assert hb.lib().hils_select_noalloc_max_bytes() == 8 << 20
