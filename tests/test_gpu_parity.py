"""CUDA path vs the fp64 oracle, through the C ABI (libhils.so) on a B200.

Every case compares element by element against the oracle on the same seeded inputs: every query
for sizes the oracle finishes in seconds (several tiles and a ragged tail), sampled rows at the
full workload sizes in the benchmark's launch configuration.
"""
import math
import zlib

import numpy as np
import pytest
import torch

import oracle
import parity
from hierarchical_chunk_sparse_scoring_b200 import binding as hb
from hierarchical_chunk_sparse_scoring_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _run(wl, **kw):
    out, lse, idx = hb.forward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, **wl.kwargs(), **kw)
    torch.cuda.synchronize()
    return out, lse, idx


def _free():
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def test_library_loads():
    assert hb.version().startswith("hils-b200")


SMALL_CASES = [
    ("tiny_fp32", {}),                                          # the fp32 correctness workload
    ("small_mha_bf16", dict(B=2, Hq=4, Hkv=4, N=2048)),         # MHA, K=8
    ("gqa7b_prefill", dict(N=4096)),                            # GQA G=4, d=128, K=16
    ("extreme", dict(N=8192)),                                  # G=8, S=128, W=2048
    ("long_decode", dict(B=4, N=16384)),                        # decode, split selection
    ("small_mha_bf16", dict(B=1, Hq=2, Hkv=2, N=1000)),         # ragged tail (partial chunk)
    ("gqa7b_prefill", dict(N=3000, dtype=torch.float32)),       # fp32, GQA, ragged
    ("long_decode", dict(B=2, N=20000, dtype=torch.float32)),   # fp32 decode
]


@pytest.mark.parametrize("name,kw", SMALL_CASES, ids=lambda x: x if isinstance(x, str) else
                         ",".join("%s=%s" % (k, v) for k, v in x.items()))
def test_forward_every_query(name, kw):
    wl = W.make(name, "cuda", **kw)
    out, lse, idx = _run(wl)
    errs = parity.full_check(wl, out, lse, idx)
    assert errs["exact_rows"] + errs["tie_rows"] == idx.shape[0] * idx.shape[1] * idx.shape[2]


def _random_case(B, Hq, Hkv, N, d, S, K, W_, dtype, seed, q_pos0=0, N_q=None, neg_inf=False):
    g = torch.Generator(device="cuda").manual_seed(seed)
    N_q = N - q_pos0 if N_q is None else N_q
    C = N // S
    r = lambda *s: (torch.randn(s, generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    b_lm = torch.rand((B, Hkv, C), generator=g, device="cuda") * 2 - 1
    if neg_inf and C > 2:
        b_lm[..., 1] = -math.inf
        b_lm[..., C // 2] = -math.inf
    return W.Workload("random", r(B, Hq, N_q, d), r(B, Hq, N_q, d), r(B, Hkv, N, d),
                      r(B, Hkv, N, d), r(B, Hkv, C, d), b_lm, S, K, W_, q_pos0)


EDGE_CASES = {
    "k0": dict(B=1, Hq=2, Hkv=1, N=700, d=64, S=64, K=0, W_=128),
    "fewer_chunks_than_k": dict(B=1, Hq=2, Hkv=2, N=600, d=64, S=64, K=16, W_=128),
    "window_covers_all": dict(B=2, Hq=2, Hkv=1, N=300, d=64, S=64, K=4, W_=512),
    "s1": dict(B=1, Hq=2, Hkv=1, N=96, d=32, S=1, K=8, W_=4),
    "w1": dict(B=1, Hq=2, Hkv=2, N=512, d=64, S=16, K=3, W_=1),
    "g3": dict(B=1, Hq=6, Hkv=2, N=1024, d=64, S=32, K=5, W_=100),
    "g16": dict(B=1, Hq=16, Hkv=1, N=1024, d=64, S=64, K=4, W_=128),
    "d96": dict(B=1, Hq=4, Hkv=2, N=777, d=96, S=32, K=6, W_=64),
    "d8": dict(B=1, Hq=2, Hkv=1, N=400, d=8, S=16, K=4, W_=32),
    "k32": dict(B=1, Hq=2, Hkv=1, N=4096, d=64, S=32, K=32, W_=256),
    "k1": dict(B=1, Hq=2, Hkv=1, N=1024, d=64, S=64, K=1, W_=128),
    "neg_inf_bias": dict(B=1, Hq=4, Hkv=2, N=1024, d=64, S=64, K=12, W_=64, neg_inf=True),
    "decode_multi_query": dict(B=3, Hq=8, Hkv=2, N=5000, d=128, S=64, K=8, W_=256,
                               q_pos0=4996, N_q=4),
    "decode_one_query_d64": dict(B=5, Hq=4, Hkv=4, N=9000, d=64, S=64, K=16, W_=512,
                                 q_pos0=8999, N_q=1),
    "decode_short": dict(B=2, Hq=4, Hkv=1, N=100, d=128, S=64, K=4, W_=64, q_pos0=99, N_q=1),
    "decode_k32_g8": dict(B=2, Hq=8, Hkv=1, N=40000, d=128, S=32, K=32, W_=128,
                          q_pos0=39999, N_q=1),
    # decode streaming scorer on the tensor core (bf16): 16 heads per group, and streams whose
    # CTAs cross rows with ragged eligible counts per query
    "decode_g16_d64": dict(B=2, Hq=16, Hkv=1, N=20000, d=64, S=64, K=8, W_=256,
                           q_pos0=19999, N_q=1),
    "decode_multi_query_tiles": dict(B=3, Hq=4, Hkv=2, N=70020, d=128, S=64, K=16, W_=512,
                                     q_pos0=70013, N_q=3),
    # tensor-core selection shapes (bf16): ragged query tiles, every group size, K=32, S=128
    "tc_g2_d128": dict(B=1, Hq=4, Hkv=2, N=3000, d=128, S=64, K=8, W_=128),
    "tc_g8_d64": dict(B=1, Hq=8, Hkv=1, N=2500, d=64, S=32, K=16, W_=64),
    "tc_g1_d128": dict(B=2, Hq=2, Hkv=2, N=5000, d=128, S=64, K=16, W_=256),
    # one head per group with K > 16: the attention's per-row scan of the selection, scores
    # taken from the selection kernel
    "tc_g1_k24": dict(B=1, Hq=2, Hkv=2, N=5000, d=64, S=64, K=24, W_=128),
    "tc_g4_k32": dict(B=1, Hq=8, Hkv=2, N=6000, d=128, S=64, K=32, W_=128),
    "tc_s128": dict(B=1, Hq=4, Hkv=1, N=9000, d=128, S=128, K=16, W_=256),
    "tc_many_tiles": dict(B=1, Hq=4, Hkv=4, N=20000, d=64, S=16, K=8, W_=64),
    # eight heads of 128 dimensions (head-pair scoring), with S = 64 and the extreme shape S = 128
    "tc_g8_d128": dict(B=1, Hq=8, Hkv=1, N=3000, d=128, S=64, K=16, W_=128),
    "tc_g8_d128_s128": dict(B=1, Hq=8, Hkv=1, N=6000, d=128, S=128, K=16, W_=256),
    "tc_g8_d128_k8_b2": dict(B=2, Hq=16, Hkv=2, N=2100, d=128, S=64, K=8, W_=64),
    # decode units of S = 128 tokens on the tensor core (bf16): a ragged last window piece,
    # more selected slots than eligible chunks (empty units), several queries with their own
    # windows, and 16 heads per group
    "decode_s128_window": dict(B=2, Hq=8, Hkv=1, N=9000, d=128, S=128, K=16, W_=300,
                               q_pos0=8999, N_q=1),
    "decode_s128_k_gt_n": dict(B=1, Hq=4, Hkv=1, N=700, d=128, S=128, K=16, W_=256,
                               q_pos0=699, N_q=1),
    "decode_s128_multi": dict(B=2, Hq=16, Hkv=2, N=5000, d=128, S=128, K=8, W_=129,
                              q_pos0=4991, N_q=5),
    "decode_s128_g16": dict(B=1, Hq=16, Hkv=1, N=12345, d=128, S=128, K=12, W_=2048,
                            q_pos0=12344, N_q=1),
    # rows of at least 16384 eligible chunks: the two-level top-K (group maxima), two queries
    "decode_long_rows": dict(B=1, Hq=4, Hkv=1, N=560000, d=64, S=32, K=16, W_=300,
                             q_pos0=559998, N_q=2),
    # the tensor-core units kernel's head bounds (4, 8, 16) at S = 64, with G below its bound
    "decode_s64_g3": dict(B=2, Hq=6, Hkv=2, N=7000, d=128, S=64, K=16, W_=300,
                          q_pos0=6999, N_q=1),
    "decode_s64_g6": dict(B=1, Hq=12, Hkv=2, N=9100, d=128, S=64, K=10, W_=700,
                          q_pos0=9097, N_q=3),
    "decode_s64_g16": dict(B=1, Hq=16, Hkv=1, N=8000, d=128, S=64, K=16, W_=1024,
                           q_pos0=7999, N_q=1),
}


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("case", sorted(EDGE_CASES))
def test_edge_cases(case, dtype):
    wl = _random_case(**EDGE_CASES[case], dtype=dtype, seed=zlib.crc32(case.encode()) % 1000)
    out, lse, idx = _run(wl)
    parity.full_check(wl, out, lse, idx)


def test_empty_inputs_launch_nothing():
    wl = _random_case(B=1, Hq=2, Hkv=1, N=256, d=64, S=64, K=4, W_=64, dtype=torch.bfloat16,
                      seed=3)
    for q_slice in (slice(0, 0),):
        q = wl.q[:, :, q_slice].contiguous()
        out, lse, idx = hb.forward(q, q.clone(), wl.K, wl.V, wl.k_lm, wl.b_lm, S=64, K_top=4, W=64)
        assert out.numel() == 0
    empty = lambda t: t[:0].contiguous()
    out, _, _ = hb.forward(empty(wl.q), empty(wl.q_cal), empty(wl.K), empty(wl.V),
                           empty(wl.k_lm), empty(wl.b_lm), S=64, K_top=4, W=64)
    assert out.shape[0] == 0


def test_selection_is_deterministic():
    wl = W.make("gqa7b_prefill", "cuda", N=4096)
    a = _run(wl)[2].clone()
    b = _run(wl)[2]
    assert torch.equal(a, b)
    dec = W.make("long_decode", "cuda", B=2, N=32768)
    a = _run(dec)[2].clone()
    assert torch.equal(a, _run(dec)[2])


@pytest.mark.parametrize("name,kw", [("gqa7b_prefill", dict(N=4096)),
                                     # landmark-major scoring: per-head scores from its epilogue
                                     ("extreme", dict(N=16384)),
                                     ("small_mha_bf16", dict(B=1, Hq=4, Hkv=4, N=2048)),
                                     ("long_decode", dict(B=3, N=40000)),
                                     ("tiny_fp32", {})])
def test_select_step(name, kw):
    wl = W.make(name, "cuda", **kw)
    d = wl.dims
    idx, s_sel = hb.select(wl.q_cal, wl.k_lm, wl.b_lm, N_kv=d["N_kv"], Hkv=d["Hkv"],
                           **wl.kwargs())
    torch.cuda.synchronize()
    arrs = [parity.f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    kw2 = dict(S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0)
    own = oracle.forward(*arrs, **kw2)
    gidx = idx.cpu().numpy()
    forced = oracle.forward(*arrs, idx_in=gidx, **kw2)
    Kt = wl.K_top
    n = np.array([parity.eligible(wl.q_pos0 + i, wl.S, wl.W) for i in range(d["N_q"])])
    parity.check_selection(gidx.reshape(-1, Kt), own["idx"].reshape(-1, Kt),
                           own["gap"].reshape(-1), forced["sigma"].reshape(-1, Kt),
                           own["sigma"].reshape(-1, Kt), np.tile(n, d["B"] * d["Hkv"]))
    got = s_sel.cpu().double().numpy()
    ref = forced["s_sel"]
    fin = np.isfinite(ref)
    assert (np.isfinite(got) == fin).all()
    tol = 1e-5 if wl.q.dtype == torch.float32 else 1e-4
    assert np.abs(got[fin] - ref[fin]).max(initial=0) <= tol * max(1.0, np.abs(ref[fin]).max())


@pytest.mark.parametrize("name,kw", [("gqa7b_prefill", dict(N=2048)), ("tiny_fp32", {}),
                                     ("long_decode", dict(B=2, N=8192))])
def test_chunk_attn_and_fuse_steps(name, kw):
    wl = W.make(name, "cuda", **kw)
    arrs = [parity.f64(t) for t in (wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm)]
    ref = oracle.forward(*arrs, S=wl.S, K_top=wl.K_top, W=wl.W, q_pos0=wl.q_pos0, units=True)
    idx = torch.from_numpy(ref["idx"]).cuda()
    unit_o, unit_lse = hb.chunk_attn(wl.q, wl.K, wl.V, idx, **wl.kwargs())
    torch.cuda.synchronize()
    valid = np.isfinite(ref["unit_lse"])
    got_l = unit_lse.cpu().double().numpy()
    assert (np.isfinite(got_l) == valid).all()
    tol = 1e-5 if wl.q.dtype == torch.float32 else 1e-4
    assert np.abs(got_l[valid] - ref["unit_lse"][valid]).max() <= tol * 10
    got_o = unit_o.cpu().double().numpy()
    assert np.abs(got_o - ref["unit_o"]).max() <= tol * max(1, np.abs(ref["unit_o"]).max())
    # step 4 alone, fed the oracle's own units and scores
    d = wl.dims
    out, lse = hb.fuse(torch.from_numpy(ref["s_sel"]).float().cuda(),
                       torch.from_numpy(ref["unit_o"]).float().cuda(),
                       torch.from_numpy(ref["unit_lse"]).float().cuda(), Hkv=d["Hkv"],
                       N_kv=d["N_kv"], dtype=wl.q.dtype, **wl.kwargs())
    torch.cuda.synchronize()
    parity.compare_outputs(parity.f64(out), ref["out"], parity.f64(lse), ref["lse"], wl.q.dtype)


def test_device_status_clear_after_forward():
    wl = W.make("gqa7b_prefill", "cuda", N=2048)
    p = hb.params_for(wl.q, wl.K, **wl.kwargs())
    ws = hb.workspace(p, wl.q.device)
    _run(wl, ws=ws)
    assert hb.device_status(ws) == 0


def test_bounded_wait_gives_up_and_reports():
    # the bounded mbarrier wait of the tensor-core kernels: a phase that nothing completes makes
    # the wait give up after its poll limit, record HILS_ERR_TIMEOUT and let the kernel return;
    # a completed phase records nothing; the context stays usable either way
    wl = W.make("gqa7b_prefill", "cuda", N=2048)
    p = hb.params_for(wl.q, wl.K, **wl.kwargs())
    ws = hb.workspace(p, wl.q.device)
    assert hb.device_status(ws) == 0
    hb.wait_check(1000, True, ws)
    assert hb.device_status(ws) == 0
    hb.wait_check(1000, False, ws)
    assert hb.device_status(ws) == 6
    assert hb.device_status(ws) == 0          # reading cleared it
    out, lse, idx = _run(wl, ws=ws)           # and the next forward runs normally
    parity.full_check(wl, out, lse, idx)
    assert hb.device_status(ws) == 0


def test_invalid_arguments_raise_before_launch():
    wl = W.make("gqa7b_prefill", "cuda", N=2048)
    with pytest.raises(hb.HilsError) as e:
        hb.forward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, S=64, K_top=33, W=1024)
    assert e.value.status == 2
    with pytest.raises(hb.HilsError) as e:
        hb.forward(wl.q, wl.q_cal, wl.K, wl.V, wl.k_lm, wl.b_lm, S=64, K_top=16, W=0)
    assert e.value.status == 1


# ------------------------------------------------------------------- full workload sizes
FULL = [("small_mha_bf16", 2048, {}), ("gqa7b_prefill", 512, {}), ("long_decode", 64, {}),
        ("extreme", 256, {}), ("extreme", 256, dict(N=1 << 20)), ("extreme", 256, dict(N=1 << 22)),
        # four heads per group over 8192 chunks: the landmark-major scoring kernel at G = 4
        ("gqa7b_prefill", 256, dict(N=1 << 19))]


@pytest.mark.parametrize("name,rows,kw", FULL,
                         ids=lambda x: x if isinstance(x, str) else (
                             "N=%d" % x["N"] if isinstance(x, dict) and "N" in x else
                             ("full" if isinstance(x, dict) else str(x))))
def test_full_size_sampled(name, rows, kw):
    wl = W.make(name, "cuda", **kw)
    out, lse, idx = _run(wl)
    sample = parity.sample_rows(wl, rows, seed=7)
    errs = parity.sampled_check(wl, out, lse, idx, sample)
    assert errs["rows"] >= rows
    _every_row_properties(wl, out, lse, idx)
    if name == "extreme":
        # the decode step of the sequence's last query (the extreme sweep's decode point)
        del out, lse, idx
        _free()
        dec = W.decode_view(wl)
        out, lse, idx = _run(dec)
        parity.sampled_check(dec, out, lse, idx, [(0, 0, 0)])
        _every_row_properties(dec, out, lse, idx)
    del wl, out, lse, idx
    _free()


def _every_row_properties(wl, out, lse, idx):
    """Properties that hold at any size, on every row."""
    Kt = wl.K_top
    pos = torch.arange(wl.q.shape[2], device="cuda", dtype=torch.int64) + wl.q_pos0
    first = pos - wl.W + 1
    n = torch.where(first > 0, torch.div(first, wl.S, rounding_mode="floor"),
                    torch.zeros_like(first))
    k = torch.clamp(n, max=Kt)
    valid = idx >= 0
    assert torch.equal(valid.sum(-1), k.expand_as(valid.sum(-1)).to(valid.sum(-1).dtype))
    assert bool((idx < n[None, None, :, None]).all())
    srt = torch.sort(idx, dim=-1).values
    dup = (srt[..., 1:] == srt[..., :-1]) & (srt[..., 1:] >= 0)
    assert not bool(dup.any())
    assert bool(torch.isfinite(out.float()).all()) and bool(torch.isfinite(lse).all())
