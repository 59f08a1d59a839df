"""The C ABI without a GPU: the library loads, exports every function include/hils.h declares,
the header is plain C, and host-side argument checks answer before anything touches a device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from hierarchical_chunk_sparse_scoring_b200 import binding as hb
from hierarchical_chunk_sparse_scoring_b200 import build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hils.h")


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return hb.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hils_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ("hils_forward", "hils_select", "hils_chunk_attn", "hils_fuse",
                 "hils_workspace_size"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", hb.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(hils_\w+)", out))
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    assert set(hb.SIGNATURES) == set(_declared())


def test_header_is_plain_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "hils.h"\nint main(void){hils_params p={0};(void)p;return 0;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-fsyntax-only", "-I",
                    os.path.dirname(HEADER), str(src)], check=True)


def _params(**kw):
    base = dict(B=1, Hq=8, Hkv=2, N_q=4096, N_kv=4096, d=128, S=64, K_top=16, W=1024)
    base.update(kw)
    B, Hq, Hkv, N_q, N_kv, d = (base.pop(k) for k in ("B", "Hq", "Hkv", "N_q", "N_kv", "d"))
    return hb.make_params(B, Hq, Hkv, N_q, N_kv, d, **base)


def test_workspace_size(lib):
    p = _params()
    ws = hb.workspace_size(p)
    assert ws >= 256 and ws % 256 == 0
    assert hb.workspace_size(_params(N_q=8192, N_kv=8192)) > ws
    dec = hb.workspace_size(_params(N_q=1, N_kv=524288, q_pos0=524287))
    assert dec > 256
    assert hb.workspace_size(_params(K_top=33)) == 0      # unsupported -> 0
    assert hb.workspace_size(_params(Hq=6, Hkv=4)) == 0   # Hq % Hkv != 0


def test_decode_group_maxima_region(lib):
    # rows of 1024 eligible chunks or more on the tensor-core streaming scorer (bf16) get the
    # two-level top-K's group maxima (4 per 128-chunk tile, one aligned region); fp32 decode
    # streams on the CUDA cores and has none.  n = 1023 and 1024 share every other region
    # (same sigma row stride, same 1024-token window).
    def dec(n, dtype=torch.bfloat16):
        pos = n * 64 + 1024 - 1
        return hb.workspace_size(_params(B=1, Hq=8, Hkv=2, N_q=1, N_kv=pos + 1, q_pos0=pos,
                                         dtype=dtype))
    rows, g_stride = 1 * 2 * 1, (1024 + 127) // 128 * 4
    region = (rows * g_stride * 4 + 255) // 256 * 256
    assert dec(1024) - dec(1023) == region
    assert dec(1024, torch.float32) == dec(1023, torch.float32)


def test_prefill_workspace_layout(lib):
    # status word, then idx [B, Hkv, N_q, K]; per-head scores [B, Hq, N_q, K] only where the
    # tensor-core attention does not score the selected chunks itself: one head per KV group
    # (it takes the scoring kernel's sigma of the winners), the d = 128, K <= 16 attention that
    # runs two CTAs per SM (it takes every head's scores from the selection step), or no
    # tensor-core path (fp32)
    def rup(x):
        return (x + 255) // 256 * 256
    nq, k = 4096, 16
    gqa = hb.workspace_size(_params(Hq=8, Hkv=2, N_q=nq, N_kv=nq, K_top=k))
    assert gqa == 256 + rup(2 * nq * k * 4) + rup(8 * nq * k * 4)
    # (K = 32 at d = 128: the attention CTA scores the selected chunks per head itself)
    gqa32 = hb.workspace_size(_params(Hq=8, Hkv=2, N_q=nq, N_kv=nq, K_top=32))
    assert gqa32 == 256 + rup(2 * nq * 32 * 4)
    gqa64 = hb.workspace_size(_params(Hq=8, Hkv=2, N_q=nq, N_kv=nq, K_top=k, d=64))
    assert gqa64 == 256 + rup(2 * nq * k * 4)
    mha = hb.workspace_size(_params(Hq=8, Hkv=8, N_q=nq, N_kv=nq, K_top=k))
    assert mha == 256 + rup(8 * nq * k * 4) + rup(8 * nq * k * 4)
    f32 = hb.workspace_size(_params(Hq=8, Hkv=2, N_q=nq, N_kv=nq, K_top=k, dtype=torch.float32))
    assert f32 == 256 + rup(2 * nq * k * 4) + rup(8 * nq * k * 4)
    # rows beyond 32-bit TMA coordinates (B * Hkv * N_kv >= 2^31): the CUDA-core kernels, which
    # take the per-head scores from the workspace
    big = 1 << 28
    ws = hb.workspace_size(_params(Hq=32, Hkv=8, N_q=big, N_kv=big, K_top=k))
    assert ws == 256 + rup(8 * big * k * 4) + rup(32 * big * k * 4)


BAD = [
    (dict(K_top=33), 2), (dict(d=130), 2), (dict(d=6), 2), (dict(Hq=64, Hkv=2), 2),
    (dict(Hq=6, Hkv=4), 1), (dict(W=0), 1), (dict(S=0), 1), (dict(K_top=-1), 1),
    (dict(N_q=10, N_kv=8, q_pos0=0), 1), (dict(N_q=1, N_kv=100, q_pos0=100), 1),
    (dict(B=-1), 1), (dict(Hkv=0), 1),
]


@pytest.mark.parametrize("kw,status", BAD, ids=[str(b[0]) for b in BAD])
def test_bad_params_rejected_on_host(lib, kw, status):
    p = _params(**kw)
    dummy = ctypes.c_void_p(4096)
    args = [ctypes.byref(p)] + [dummy] * 6 + [dummy, None, None, dummy, 1 << 40, None]
    assert lib.hils_forward(*args) == status
    assert lib.hils_select(ctypes.byref(p), dummy, dummy, dummy, dummy, None, dummy, 1 << 40,
                           None) == status


def test_null_and_misaligned_pointers_rejected(lib):
    p = _params()
    ok = ctypes.c_void_p(4096)
    big = 1 << 40
    assert lib.hils_forward(ctypes.byref(p), None, ok, ok, ok, ok, ok, ok, None, None, ok, big,
                            None) == 1
    assert lib.hils_forward(ctypes.byref(p), ctypes.c_void_p(4100), ok, ok, ok, ok, ok, ok, None,
                            None, ok, big, None) == 1
    assert lib.hils_forward(ctypes.byref(p), ok, ok, ok, ok, ok, ok, ok, None, None, ok, 100,
                            None) == 3
    assert lib.hils_forward(ctypes.byref(p), ok, ok, ok, ok, ok, ok, ok, None, None, None, big,
                            None) == 3
    assert lib.hils_chunk_attn(ctypes.byref(p), ok, ok, ok, None, ok, ok, None) == 1
    assert lib.hils_fuse(ctypes.byref(p), ok, ok, ok, None, None, None) == 1


def test_empty_problem_is_a_no_op_without_device(lib):
    p = _params(N_q=0)
    ws = ctypes.c_void_p(4096)
    assert lib.hils_forward(ctypes.byref(p), None, None, None, None, None, None, None, None,
                            None, ws, 1 << 20, None) == 0


def test_status_strings(lib):
    for code in range(7):
        assert lib.hils_status_string(code).decode() == hb.STATUS[code]
    assert hb.version().startswith("hils-b200")
