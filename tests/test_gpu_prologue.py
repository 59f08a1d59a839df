"""Query prologue (hils_qcal_hope, hils_hope_rotate) against the fp64 oracle, through the C ABI.

q_out = HoPE(q) and q_cal = HoPE(q + W_up (W_down hidden)); keys HoPE(K) at their positions
([Reader] "Implementation and Training Recipes": Q-Cal and HoPE; reading R17 of the oracle).

Tolerance.  The down-projection multiplies bf16 operands exactly and accumulates in fp32 over
d_model terms; the correction, the sum and the rotation are fp32, with the angle reduced modulo
2 pi in fp64 first (so positions up to 2^22 lose nothing there).  fp32 outputs: per row
max |x - ref| <= 1e-5 max |ref| (fp32 sums of up to 4096 products and a few rounding steps).
bf16 outputs add one rounding to bf16 (half an ulp, 2^-9 relative): |x - ref| <= 2^-8 |ref| +
1e-4 max_row |ref|.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from hierarchical_chunk_sparse_scoring_b200 import binding as hb

pytestmark = pytest.mark.gpu


def _inputs(B, Hq, N_q, d, d_model, r, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = (torch.randn((B, Hq, N_q, d), generator=g, device="cuda") / math.sqrt(d)).to(dtype)
    hidden = torch.randn((B, N_q, d_model), generator=g, device="cuda").to(torch.bfloat16)
    W_down = (torch.randn((Hq, r, d_model), generator=g, device="cuda") /
              math.sqrt(d_model)).to(torch.bfloat16)
    W_up = (0.1 * torch.randn((Hq, d, r), generator=g, device="cuda") /
            math.sqrt(max(r, 1))).to(dtype)
    return q, hidden, W_down, W_up


def _check(got, ref, dtype):
    got = parity.f64(got)
    assert np.isfinite(got).all()
    rowmax = np.abs(ref).max(-1, keepdims=True)
    if dtype == torch.float32:
        assert (np.abs(got - ref) <= 1e-5 * rowmax).all(), float(np.abs(got - ref).max())
    else:
        assert (np.abs(got - ref) <= 2 ** -8 * np.abs(ref) + 1e-4 * rowmax).all(), float(
            np.abs(got - ref).max())


CASES = {
    # name: (B, Hq, N_q, d, d_model, r, q_pos0, base, train_len, dtype)
    "bf16_d128_r16": (1, 8, 300, 128, 512, 16, 1000, 10000.0, 8192.0, torch.bfloat16),
    "bf16_n512_dm4096": (1, 32, 1000, 128, 4096, 16, 0, 10000.0, 32768.0, torch.bfloat16),
    # tensor-core up-projection: two sequences, r = 32 (two k steps), a ragged token block
    "bf16_b2_r32": (2, 4, 200, 128, 256, 32, 50, 10000.0, 8192.0, torch.bfloat16),
    "fp32_d64_r16": (2, 4, 77, 64, 128, 16, 5, 10000.0, 4096.0, torch.float32),
    "fp32_d128_r8_far": (1, 8, 200, 128, 256, 8, (1 << 22) - 200, 500000.0, 1e7,
                         torch.float32),
    "bf16_r0_rope_all": (2, 2, 50, 64, 64, 0, 17, 10000.0, 1e30, torch.bfloat16),
    "fp32_r64_nope": (1, 2, 130, 128, 192, 64, 0, 10000.0, 0.0, torch.float32),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_qcal_hope_matches_oracle(case):
    B, Hq, N_q, d, dm, r, pos0, base, L, dtype = CASES[case]
    q, hidden, W_down, W_up = _inputs(B, Hq, N_q, d, dm, r, dtype, seed=len(case))
    if r == 0:
        q_out, q_cal = hb.qcal_hope(q, None, None, None, rope_base=base, train_len=L, q_pos0=pos0)
        ref_q = oracle.hope_rotate(parity.f64(q), base=base, train_len=L, pos0=pos0)
        ref_c = ref_q
    else:
        q_out, q_cal = hb.qcal_hope(q, hidden, W_down, W_up, rope_base=base, train_len=L,
                                    q_pos0=pos0)
        ref_q, ref_c = oracle.qcal_hope(parity.f64(q), parity.f64(hidden), parity.f64(W_down),
                                        parity.f64(W_up), base=base, train_len=L, pos0=pos0)
    torch.cuda.synchronize()
    _check(q_out, ref_q, dtype)
    _check(q_cal, ref_c, dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("pos0", [0, (1 << 22) - 1000])
def test_hope_rotate_keys(dtype, pos0):
    g = torch.Generator(device="cuda").manual_seed(9)
    x = (torch.randn((2, 3, 1000, 128), generator=g, device="cuda") / math.sqrt(128)).to(dtype)
    got = hb.hope_rotate(x, rope_base=10000.0, train_len=65536.0, pos0=pos0)
    torch.cuda.synchronize()
    ref = oracle.hope_rotate(parity.f64(x), base=10000.0, train_len=65536.0, pos0=pos0)
    _check(got, ref, dtype)
    # in place gives the same
    y = x.clone()
    hb.hope_rotate(y, rope_base=10000.0, train_len=65536.0, pos0=pos0, out=y)
    torch.cuda.synchronize()
    assert torch.equal(y, got)
