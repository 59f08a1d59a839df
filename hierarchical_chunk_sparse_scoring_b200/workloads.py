"""Seeded synthetic inputs for the HiLS forward pass.

This module only draws random numbers and plants structure (needle keys, chunk means); it holds
none of the method's arithmetic.  Both the CUDA path and the CPU oracle consume what it returns.

Values are drawn in fp32 with a torch.Generator on the requested device, then rounded once to
the workload dtype.  Notation: N(0, 1/d) per component is written `nd`.  A "planted logit tau"
for a query direction u is a key tau * sqrt(d) * u with |u| = 1, so u . key / sqrt(d) = tau.

Workloads (shapes of the pages' settings: a 345M-like MHA model, a 7B-like GQA model,
long-context decode and an extreme-length sweep; chunk 64, top-k, local window):
  tiny_fp32         B=1, Hq=Hkv=2, d=64, N=2048, S=64, K=4, W=128, fp32.  Every query with at
                    least one eligible chunk plants one key (tau=8 along the query, + 3*nd noise)
                    in a random earlier chunk (later plants overwrite earlier ones).
  small_mha_bf16    B=4, Hq=Hkv=16, d=64, N=8192, S=64, K=8, W=512.  1% needle chunks (at least one
                    per (b,h)): key tau=8 along a unit u, landmark += 2*sqrt(d)*u, and every query
                    of one probe query chunk where the needle is eligible gets q += u, q_cal += u.
  gqa7b_prefill     B=1, Hq=32, Hkv=8, d=128, N=131072, S=64, K=16, W=1024.  Per (g, chunk) a key
                    mean m_c and value mean; K_j = m_c + nd, V_j = mv_c + nd; per (h, query
                    chunk) a target eligible chunk c*, q = 2*sqrt(d)*m_c* + nd; landmark = the
                    chunk's mean key + 0.1*nd; b ~ N(0, variance 0.5).
  long_decode       B=32, Hq=32, Hkv=8, d=128, N_kv=524288, S=64, K=16, W=1024, one query per
                    sequence at position N_kv-1; one needle chunk per sequence (per KV head a
                    unit u: key tau=8, landmark += 2*sqrt(d)*u, the group's query heads += u).
  extreme           B=1, Hq=8, Hkv=1, d=128, S=128, K=16, W=2048, N in {2^18, 2^20, 2^22}; as
                    small_mha_bf16 plus one needle probed by the last query (the decode query).
In every workload q_cal = q + 0.1*nd (plus the needle directions) unless stated, and
b ~ U(-1, 1) unless stated.  All sizes can be overridden to get smaller cases of the same recipe.
"""
import math
from dataclasses import dataclass, field

import torch

SPECS = {
    "tiny_fp32": dict(B=1, Hq=2, Hkv=2, d=64, N=2048, S=64, K_top=4, W=128,
                      dtype=torch.float32, seed=1001),
    "small_mha_bf16": dict(B=4, Hq=16, Hkv=16, d=64, N=8192, S=64, K_top=8, W=512,
                           dtype=torch.bfloat16, seed=1002),
    "gqa7b_prefill": dict(B=1, Hq=32, Hkv=8, d=128, N=131072, S=64, K_top=16, W=1024,
                          dtype=torch.bfloat16, seed=1003),
    "long_decode": dict(B=32, Hq=32, Hkv=8, d=128, N=524288, S=64, K_top=16, W=1024,
                        dtype=torch.bfloat16, seed=1004, decode=True),
    "extreme": dict(B=1, Hq=8, Hkv=1, d=128, N=262144, S=128, K_top=16, W=2048,
                    dtype=torch.bfloat16, seed=1005, decode_needle=True),
}

TAU = 8.0      # planted needle logit
GAMMA = 2.0    # landmark boost of a needle chunk (selection margin)
LAMBDA = 2.0   # gqa7b_prefill: query = LAMBDA * sqrt(d) * target chunk mean + noise
NEEDLE_P = 0.01


@dataclass
class Workload:
    name: str
    q: torch.Tensor
    q_cal: torch.Tensor
    K: torch.Tensor
    V: torch.Tensor
    k_lm: torch.Tensor
    b_lm: torch.Tensor
    S: int
    K_top: int
    W: int
    q_pos0: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def dims(self):
        B, Hq, N_q, d = self.q.shape
        return dict(B=B, Hq=Hq, Hkv=self.K.shape[1], N_q=N_q, N_kv=self.K.shape[2], d=d)

    def kwargs(self):
        return dict(S=self.S, K_top=self.K_top, W=self.W, q_pos0=self.q_pos0)


def _eligible(pos, S, W):
    first = pos - W + 1
    return 0 if first <= 0 else first // S


class _Gen:
    def __init__(self, device, seed):
        self.device = torch.device(device)
        self.g = torch.Generator(device=self.device)
        self.g.manual_seed(int(seed))

    def randn(self, *shape):
        return torch.randn(shape, generator=self.g, device=self.device, dtype=torch.float32)

    def rand(self, *shape):
        return torch.rand(shape, generator=self.g, device=self.device, dtype=torch.float32)

    def randint(self, lo, hi, shape):
        return torch.randint(lo, hi, shape, generator=self.g, device=self.device)

    def unit(self, *shape):
        u = self.randn(*shape)
        return u / u.norm(dim=-1, keepdim=True)


def _fill_nd(gen, out, d, chunk_rows=1 << 22):
    """out (any dtype) <- N(0, 1/d) drawn in fp32, written slice by slice along dim 0..1."""
    flat = out.view(-1, out.shape[-1])
    rows = flat.shape[0]
    s = 1.0 / math.sqrt(d)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        flat[r0:r1] = (gen.randn(r1 - r0, out.shape[-1]) * s).to(out.dtype)
    return out


def make(name, device="cuda", *, seed=None, dtype=None, **overrides):
    """Builds the named workload (optionally resized) on `device`."""
    spec = dict(SPECS[name])
    spec.update({k: v for k, v in overrides.items() if v is not None})
    if dtype is not None:
        spec["dtype"] = dtype
    if seed is not None:
        spec["seed"] = seed
    gen = _Gen(device, spec["seed"])
    build = {"tiny_fp32": _tiny, "small_mha_bf16": _needles, "gqa7b_prefill": _gqa_mixture,
             "long_decode": _long_decode, "extreme": _needles}[name]
    wl = build(gen, spec)
    wl.name = name
    wl.meta.update({k: (str(v) if isinstance(v, torch.dtype) else v) for k, v in spec.items()})
    return wl


def _finish(name, spec, q, q_cal, K, V, k_lm, b_lm, q_pos0=0, meta=None):
    dt = spec["dtype"]
    return Workload(name, q.to(dt).contiguous(), q_cal.to(dt).contiguous(), K, V,
                    k_lm.to(dt).contiguous(), b_lm.float().contiguous(), spec["S"],
                    spec["K_top"], spec["W"], q_pos0, meta or {})


def _tiny(gen, spec):
    B, Hq, Hkv, d, N, S, W = (spec[k] for k in ("B", "Hq", "Hkv", "d", "N", "S", "W"))
    assert Hq == Hkv, "the tiny workload plants per head and needs Hq == Hkv"
    nd = 1.0 / math.sqrt(d)
    q = gen.randn(B, Hq, N, d) * nd
    K = gen.randn(B, Hkv, N, d) * nd
    V = gen.randn(B, Hkv, N, d) * nd
    q_cal = gen.randn(B, Hq, N, d) * nd
    C = N // S
    k_lm = gen.randn(B, Hkv, C, d) * nd
    b_lm = gen.rand(B, Hkv, C) * 2 - 1
    # one planted key per query with n >= 1, in a random eligible chunk; later queries win
    n = torch.tensor([_eligible(i, S, W) for i in range(N)], device=gen.device)
    has = n >= 1
    c = (gen.rand(B, Hq, N) * n.clamp(min=1)).long().clamp(max=C - 1)
    j = c * S + gen.randint(0, S, (B, Hq, N))
    noise = gen.randn(B, Hq, N, d) * (3 * nd)
    qn = q / (q.norm(dim=-1, keepdim=True) ** 2)
    planted = TAU * math.sqrt(d) * qn + noise
    i_idx = torch.arange(N, device=gen.device).expand(B, Hq, N)
    winner = torch.full((B, Hkv, N), -1, dtype=torch.long, device=gen.device)
    winner.scatter_reduce_(2, torch.where(has, j, torch.zeros_like(j)),
                           torch.where(has, i_idx, torch.full_like(i_idx, -1)), "amax")
    for b in range(B):
        for h in range(Hq):
            rows = (winner[b, h] >= 0).nonzero().squeeze(1)
            K[b, h, rows] = planted[b, h, winner[b, h, rows]]
    return _finish("tiny_fp32", spec, q, q_cal, K.to(spec["dtype"]), V.to(spec["dtype"]), k_lm,
                   b_lm)


def _needles(gen, spec):
    B, Hq, Hkv, d, N, S, W = (spec[k] for k in ("B", "Hq", "Hkv", "d", "N", "S", "W"))
    G = Hq // Hkv
    dt = spec["dtype"]
    nd = 1.0 / math.sqrt(d)
    C = N // S
    K = _fill_nd(gen, torch.empty((B, Hkv, N, d), dtype=dt, device=gen.device), d)
    V = _fill_nd(gen, torch.empty((B, Hkv, N, d), dtype=dt, device=gen.device), d)
    q = _fill_nd(gen, torch.empty((B, Hq, N, d), dtype=torch.float32, device=gen.device), d)
    q_cal = q + 0.1 * _fill_nd(gen, torch.empty_like(q), d)
    k_lm = gen.randn(B, Hkv, C, d) * nd
    b_lm = gen.rand(B, Hkv, C) * 2 - 1
    # query chunk t sees chunk c iff c < n(first query of t)
    n_first = torch.tensor([_eligible(t * S, S, W) for t in range(C)])
    is_needle = (gen.rand(B, Hkv, C) < NEEDLE_P).cpu()
    for b in range(B):
        for g in range(Hkv):
            if not bool(is_needle[b, g].any()):
                is_needle[b, g, int(gen.randint(0, max(1, C // 2), (1,)))] = True
    needles = is_needle.nonzero().tolist()
    probes = []
    for (b, g, c) in needles:
        ok = (n_first > c).nonzero().squeeze(1)
        probes.append(int(ok[int(gen.randint(0, len(ok), (1,)))]) if len(ok) else -1)
    if spec.get("decode_needle", False) and N // S > 0:
        # one more needle probed by the last query (the decode query of this sequence)
        n_last = _eligible(N - 1, S, W)
        if n_last > 0:
            for b in range(B):
                for g in range(Hkv):
                    c = int(gen.randint(0, n_last, (1,)))
                    needles.append([b, g, c])
                    probes.append(-2)
    us = gen.unit(max(1, len(needles)), d)
    slots = gen.randint(0, S, (max(1, len(needles)),)).tolist()
    for k, ((b, g, c), t) in enumerate(zip(needles, probes)):
        u = us[k]
        K[b, g, c * S + slots[k]] = (TAU * math.sqrt(d) * u).to(dt)
        k_lm[b, g, c] += GAMMA * math.sqrt(d) * u
        if t == -1:
            continue
        rows = slice(t * S, (t + 1) * S) if t >= 0 else slice(N - 1, N)
        q[b, g * G:(g + 1) * G, rows] += u
        q_cal[b, g * G:(g + 1) * G, rows] += u
    meta = {"needles": len(needles)}
    return _finish("needles", spec, q, q_cal, K, V, k_lm, b_lm, meta=meta)


def _gqa_mixture(gen, spec):
    B, Hq, Hkv, d, N, S, W = (spec[k] for k in ("B", "Hq", "Hkv", "d", "N", "S", "W"))
    G = Hq // Hkv
    dt = spec["dtype"]
    nd = 1.0 / math.sqrt(d)
    C = N // S
    dev = gen.device
    K = torch.empty((B, Hkv, N, d), dtype=dt, device=dev)
    V = torch.empty((B, Hkv, N, d), dtype=dt, device=dev)
    k_lm = torch.empty((B, Hkv, C, d), dtype=torch.float32, device=dev)
    mk = gen.randn(B, Hkv, C, d) * nd
    for b in range(B):
        for g in range(Hkv):
            kf = mk[b, g].repeat_interleave(S, 0)
            kf = torch.cat([kf, torch.zeros((N - C * S, d), device=dev)]) + gen.randn(N, d) * nd
            K[b, g] = kf.to(dt)
            k_lm[b, g] = K[b, g, :C * S].float().view(C, S, d).mean(1) + 0.1 * nd * gen.randn(C, d)
            mv = gen.randn(C, d) * nd
            vf = torch.cat([mv.repeat_interleave(S, 0), torch.zeros((N - C * S, d), device=dev)])
            V[b, g] = (vf + gen.randn(N, d) * nd).to(dt)
    b_lm = gen.randn(B, Hkv, C) * math.sqrt(0.5)
    q = torch.empty((B, Hq, N, d), dtype=torch.float32, device=dev)
    T = (N + S - 1) // S
    n_first = torch.tensor([_eligible(t * S, S, W) for t in range(T)], device=dev)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            tgt = (gen.rand(T) * n_first.clamp(min=1)).long().clamp(max=max(C - 1, 0))
            means = mk[b, g][tgt] * (LAMBDA * math.sqrt(d))
            means = torch.where((n_first > 0)[:, None], means, torch.zeros_like(means))
            qh = means.repeat_interleave(S, 0)[:N] + gen.randn(N, d) * nd
            q[b, h] = qh
    q_cal = q + 0.1 * nd * gen.randn(B, Hq, N, d)
    return _finish("gqa7b_prefill", spec, q, q_cal, K, V, k_lm, b_lm)


def _long_decode(gen, spec):
    B, Hq, Hkv, d, N, S, W = (spec[k] for k in ("B", "Hq", "Hkv", "d", "N", "S", "W"))
    G = Hq // Hkv
    dt = spec["dtype"]
    nd = 1.0 / math.sqrt(d)
    C = N // S
    dev = gen.device
    K = _fill_nd(gen, torch.empty((B, Hkv, N, d), dtype=dt, device=dev), d)
    V = _fill_nd(gen, torch.empty((B, Hkv, N, d), dtype=dt, device=dev), d)
    q = gen.randn(B, Hq, 1, d) * nd
    q_cal = q + 0.1 * nd * gen.randn(B, Hq, 1, d)
    k_lm = gen.randn(B, Hkv, C, d) * nd
    b_lm = gen.rand(B, Hkv, C) * 2 - 1
    n = _eligible(N - 1, S, W)
    needle_chunks = []
    if n > 0:
        cb = gen.randint(0, n, (B,)).tolist()
        us = gen.unit(B, Hkv, d)
        slots = gen.randint(0, S, (B, Hkv)).tolist()
        for b in range(B):
            c = cb[b]
            needle_chunks.append(c)
            for g in range(Hkv):
                u = us[b, g]
                K[b, g, c * S + slots[b][g]] = (TAU * math.sqrt(d) * u).to(dt)
                k_lm[b, g, c] += GAMMA * math.sqrt(d) * u
                q[b, g * G:(g + 1) * G, 0] += u
                q_cal[b, g * G:(g + 1) * G, 0] += u
    return _finish("long_decode", spec, q, q_cal, K, V, k_lm, b_lm, q_pos0=N - 1,
                   meta={"needle_chunks": needle_chunks})


def decode_view(wl, query_index=None):
    """The decode problem of a prefill workload: one query per sequence at the last position."""
    i = wl.q.shape[2] - 1 if query_index is None else query_index
    return Workload(wl.name + "_decode", wl.q[:, :, i:i + 1].contiguous(),
                    wl.q_cal[:, :, i:i + 1].contiguous(), wl.K, wl.V, wl.k_lm, wl.b_lm, wl.S,
                    wl.K_top, wl.W, wl.q_pos0 + i, dict(wl.meta))
