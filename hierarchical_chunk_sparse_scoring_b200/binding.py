"""Thin Python binding of libhils.so (the C ABI in include/hils.h).

Argument marshalling only: tensors are checked for device, dtype and contiguity, outputs and the
workspace are allocated with PyTorch, and every step of the computation runs in the library's
CUDA kernels.  There is no CPU path: if the library is missing, importing this module's functions
raises.
"""
import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhils.so")

HILS_F32, HILS_BF16 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration",
          3: "workspace missing or too small", 4: "CUDA error", 5: "device-side check failed",
          6: "bounded on-chip wait timed out"}


class HilsError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, STATUS.get(status, "?"), status))


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("Hq", ctypes.c_int64), ("Hkv", ctypes.c_int64),
                ("N_q", ctypes.c_int64), ("N_kv", ctypes.c_int64), ("d", ctypes.c_int64),
                ("q_pos0", ctypes.c_int64), ("S", ctypes.c_int32), ("K_top", ctypes.c_int32),
                ("W", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class PrologueParams(ctypes.Structure):
    """hils_prologue_params (include/hils.h)."""
    _fields_ = [("d_model", ctypes.c_int64), ("r", ctypes.c_int32),
                ("rope_base", ctypes.c_double), ("train_len", ctypes.c_double)]


# every function the header declares, with its ctypes signature
_P = ctypes.POINTER(Params)
_V = ctypes.c_void_p
SIGNATURES = {
    "hils_workspace_size": (ctypes.c_size_t, [_P]),
    "hils_forward": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V, ctypes.c_size_t, _V]),
    "hils_forward_timed": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V, _V, _V, _V,
                                          ctypes.c_size_t, _V, ctypes.POINTER(_V), ctypes.c_int]),
    "hils_forward_phases": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_char_p), ctypes.c_int]),
    "hils_select": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, ctypes.c_size_t, _V]),
    "hils_select_noalloc": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V]),
    "hils_select_noalloc_max_bytes": (ctypes.c_size_t, []),
    "hils_select_noalloc_status": (ctypes.c_int, [_V, ctypes.POINTER(ctypes.c_int32)]),
    "hils_landmarks": (ctypes.c_int, [_P, _V, _V, _V, _V, _V]),
    "hils_decode_step": (ctypes.c_int, [_P] + [_V] * 13 + [ctypes.c_size_t, _V]),
    "hils_wait_check": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_int, _V, ctypes.c_size_t, _V]),
    "hils_backward_workspace_size": (ctypes.c_size_t, [_P]),
    "hils_qcal_workspace_size": (ctypes.c_size_t, [_P, ctypes.POINTER(PrologueParams)]),
    "hils_qcal_hope": (ctypes.c_int, [_P, ctypes.POINTER(PrologueParams)] + [_V] * 7 +
                       [ctypes.c_size_t, _V]),
    "hils_hope_rotate": (ctypes.c_int, [_P, ctypes.POINTER(PrologueParams), ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _V, _V,
                                        _V]),
    "hils_backward": (ctypes.c_int, [_P] + [_V] * 16 + [ctypes.c_size_t, _V]),
    "hils_chunk_attn": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V, _V]),
    "hils_fuse": (ctypes.c_int, [_P, _V, _V, _V, _V, _V, _V]),
    "hils_workspace_init": (ctypes.c_int, [_V, ctypes.c_size_t, _V]),
    "hils_device_status": (ctypes.c_int, [_V, _V, ctypes.POINTER(ctypes.c_int32)]),
    "hils_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "hils_version": (ctypes.c_char_p, []),
}

_lib = None
_lock = threading.Lock()


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        "libhils.so is not built (%s); run `python -m "
                        "hierarchical_chunk_sparse_scoring_b200.build`" % LIB_PATH)
                l = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(l, name)
                    f.restype = res
                    f.argtypes = args
                _lib = l
    return _lib


def _dtype_code(t):
    if t == torch.float32:
        return HILS_F32
    if t == torch.bfloat16:
        return HILS_BF16
    raise TypeError("HiLS tensors must be float32 or bfloat16, got %s" % t)


def make_params(B, Hq, Hkv, N_q, N_kv, d, *, S, K_top, W, q_pos0=0, dtype=torch.bfloat16,
                scale=0.0):
    return Params(B, Hq, Hkv, N_q, N_kv, d, q_pos0, S, K_top, W, _dtype_code(dtype), float(scale))


def params_for(q, K, *, S, K_top, W, q_pos0=0, scale=0.0):
    B, Hq, N_q, d = q.shape
    _, Hkv, N_kv, _ = K.shape
    return make_params(B, Hq, Hkv, N_q, N_kv, d, S=S, K_top=K_top, W=W, q_pos0=q_pos0,
                       dtype=q.dtype, scale=scale)


def workspace_size(p):
    return int(lib().hils_workspace_size(ctypes.byref(p)))


def _ptr(t):
    return None if t is None or t.numel() == 0 else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, where):
    if status != 0:
        raise HilsError(status, where)


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must live on a CUDA device (there is no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    return t


_ws_cache = {}


def workspace(p, device, stream=None):
    """A workspace of at least workspace_size(p) bytes for `device`, reused across calls made
    from the same stream."""
    need = workspace_size(p)
    if need == 0:
        # invalid or unsupported parameters: the library call reports which, before any launch
        return torch.empty(0, dtype=torch.uint8, device=device)
    st = stream if stream is not None else torch.cuda.current_stream(device)
    key = (torch.device(device).index, st.cuda_stream)
    buf = _ws_cache.get(key)
    if buf is None or buf.numel() < need:
        buf = torch.empty(need, dtype=torch.uint8, device=device)
        _check(lib().hils_workspace_init(_ptr(buf), buf.numel(), _stream(st)), "hils_workspace_init")
        _ws_cache[key] = buf
    return buf


def forward(q, q_cal, K, V, k_lm, b_lm, *, S, K_top, W, q_pos0=0, scale=0.0, out=None,
            lse=None, idx=None, ws=None, stream=None):
    """The whole HiLS forward (steps 1-4).  Returns (out, lse, idx)."""
    B, Hq, N_q, d = q.shape
    _, Hkv, N_kv, _ = K.shape
    C = N_kv // S
    dt = q.dtype
    _need(q, "q", dt)
    _need(q_cal, "q_cal", dt, q.shape)
    _need(K, "K", dt)
    _need(V, "V", dt, K.shape)
    _need(k_lm, "k_lm", dt, (B, Hkv, C, d))
    _need(b_lm, "b_lm", torch.float32, (B, Hkv, C))
    p = params_for(q, K, S=S, K_top=K_top, W=W, q_pos0=q_pos0, scale=scale)
    out = torch.empty_like(q) if out is None else _need(out, "out", dt, q.shape)
    if lse is None:
        lse = torch.empty((B, Hq, N_q), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hkv, N_q, K_top), dtype=torch.int32, device=q.device)
    ws = workspace(p, q.device, stream) if ws is None else ws
    st = lib().hils_forward(ctypes.byref(p), _ptr(q), _ptr(q_cal), _ptr(K), _ptr(V), _ptr(k_lm),
                            _ptr(b_lm), _ptr(out), _ptr(lse), _ptr(idx), _ptr(ws), ws.numel(),
                            _stream(stream))
    _check(st, "hils_forward")
    return out, lse, idx


def select(q_cal, k_lm, b_lm, *, N_kv, Hkv, S, K_top, W, q_pos0=0, scale=0.0, stream=None):
    """Steps 1-2.  Returns (idx [B,Hkv,N_q,K] int32, s_sel [B,Hq,N_q,K] fp32)."""
    B, Hq, N_q, d = q_cal.shape
    _need(q_cal, "q_cal")
    _need(k_lm, "k_lm", q_cal.dtype, (B, Hkv, N_kv // S, d))
    _need(b_lm, "b_lm", torch.float32, (B, Hkv, N_kv // S))
    p = make_params(B, Hq, Hkv, N_q, N_kv, d, S=S, K_top=K_top, W=W, q_pos0=q_pos0,
                    dtype=q_cal.dtype, scale=scale)
    idx = torch.empty((B, Hkv, N_q, K_top), dtype=torch.int32, device=q_cal.device)
    s_sel = torch.empty((B, Hq, N_q, K_top), dtype=torch.float32, device=q_cal.device)
    ws = workspace(p, q_cal.device, stream)
    _check(lib().hils_select(ctypes.byref(p), _ptr(q_cal), _ptr(k_lm), _ptr(b_lm), _ptr(idx),
                             _ptr(s_sel), _ptr(ws), ws.numel(), _stream(stream)), "hils_select")
    return idx, s_sel


def chunk_attn(q, K, V, idx, *, S, K_top, W, q_pos0=0, scale=0.0, stream=None):
    """Step 3.  Returns (unit_o [B,Hq,N_q,K+1,d] fp32, unit_lse [B,Hq,N_q,K+1] fp32)."""
    B, Hq, N_q, d = q.shape
    _, Hkv, N_kv, _ = K.shape
    _need(q, "q")
    _need(K, "K", q.dtype)
    _need(V, "V", q.dtype, K.shape)
    _need(idx, "idx", torch.int32, (B, Hkv, N_q, K_top))
    p = params_for(q, K, S=S, K_top=K_top, W=W, q_pos0=q_pos0, scale=scale)
    unit_o = torch.empty((B, Hq, N_q, K_top + 1, d), dtype=torch.float32, device=q.device)
    unit_lse = torch.empty((B, Hq, N_q, K_top + 1), dtype=torch.float32, device=q.device)
    _check(lib().hils_chunk_attn(ctypes.byref(p), _ptr(q), _ptr(K), _ptr(V), _ptr(idx),
                                 _ptr(unit_o), _ptr(unit_lse), _stream(stream)), "hils_chunk_attn")
    return unit_o, unit_lse


def fuse(s_sel, unit_o, unit_lse, *, Hkv, N_kv, S, K_top, W, q_pos0=0, dtype=torch.bfloat16,
         stream=None):
    """Step 4.  Returns (out [B,Hq,N_q,d] dtype, lse [B,Hq,N_q] fp32)."""
    B, Hq, N_q, _, d = unit_o.shape
    _need(s_sel, "s_sel", torch.float32, (B, Hq, N_q, K_top))
    _need(unit_o, "unit_o", torch.float32, (B, Hq, N_q, K_top + 1, d))
    _need(unit_lse, "unit_lse", torch.float32, (B, Hq, N_q, K_top + 1))
    p = make_params(B, Hq, Hkv, N_q, N_kv, d, S=S, K_top=K_top, W=W, q_pos0=q_pos0, dtype=dtype)
    out = torch.empty((B, Hq, N_q, d), dtype=dtype, device=unit_o.device)
    lse = torch.empty((B, Hq, N_q), dtype=torch.float32, device=unit_o.device)
    _check(lib().hils_fuse(ctypes.byref(p), _ptr(s_sel), _ptr(unit_o), _ptr(unit_lse), _ptr(out),
                           _ptr(lse), _stream(stream)), "hils_fuse")
    return out, lse


def device_status(ws, stream=None):
    code = ctypes.c_int32(0)
    _check(lib().hils_device_status(_ptr(ws), _stream(stream), ctypes.byref(code)),
           "hils_device_status")
    return int(code.value)


def landmarks(q_lm, K, *, S, scale=0.0, k_lm=None, b_lm=None, stream=None):
    """Landmark construction: q_lm [B,Hkv,C,d] landmark queries, K [B,Hkv,N_kv,d] keys with
    C = N_kv // S.  Returns (k_lm [B,Hkv,C,d] in K's dtype, b_lm [B,Hkv,C] fp32)."""
    B, Hkv, N_kv, d = K.shape
    C = N_kv // S
    _need(K, "K")
    _need(q_lm, "q_lm", K.dtype, (B, Hkv, C, d))
    if k_lm is None:
        k_lm = torch.empty((B, Hkv, C, d), dtype=K.dtype, device=K.device)
    if b_lm is None:
        b_lm = torch.empty((B, Hkv, C), dtype=torch.float32, device=K.device)
    _need(k_lm, "k_lm", K.dtype, (B, Hkv, C, d))
    _need(b_lm, "b_lm", torch.float32, (B, Hkv, C))
    p = make_params(B, Hkv, Hkv, 0, N_kv, d, S=S, K_top=0, W=1, dtype=K.dtype, scale=scale)
    _check(lib().hils_landmarks(ctypes.byref(p), _ptr(q_lm), _ptr(K), _ptr(k_lm), _ptr(b_lm),
                                _stream(stream)), "hils_landmarks")
    return k_lm, b_lm


def decode_step(q, q_cal, k_new, v_new, q_lm_new, K, V, k_lm, b_lm, *, pos, S, K_top, W,
                scale=0.0, out=None, lse=None, idx=None, ws=None, stream=None):
    """One decode step over a cache of capacity K.shape[2]: appends (k_new, v_new) at `pos`,
    builds the landmark of the chunk the token completes (q_lm_new, may be None otherwise) and
    runs the forward for the query at `pos`.  Returns (out, lse, idx)."""
    B, Hq, N_q, d = q.shape
    _, Hkv, N_cap, _ = K.shape
    p = make_params(B, Hq, Hkv, N_q, N_cap, d, S=S, K_top=K_top, W=W, q_pos0=pos,
                    dtype=q.dtype, scale=scale)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, Hq, N_q), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((B, Hkv, N_q, K_top), dtype=torch.int32, device=q.device)
    if ws is None:
        ws = workspace(p, q.device, stream)
    _check(lib().hils_decode_step(ctypes.byref(p), _ptr(q), _ptr(q_cal), _ptr(k_new),
                                  _ptr(v_new), _ptr(q_lm_new) if q_lm_new is not None else None,
                                  _ptr(K), _ptr(V), _ptr(k_lm), _ptr(b_lm), _ptr(out), _ptr(lse),
                                  _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)),
           "hils_decode_step")
    return out, lse, idx


def qcal_hope(q, hidden, W_down, W_up, *, rope_base, train_len, q_pos0=0, q_out=None,
              q_cal_out=None, ws=None, stream=None):
    """hils_qcal_hope: (HoPE(q), HoPE(q + W_up W_down hidden)) for query i at q_pos0 + i.
    q [B,Hq,N_q,d] and W_up [Hq,d,r] in the model dtype; hidden [B,N_q,d_model] and W_down
    [Hq,r,d_model] bf16 (W_down / W_up may be None for r = 0)."""
    B, Hq, N_q, d = q.shape
    _need(q, "q")
    r = 0 if W_down is None else W_down.shape[1]
    d_model = 0 if hidden is None else hidden.shape[2]
    if r > 0:
        _need(hidden, "hidden", torch.bfloat16, (B, N_q, d_model))
        _need(W_down, "W_down", torch.bfloat16, (Hq, r, d_model))
        _need(W_up, "W_up", q.dtype, (Hq, d, r))
    p = make_params(B, Hq, Hq, N_q, max(N_q + q_pos0, 1), d, S=1, K_top=0, W=1, q_pos0=q_pos0,
                    dtype=q.dtype)
    c = PrologueParams(d_model, r, float(rope_base), float(train_len))
    if q_out is None:
        q_out = torch.empty_like(q)
    if q_cal_out is None:
        q_cal_out = torch.empty_like(q)
    if ws is None:
        need = int(lib().hils_qcal_workspace_size(ctypes.byref(p), ctypes.byref(c)))
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().hils_qcal_hope(ctypes.byref(p), ctypes.byref(c), _ptr(q), _ptr(hidden),
                                _ptr(W_down), _ptr(W_up), _ptr(q_out), _ptr(q_cal_out), _ptr(ws),
                                ws.numel(), _stream(stream)), "hils_qcal_hope")
    return q_out, q_cal_out


def hope_rotate(x, *, rope_base, train_len, pos0=0, out=None, stream=None):
    """hils_hope_rotate: HoPE of x [B,H,N,d], token n at position pos0 + n."""
    B, H, N, d = x.shape
    _need(x, "x")
    p = make_params(1, 1, 1, 1, 1, d, S=1, K_top=0, W=1, dtype=x.dtype)
    c = PrologueParams(0, 0, float(rope_base), float(train_len))
    if out is None:
        out = torch.empty_like(x)
    _check(lib().hils_hope_rotate(ctypes.byref(p), ctypes.byref(c), B, H, N, pos0, _ptr(x),
                                  _ptr(out), _stream(stream)), "hils_hope_rotate")
    return out


def backward_workspace(p, device):
    need = int(lib().hils_backward_workspace_size(ctypes.byref(p)))
    if need == 0:
        return None   # invalid or unsupported: hils_backward says which
    return torch.empty(need, dtype=torch.uint8, device=device)


def backward(q, q_cal, K, V, k_lm, b_lm, idx, dout, dlse=None, *, S, K_top, W, q_pos0=0,
             scale=0.0, ws=None, out=None, stream=None):
    """hils_backward: gradients of sum(dout * out) + sum(dlse * lse) with the selection `idx`
    held fixed.  Returns a dict of fp32 tensors dq, dq_cal, dK, dV, dk_lm, db_lm."""
    B, Hq, N_q, d = q.shape
    _, Hkv, N_kv, _ = K.shape
    C = N_kv // S
    _need(q, "q")
    _need(q_cal, "q_cal", q.dtype, q.shape)
    _need(K, "K", q.dtype)
    _need(V, "V", q.dtype, K.shape)
    _need(k_lm, "k_lm", q.dtype, (B, Hkv, C, d))
    _need(b_lm, "b_lm", torch.float32, (B, Hkv, C))
    _need(idx, "idx", torch.int32, (B, Hkv, N_q, K_top))
    _need(dout, "dout", q.dtype, q.shape)
    if dlse is not None:
        _need(dlse, "dlse", torch.float32, (B, Hq, N_q))
    p = make_params(B, Hq, Hkv, N_q, N_kv, d, S=S, K_top=K_top, W=W, q_pos0=q_pos0,
                    dtype=q.dtype, scale=scale)
    if ws is None:
        ws = backward_workspace(p, q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = out if out is not None else {
        "dq": torch.empty(q.shape, **f32), "dq_cal": torch.empty(q.shape, **f32),
        "dK": torch.empty(K.shape, **f32), "dV": torch.empty(K.shape, **f32),
        "dk_lm": torch.empty(k_lm.shape, **f32), "db_lm": torch.empty(b_lm.shape, **f32)}
    _check(lib().hils_backward(ctypes.byref(p), _ptr(q), _ptr(q_cal), _ptr(K), _ptr(V),
                               _ptr(k_lm), _ptr(b_lm), _ptr(idx), _ptr(dout), _ptr(dlse),
                               _ptr(g["dq"]), _ptr(g["dq_cal"]), _ptr(g["dK"]), _ptr(g["dV"]),
                               _ptr(g["dk_lm"]), _ptr(g["db_lm"]), _ptr(ws),
                               0 if ws is None else ws.numel(), _stream(stream)),
           "hils_backward")
    return g


def select_noalloc(q_cal, k_lm, b_lm, *, N_kv, Hkv, S, K_top, W, q_pos0=0, scale=0.0,
                   stream=None):
    """hils_select_noalloc: steps 1-2 with the library's fixed scratch array (no workspace).
    Returns (idx, s_sel)."""
    B, Hq, N_q, d = q_cal.shape
    p = make_params(B, Hq, Hkv, N_q, N_kv, d, S=S, K_top=K_top, W=W, q_pos0=q_pos0,
                    dtype=q_cal.dtype, scale=scale)
    idx = torch.empty((B, Hkv, N_q, K_top), dtype=torch.int32, device=q_cal.device)
    s_sel = torch.empty((B, Hq, N_q, K_top), dtype=torch.float32, device=q_cal.device)
    _check(lib().hils_select_noalloc(ctypes.byref(p), _ptr(q_cal), _ptr(k_lm), _ptr(b_lm),
                                     _ptr(idx), _ptr(s_sel), _stream(stream)),
           "hils_select_noalloc")
    return idx, s_sel


def select_noalloc_status(stream=None):
    """Reads and clears this device's hils_select_noalloc status word."""
    code = ctypes.c_int32(0)
    _check(lib().hils_select_noalloc_status(_stream(stream), ctypes.byref(code)),
           "hils_select_noalloc_status")
    return int(code.value)


def wait_check(polls, complete, ws, stream=None):
    """hils_wait_check: one bounded mbarrier wait on the device (see include/hils.h)."""
    _check(lib().hils_wait_check(int(polls), int(bool(complete)), _ptr(ws), ws.numel(),
                                 _stream(stream)), "hils_wait_check")


def version():
    return lib().hils_version().decode()


def phases(p):
    """Names of the kernels hils_forward launches for params p, in launch order."""
    n = lib().hils_forward_phases(ctypes.byref(p), None, 0)
    if n < 0:
        raise HilsError(1, "hils_forward_phases")
    arr = (ctypes.c_char_p * max(n, 1))()
    lib().hils_forward_phases(ctypes.byref(p), arr, n)
    return [arr[i].decode() for i in range(n)]


def forward_raw(p, q, q_cal, K, V, k_lm, b_lm, out, lse, idx, ws, stream=None, events=None):
    """hils_forward on preallocated tensors (no Python-side checks).  `events`: torch.cuda.Event
    objects already recorded once (so their CUDA handles exist); the library records them before
    the first kernel and after each kernel."""
    if events is None:
        st = lib().hils_forward(ctypes.byref(p), _ptr(q), _ptr(q_cal), _ptr(K), _ptr(V),
                                _ptr(k_lm), _ptr(b_lm), _ptr(out), _ptr(lse), _ptr(idx),
                                _ptr(ws), ws.numel(), _stream(stream))
    else:
        handles = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        st = lib().hils_forward_timed(ctypes.byref(p), _ptr(q), _ptr(q_cal), _ptr(K), _ptr(V),
                                      _ptr(k_lm), _ptr(b_lm), _ptr(out), _ptr(lse), _ptr(idx),
                                      _ptr(ws), ws.numel(), _stream(stream), handles,
                                      len(events))
    _check(st, "hils_forward")
