"""fp64 CPU oracle for KDA prefill and the context-parallel segment scan.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA library and its Python binding never do.

``kda_oracle.c`` is the token-by-token definition (see its header for the citations);
``chunked.py`` restates the chunk-parallel algebra in numpy to check that algebra against
the recurrence.  All arithmetic is float64 on inputs widened exactly from bf16/fp32.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

GATE_SAFE = 1
BETA_PROB = 2
V_FIRST = 4

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lib.kda_oracle_forward.restype = ctypes.c_int
        lib.kda_oracle_forward.argtypes = [dp, dp, dp, dp, dp, dp, dp, ip, ctypes.c_int32,
                                           ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, ctypes.c_int32, dp, ctypes.c_int32, ip,
                                           dp, ctypes.c_uint32, ctypes.c_double]
        lib.kda_oracle_segment_summary.restype = ctypes.c_int
        lib.kda_oracle_segment_summary.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.c_int64,
                                                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                   ctypes.c_int32, ip, ctypes.c_int32, dp, dp,
                                                   ctypes.c_uint32, ctypes.c_double]
        lib.kda_oracle_affine_scan.restype = ctypes.c_int
        lib.kda_oracle_affine_scan.argtypes = [dp, dp, dp, ctypes.c_int32, ctypes.c_int32,
                                               ctypes.c_int32, ctypes.c_int32, ctypes.c_uint32,
                                               dp, dp, dp]
        lib.kda_oracle_compose.restype = None
        lib.kda_oracle_compose.argtypes = [dp, dp, dp, dp, ctypes.c_int32, ctypes.c_int32, dp, dp]
        lib.kda_oracle_gate.restype = ctypes.c_double
        lib.kda_oracle_gate.argtypes = [ctypes.c_double, ctypes.c_double, ctypes.c_double,
                                        ctypes.c_uint32, ctypes.c_double]
        lib.kda_oracle_beta.restype = ctypes.c_double
        lib.kda_oracle_beta.argtypes = [ctypes.c_double, ctypes.c_uint32]
        lib.kda_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening to a contiguous float64 array (bf16 and fp32 are exact in fp64)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.int32).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _dp(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def flags_of(gate_mode="original", beta_mode="logits", state_layout="K_FIRST") -> int:
    if gate_mode not in ("original", "safe"):
        raise ValueError(gate_mode)
    if beta_mode not in ("logits", "probability"):
        raise ValueError(beta_mode)
    if state_layout not in ("K_FIRST", "V_FIRST"):
        raise ValueError(state_layout)
    f = 0
    if gate_mode == "safe":
        f |= GATE_SAFE
    if beta_mode == "probability":
        f |= BETA_PROB
    if state_layout == "V_FIRST":
        f |= V_FIRST
    return f


def num_threads() -> int:
    return int(_load().kda_oracle_num_threads())


def gate(raw, a_log, dt_bias, gate_mode="original", lower_bound=-5.0) -> float:
    return float(_load().kda_oracle_gate(float(raw), float(a_log), float(dt_bias),
                                         flags_of(gate_mode), float(lower_bound)))


def beta(logit, beta_mode="logits") -> float:
    return float(_load().kda_oracle_beta(float(logit), flags_of(beta_mode=beta_mode)))


def kda_forward(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu_seqlens, state_pool,
                state_indices=None, *, gate_mode="original", beta_mode="logits",
                state_layout="K_FIRST", gate_lower_bound=-5.0, with_output=True):
    """Token-by-token fp64 prefill.  Returns (out [T,Hv,dv] or None, new_state_pool)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    raw_gate, beta_logits = _f64(raw_gate), _f64(beta_logits)
    a_log, dt_bias = _f64(a_log), _f64(dt_bias)
    cu = _i32(cu_seqlens)
    pool = _f64(state_pool).copy()
    T, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    B = cu.size - 1
    idx = _i32(state_indices) if state_indices is not None else np.arange(B, dtype=np.int32)
    out = np.zeros((T, Hv, dv), dtype=np.float64) if with_output else None
    rc = _load().kda_oracle_forward(_dp(q), _dp(k), _dp(v), _dp(raw_gate), _dp(beta_logits),
                                    _dp(a_log), _dp(dt_bias), _ip(cu), B, T, Hk, Hv, dk, dv,
                                    _dp(pool), pool.shape[0], _ip(idx),
                                    _dp(out) if out is not None else None,
                                    flags_of(gate_mode, beta_mode, state_layout),
                                    float(gate_lower_bound))
    if rc != 0:
        raise ValueError(f"oracle forward rejected its inputs (code {rc})")
    return out, pool


def kda_decode(q, k, v, raw_gate, beta_logits, a_log, dt_bias, state_pool, state_indices=None, *,
               gate_mode="original", beta_mode="logits", state_layout="K_FIRST", gate_lower_bound=-5.0):
    """One token per sequence: the token-by-token definition on a batch of one-token sequences
    (q, k [B,Hk,dk], v [B,Hv,dv], ...).  Returns (out [B,Hv,dv], new_state_pool)."""
    B = int(np.asarray(q.shape)[0])
    cu = np.arange(B + 1, dtype=np.int32)
    return kda_forward(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu, state_pool, state_indices,
                       gate_mode=gate_mode, beta_mode=beta_mode, state_layout=state_layout,
                       gate_lower_bound=gate_lower_bound)


def kda_segment_summary(k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, *,
                        num_v_heads=None, gate_mode="original", beta_mode="logits",
                        state_layout="K_FIRST", gate_lower_bound=-5.0):
    """(M [N,Hv,dk,dk], U [N,Hv,dk,dv] or [N,Hv,dv,dk]) by replaying each segment."""
    k, v = _f64(k), _f64(v)
    raw_gate, beta_logits = _f64(raw_gate), _f64(beta_logits)
    a_log, dt_bias = _f64(a_log), _f64(dt_bias)
    offs = _i32(seg_offsets)
    T, Hk, dk = k.shape
    Hv, dv = v.shape[1], v.shape[2]
    N = offs.size - 1
    M = np.zeros((N, Hv, dk, dk))
    U = np.zeros((N, Hv, dk, dv) if state_layout == "K_FIRST" else (N, Hv, dv, dk))
    rc = _load().kda_oracle_segment_summary(_dp(k), _dp(v), _dp(raw_gate), _dp(beta_logits),
                                            _dp(a_log), _dp(dt_bias), T, Hk, Hv, dk, dv,
                                            _ip(offs), N, _dp(M), _dp(U),
                                            flags_of(gate_mode, beta_mode, state_layout),
                                            float(gate_lower_bound))
    if rc != 0:
        raise ValueError(f"oracle segment summary rejected its inputs (code {rc})")
    return M, U


def kda_affine_scan(M, U, initial_state, *, state_layout="K_FIRST"):
    """The exclusive scan.  Returns dict(incoming_states, outgoing_states, final_state)."""
    M, U, init = _f64(M), _f64(U), _f64(initial_state)
    squeeze = False
    if M.ndim == 3:  # no head axis: (N, dk, dk), (N, dk, dv), (dk, dv)
        M, U, init, squeeze = M[:, None], U[:, None], init[None], True
        M, U, init = (np.ascontiguousarray(a) for a in (M, U, init))
    N, H, dk = M.shape[0], M.shape[1], M.shape[2]
    dv = U.shape[3] if state_layout == "K_FIRST" else U.shape[2]
    inc = np.zeros_like(U)
    outg = np.zeros_like(U)
    fin = np.zeros_like(init)
    rc = _load().kda_oracle_affine_scan(_dp(M), _dp(U), _dp(init), N, H, dk, dv,
                                        flags_of(state_layout=state_layout), _dp(inc), _dp(outg),
                                        _dp(fin))
    if rc != 0:
        raise ValueError(f"oracle scan rejected its inputs (code {rc})")
    if squeeze:
        inc, outg, fin = inc[:, 0], outg[:, 0], fin[0]
    return {"incoming_states": inc, "outgoing_states": outg, "final_state": fin}


def kda_compose(later, earlier):
    """(M2,U2) o (M1,U1) = (M2 M1, M2 U1 + U2); ``later`` = (M2,U2), ``earlier`` = (M1,U1)."""
    M2, U2 = (np.atleast_2d(_f64(x)) for x in later)
    M1, U1 = (np.atleast_2d(_f64(x)) for x in earlier)
    dk, dv = M2.shape[0], U2.shape[1]
    Mo = np.zeros((dk, dk))
    Uo = np.zeros((dk, dv))
    _load().kda_oracle_compose(_dp(M2), _dp(U2), _dp(M1), _dp(U1), dk, dv, _dp(Mo), _dp(Uo))
    return Mo, Uo
