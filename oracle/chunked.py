"""Chunk-parallel restatement of the KDA recurrence in float64 numpy (test infrastructure).

This is not a second oracle: it exists to check, against the token-by-token definition in
``kda_oracle.c``, the chunk algebra that a chunk-parallel prefill relies on (the
"Chunked processing algorithm" of the pages: the same recurrence evaluated over fixed-size
chunks -- ``max.nn.state_space.kda_chunk`` describes 16-token chunks; the GStar assignment
builds it from a gate prefix scan, a triangular inverse and a score builder).

Derivation (by induction on the per-token step S <- Diag(a_t)S; S += k_t b_t (v_t - k_t^T S)^T;
o_t = q_t^T S, with a_t = exp(g_t)).  Inside a chunk with incoming state S0 and positions
r, s = 1..C, let G_r = sum_{u<=r} g_u (per channel) and Gamma_r = exp(G_r).  Then

    delta_s = b_s (v_s - S0^T(Gamma_s * k_s) - sum_{u<s} A_su delta_u),
    A_su    = sum_i k_si k_ui exp(G_si - G_ui)              (u < s)

so with T = (I + diag(b) A)^{-1} diag(b):
    Delta = T (V - (K*Gamma) S0)
    O     = (Q*Gamma) S0 + (P masked to u <= r) Delta,   P_ru = sum_i q_ri k_ui exp(G_ri - G_ui)
    S_C   = Diag(Gamma_C) S0 + (K * exp(G_C - G))^T Delta
Every exponent above is <= 0 (g <= 0 and r >= u), so no term can overflow.
"""
from __future__ import annotations

import numpy as np

from . import _f64, _i32


def _gates(raw, a_log, dt_bias, safe, lb):
    x = raw + dt_bias
    sp = np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))
    g = -np.exp(a_log) * sp
    if safe:
        g = np.maximum(g, lb)
    return g


def _betas(logits, prob):
    if prob:
        return logits.copy()
    return np.where(logits >= 0, 1.0 / (1.0 + np.exp(-np.abs(logits))),
                    np.exp(-np.abs(logits)) / (1.0 + np.exp(-np.abs(logits))))


def chunk_step(S0, Q, K, V, g, b):
    """One chunk: S0 [dk,dv]; Q,K [C,dk]; V [C,dv]; g [C,dk]; b [C].  Returns (O, S_C)."""
    C = K.shape[0]
    G = np.cumsum(g, axis=0)
    D = G[:, None, :] - G[None, :, :]            # D[r,u,i] = G_ri - G_ui
    low = np.tril(np.ones((C, C), dtype=bool), -1)
    incl = np.tril(np.ones((C, C), dtype=bool), 0)
    E = np.exp(np.where(incl[:, :, None], D, 0.0))  # only r >= u is used (exponent <= 0)
    A = np.einsum("ri,ui,rui->ru", K, K, E) * low
    P = np.einsum("ri,ui,rui->ru", Q, K, E) * incl
    Tm = np.linalg.solve(np.eye(C) + b[:, None] * A, np.diag(b))
    Gam = np.exp(G)
    Delta = Tm @ (V - (K * Gam) @ S0)
    O = (Q * Gam) @ S0 + P @ Delta
    Kp = K * np.exp(G[-1][None, :] - G)
    S = Gam[-1][:, None] * S0 + Kp.T @ Delta
    return O, S


def kda_forward_chunked(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu_seqlens, state_pool,
                        state_indices=None, *, chunk=16, gate_mode="original", beta_mode="logits",
                        state_layout="K_FIRST", gate_lower_bound=-5.0):
    q, k, v = _f64(q), _f64(k), _f64(v)
    raw_gate, beta_logits = _f64(raw_gate), _f64(beta_logits)
    a_log, dt_bias = _f64(a_log), _f64(dt_bias)
    cu = _i32(cu_seqlens)
    pool = _f64(state_pool).copy()
    T, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    group = Hv // Hk
    B = cu.size - 1
    idx = _i32(state_indices) if state_indices is not None else np.arange(B, dtype=np.int32)
    out = np.zeros((T, Hv, dv))
    safe = gate_mode == "safe"
    prob = beta_mode == "probability"
    for bi in range(B):
        t0, t1 = int(cu[bi]), int(cu[bi + 1])
        for h in range(Hv):
            kh = h // group
            blk = pool[idx[bi], h]
            S = blk.T.copy() if state_layout == "V_FIRST" else blk.copy()
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                g = _gates(raw_gate[c0:c1, h], a_log[h], dt_bias[h], safe, gate_lower_bound)
                b = _betas(beta_logits[c0:c1, h], prob)
                O, S = chunk_step(S, q[c0:c1, kh], k[c0:c1, kh], v[c0:c1, h], g, b)
                out[c0:c1, h] = O
            pool[idx[bi], h] = S.T if state_layout == "V_FIRST" else S
    return out, pool
