"""Pins for the fp64 oracle: each test checks it against something other than itself.

Sources of the pinned facts:
  * "KDA Context Parallelism" -- the scalar three-segment example, the composition rule,
    the exclusive-prefix definition, the listed common mistakes and the requirements.
  * "nx_nofloat_kda.nx source" -- the delta-rule overwrite invariant and the per-token order
    (gate, then delta write predicting from the decayed state, then readout).
  * Closed forms that follow from the recurrence: identity case, beta = 0, q = k with beta = 1,
    the scalar (dk = dv = 1) recurrence, and the transition-matrix form of one step.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import kda_workloads as W
import oracle
from oracle import chunked

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def tiny(lengths, Hk=1, Hv=1, dk=4, dv=3, seed=0, state_std=0.5, **kw):
    return W.random_inputs(lengths, Hk, Hv, dk, dv, seed=seed, qkv_dtype=torch.float32,
                           state_std=state_std, **kw)


def run(w, **kw):
    return oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                              w.cu_seqlens, w.state_pool, w.state_indices, gate_mode=w.gate_mode,
                              beta_mode=w.beta_mode, state_layout=w.state_layout,
                              gate_lower_bound=w.gate_lower_bound, **kw)


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    n = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (n if n > 0 else 1.0)


# ------------------------------------------------------------------------------------------
# Segment scan: the page's scalar example, composition, requirements, planted mistakes
# ------------------------------------------------------------------------------------------

def _gold():
    with open(os.path.join(GOLD, "scalar_three_segments.json")) as f:
        return json.load(f)


def test_scalar_three_segment_example():
    g = _gold()
    M = np.array([[[m]] for m, _ in g["maps"]])
    U = np.array([[[u]] for _, u in g["maps"]])
    init = np.array([[g["initial_state"]]])
    res = oracle.kda_affine_scan(M, U, init)
    assert set(res) == {"incoming_states", "outgoing_states", "final_state"}
    assert res["incoming_states"].shape[0] == 3 and res["outgoing_states"].shape[0] == 3
    assert res["incoming_states"].ravel().tolist() == g["incoming_states"]
    assert res["outgoing_states"].ravel().tolist() == g["outgoing_states"]
    assert res["final_state"].item() == g["final_state"]


def test_composition_order():
    g = _gold()
    (m0, u0), (m1, u1) = g["maps"][0], g["maps"][1]
    Mo, Uo = oracle.kda_compose((m1, u1), (m0, u0))  # segment 1 applied after segment 0
    assert [Mo.item(), Uo.item()] == g["compose_second_after_first"]
    assert Mo.item() * g["initial_state"] + Uo.item() == g["compose_second_after_first_applied_to_initial"]
    Mr, Ur = oracle.kda_compose((m0, u0), (m1, u1))
    assert [Mr.item(), Ur.item()] == g["compose_first_after_second"]


def test_composition_associative_not_commutative():
    rng = np.random.default_rng(1)
    maps = [(rng.normal(size=(3, 3)), rng.normal(size=(3, 2))) for _ in range(3)]
    a = oracle.kda_compose(maps[2], oracle.kda_compose(maps[1], maps[0]))
    b = oracle.kda_compose(oracle.kda_compose(maps[2], maps[1]), maps[0])
    assert rel(a[0], b[0]) < 1e-14 and rel(a[1], b[1]) < 1e-14
    c = oracle.kda_compose(maps[0], maps[1])
    d = oracle.kda_compose(maps[1], maps[0])
    assert rel(c[0], d[0]) > 1e-3


def test_scan_matches_applying_maps_and_does_not_mutate():
    rng = np.random.default_rng(2)
    N, H, dk, dv = 4, 2, 3, 2
    M, U = rng.normal(size=(N, H, dk, dk)), rng.normal(size=(N, H, dk, dv))
    init = rng.normal(size=(H, dk, dv))
    copies = [x.copy() for x in (M, U, init)]
    res = oracle.kda_affine_scan(M, U, init)
    for x, c in zip((M, U, init), copies):
        assert np.array_equal(x, c)
    for h in range(H):
        s = init[h]
        for i in range(N):
            assert rel(res["incoming_states"][i, h], s) < 1e-15
            s = M[i, h] @ s + U[i, h]
            assert rel(res["outgoing_states"][i, h], s) < 1e-14
        assert rel(res["final_state"][h], s) < 1e-14
    # V_FIRST stores every state transposed; the math is unchanged
    resv = oracle.kda_affine_scan(M, np.swapaxes(U, 2, 3).copy(), np.swapaxes(init, 1, 2).copy(),
                                  state_layout="V_FIRST")
    assert rel(np.swapaxes(resv["outgoing_states"], 2, 3), res["outgoing_states"]) < 1e-15


def _mistaken_scans():
    """The page's list of common mistakes, each as a broken scalar scan."""
    def inclusive(maps, s0):
        inc, out, s = [], [], s0
        for m, u in maps:
            s_new = m * s + u
            inc.append(s_new)
            out.append(s_new)
            s = s_new
        return inc, out, s

    def no_transitions(maps, s0):
        inc, out, s = [], [], s0
        for m, u in maps:
            inc.append(s)
            s = s + u
            out.append(s)
        return inc, out, s

    def reversed_order(maps, s0):
        inc, out, s = [], [], s0
        for m, u in reversed(maps):
            inc.append(s)
            s = m * s + u
            out.append(s)
        return inc, out, s

    def zero_start(maps, s0):
        inc, out, s = [], [], 0.0
        for m, u in maps:
            inc.append(s)
            s = m * s + u
            out.append(s)
        return inc, out, s

    def final_only(maps, s0):
        s = s0
        for m, u in maps:
            s = m * s + u
        return [], [], s

    return [inclusive, no_transitions, reversed_order, zero_start, final_only]


@pytest.mark.parametrize("mistake", _mistaken_scans(), ids=lambda f: f.__name__)
def test_scalar_example_rejects_each_listed_mistake(mistake):
    g = _gold()
    inc, out, fin = mistake([tuple(x) for x in g["maps"]], g["initial_state"])
    ok = (inc == g["incoming_states"] and out == g["outgoing_states"] and fin == g["final_state"])
    assert not ok


def test_matrix_scan_rejects_right_multiplication():
    rng = np.random.default_rng(3)
    M, U = rng.normal(size=(3, 1, 3, 3)), rng.normal(size=(3, 1, 3, 3))
    init = rng.normal(size=(1, 3, 3))
    res = oracle.kda_affine_scan(M, U, init)
    s = init[0]
    for i in range(3):
        s = s @ M[i, 0] + U[i, 0]  # the "S M_i" mistake
    assert rel(res["final_state"][0], s) > 1e-3


# ------------------------------------------------------------------------------------------
# Gate and beta activations
# ------------------------------------------------------------------------------------------

def test_gate_special_values():
    assert oracle.gate(0.0, 0.0, 0.0) == pytest.approx(-math.log(2.0), rel=1e-15)
    # large pre-activation: softplus(x) -> x
    assert oracle.gate(40.0, 1.5, 0.0) == pytest.approx(-math.exp(1.5) * 40.0, rel=1e-15)
    # very negative pre-activation: softplus(x) -> e^x
    assert oracle.gate(-40.0, 0.7, 0.0) == pytest.approx(-math.exp(0.7) * math.exp(-40.0), rel=1e-12)
    # softplus(x) - softplus(-x) = x
    for x in (-3.0, -0.25, 0.5, 7.0):
        assert oracle.gate(x, 0.0, 0.0) - oracle.gate(-x, 0.0, 0.0) == pytest.approx(-x, abs=1e-14)
    # raw_gate is the pre-activation BEFORE dt_bias: only their sum matters
    assert oracle.gate(0.3, 0.2, -1.1) == oracle.gate(-0.8, 0.2, 0.0)
    # a_log scales by exp(a_log)
    assert oracle.gate(0.9, math.log(16.0), 0.0) == pytest.approx(16.0 * oracle.gate(0.9, 0.0, 0.0), rel=1e-14)
    # far below: exp underflow gives an exactly zero log-gate (alpha = 1)
    assert oracle.gate(-800.0, 0.0, 0.0) == 0.0


def test_gate_safe_mode_clamps():
    assert oracle.gate(5.0, math.log(16.0), 0.0, "safe", -5.0) == -5.0
    unclamped = oracle.gate(-2.0, 0.0, 0.0)
    assert unclamped > -5.0
    assert oracle.gate(-2.0, 0.0, 0.0, "safe", -5.0) == unclamped
    for x in np.linspace(-10, 10, 41):
        assert oracle.gate(float(x), 2.0, 0.0, "safe", -5.0) >= -5.0


def test_beta_modes():
    assert oracle.beta(0.0) == 0.5
    for x in (-30.0, -2.0, 0.3, 4.0, 30.0):
        assert oracle.beta(x) + oracle.beta(-x) == pytest.approx(1.0, abs=1e-15)
        assert 0.0 <= oracle.beta(x) <= 1.0
    assert oracle.beta(0.37, "probability") == 0.37


# ------------------------------------------------------------------------------------------
# The recurrence
# ------------------------------------------------------------------------------------------

def _unit(rng, d):
    x = rng.normal(size=d)
    return x / np.linalg.norm(x)


def _one_seq(q, k, v, raw, beta_logits, S0, a_log=0.0, beta_mode="logits", gate_mode="original",
             lb=-5.0):
    T, dk = k.shape
    dv = v.shape[1]
    out, pool = oracle.kda_forward(q[:, None], k[:, None], v[:, None], raw[:, None],
                                   np.asarray(beta_logits)[:, None], np.array([a_log]),
                                   np.zeros((1, dk)), np.array([0, T]), S0[None, None],
                                   np.array([0]), beta_mode=beta_mode, gate_mode=gate_mode,
                                   gate_lower_bound=lb)
    return out[:, 0], pool[0, 0]


def test_overwrite_invariant():
    """Writing the same unit key twice with beta = 1 overwrites the stored value."""
    rng = np.random.default_rng(4)
    dk, dv = 5, 3
    k1 = _unit(rng, dk)
    v1, v2 = rng.normal(size=dv), rng.normal(size=dv)
    S0 = rng.normal(size=(dk, dv))
    raw = np.full((2, dk), -800.0)  # log-gate exactly 0: no decay
    ones = np.ones(2)
    # (k, v1) then (k, v2): reading along k gives v2, not v1 + v2
    out, S = _one_seq(np.stack([k1, k1]), np.stack([k1, k1]), np.stack([v1, v2]), raw, ones, S0,
                      beta_mode="probability")
    assert rel(out[0], v1) < 1e-14
    assert rel(out[1], v2) < 1e-14
    assert rel(k1 @ S, v2) < 1e-14
    # (k, v1) twice: the second write changes nothing
    _, S_once = _one_seq(k1[None], k1[None], v1[None], raw[:1], ones[:1], S0, beta_mode="probability")
    _, S_twice = _one_seq(np.stack([k1, k1]), np.stack([k1, k1]), np.stack([v1, v1]), raw, ones, S0,
                          beta_mode="probability")
    assert rel(S_twice, S_once) < 1e-14
    assert rel(k1 @ S_twice, v1) < 1e-14  # not 2 * v1
    # directions orthogonal to k keep their old content
    w = rng.normal(size=dk)
    w -= (w @ k1) * k1
    assert rel(w @ S_twice, w @ S0) < 1e-13


def test_identity_case():
    """alpha = 1 and beta = 0: the state never changes and o_t = q_t^T S0."""
    rng = np.random.default_rng(5)
    T, dk, dv = 7, 4, 6
    q, k, v = rng.normal(size=(T, dk)), rng.normal(size=(T, dk)), rng.normal(size=(T, dv))
    S0 = rng.normal(size=(dk, dv))
    out, S = _one_seq(q, k, v, np.full((T, dk), -800.0), np.zeros(T), S0, beta_mode="probability")
    assert np.array_equal(S, S0)
    assert rel(out, q @ S0) < 1e-15


def test_beta_zero_is_pure_decay():
    """beta = 0: S_t = Diag(exp(G_t)) S0, with G_t the running sum of log-gates."""
    rng = np.random.default_rng(6)
    T, dk, dv = 9, 4, 3
    q, k, v = rng.normal(size=(T, dk)), rng.normal(size=(T, dk)), rng.normal(size=(T, dv))
    raw = rng.normal(size=(T, dk))
    S0 = rng.normal(size=(dk, dv))
    a_log = 0.8
    out, S = _one_seq(q, k, v, raw, np.zeros(T), S0, a_log=a_log, beta_mode="probability")
    g = np.array([[oracle.gate(raw[t, i], a_log, 0.0) for i in range(dk)] for t in range(T)])
    G = np.cumsum(g, axis=0)
    for t in range(T):
        assert rel(out[t], (q[t] * np.exp(G[t])) @ S0) < 1e-13
    assert rel(S, np.exp(G[-1])[:, None] * S0) < 1e-13


def test_readout_of_written_key_with_beta_one():
    """q = k (unit) and beta = 1: the readout returns exactly the value just written."""
    rng = np.random.default_rng(7)
    T, dk, dv = 12, 6, 5
    k = np.stack([_unit(rng, dk) for _ in range(T)])
    v = rng.normal(size=(T, dv))
    out, _ = _one_seq(k, k, v, rng.normal(size=(T, dk)) * 2, np.ones(T), rng.normal(size=(dk, dv)),
                      a_log=1.3, beta_mode="probability")
    assert rel(out, v) < 1e-13


def test_transition_matrix_form():
    """Each step equals S <- (I - b k k^T) Diag(a) S + b k v^T, o = S^T q (brute force)."""
    rng = np.random.default_rng(8)
    T, dk, dv = 10, 5, 4
    q, k, v = rng.normal(size=(T, dk)), rng.normal(size=(T, dk)), rng.normal(size=(T, dv))
    raw, logits = rng.normal(size=(T, dk)), rng.normal(size=T)
    S0 = rng.normal(size=(dk, dv))
    a_log = 0.4
    out, S = _one_seq(q, k, v, raw, logits, S0, a_log=a_log)
    s = S0.copy()
    for t in range(T):
        # gate and beta written out independently with the math module
        alpha = np.array([math.exp(-math.exp(a_log) * math.log1p(math.exp(raw[t, i]))) for i in range(dk)])
        b = 1.0 / (1.0 + math.exp(-logits[t]))
        s = (np.eye(dk) - b * np.outer(k[t], k[t])) @ np.diag(alpha) @ s + b * np.outer(k[t], v[t])
        assert rel(out[t], s.T @ q[t]) < 1e-12
    assert rel(S, s) < 1e-12


def test_scalar_recurrence_by_hand():
    """dk = dv = 1 in plain Python floats."""
    rng = np.random.default_rng(9)
    T = 20
    q, k, v = rng.normal(size=(T, 1)), rng.normal(size=(T, 1)), rng.normal(size=(T, 1))
    raw, logits = rng.normal(size=(T, 1)), rng.normal(size=T)
    out, S = _one_seq(q, k, v, raw, logits, np.array([[0.7]]), a_log=0.2)
    s = 0.7
    for t in range(T):
        a = math.exp(-math.exp(0.2) * math.log1p(math.exp(raw[t, 0])))
        b = 1.0 / (1.0 + math.exp(-logits[t]))
        s = a * s
        pred = k[t, 0] * s
        s = s + k[t, 0] * b * (v[t, 0] - pred)
        assert out[t, 0] == pytest.approx(q[t, 0] * s, rel=1e-13, abs=1e-15)
    assert S[0, 0] == pytest.approx(s, rel=1e-13)


def test_prediction_uses_decayed_state():
    """A mistaken order (predict before decaying) differs from the oracle."""
    rng = np.random.default_rng(10)
    dk, dv = 3, 2
    k = _unit(rng, dk)
    v = rng.normal(size=dv)
    S0 = rng.normal(size=(dk, dv))
    raw = np.full((1, dk), 1.0)
    out, S = _one_seq(k[None], k[None], v[None], raw, np.ones(1), S0, beta_mode="probability")
    a = np.exp([oracle.gate(1.0, 0.0, 0.0)] * dk)
    wrong = np.diag(a) @ S0 + np.outer(k, v - k @ S0)
    assert rel(out[0], v) < 1e-14          # decayed prediction: exact overwrite along k
    assert rel(S, wrong) > 1e-3


# ------------------------------------------------------------------------------------------
# Varlen, pool, layouts, heads, resume
# ------------------------------------------------------------------------------------------

def test_varlen_pool_independence_and_untouched_slots():
    w = tiny([5, 0, 9, 1], Hk=1, Hv=2, dk=4, dv=3, seed=11, max_slots=7,
             state_indices=torch.tensor([3, 0, 6, 2], dtype=torch.int32))
    out, pool = run(w)
    pool0 = w.state_pool.double().numpy()
    for s in (1, 4, 5):
        assert np.array_equal(pool[s], pool0[s])
    assert np.array_equal(pool[0], pool0[0])  # zero-length sequence: slot unchanged
    cu = w.cu_seqlens.tolist()
    for b, slot in enumerate(w.state_indices.tolist()):
        t0, t1 = cu[b], cu[b + 1]
        if t1 == t0:
            continue
        o1, p1 = oracle.kda_forward(w.q[t0:t1], w.k[t0:t1], w.v[t0:t1], w.raw_gate[t0:t1],
                                    w.beta_logits[t0:t1], w.a_log, w.dt_bias, [0, t1 - t0],
                                    w.state_pool[slot:slot + 1], [0])
        assert np.array_equal(out[t0:t1], o1)
        assert np.array_equal(pool[slot], p1[0])


def test_v_first_is_transposed_k_first():
    wk = tiny([13, 6], Hv=2, seed=12, max_slots=3, state_indices=torch.tensor([2, 0], dtype=torch.int32))
    wv = tiny([13, 6], Hv=2, seed=12, max_slots=3, state_indices=torch.tensor([2, 0], dtype=torch.int32),
              state_layout="V_FIRST")
    wv.state_pool = wk.state_pool.transpose(2, 3).contiguous()
    ok, pk = run(wk)
    ov, pv = run(wv)
    assert np.array_equal(ok, ov)
    assert np.array_equal(np.swapaxes(pk, 2, 3), pv)


def test_grouped_heads_map_to_contiguous_groups():
    w = tiny([11], Hk=2, Hv=4, seed=13)
    out, pool = run(w)
    w2 = tiny([11], Hk=2, Hv=4, seed=13)
    w2.q = w.q.repeat_interleave(2, dim=1)
    w2.k = w.k.repeat_interleave(2, dim=1)
    out2, pool2 = run(w2)
    assert np.array_equal(out, out2) and np.array_equal(pool, pool2)


def test_split_call_resumes_from_pool():
    w = tiny([40], Hv=2, seed=14)
    out, pool = run(w)
    for t1 in (16, 23):
        o_a, p_a = oracle.kda_forward(w.q[:t1], w.k[:t1], w.v[:t1], w.raw_gate[:t1],
                                      w.beta_logits[:t1], w.a_log, w.dt_bias, [0, t1], w.state_pool)
        o_b, p_b = oracle.kda_forward(w.q[t1:], w.k[t1:], w.v[t1:], w.raw_gate[t1:],
                                      w.beta_logits[t1:], w.a_log, w.dt_bias, [0, 40 - t1], p_a)
        assert rel(np.concatenate([o_a, o_b]), out) < 1e-14
        assert rel(p_b, pool) < 1e-14


def test_decode_steps_equal_the_prefill():
    # kda_decode is the single-token path of the same recurrence ("max.nn.state_space.kda_chunk"):
    # stepping each sequence one token at a time through its pool slot equals one prefill call
    w = tiny([9, 9, 9], Hk=1, Hv=2, dk=5, dv=4, seed=31, max_slots=4,
             state_indices=torch.tensor([3, 0, 2], dtype=torch.int32), state_layout="V_FIRST")
    out, pool = run(w)
    p = w.state_pool
    steps = []
    for t in range(9):
        rows = [0 + t, 9 + t, 18 + t]
        o, p = oracle.kda_decode(w.q[rows], w.k[rows], w.v[rows], w.raw_gate[rows], w.beta_logits[rows], w.a_log,
                                 w.dt_bias, p, w.state_indices, state_layout="V_FIRST")
        steps.append(o)
    got = np.stack(steps, axis=1).reshape(27, 2, 4)
    assert rel(got, out) < 1e-14
    assert rel(p, pool) < 1e-14
    assert np.array_equal(p[1], np.asarray(w.state_pool[1], np.float64))  # unnamed slot untouched


@pytest.mark.parametrize("chunk", [1, 2, 4, 16])
@pytest.mark.parametrize("gate_mode,raw_std", [("original", 1.0), ("original", 3.0), ("safe", 2.0)])
def test_chunked_algebra_equals_recurrence(chunk, gate_mode, raw_std):
    w = tiny([1, 15, 16, 17, 64], Hk=1, Hv=2, dk=6, dv=5, seed=15 + chunk, raw_std=raw_std,
             gate_mode=gate_mode, max_slots=6,
             state_indices=torch.tensor([4, 1, 0, 5, 2], dtype=torch.int32))
    o_r, p_r = run(w)
    o_c, p_c = chunked.kda_forward_chunked(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log,
                                           w.dt_bias, w.cu_seqlens, w.state_pool, w.state_indices,
                                           chunk=chunk, gate_mode=gate_mode,
                                           gate_lower_bound=w.gate_lower_bound)
    assert rel(o_c, o_r) < 1e-12
    assert rel(p_c, p_r) < 1e-12


# ------------------------------------------------------------------------------------------
# Segment summaries
# ------------------------------------------------------------------------------------------

def _segments(T=50, N=4, Hv=2, dk=4, dv=3, seed=20, layout="K_FIRST", **kw):
    w = tiny([T], Hk=1, Hv=Hv, dk=dk, dv=dv, seed=seed, state_layout=layout, **kw)
    offs = np.array([0, 9, 9 + 16, 9 + 16 + 1, T][: N + 1])
    offs[-1] = T
    M, U = oracle.kda_segment_summary(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs,
                                      gate_mode=w.gate_mode, state_layout=layout)
    return w, offs, M, U


def test_segment_map_is_affine_in_the_incoming_state():
    w, offs, M, U = _segments()
    rng = np.random.default_rng(21)
    for i in range(len(offs) - 1):
        t0, t1 = offs[i], offs[i + 1]
        S = rng.normal(size=(1, 2, 4, 3))
        _, pool = oracle.kda_forward(w.q[t0:t1], w.k[t0:t1], w.v[t0:t1], w.raw_gate[t0:t1],
                                     w.beta_logits[t0:t1], w.a_log, w.dt_bias, [0, t1 - t0], S)
        for h in range(2):
            assert rel(pool[0, h], M[i, h] @ S[0, h] + U[i, h]) < 1e-12


def test_segment_transition_with_beta_zero_is_diagonal_decay():
    w, offs, M, U = _segments(beta_mode="probability")
    w.beta_logits.zero_()
    M, U = oracle.kda_segment_summary(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs,
                                      beta_mode="probability")
    assert np.all(U == 0.0)
    for i in range(len(offs) - 1):
        for h in range(2):
            g = [[oracle.gate(float(w.raw_gate[t, h, c]), float(w.a_log[h]), float(w.dt_bias[h, c]))
                  for c in range(4)] for t in range(offs[i], offs[i + 1])]
            diag = np.exp(np.sum(np.array(g).reshape(-1, 4), axis=0))
            assert rel(M[i, h], np.diag(diag)) < 1e-13


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_sequential_equals_scanned(layout):
    w, offs, M, U = _segments(layout=layout, state_std=0.7)
    S_init = w.state_pool[0].double().numpy()
    out_straight, pool_straight = run(w)
    res = oracle.kda_affine_scan(M, U, S_init, state_layout=layout)
    assert rel(res["final_state"], pool_straight[0]) < 1e-12
    # second pass: every segment as its own sequence, its incoming state as its pool slot
    N = len(offs) - 1
    out_cp, pool_cp = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log,
                                         w.dt_bias, offs, res["incoming_states"], np.arange(N),
                                         state_layout=layout)
    assert rel(out_cp, out_straight) < 1e-12
    assert rel(pool_cp, res["outgoing_states"]) < 1e-12


def test_planted_scan_mistakes_fail_the_segment_check():
    # slow decay and weak writes so the incoming state still matters at the sequence end
    w, offs, M, U = _segments(state_std=0.7, a_log_range=(-3.0, -2.0), beta_mean=-3.0)
    S_init = w.state_pool[0].double().numpy()
    _, pool_straight = run(w)
    target = pool_straight[0]
    N = len(offs) - 1

    def scan(step, start):
        s = start.copy()
        for i in range(N):
            s = np.stack([step(M[i, h], U[i, h], s[h]) for h in range(2)])
        return s

    good = scan(lambda m, u, s: m @ s + u, S_init)
    assert rel(good, target) < 1e-12
    assert rel(scan(lambda m, u, s: s + u, S_init), target) > 1e-3          # no transitions
    assert rel(scan(lambda m, u, s: m @ s + u, np.zeros_like(S_init)), target) > 1e-3  # zero start
    rev = S_init.copy()
    for i in reversed(range(N)):
        rev = np.stack([M[i, h] @ rev[h] + U[i, h] for h in range(2)])
    assert rel(rev, target) > 1e-3                                            # reversed order
