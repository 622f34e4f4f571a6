"""GPU parity of the segment summaries, the exclusive scan and the context-parallel prefill.

Against the fp64 oracle: M_i (recurrence from I with zero values), U_i (recurrence from 0),
the scan's incoming / outgoing / final states, and the second pass (every segment as its own
sequence, starting from its incoming state) against the straight token-by-token recurrence.
"""
import json
import os

import numpy as np
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def rel_l2(x, ref):
    x = x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def test_scalar_three_segment_example_on_gpu():
    with open(os.path.join(GOLD, "scalar_three_segments.json")) as f:
        g = json.load(f)
    M = torch.tensor([[[m]] for m, _ in g["maps"]], dtype=torch.float32, device="cuda")
    U = torch.tensor([[[u]] for _, u in g["maps"]], dtype=torch.float32, device="cuda")
    S0 = torch.tensor([[g["initial_state"]]], dtype=torch.float32, device="cuda")
    copies = [t.clone() for t in (M, U, S0)]
    res = kda.kda_context_parallel(M, U, S0)
    torch.cuda.synchronize()
    assert set(res) == {"incoming_states", "outgoing_states", "final_state"}
    assert res["incoming_states"].flatten().tolist() == g["incoming_states"]
    assert res["outgoing_states"].flatten().tolist() == g["outgoing_states"]
    assert res["final_state"].item() == g["final_state"]
    assert res["final_state"].dtype == torch.float32 and res["final_state"].device.type == "cuda"
    for t, c in zip((M, U, S0), copies):
        assert torch.equal(t, c)


def test_scan_only_matches_oracle_scan():
    rng = np.random.default_rng(0)
    N, H, dk, dv = 5, 3, 128, 128
    M = rng.normal(size=(N, H, dk, dk)) / np.sqrt(dk)
    U = rng.normal(size=(N, H, dk, dv))
    S0 = rng.normal(size=(H, dk, dv))
    ref = oracle.kda_affine_scan(M, U, S0)
    cu = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda")  # noqa: E731
    res = kda.kda_context_parallel(cu(M), cu(U), cu(S0))
    for key in ref:
        parity.check_states(f"scan only: {key}", res[key], ref[key], 1e-5)


CASES = [
    (torch.float32, 16, "K_FIRST", 1e-4),
    (torch.float32, 32, "V_FIRST", 1e-4),
    (torch.bfloat16, 128, "K_FIRST", 1e-2),
    (torch.bfloat16, 128, "V_FIRST", 1e-2),
]


@pytest.mark.parametrize("dtype,d,layout,tol", CASES)
def test_segment_summaries_and_scan(dtype, d, layout, tol):
    T = 300
    w = W.random_inputs([T], 2, 2, d, d, seed=d, qkv_dtype=dtype, state_std=0.2, state_layout=layout,
                        output_dtype=dtype)
    offs = torch.tensor([0, 37, 100, 164, 300], dtype=torch.int32)
    wd = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = kda.kda_segment_summarize_and_scan(wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias,
                                             offs.cuda(), wd.state_pool[0].contiguous(), state_layout=layout,
                                             device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    M, U = oracle.kda_segment_summary(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs,
                                      state_layout=layout)
    ref = oracle.kda_affine_scan(M, U, w.state_pool[0], state_layout=layout)
    lab = f"segment summaries {'fp32' if dtype == torch.float32 else 'bf16'}"
    parity.check_maps(f"{lab}: M", res["transition_matrices"], M, tol)
    parity.check_states(f"{lab}: U", res["local_contributions"], U, tol)
    parity.check_states(f"{lab}: incoming", res["incoming_states"], ref["incoming_states"], tol)
    parity.check_states(f"{lab}: outgoing", res["outgoing_states"], ref["outgoing_states"], tol)
    parity.check_states(f"{lab}: final", res["final_state"], ref["final_state"], tol)


def _cp_prefill(wd, offs, init, layout="K_FIRST", gate_mode="original", lb=-5.0):
    N = offs.numel() - 1
    res = kda.kda_segment_summarize_and_scan(wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, offs,
                                             init, state_layout=layout, gate_mode=gate_mode, gate_lower_bound=lb)
    pool = res["incoming_states"].clone()
    out = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, offs, pool,
                            torch.arange(N, dtype=torch.int32, device=wd.q.device), state_layout=layout,
                            gate_mode=gate_mode, gate_lower_bound=lb)
    torch.cuda.synchronize()
    return out, pool, res


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_context_parallel_prefill_matches_straight_recurrence(layout):
    w = W.random_inputs([1000], 2, 2, 128, 128, seed=3, state_std=0.1, state_layout=layout)
    wd = w.to("cuda")
    offs = torch.tensor([0, 250, 500, 777, 1000], dtype=torch.int32, device="cuda")
    out, pool, res = _cp_prefill(wd, offs, wd.state_pool[0].contiguous(), layout)
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices, state_layout=layout)
    parity.check_rows("two-pass context parallel: out", out, o_ref, 1e-2)
    parity.check_states("two-pass context parallel: final", res["final_state"], p_ref[0], 1e-2)
    parity.check_states("two-pass context parallel: final", pool[-1], p_ref[0], 1e-2)
    # the second pass ends every segment in the scan's outgoing state
    parity.check_states("two-pass: pass 2 vs scan outgoing", pool, res["outgoing_states"], 1e-2)


def test_full_size_context_parallel_sampled_heads():
    """The benchmark's launch configuration: 131072 tokens, 32 heads, 16 segments of 8192."""
    w = W.make("long_T131072_H32_cp16", device="cuda")
    out, pool, res = _cp_prefill(w, w.seg_offsets, w.state_pool[0])
    heads = [2, 21]
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    o_ref, p_ref = oracle.kda_forward(cpu(w.q)[:, heads], cpu(w.k)[:, heads], cpu(w.v)[:, heads],
                                      cpu(w.raw_gate)[:, heads], cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads],
                                      cpu(w.dt_bias)[heads], cpu(w.cu_seqlens), cpu(w.state_pool)[:, heads],
                                      cpu(w.state_indices))
    parity.check_rows("long_T131072_H32_cp16 two-pass: out", out[:, heads], o_ref, 1e-2)
    parity.check_states("long_T131072_H32_cp16 two-pass: final", res["final_state"][heads], p_ref[0], 1e-2)


@pytest.mark.parametrize("layout,out_dtype", [("K_FIRST", torch.bfloat16), ("V_FIRST", torch.float32)])
def test_context_parallel_prefill_entry_point(layout, out_dtype):
    w = W.random_inputs([1000], 2, 2, 128, 128, seed=4, state_std=0.1, state_layout=layout)
    wd = w.to("cuda")
    offs = torch.tensor([0, 64, 300, 301, 777, 1000], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = kda.kda_context_parallel_prefill(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias,
                                           offs, wd.state_pool[0].contiguous(), output_dtype=out_dtype,
                                           state_layout=layout, device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices, state_layout=layout)
    assert res["out"].dtype == out_dtype
    parity.check_rows("context-parallel prefill: out", res["out"], o_ref, 1e-2)
    parity.check_states("context-parallel prefill: final", res["final_state"], p_ref[0], 1e-2)
    M, U = oracle.kda_segment_summary(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs.cpu(),
                                      state_layout=layout)
    parity.check_maps("context-parallel prefill: M", res["transition_matrices"], M, 1e-2)
    parity.check_states("context-parallel prefill: U", res["local_contributions"], U, 1e-2)


def test_full_size_context_parallel_prefill_sampled_heads():
    """The benchmark's step: 131072 tokens, 32 heads, 16 segments, one entry point.  Besides the
    outputs and the final state, every segment's M_i, U_i and its incoming and outgoing states
    are compared with the oracle's own summaries (each segment replayed from I and from 0) and
    its scan -- on the sampled heads, at full length."""
    w = W.make("long_T131072_H32_cp16", device="cuda")
    res = kda.kda_context_parallel_prefill(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                           w.seg_offsets, w.state_pool[0])
    torch.cuda.synchronize()
    heads = [9, 30]
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    o_ref, p_ref = oracle.kda_forward(cpu(w.q)[:, heads], cpu(w.k)[:, heads], cpu(w.v)[:, heads],
                                      cpu(w.raw_gate)[:, heads], cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads],
                                      cpu(w.dt_bias)[heads], cpu(w.cu_seqlens), cpu(w.state_pool)[:, heads],
                                      cpu(w.state_indices))
    lab = "long_T131072_H32_cp16"
    parity.check_rows(f"{lab}: out", res["out"][:, heads], o_ref, 1e-2)
    parity.check_states(f"{lab}: final", res["final_state"][heads], p_ref[0], 1e-2)
    M, U = oracle.kda_segment_summary(cpu(w.k)[:, heads], cpu(w.v)[:, heads], cpu(w.raw_gate)[:, heads],
                                      cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads], cpu(w.dt_bias)[heads],
                                      cpu(w.seg_offsets))
    scan = oracle.kda_affine_scan(M, U, cpu(w.state_pool)[0, heads])
    parity.check_maps(f"{lab}: M", res["transition_matrices"][:, heads], M, 1e-2)
    parity.check_states(f"{lab}: U", res["local_contributions"][:, heads], U, 1e-2)
    parity.check_states(f"{lab}: incoming", res["incoming_states"][:, heads], scan["incoming_states"], 1e-2)
    parity.check_states(f"{lab}: outgoing", res["outgoing_states"][:, heads], scan["outgoing_states"], 1e-2)


# ------------------------------------------------------------------------------------------
# Segments built as pieces: boundaries, composition, and the split prefill
# ------------------------------------------------------------------------------------------

def _piece_rule(offs, k):
    """The documented boundaries: piece p of [s0, s1) starts at s0 + 64 floor(nch p / k)."""
    out = []
    for i in range(len(offs) - 1):
        s0, s1 = offs[i], offs[i + 1]
        nch = (s1 - s0 + 63) // 64 if s1 > s0 else 0
        out += [min(s0 + 64 * ((nch * p) // k), s1) if s1 > s0 else s0 for p in range(k)]
    return out + [offs[-1]]


@pytest.mark.parametrize("k", [1, 2, 3, 8])
def test_piece_offsets_follow_the_documented_rule(k):
    offs = [0, 0, 1, 64, 65, 1000, 8192, 8200]
    d = torch.tensor(offs, dtype=torch.int32, device="cuda")
    got = kda.kda_context_parallel_piece_offsets(d, k)
    torch.cuda.synchronize()
    assert got.cpu().tolist() == _piece_rule(offs, k)


@pytest.mark.parametrize("dk,dv,layout", [(128, 128, "K_FIRST"), (40, 24, "V_FIRST")])
def test_compose_matches_oracle_composition(dk, dv, layout):
    rng = np.random.default_rng(dk + dv)
    N, k, H = 3, 3, 2
    st = (dk, dv) if layout == "K_FIRST" else (dv, dk)
    Mp = rng.normal(size=(N * k, H, dk, dk)) / np.sqrt(dk)
    Up = rng.normal(size=(N * k, H, *st))
    Ip = rng.normal(size=(N * k + 1, H, *st))
    fin = rng.normal(size=(H, *st))
    cu = lambda x: torch.tensor(x, dtype=torch.float32, device="cuda")  # noqa: E731
    res = kda.kda_segment_compose(cu(Mp), cu(Up), cu(Ip), cu(fin), k, state_layout=layout)
    torch.cuda.synchronize()
    kf = (lambda u: u) if layout == "K_FIRST" else (lambda u: u.T)  # noqa: E731
    for i in range(N):
        for h in range(H):
            Mc, Uc = Mp[i * k, h], kf(Up[i * k, h])
            for p in range(1, k):
                Mc, Uc = oracle.kda_compose((Mp[i * k + p, h], kf(Up[i * k + p, h])), (Mc, Uc))
            assert rel_l2(res["transition_matrices"][i, h], Mc) < 1e-5
            assert rel_l2(kf(res["local_contributions"][i, h].cpu().double().numpy()), Uc) < 1e-5
            assert torch.equal(res["incoming_states"][i, h].cpu(), cu(Ip[i * k, h]).cpu())
            nxt = Ip[(i + 1) * k, h] if i + 1 < N else fin[h]
            assert torch.equal(res["outgoing_states"][i, h].cpu(), cu(nxt).cpu())


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_split_prefill_matches_oracle_and_unsplit(layout):
    """4096 tokens, 2 heads, 4 segments (one of a single token): 8 chains, so every segment is
    built as several pieces; results against the oracle and against the unsplit prefill."""
    T, H = 4096, 2
    w = W.random_inputs([T], H, H, 128, 128, seed=12, state_std=0.1, state_layout=layout)
    wd = w.to("cuda")
    offs = torch.tensor([0, 1000, 1001, 2500, T], dtype=torch.int32, device="cuda")
    N = offs.numel() - 1
    pieces = kda.kda_context_parallel_pieces(T, N, H)
    assert pieces > 1
    init = wd.state_pool[0].contiguous()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    split = kda.kda_context_parallel_prefill(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias,
                                             offs, init, state_layout=layout, device_status=status)
    ws = torch.empty(kda.kda_context_parallel_workspace_size(T, H, 128), dtype=torch.uint8, device="cuda")
    assert ws.numel() < kda.kda_context_parallel_workspace_preferred(T, N, H, 128)
    whole = kda.kda_context_parallel_prefill(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias,
                                             offs, init, state_layout=layout, workspace=ws, device_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices, state_layout=layout)
    M, U = oracle.kda_segment_summary(w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs.cpu(),
                                      state_layout=layout)
    scan = oracle.kda_affine_scan(M, U, w.state_pool[0].double().numpy(), state_layout=layout)
    for name, res in (("pieces", split), ("whole segments", whole)):
        lab = f"context parallel ({name})"
        parity.check_rows(f"{lab}: out", res["out"], o_ref, 1e-2)
        parity.check_states(f"{lab}: final", res["final_state"], p_ref[0], 1e-2)
        parity.check_maps(f"{lab}: M", res["transition_matrices"], M, 1e-2)
        parity.check_states(f"{lab}: U", res["local_contributions"], U, 1e-2)
        parity.check_states(f"{lab}: incoming", res["incoming_states"], scan["incoming_states"], 1e-2)
        parity.check_states(f"{lab}: outgoing", res["outgoing_states"], scan["outgoing_states"], 1e-2)
    assert rel_l2(split["out"], whole["out"].double().cpu().numpy()) < 1e-2


@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_head_major_readouts_equal_token_major(out_dtype):
    """KDA_READOUT_HEAD_MAJOR stores the same readouts as [Hv, T, 128]: bit for bit the
    token-major ones transposed, and the apply gives the same outputs from either layout
    (ragged segments: partial chunks in the build, partial tiles in the apply)."""
    w = W.random_inputs([1500], 2, 4, 128, 128, seed=31, state_std=0.1)
    wd = w.to("cuda")
    offs = torch.tensor([0, 130, 131, 700, 1500], dtype=torch.int32, device="cuda")
    init = wd.state_pool[0].contiguous()
    res = {}
    for layout in ("token_major", "head_major"):
        r = kda.kda_segment_summarize_and_scan(wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, offs,
                                               init, q=wd.q, readout_layout=layout)
        out = kda.kda_context_parallel_apply(r["readout_m"], r["readout_u"], r["incoming_states"], offs,
                                             output_dtype=out_dtype, readout_layout=layout)
        res[layout] = (r, out)
    torch.cuda.synchronize()
    (rt, ot), (rh, oh) = res["token_major"], res["head_major"]
    assert rh["readout_m"].shape == (4, 1500, 128)
    assert torch.equal(rh["readout_m"], rt["readout_m"].transpose(0, 1))
    assert torch.equal(rh["readout_u"], rt["readout_u"].transpose(0, 1))
    assert torch.equal(oh, ot)
    o_ref, _ = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                  w.state_pool, w.state_indices)
    parity.check_rows("head-major readouts: out", oh, o_ref, 1e-2)
