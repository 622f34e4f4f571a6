"""GPU parity of the per-rank context-parallel calls (kda_context_parallel_range_summary /
kda_context_parallel_range_finish, through the C ABI) against the fp64 oracle.

Several ranks are emulated on one GPU at the level of the calls: every rank's range summary,
then the gather (a stack, as the all-gather would leave it on every rank), the scan over the
ranks, and every rank's finish.  No kernel waits on another rank.  One test runs the real
exchange (``distributed.context_parallel_prefill``) in a one-rank NCCL group.  Tolerances as
for the single-GPU context-parallel prefill: relative L2 1e-2 (bf16 q/k/v and readouts).
"""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity
from kimi_delta_attention_23_b200 import distributed as D

pytestmark = pytest.mark.gpu

TOL = 1e-2


def rel_l2(x, ref):
    x = x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = ref.double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def local_offsets(n, fracs=(0.37,), short=False):
    # the range's own segments; with short=True one of them is a single token (with this gate
    # distribution only a short segment keeps a transition far from zero: a long one decays to
    # below fp32's range, and then relative errors of M say nothing)
    cuts = [0] + [64 * int(n * f / 64) for f in fracs] + [n]
    if short and n > 65:
        cuts = sorted(cuts + [64, 65])
    return torch.tensor(cuts, dtype=torch.int32, device="cuda")


def emulate(w, world, layout, fracs=(0.37,), gate_mode="original", lb=-5.0, output_dtype=torch.bfloat16,
            short=False):
    """Every rank's calls, in the order a real run makes them, on one GPU."""
    T = w.q.shape[0]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    kw = dict(state_layout=layout, gate_mode=gate_mode, gate_lower_bound=lb, device_status=st)
    ranges = D.rank_ranges(T, world)
    sums = []
    for s, e in ranges:
        offs = local_offsets(e - s, fracs, short)
        r = kda.kda_context_parallel_range_summary(w.q[s:e], w.k[s:e], w.v[s:e], w.raw_gate[s:e],
                                                   w.beta_logits[s:e], w.a_log, w.dt_bias, offs, **kw)
        sums.append((r, offs))
    M_all = torch.stack([r["range_transition"] for r, _ in sums])
    U_all = torch.stack([r["range_contribution"] for r, _ in sums])
    scan = kda.kda_context_parallel(M_all, U_all, w.state_pool[0].contiguous(), state_layout=layout)
    fins = []
    for i, ((s, e), (r, offs)) in enumerate(zip(ranges, sums)):
        fins.append(kda.kda_context_parallel_range_finish(scan["incoming_states"][i].contiguous(), r["workspace"],
                                                          offs, e - s, output_dtype=output_dtype,
                                                          state_layout=layout, device_status=st))
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    return ranges, sums, scan, fins


def straight(w, layout, heads=None, gate_mode="original", lb=-5.0, upto=None):
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    T = w.q.shape[0] if upto is None else upto
    Hv, Hk = w.v.shape[1], w.q.shape[1]
    heads = list(range(Hv)) if heads is None else heads
    kh = [h // (Hv // Hk) for h in heads]
    return oracle.kda_forward(cpu(w.q)[:T, kh], cpu(w.k)[:T, kh], cpu(w.v)[:T, heads], cpu(w.raw_gate)[:T, heads],
                              cpu(w.beta_logits)[:T, heads], cpu(w.a_log)[heads], cpu(w.dt_bias)[heads],
                              np.array([0, T], np.int32), cpu(w.state_pool)[:, heads], np.array([0], np.int32),
                              state_layout=layout, gate_mode=gate_mode, gate_lower_bound=lb)


@pytest.mark.parametrize("world,T,layout", [(1, 1500, "K_FIRST"), (2, 1500, "V_FIRST"), (4, 3000, "K_FIRST"),
                                            (3, 100, "K_FIRST")])
def test_emulated_ranks_match_the_straight_recurrence(cuda_device, world, T, layout):
    w = W.random_inputs([T], 2, 4, 128, 128, seed=T + world, state_std=0.1, state_layout=layout).to("cuda")
    ranges, sums, scan, fins = emulate(w, world, layout)
    out = torch.cat([f["out"] for f in fins])
    o_ref, p_ref = straight(w, layout)
    parity.check_rows("emulated ranks: out", out, o_ref, TOL)
    parity.check_states("emulated ranks: final", scan["final_state"], p_ref[0], TOL)
    for i, ((s, e), f) in enumerate(zip(ranges, fins)):
        assert rel_l2(f["range_outgoing"], scan["outgoing_states"][i]) < 1e-4  # the range's end, two ways
        if s > 0:
            _, p_s = straight(w, layout, upto=s)
            parity.check_states("emulated ranks: incoming of a rank", scan["incoming_states"][i], p_s[0], TOL)


def test_range_segments_match_oracle_summaries(cuda_device):
    # a rank's own segments: their maps and states, from the state entering the range
    layout = "K_FIRST"
    w = W.random_inputs([2000], 2, 2, 128, 128, seed=5, state_std=0.1).to("cuda")
    ranges, sums, scan, fins = emulate(w, 2, layout, fracs=(0.25, 0.6), short=True)
    for i, ((s, e), (_, offs), f) in enumerate(zip(ranges, sums, fins)):
        cpu = lambda t: t.detach().cpu()  # noqa: E731
        M, U = oracle.kda_segment_summary(cpu(w.k)[s:e], cpu(w.v)[s:e], cpu(w.raw_gate)[s:e],
                                          cpu(w.beta_logits)[s:e], cpu(w.a_log), cpu(w.dt_bias), cpu(offs))
        sc = oracle.kda_affine_scan(M, U, cpu(scan["incoming_states"][i]).double().numpy())
        parity.check_maps("rank segments: M", f["transition_matrices"], M, TOL)
        parity.check_states("rank segments: U", f["local_contributions"], U, TOL)
        parity.check_states("rank segments: incoming", f["incoming_states"], sc["incoming_states"], TOL)
        parity.check_states("rank segments: outgoing", f["outgoing_states"], sc["outgoing_states"], TOL)
        # the whole range's map is its segments' composed in order; over a thousand tokens the
        # transition has decayed to (fp32) zero, so it is checked in absolute terms
        Mr, Ur = oracle.kda_segment_summary(cpu(w.k)[s:e], cpu(w.v)[s:e], cpu(w.raw_gate)[s:e],
                                            cpu(w.beta_logits)[s:e], cpu(w.a_log), cpu(w.dt_bias),
                                            np.array([0, e - s], np.int32))
        assert np.abs(cpu(sums[i][0]["range_transition"]).double().numpy() - Mr[0]).max() < 1e-6
        parity.check_states("rank map: U", sums[i][0]["range_contribution"], Ur[0], TOL)


def test_safe_gate_fp32_output(cuda_device):
    w = W.random_inputs([1200], 2, 2, 128, 128, seed=9, state_std=0.1, raw_std=2.0, beta_mean=2.0,
                        gate_mode="safe").to("cuda")
    ranges, sums, scan, fins = emulate(w, 2, "K_FIRST", gate_mode="safe", output_dtype=torch.float32)
    out = torch.cat([f["out"] for f in fins])
    assert out.dtype == torch.float32
    o_ref, p_ref = straight(w, "K_FIRST", gate_mode="safe")
    parity.check_rows("emulated ranks, safe gate: out", out, o_ref, TOL)
    parity.check_states("emulated ranks, safe gate: final", scan["final_state"], p_ref[0], TOL)


def test_one_rank_equals_the_single_gpu_prefill(cuda_device):
    w = W.random_inputs([2500], 2, 4, 128, 128, seed=13, state_std=0.1).to("cuda")
    offs = local_offsets(2500)
    ranges, sums, scan, fins = emulate(w, 1, "K_FIRST")
    ref = kda.kda_context_parallel_prefill(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs,
                                           w.state_pool[0].contiguous())
    torch.cuda.synchronize()
    assert rel_l2(fins[0]["out"], ref["out"]) < 1e-2
    assert rel_l2(scan["final_state"], ref["final_state"]) < 1e-4
    for key in ("incoming_states", "outgoing_states", "transition_matrices", "local_contributions"):
        assert rel_l2(fins[0][key], ref[key]) < 1e-4, key


def test_full_size_eight_ranks_sampled_heads(cuda_device):
    """The 131072-token, 32-head sequence over eight emulated ranks, two segments each (the
    16-segment cut of the single-GPU benchmark); the oracle replays two heads."""
    w = W.make("long_T131072_H32_cp16", device="cuda")
    ranges, sums, scan, fins = emulate(w, 8, "K_FIRST", fracs=(0.5,))
    out = torch.cat([f["out"] for f in fins])
    heads = [0, 31]
    o_ref, p_ref = straight(w, "K_FIRST", heads=heads)
    parity.check_rows("long_T131072_H32 over 8 ranks: out", out[:, heads], o_ref, TOL)
    parity.check_states("long_T131072_H32 over 8 ranks: final", scan["final_state"][heads], p_ref[0], TOL)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_distributed_entry_in_a_one_rank_nccl_group(cuda_device):
    w = W.random_inputs([1000], 2, 2, 128, 128, seed=17, state_std=0.1).to("cuda")
    dist.init_process_group("nccl", rank=0, world_size=1, init_method=f"tcp://127.0.0.1:{_free_port()}",
                            device_id=torch.device("cuda:0"))
    try:
        res = D.context_parallel_prefill(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                         local_offsets(1000), w.state_pool[0].contiguous())
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    o_ref, p_ref = straight(w, "K_FIRST")
    parity.check_rows("one-rank NCCL group: out", res["out"], o_ref, TOL)
    parity.check_states("one-rank NCCL group: final", res["final_state"], p_ref[0], TOL)
    assert rel_l2(res["range_incoming"], w.state_pool[0]) == 0.0
