"""kda_chunk_fwd's split route: sequences cut into pieces, built in parallel, applied in order
from their pool slots.  Against the fp64 oracle (bf16 tolerance), against the plain route, and
with the device-side checks that send a batch back to the plain route.

Which route ran is read from the planner's flag, the first word of the workspace's last
256-byte block (0: the pieces ran, 1: the plain kernel ran).
"""
import numpy as np
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu

TOL = 1e-2


def rel_l2(x, ref):
    x = x.double().cpu().numpy() if isinstance(x, torch.Tensor) else np.asarray(x, np.float64)
    ref = ref.double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def run(w, workspace=None, status=None):
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    if workspace is None:
        T, Hk, dk = wd.q.shape
        need = kda.kda_workspace_size(T, wd.batch, Hk, wd.num_v_heads, dk, wd.dv)
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    out = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens,
                            pool, wd.state_indices, output_dtype=w.output_dtype, gate_mode=w.gate_mode,
                            beta_mode=w.beta_mode, state_layout=w.state_layout,
                            gate_lower_bound=w.gate_lower_bound, workspace=workspace, device_status=status)
    torch.cuda.synchronize()
    return out, pool, workspace


def split_ran(ws):
    return ws.numel() > 0 and int(ws[-256:-252].view(torch.int32).item()) == 0


def check_against_oracle(w, out, pool, label="split route"):
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                                      state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    cu = w.cu_seqlens.tolist()
    s, e = cu[0], cu[-1]
    parity.check_rows(f"{label}: out", out[s:e], o_ref[s:e], TOL, cu=[c - s for c in cu])
    touched = sorted(set(w.state_indices.tolist()))
    parity.check_states(f"{label}: final state", pool[touched], p_ref[touched], TOL)
    untouched = [i for i in range(w.state_pool.shape[0]) if i not in touched]
    if untouched:
        assert torch.equal(pool[untouched].cpu(), w.state_pool[untouched])


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_single_long_sequence_takes_the_split_route(layout):
    w = W.random_inputs([4000], 4, 4, 128, 128, seed=21, state_std=0.1, state_layout=layout, max_slots=3,
                        state_indices=torch.tensor([2], dtype=torch.int32))
    out, pool, ws = run(w)
    assert split_ran(ws)
    check_against_oracle(w, out, pool, f"split route, one sequence ({layout})")
    plain_out, plain_pool, _ = run(w, workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    assert rel_l2(out, plain_out) <= TOL
    assert rel_l2(pool, plain_pool) <= TOL


def test_uneven_varlen_batch_with_empty_sequences():
    lengths = [3000, 0, 1, 700, 64, 2500, 0, 129]
    w = W.random_inputs(lengths, 2, 4, 128, 128, seed=22, state_std=0.1, max_slots=10,  # Hk = 2, Hv = 4
                        state_indices=torch.randperm(10, generator=torch.Generator().manual_seed(5))[:8].to(
                            torch.int32), output_dtype=torch.float32)
    out, pool, ws = run(w)
    assert split_ran(ws)
    assert out.dtype == torch.float32
    check_against_oracle(w, out, pool, "split route, uneven varlen")


def test_safe_gate_and_probability_beta_on_the_split_route():
    w = W.random_inputs([2100, 1900], 4, 4, 128, 128, seed=23, state_std=0.1, raw_std=2.0, beta_mean=2.0,
                        gate_mode="safe", gate_lower_bound=-5.0)
    w.beta_mode = "probability"
    w.beta_logits = torch.rand(w.beta_logits.shape, generator=torch.Generator().manual_seed(8))
    out, pool, ws = run(w)
    assert split_ran(ws)
    check_against_oracle(w, out, pool, "split route, safe gate")


def test_balanced_batch_gets_no_split_workspace():
    # 4 x 2048 tokens x 32 heads: 128 chains, more than half as many as SMs: no split is offered
    w = W.make("batch4_T2048_H32", device="cpu")
    assert kda.kda_workspace_size(w.total_tokens, w.batch, 32, 32, 128, 128) == 0


def test_short_sequences_keep_the_plain_route():
    # 8 chains of 5 chunks: the host offers the split, the planner (real lengths) refuses it
    w = W.random_inputs([300] * 4, 2, 2, 128, 128, seed=25, state_std=0.1)
    out, pool, ws = run(w)
    assert ws.numel() > 0 and not split_ran(ws)
    check_against_oracle(w, out, pool, "planner keeps the plain route")


def test_bad_slot_falls_back_to_the_plain_route_and_is_reported():
    w = W.random_inputs([3000, 500], 4, 4, 128, 128, seed=24, state_std=0.1, max_slots=3,
                        state_indices=torch.tensor([7, 1], dtype=torch.int32))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, pool, ws = run(w, status=status)
    assert not split_ran(ws)
    assert int(status.item()) == 5  # KDA_ERR_DEVICE_CHECK
    # the valid sequence (slot 1) ran, the bad one left everything untouched
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                      torch.tensor([3000, 3500], dtype=torch.int32), w.state_pool,
                                      torch.tensor([1], dtype=torch.int32))
    parity.check_rows("bad slot (split workspace): the valid sequence", out[3000:3500], o_ref[3000:3500], TOL)
    parity.check_states("bad slot (split workspace): its state", pool[1:2], p_ref[1:2], TOL)
    assert torch.equal(pool[0].cpu(), w.state_pool[0]) and torch.equal(pool[2].cpu(), w.state_pool[2])
