"""The bounded waits' error path, made to run out on purpose without a fault or a hang.

Every wait inside the fused bf16 kernel gives up after about one second, records
KDA_ERR_DEVICE_TIMEOUT in ``device_status`` and lets both warp teams leave their chunk loops, wait
(again bounded) for their own copies and products in flight, and free the tensor memory.  The
test hook ``DEBUG_WITHHOLD_HANDOFF`` withholds the key team's first "scores ready" signal in every
chain, so the state team's wait has nothing to wait for: the call must come back with the status,
and the next call on the same context must be correct (checked against the fp64 oracle).
"""
import time

import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu


def _run(w, debug_flags, pool):
    wd = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    no_split = torch.empty(0, dtype=torch.uint8, device="cuda")  # the fused kernel alone
    out = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens,
                            pool, wd.state_indices, output_dtype=w.output_dtype, state_layout=w.state_layout,
                            workspace=no_split, device_status=status, _debug_flags=debug_flags)
    torch.cuda.synchronize()
    return out, int(status.item())


def test_withheld_handoff_times_out_and_the_context_stays_usable():
    w = W.random_inputs([200, 77], 2, 2, 128, 128, seed=61, state_std=0.1)
    pool = w.state_pool.to("cuda").clone()
    t0 = time.monotonic()
    _, status = _run(w, kda.DEBUG_WITHHOLD_HANDOFF, pool)
    elapsed = time.monotonic() - t0
    assert status == kda.ERR_DEVICE_TIMEOUT, status
    assert elapsed < 30.0, elapsed  # the waits are bounded (about a second each, concurrently)
    # same context, same inputs, no hook: a correct result
    pool = w.state_pool.to("cuda").clone()
    out, status = _run(w, 0, pool)
    assert status == 0
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias,
                                      w.cu_seqlens, w.state_pool, w.state_indices, gate_mode=w.gate_mode,
                                      beta_mode=w.beta_mode, state_layout=w.state_layout,
                                      gate_lower_bound=w.gate_lower_bound)
    parity.check_rows("bounded-wait recovery out", out.double().cpu().numpy(), o_ref, 1e-2, cu=w.cu_seqlens)
    touched = sorted(set(w.state_indices.tolist()))
    parity.check_states("bounded-wait recovery state", pool.double().cpu().numpy()[touched], p_ref[touched], 1e-2)


def test_withheld_handoff_flag_is_accepted_by_the_fp32_kernel_and_ignored():
    w = W.random_inputs([70, 33], 1, 2, 32, 32, seed=62, qkv_dtype=torch.float32, state_std=0.2,
                        output_dtype=torch.float32)
    pool = w.state_pool.to("cuda").clone()
    out, status = _run(w, kda.DEBUG_WITHHOLD_HANDOFF, pool)
    assert status == 0
    o_ref, _ = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                  w.state_pool, w.state_indices, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                                  state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    parity.check_rows("fp32 with the wait hook out", out.double().cpu().numpy(), o_ref, 1e-4, cu=w.cu_seqlens)
