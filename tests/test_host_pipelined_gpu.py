"""kda_prefill_host_pipelined (through the C ABI): one sequence in pinned host memory, copies
pipelined with the kernels in segments.  Segment boundaries fall on chunk boundaries, so the
outputs and the final state must equal the plain chunk kernel's on the whole sequence bit for
bit (kda_chunk_fwd without a workspace); one
case is also checked against the fp64 oracle (relative L2 1e-2, bf16 q/k/v)."""
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu


def pinned(t):
    return t.detach().cpu().contiguous().pin_memory()


def run_both(w, segment_tokens, output_dtype=torch.bfloat16):
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    # the plain chunk kernel (an empty workspace keeps kda_chunk_fwd off its split route for few chains)
    ref = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens, pool,
                            wd.state_indices, output_dtype=output_dtype, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                            state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound,
                            workspace=torch.empty(0, dtype=torch.uint8, device="cuda"))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = kda.kda_prefill_host_pipelined(pinned(w.q), pinned(w.k), pinned(w.v), pinned(w.raw_gate),
                                         pinned(w.beta_logits), pinned(w.a_log), pinned(w.dt_bias),
                                         pinned(w.state_pool[0]), segment_tokens=segment_tokens,
                                         output_dtype=output_dtype, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                                         state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound,
                                         device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return ref.cpu(), pool[0].cpu(), res


@pytest.mark.parametrize("T,segment,layout", [(5000, 1024, "K_FIRST"), (5000, 1024, "V_FIRST"), (640, 4096, "K_FIRST"),
                                              (4096, 64, "K_FIRST"), (4097, 2048, "V_FIRST")])
def test_equals_chunk_fwd_bit_for_bit(cuda_device, T, segment, layout):
    w = W.random_inputs([T], 2, 4, 128, 128, seed=T + segment, state_std=0.1, state_layout=layout)
    ref, ref_state, res = run_both(w, segment)
    assert torch.equal(res["out"], ref)
    assert torch.equal(res["final_state"], ref_state)


def test_safe_gate_fp32_output(cuda_device):
    w = W.random_inputs([3000], 2, 2, 128, 128, seed=5, state_std=0.1, raw_std=2.0, beta_mean=2.0, gate_mode="safe")
    ref, ref_state, res = run_both(w, 512, output_dtype=torch.float32)
    assert res["out"].dtype == torch.float32
    assert torch.equal(res["out"], ref)
    assert torch.equal(res["final_state"], ref_state)


def test_matches_oracle(cuda_device):
    w = W.random_inputs([2000], 2, 2, 128, 128, seed=9, state_std=0.1)
    _, _, res = run_both(w, 512)
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices)
    parity.check_rows("host-pipelined prefill: out", res["out"], o_ref, 1e-2)
    parity.check_states("host-pipelined prefill: final", res["final_state"], p_ref[0], 1e-2)


def test_empty_sequence_passes_the_state_through(cuda_device):
    w = W.random_inputs([0], 2, 2, 128, 128, seed=1, state_std=0.1)
    res = kda.kda_prefill_host_pipelined(pinned(w.q), pinned(w.k), pinned(w.v), pinned(w.raw_gate),
                                         pinned(w.beta_logits), pinned(w.a_log), pinned(w.dt_bias),
                                         pinned(w.state_pool[0]), segment_tokens=256)
    torch.cuda.synchronize()
    assert res["out"].shape == (0, 2, 128)
    assert torch.equal(res["final_state"], w.state_pool[0])


def test_refuses_unpinned_host_tensors(cuda_device):
    w = W.random_inputs([128], 1, 1, 128, 128, seed=2)
    with pytest.raises(ValueError, match="pinned"):
        kda.kda_prefill_host_pipelined(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.state_pool[0])
