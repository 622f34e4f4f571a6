"""Wrappers launched on a side stream: the memory they allocate themselves (results and scratch)
must not go to other work while their kernels still run there.  Each call runs on a side stream,
and straight afterwards the current stream allocates and overwrites as much memory as the call
took; the results must equal, bit for bit, those of the same call on the current stream."""
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda

pytestmark = pytest.mark.gpu


def _scribble(nbytes):
    # the current stream takes (and overwrites) freshly allocated memory of about this size
    junk = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    junk.fill_(0x7F)
    return junk


def test_context_parallel_prefill_on_a_side_stream(cuda_device):
    w = W.random_inputs([8192], 8, 8, 128, 128, seed=61, state_std=0.1, device="cuda")
    offs = torch.tensor([0, 2048, 4096, 6000, 8192], dtype=torch.int32, device="cuda")
    init = w.state_pool[0].contiguous()
    args = (w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs, init)
    ref = kda.kda_context_parallel_prefill(*args)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    res = kda.kda_context_parallel_prefill(*args, stream=side)
    junk = _scribble(kda.kda_context_parallel_workspace_preferred(8192, 4, 8, 128))
    side.synchronize()
    torch.cuda.synchronize()
    del junk
    for key in ("out", "final_state", "incoming_states", "outgoing_states"):
        assert torch.equal(res[key], ref[key]), key


def test_chunk_fwd_split_workspace_on_a_side_stream(cuda_device):
    # one long sequence: the split route's scratch is allocated by the wrapper and dropped at return
    w = W.random_inputs([6000], 4, 4, 128, 128, seed=62, state_std=0.1, device="cuda")
    T, Hk, dk = w.q.shape
    need = kda.kda_workspace_size(T, 1, Hk, 4, 128, 128)
    assert need > 0
    pool_ref = w.state_pool.clone()
    ref = kda.kda_chunk_fwd(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens, pool_ref,
                            w.state_indices)
    pool = w.state_pool.clone()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    out = kda.kda_chunk_fwd(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens, pool,
                            w.state_indices, stream=side)
    junk = _scribble(need + T * 4 * 128 * 2)
    side.synchronize()
    torch.cuda.synchronize()
    del junk
    assert torch.equal(out, ref)
    assert torch.equal(pool, pool_ref)
