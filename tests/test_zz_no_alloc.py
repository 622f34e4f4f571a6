"""The allocation-free context-parallel prefill, called through the C ABI.

kda_context_parallel_prefill_static serves callers that cannot allocate device memory where
they run the prefill: it keeps its scratch in a fixed array inside the library instead of a
caller-supplied workspace.  Two calls in a row (different inputs, so the second cannot lean on
what the first left in the shared array) must each match the fp64 oracle, and
kda_context_parallel_prefill (the entry point with a caller workspace), within the bf16
tolerance of the other parity tests.  One call sits exactly at the array's limit (2048 tokens
x 32 heads = 65536 token-heads, several segments), and across the calls neither torch's
allocator nor the device's free memory moves.
This file is collected last so that a run stopping at the first failure has run the rest.
"""
import ctypes

import numpy as np
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu

TOL = 1e-2
_CALLS = []  # return codes of the calls made so far in this process


def _rel(x, ref):
    x, ref = x.double().cpu().numpy(), ref.double().cpu().numpy()
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))


def _static_entry():
    lib = kda.load_library()
    fn = lib.kda_context_parallel_prefill_static
    vp, i32, i64, u32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i64, i32, i32, i32, i32, vp, i32, vp, vp, ctypes.c_int,
                   vp, vp, vp, vp, vp, u32, ctypes.c_float, vp, vp]
    return fn


def _call_static(fn, w, offs, init, out, fin):
    dev = w.q.device
    T, Hv = w.total_tokens, w.num_v_heads
    N = offs.numel() - 1
    M = torch.empty((N, Hv, 128, 128), device=dev)
    U, inc, outg = (torch.empty((N, Hv, 128, 128), device=dev) for _ in range(3))
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    torch.cuda.synchronize()
    alloc0 = torch.cuda.memory_allocated()
    # the first call in a process may load the library's module (and with it the array itself)
    free0 = torch.cuda.mem_get_info()[0] if _CALLS else None
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = fn(p(w.q), p(w.k), p(w.v), 1, p(w.raw_gate), p(w.beta_logits), p(w.a_log), p(w.dt_bias), T,
            w.num_k_heads, Hv, 128, 128, p(offs), N, p(init), p(out), 1, p(fin), p(M), p(U), p(inc), p(outg), 0,
            -5.0, p(status), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    _CALLS.append(rc)
    assert torch.cuda.memory_allocated() == alloc0
    if free0 is not None:
        # a kernel's first launch may still load its module (code, a few hundred KB): far below the
        # 16 MiB and more that any scratch for these calls would take
        assert torch.cuda.mem_get_info()[0] >= free0 - (4 << 20), "the call took device memory"
    assert rc == 0, kda.kda_status_string(rc)
    assert int(status.item()) == 0


def _oracle(w, cuts, heads):
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    T = w.total_tokens
    o_ref, p_ref = oracle.kda_forward(cpu(w.q)[:, heads], cpu(w.k)[:, heads], cpu(w.v)[:, heads],
                                      cpu(w.raw_gate)[:, heads], cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads],
                                      cpu(w.dt_bias)[heads], np.array([0, T], np.int32),
                                      cpu(w.state_pool)[:1, heads], np.array([0], np.int32))
    return o_ref, p_ref[0]


def test_static_scratch_prefill_matches_the_oracle_and_the_workspace_entry_point_twice():
    fn = _static_entry()
    cases = [
        (W.random_inputs([1500], 4, 4, 128, 128, seed=31, state_std=0.1, device="cuda"), [0, 300, 700, 1500],
         [0, 1, 2, 3]),
        # exactly at the limit: 2048 tokens x 32 heads fill the whole array (too full for the pieces)
        (W.random_inputs([2048], 32, 32, 128, 128, seed=32, state_std=0.2, device="cuda"),
         [0, 64, 1000, 1001, 2048], [0, 13, 31]),
    ]
    assert 2 * 2048 * 32 * 128 * 2 == 32 << 20
    outs = []
    for w, cuts, heads in cases:
        T, Hv = w.total_tokens, w.num_v_heads
        offs = torch.tensor(cuts, dtype=torch.int32, device="cuda")
        init = w.state_pool[0].contiguous()
        out_s = torch.empty((T, Hv, 128), dtype=torch.bfloat16, device="cuda")
        fin_s = torch.empty((Hv, 128, 128), device="cuda")
        _call_static(fn, w, offs, init, out_s, fin_s)
        outs.append((w, cuts, heads, offs, init, out_s, fin_s))
    for w, cuts, heads, offs, init, out_s, fin_s in outs:
        o_ref, s_ref = _oracle(w, cuts, heads)
        lab = f"allocation-free prefill T={w.total_tokens} H={w.num_v_heads}"
        parity.check_rows(f"{lab}: out", out_s[:, heads], o_ref, TOL)
        parity.check_states(f"{lab}: final", fin_s[heads], s_ref, TOL)
        ref = kda.kda_context_parallel_prefill(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, offs,
                                               init)
        torch.cuda.synchronize()
        assert _rel(out_s, ref["out"]) <= TOL
        assert _rel(fin_s, ref["final_state"]) <= TOL


def test_static_scratch_prefill_refuses_calls_beyond_its_array():
    fn = _static_entry()
    # 65537 token-heads need more than the 32 MiB array; refused before any GPU work
    null = ctypes.c_void_p(16)
    rc = fn(null, null, null, 1, null, null, null, null, 65537, 1, 1, 128, 128, null, 1, null, null, 1, null, null,
            null, null, null, 0, -5.0, None, None)
    assert rc == 3  # KDA_ERR_WORKSPACE
