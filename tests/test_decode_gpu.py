"""GPU parity of the single-token step (kda_decode, through the C ABI) against the fp64 oracle.

The oracle's decode is its token-by-token definition on a batch of one-token sequences.
Tolerances as for the prefill: relative L2 error over the whole output and, separately, over
every touched pool slot -- 1e-4 for fp32 q/k/v, 1e-2 for bf16 q/k/v (fp32 gates and state).
"""
import numpy as np
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_BF16 = 1e-2


def rel_l2(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def gpu_decode(w, pool=None, status=None):
    wd = w.to("cuda")
    pool = (wd.state_pool if pool is None else pool).clone()
    st = torch.zeros(1, dtype=torch.int32, device="cuda") if status is None else status
    out = kda.kda_decode(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, pool,
                         wd.state_indices, output_dtype=w.output_dtype, gate_mode=w.gate_mode,
                         beta_mode=w.beta_mode, state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound,
                         device_status=st)
    torch.cuda.synchronize()
    if status is None:
        assert int(st.item()) == 0
    return out, pool


def oracle_decode(w, heads=None):
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    if heads is None:
        return oracle.kda_decode(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.state_pool,
                                 w.state_indices, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                                 state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    group = w.num_v_heads // w.num_k_heads
    kh = [h // group for h in heads]
    return oracle.kda_decode(cpu(w.q)[:, kh], cpu(w.k)[:, kh], cpu(w.v)[:, heads], cpu(w.raw_gate)[:, heads],
                             cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads], cpu(w.dt_bias)[heads],
                             cpu(w.state_pool)[:, heads], cpu(w.state_indices), gate_mode=w.gate_mode,
                             beta_mode=w.beta_mode, state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)


def check(w, out, pool, tol, heads=None, label="decode"):
    o_ref, p_ref = oracle_decode(w, heads)
    out, pool, base = out.cpu(), pool.cpu(), w.state_pool.cpu()
    if heads is not None:
        out, pool, base = out[:, heads], pool[:, heads], base[:, heads]
    out, pool, base = out.double().numpy(), pool.double().numpy(), base.double().numpy()
    touched = sorted(set(w.state_indices.tolist()))
    # every sequence is one token: its chain is one output row per head
    parity.check_rows(f"{label}: out", out, o_ref, tol, cu=np.arange(out.shape[0] + 1))
    parity.check_states(f"{label}: state", pool[touched], p_ref[touched], tol)
    for s in range(pool.shape[0]):
        if s not in touched:
            assert np.array_equal(pool[s], base[s]), f"untouched slot {s} changed"


def one_token_batch(B, Hk, Hv, dk, dv, seed, qkv_dtype=torch.float32, output_dtype=torch.float32, **kw):
    slots = kw.pop("max_slots", B + 3)
    g = torch.Generator().manual_seed(500 + seed)
    idx = torch.randperm(slots, generator=g)[:B].to(torch.int32)
    return W.random_inputs([1] * B, Hk, Hv, dk, dv, seed=seed, qkv_dtype=qkv_dtype, output_dtype=output_dtype,
                           state_std=0.3, max_slots=slots, state_indices=idx, **kw)


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
@pytest.mark.parametrize("dk,dv", [(16, 16), (128, 128), (7, 33), (128, 100), (65, 128), (1, 1)])
def test_decode_fp32_matches_oracle(cuda_device, layout, dk, dv):
    w = one_token_batch(5, 1, 2, dk, dv, seed=dk + dv, state_layout=layout)
    out, pool = gpu_decode(w)
    check(w, out, pool, TOL_F32, label="decode fp32")


@pytest.mark.parametrize("gate_mode,beta_mode", [("safe", "logits"), ("original", "probability")])
def test_decode_gate_and_beta_modes(cuda_device, gate_mode, beta_mode):
    w = one_token_batch(6, 2, 4, 32, 48, seed=3, gate_mode=gate_mode, beta_mode=beta_mode, raw_std=2.0,
                        beta_mean=0.5 if beta_mode == "probability" else 0.0,
                        beta_std=0.2 if beta_mode == "probability" else 1.0)
    out, pool = gpu_decode(w)
    check(w, out, pool, TOL_F32, label="decode fp32 modes")


@pytest.mark.parametrize("layout,out_dtype", [("K_FIRST", torch.bfloat16), ("V_FIRST", torch.float32)])
def test_decode_bf16(cuda_device, layout, out_dtype):
    w = one_token_batch(9, 4, 8, 128, 128, seed=11, qkv_dtype=torch.bfloat16, output_dtype=out_dtype,
                        state_layout=layout)
    out, pool = gpu_decode(w)
    assert out.dtype == out_dtype
    check(w, out, pool, TOL_BF16, label="decode bf16")


def test_decode_steps_equal_prefill(cuda_device):
    # T decode steps through the slots equal one prefill call over the T-token sequences
    B, T = 3, 20
    w = W.random_inputs([T] * B, 2, 2, 128, 128, seed=21, qkv_dtype=torch.float32, output_dtype=torch.float32,
                        state_std=0.2, max_slots=4, state_indices=torch.tensor([2, 0, 3], dtype=torch.int32))
    wd = w.to("cuda")
    pool_p = wd.state_pool.clone()
    out_p = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens,
                              pool_p, wd.state_indices)
    pool_d = wd.state_pool.clone()
    outs = []
    for t in range(T):
        rows = torch.arange(B, device="cuda") * T + t
        outs.append(kda.kda_decode(wd.q[rows], wd.k[rows], wd.v[rows], wd.raw_gate[rows], wd.beta_logits[rows],
                                   wd.a_log, wd.dt_bias, pool_d, wd.state_indices))
    torch.cuda.synchronize()
    out_d = torch.stack(outs, dim=1).reshape(B * T, 2, 128)
    assert rel_l2(out_d.cpu(), out_p.cpu()) < 1e-5
    assert rel_l2(pool_d.cpu(), pool_p.cpu()) < 1e-5
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices)
    parity.check_rows("decode steps = prefill: out", out_d, o_ref, TOL_F32, cu=w.cu_seqlens)
    parity.check_states("decode steps = prefill: state", pool_d, p_ref, TOL_F32)


def test_decode_bad_slot_is_reported_and_skipped(cuda_device):
    w = one_token_batch(3, 1, 1, 16, 16, seed=5, max_slots=3)
    w.state_indices = torch.tensor([0, 7, 2], dtype=torch.int32)
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((3, 1, 16), 123.0, device="cuda")
    kda.kda_decode(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, pool, wd.state_indices, out,
                   device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5  # KDA_ERR_DEVICE_CHECK
    assert torch.all(out[1] == 123.0)
    assert torch.equal(pool[1], wd.state_pool[1])
    w.state_indices = torch.tensor([0, 2], dtype=torch.int32)
    rows = [0, 2]
    o_ref, p_ref = oracle.kda_decode(w.q[rows], w.k[rows], w.v[rows], w.raw_gate[rows], w.beta_logits[rows],
                                     w.a_log, w.dt_bias, w.state_pool, w.state_indices)
    parity.check_rows("decode bad slot: the valid sequences", out[rows], o_ref, TOL_F32, cu=[0, 1, 2])
    parity.check_states("decode bad slot: their states", pool[[0, 2]], p_ref[[0, 2]], TOL_F32)


@pytest.mark.parametrize("name", ["decode_B256_H32", "decode_B64_H16_safe"])
def test_decode_workloads_sampled_heads(cuda_device, name):
    # the benchmark's workloads at full size, in the benchmark's launch configuration; the oracle
    # replays three value heads of every sequence
    w = W.make(name, device="cuda")
    pool = w.state_pool.clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kda.kda_decode(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, pool, w.state_indices,
                         output_dtype=w.output_dtype, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                         state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    heads = [0, w.num_v_heads // 2, w.num_v_heads - 1]
    check(w, out, pool, TOL_BF16, heads=heads, label=name)
