"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle, element by element.

Tolerances (relative L2 error over the whole output tensor and, separately, over every final
state the call touched): 1e-4 for fp32 q/k/v, 1e-2 for bf16 q/k/v with fp32 gates and state.
The same bound holds for every (sequence, head) chain on its own -- its output rows and its
final state -- so that a short sequence or a single head cannot hide a local error under the
norm of the rest (``parity.check_rows`` / ``parity.check_states``).  Full-size workloads are
checked on sampled value heads: every (sequence, head) chain is independent, so the oracle
replays the sampled heads alone at full length.
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


def gpu_forward(w, force_simt=False, pool=None):
    wd = w.to("cuda")
    pool = (wd.state_pool if pool is None else pool.to("cuda")).clone()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens,
                            pool, wd.state_indices, output_dtype=w.output_dtype, gate_mode=w.gate_mode,
                            beta_mode=w.beta_mode, state_layout=w.state_layout,
                            gate_lower_bound=w.gate_lower_bound, force_simt=force_simt, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, pool


def oracle_forward(w, heads=None):
    """Oracle on all heads, or on the listed value heads only (returns arrays restricted to them)."""
    if heads is None:
        return oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                  w.state_pool, w.state_indices, gate_mode=w.gate_mode, beta_mode=w.beta_mode,
                                  state_layout=w.state_layout, gate_lower_bound=w.gate_lower_bound)
    group = w.num_v_heads // w.num_k_heads
    kh = [h // group for h in heads]
    cpu = lambda t: t.detach().cpu()  # noqa: E731
    return oracle.kda_forward(cpu(w.q)[:, kh], cpu(w.k)[:, kh], cpu(w.v)[:, heads], cpu(w.raw_gate)[:, heads],
                              cpu(w.beta_logits)[:, heads], cpu(w.a_log)[heads], cpu(w.dt_bias)[heads],
                              cpu(w.cu_seqlens), cpu(w.state_pool)[:, heads], cpu(w.state_indices),
                              gate_mode=w.gate_mode, beta_mode=w.beta_mode, state_layout=w.state_layout,
                              gate_lower_bound=w.gate_lower_bound)


def check(w, out, pool, tol, heads=None, label="prefill"):
    o_ref, p_ref = oracle_forward(w, heads)
    out = out.double().cpu().numpy()
    pool = pool.double().cpu().numpy()
    if heads is not None:
        out, pool = out[:, heads], pool[:, heads]
    touched = sorted(set(w.state_indices.tolist()))
    e_out, _ = parity.check_rows(f"{label} out", out, o_ref, tol, cu=w.cu_seqlens)
    e_state, _ = parity.check_states(f"{label} final state", pool[touched], p_ref[touched], tol)
    untouched = [s for s in range(pool.shape[0]) if s not in touched]
    base = w.state_pool.double().cpu().numpy()
    if heads is not None:
        base = base[:, heads]
    for s in untouched:
        assert np.array_equal(pool[s], base[s]), f"untouched slot {s} changed"
    return e_out, e_state


# ------------------------------------------------------------------------------------------
# fp32 path (1e-4)
# ------------------------------------------------------------------------------------------

def test_tiny_fp32_workload():
    w = W.make("tiny_fp32_T64_d16")
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_F32, label="tiny_fp32_T64_d16")


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 48), (128, 128), (7, 5)])
@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_fp32_ragged_varlen(dk, dv, layout):
    lengths = [1, 15, 16, 17, 0, 63, 64, 65]
    w = W.random_inputs(lengths, 2, 4, dk, dv, seed=dk * 7 + dv, qkv_dtype=torch.float32, state_std=0.3,
                        max_slots=11, state_indices=torch.tensor([9, 0, 3, 5, 10, 1, 7, 2], dtype=torch.int32),
                        state_layout=layout, output_dtype=torch.float32)
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_F32, label="fp32 ragged varlen")


@pytest.mark.parametrize("gate_mode,beta_mode", [("safe", "logits"), ("original", "probability")])
def test_fp32_modes(gate_mode, beta_mode):
    w = W.random_inputs([70, 33], 1, 2, 32, 32, seed=5, qkv_dtype=torch.float32, raw_std=2.0, state_std=0.2,
                        gate_mode=gate_mode, beta_mode=beta_mode, output_dtype=torch.float32)
    if beta_mode == "probability":
        w.beta_logits = torch.rand(w.beta_logits.shape, generator=torch.Generator().manual_seed(3))
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_F32, label="fp32 gate/beta modes")


# ------------------------------------------------------------------------------------------
# bf16 path (1e-2), reduced sizes that still span many chunks and a ragged tail
# ------------------------------------------------------------------------------------------

BF16_SMALL = [
    dict(lengths=[700], H=2, layout="K_FIRST", gate="original", state_std=0.0, raw_std=1.0, beta_mean=0.0),
    dict(lengths=[300, 1, 129, 64, 0, 511], H=2, layout="V_FIRST", gate="original", state_std=0.1, raw_std=1.0,
         beta_mean=0.0),
    dict(lengths=[257, 256], H=3, layout="K_FIRST", gate="safe", state_std=0.1, raw_std=2.0, beta_mean=2.0),
]


@pytest.mark.parametrize("case", range(len(BF16_SMALL)))
@pytest.mark.parametrize("force_simt", [False, True])
def test_bf16_small(case, force_simt):
    c = BF16_SMALL[case]
    B = len(c["lengths"])
    w = W.random_inputs(c["lengths"], c["H"], c["H"], 128, 128, seed=100 + case, state_std=c["state_std"],
                        raw_std=c["raw_std"], beta_mean=c["beta_mean"], gate_mode=c["gate"],
                        state_layout=c["layout"], max_slots=B + 2,
                        state_indices=torch.randperm(B + 2, generator=torch.Generator().manual_seed(case))[:B])
    out, pool = gpu_forward(w, force_simt=force_simt)
    check(w, out, pool, TOL_BF16, label=f"bf16 small[{case}]" + (" simt" if force_simt else ""))


def test_bf16_fp32_output():
    w = W.random_inputs([200], 2, 2, 128, 128, seed=7, state_std=0.1, output_dtype=torch.float32)
    out, pool = gpu_forward(w)
    assert out.dtype == torch.float32
    check(w, out, pool, TOL_BF16, label="bf16 in, fp32 out")


def test_bf16_grouped_heads_v_first():
    # two key heads shared by eight value heads ("max.nn.state_space.kda_chunk": num_key_heads for
    # q/k, num_value_heads for v, gates, beta and state); key head of value head h is h // 4
    w = W.random_inputs([150, 70, 64], 2, 8, 128, 128, seed=41, state_std=0.1, state_layout="V_FIRST",
                        max_slots=5, state_indices=torch.tensor([4, 0, 2], dtype=torch.int32))
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_BF16, label="bf16 grouped heads")


def test_bf16_strong_decay_original_gate():
    # raw_gate ~ N(0, 3) with exp(a_log) up to 16: single steps decay by e^-60 and more, so
    # in-chunk decay products span far beyond the fp32 range -- every factor the kernel forms
    # is a product of decays (<= 1) and must neither overflow nor lose the surviving terms
    w = W.random_inputs([333, 190], 2, 2, 128, 128, seed=42, state_std=0.1, raw_std=3.0)
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_BF16, label="bf16 strong decay")


def test_bf16_unit_query_equals_key_with_beta_one_reads_back_v():
    # closed form of the step: with q_t = k_t (unit) and beta = 1 the readout after the delta write
    # is k_t^T S_t = v_t exactly, whatever the decay and the earlier state
    w = W.random_inputs([200, 77], 2, 2, 128, 128, seed=43, state_std=0.3, raw_std=1.0)
    w.q = w.k.clone()
    w.beta_mode = "probability"
    w.beta_logits = torch.ones_like(w.beta_logits)
    out, _ = gpu_forward(w)
    parity.check_rows("q = k, beta = 1 reads back v", out, w.v, TOL_BF16, cu=w.cu_seqlens)


# ------------------------------------------------------------------------------------------
# Full-size workloads (the benchmark's launch configuration), sampled heads
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("name,heads", [
    ("single_T4096_H16", [0, 7, 15]),
    ("varlen8_H32_vfirst", [3, 30]),
    ("batch64_T2048_H16_safe", [1, 12]),
    ("long_T131072_H32_cp16", [5]),
])
def test_full_size_sampled_heads(name, heads):
    w = W.make(name, device="cuda")
    out, pool = gpu_forward(w)
    check(w, out, pool, TOL_BF16, heads=heads, label=name)


# ------------------------------------------------------------------------------------------
# Device-side checks: reported, never a fault; other sequences still run
# ------------------------------------------------------------------------------------------

def test_bad_slot_is_reported_and_skipped():
    w = W.random_inputs([20, 30], 1, 1, 16, 16, seed=9, qkv_dtype=torch.float32, state_std=0.5, max_slots=3,
                        state_indices=torch.tensor([7, 1], dtype=torch.int32), output_dtype=torch.float32)
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    out = torch.full((50, 1, 16), 123.0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens, pool,
                      wd.state_indices, out, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5  # KDA_ERR_DEVICE_CHECK
    assert torch.all(out[:20] == 123.0)
    w1 = W.random_inputs([20, 30], 1, 1, 16, 16, seed=9, qkv_dtype=torch.float32, state_std=0.5, max_slots=3,
                         state_indices=torch.tensor([0, 1], dtype=torch.int32), output_dtype=torch.float32)
    o_ref, p_ref = oracle_forward(w1)
    parity.check_rows("bad slot: the valid sequence", out[20:], o_ref[20:], TOL_F32)
    parity.check_states("bad slot: the valid sequence's state", pool[1:2], p_ref[1:2], TOL_F32)
    assert torch.equal(pool[0].cpu(), w.state_pool[0]) and torch.equal(pool[2].cpu(), w.state_pool[2])


def test_decreasing_offsets_are_reported():
    w = W.random_inputs([10, 10], 1, 1, 16, 16, seed=10, qkv_dtype=torch.float32, output_dtype=torch.float32)
    wd = w.to("cuda")
    cu = torch.tensor([0, 15, 12], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, cu,
                      wd.state_pool.clone(), wd.state_indices, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5


# ------------------------------------------------------------------------------------------
# batch order: the prefill hands block rows to sequences longest first for batches of at most
# 256 sequences (index order above that); either way every sequence is computed once
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lengths_kind", ["over_256", "exactly_256_equal", "many_ties"])
def test_batch_order_covers_every_sequence_once(lengths_kind):
    g = torch.Generator().manual_seed(41)
    if lengths_kind == "over_256":
        lengths = torch.randint(0, 200, (300,), generator=g).tolist()
    elif lengths_kind == "exactly_256_equal":
        lengths = [70] * 256
    else:
        lengths = [int(x) for x in torch.randint(0, 3, (40,), generator=g) * 64 + 5]
    B = len(lengths)
    slots = B + 7
    idx = torch.randperm(slots, generator=g)[:B].to(torch.int32)
    w = W.random_inputs(lengths, 1, 2, 128, 128, seed=B, state_std=0.2, max_slots=slots, state_indices=idx)
    out, pool = gpu_forward(w)
    check(w, out, pool, 1e-2, label="batch order")
