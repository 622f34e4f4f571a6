"""Invariants of the method on the GPU path (kda_chunk_fwd through the C ABI), each fixed by the
recurrence itself rather than by a reference run:

- overwrite ("nx_nofloat_kda.nx source": the delta rule overwrites along k): writing the same unit
  key twice with beta = 1 and no decay leaves k v2^T, not k (v1 + v2)^T;
- identity (alpha = 1, beta = 0): the state passes through unchanged, bit for bit, and every
  output is the readout of that state;
- resume: one call over a sequence equals two calls over its halves with the state carried in
  the pool (bit for bit when the cut is chunk-aligned);
- untouched slots: pool slots no sequence names are never written.
"""
import pytest
import torch

import kda_workloads as W
import kimi_delta_attention_23_b200 as kda

pytestmark = pytest.mark.gpu

NO_WS = dict(dtype=torch.uint8, device="cuda")


def plain(wd, pool, out_dtype=torch.float32, **kw):
    """The plain chunk kernel (an empty workspace keeps kda_chunk_fwd off its split route)."""
    return kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens,
                             pool, wd.state_indices, output_dtype=out_dtype, workspace=torch.empty(0, **NO_WS), **kw)


def no_decay_case(T, H=2, seed=0, beta=1.0):
    """Inputs with alpha = 1 exactly (raw gate far below zero: softplus underflows to 0) and a
    fixed probability beta."""
    w = W.random_inputs([T], H, H, 128, 128, seed=seed, state_std=0.0)
    w.raw_gate = torch.full_like(w.raw_gate, -1.0e4)
    w.beta_logits = torch.full_like(w.beta_logits, beta)
    return w


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_same_unit_key_twice_overwrites(cuda_device, layout):
    T = 70  # the two writes sit in different 64-token chunks
    w = no_decay_case(T, seed=1, beta=1.0)
    e = torch.zeros(128)
    e[5] = 1.0
    k = torch.zeros(T, 2, 128)
    k[0, :] = e
    k[66, :] = e
    w.k = k.to(torch.bfloat16)
    w.q = k.to(torch.bfloat16)  # read back along the written key
    w.state_layout = layout
    if layout == "V_FIRST":
        w.state_pool = w.state_pool.transpose(-1, -2).contiguous()
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    out = plain(wd, pool, state_layout=layout, beta_mode="probability")
    torch.cuda.synchronize()
    v = w.v.float()
    # after the first write the key reads back v[0]; after the second, v[66] (not v[0] + v[66]).
    # The second write adds v[66] - v[0] rounded to bf16 (the update's operand): |v| of a few
    # units leaves at most ~1e-2 of it.
    atol = 3e-2
    assert torch.allclose(out[0].cpu(), v[0], rtol=0, atol=atol)
    assert torch.allclose(out[66].cpu(), v[66], rtol=0, atol=atol)
    assert (out[66].cpu() - (v[0] + v[66])).abs().max() > 0.5  # and plainly not the sum
    S = pool[0].cpu() if layout == "K_FIRST" else pool[0].cpu().transpose(-1, -2)
    assert torch.allclose(S[:, 5, :], v[66], rtol=0, atol=atol)  # row of the key: the last value
    others = torch.cat([S[:, :5, :], S[:, 6:, :]], dim=1)
    assert torch.count_nonzero(others) == 0  # nothing written along any other key


@pytest.mark.parametrize("layout", ["K_FIRST", "V_FIRST"])
def test_no_decay_no_write_keeps_the_state(cuda_device, layout):
    T = 300
    w = no_decay_case(T, seed=2, beta=0.0)
    g = torch.Generator().manual_seed(3)
    w.state_pool = torch.randn(w.state_pool.shape, generator=g) * 0.3
    w.state_layout = layout
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    out = plain(wd, pool, state_layout=layout, beta_mode="probability")
    torch.cuda.synchronize()
    assert torch.equal(pool, wd.state_pool)  # bit for bit
    S = w.state_pool[0].double() if layout == "K_FIRST" else w.state_pool[0].double().transpose(-1, -2)
    ref = torch.einsum("thi,hij->thj", w.q.double(), S)  # o_t = q_t^T S0 for every token
    err = float((out.cpu().double() - ref).norm() / ref.norm())
    assert err < 1e-2


@pytest.mark.parametrize("cut", [1024, 1000])
def test_two_calls_resume_like_one(cuda_device, cut):
    T = 2048
    w = W.random_inputs([T], 2, 2, 128, 128, seed=4, state_std=0.1)
    wd = w.to("cuda")
    pool_one = wd.state_pool.clone()
    out_one = plain(wd, pool_one)
    first = W.random_inputs([cut], 2, 2, 128, 128, seed=0)
    second = W.random_inputs([T - cut], 2, 2, 128, 128, seed=0)
    for part, sl in ((first, slice(0, cut)), (second, slice(cut, T))):
        for name in ("q", "k", "v", "raw_gate", "beta_logits"):
            setattr(part, name, getattr(w, name)[sl].clone())
        part.a_log, part.dt_bias = w.a_log, w.dt_bias
    pool_two = wd.state_pool.clone()
    out_a = plain(first.to("cuda"), pool_two)
    out_b = plain(second.to("cuda"), pool_two)
    torch.cuda.synchronize()
    out_two = torch.cat([out_a, out_b])
    if cut % 64 == 0:  # the same chunks: the same arithmetic
        assert torch.equal(out_two, out_one)
        assert torch.equal(pool_two, pool_one)
    else:
        rel = lambda x, r: float((x - r).norm() / r.norm())  # noqa: E731
        assert rel(out_two, out_one) < 1e-2
        assert rel(pool_two, pool_one) < 1e-2


def test_slots_no_sequence_names_are_never_written(cuda_device):
    lengths = [300, 0, 129, 64]
    idx = torch.tensor([7, 2, 11, 4], dtype=torch.int32)
    w = W.random_inputs(lengths, 2, 4, 128, 128, seed=6, state_std=0.2, max_slots=16, state_indices=idx)
    wd = w.to("cuda")
    pool = wd.state_pool.clone()
    kda.kda_chunk_fwd(wd.q, wd.k, wd.v, wd.raw_gate, wd.beta_logits, wd.a_log, wd.dt_bias, wd.cu_seqlens, pool,
                      wd.state_indices)
    torch.cuda.synchronize()
    named = set(idx.tolist())
    for s in range(16):
        if s not in named:
            assert torch.equal(pool[s], wd.state_pool[s]), f"slot {s} changed"
    assert torch.equal(pool[2], wd.state_pool[2])  # the empty sequence's slot keeps its state
    assert not torch.equal(pool[7], wd.state_pool[7])
