"""Seeded synthetic inputs for the KDA chunked prefill and the segment scan.

This module only draws random numbers, in the shapes, dtypes and distributions of the
workloads below. It holds none of the method's arithmetic (no gate, no recurrence, no
chunk algebra), so the fp64 CPU oracle and the CUDA library can both take their inputs
from here without sharing any code with each other.

Distribution convention: ``N(m, s)`` means mean ``m`` and standard deviation ``s``
(``torch.normal`` convention); ``U(a, b)`` is uniform on ``[a, b)``.

Tensor layouts follow the ``max.nn.state_space.kda_chunk`` parameter list:
  q, k         [total_tokens, num_key_heads, key_head_dim]
  v            [total_tokens, num_value_heads, value_head_dim]
  raw_gate     [total_tokens, num_value_heads, key_head_dim]   fp32, before dt_bias
  beta_logits  [total_tokens, num_value_heads]                 fp32
  a_log        [num_value_heads]                               fp32
  dt_bias      [num_value_heads, key_head_dim]                 fp32
  cu_seqlens   [batch + 1] int32 exclusive prefix offsets
  state_pool   [max_slots, Hv, dk, dv] (K_FIRST) or [max_slots, Hv, dv, dk] (V_FIRST), fp32
  state_indices [batch] int32
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch


@dataclass
class Workload:
    name: str
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    raw_gate: torch.Tensor
    beta_logits: torch.Tensor
    a_log: torch.Tensor
    dt_bias: torch.Tensor
    cu_seqlens: torch.Tensor
    state_pool: torch.Tensor
    state_indices: torch.Tensor
    gate_mode: str = "original"
    beta_mode: str = "logits"
    state_layout: str = "K_FIRST"
    gate_lower_bound: float = -5.0
    output_dtype: torch.dtype = torch.bfloat16
    chunk: int = 64
    seg_offsets: Optional[torch.Tensor] = None  # [N+1] int32, single-sequence workloads only
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def total_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def batch(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def num_k_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def num_v_heads(self) -> int:
        return int(self.v.shape[1])

    @property
    def dk(self) -> int:
        return int(self.q.shape[2])

    @property
    def dv(self) -> int:
        return int(self.v.shape[2])

    def lengths(self) -> List[int]:
        cu = self.cu_seqlens.tolist()
        return [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]

    def to(self, device) -> "Workload":
        out = Workload(**{k: getattr(self, k) for k in self.__dataclass_fields__})
        for name in ("q", "k", "v", "raw_gate", "beta_logits", "a_log", "dt_bias",
                     "cu_seqlens", "state_pool", "state_indices", "seg_offsets"):
            t = getattr(self, name)
            if t is not None:
                setattr(out, name, t.to(device))
        return out


def _l2_rows(x: torch.Tensor) -> torch.Tensor:
    # per-token unit vectors over the last axis (input shaping only, as the workloads state)
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)


def random_inputs(lengths, num_k_heads, num_v_heads, dk, dv, *, seed, qkv_dtype=torch.bfloat16,
                  raw_std=1.0, beta_mean=0.0, beta_std=1.0, a_log_range=(0.0, math.log(16.0)),
                  dt_bias_std=0.1, state_std=0.0, max_slots=None, state_indices=None,
                  state_layout="K_FIRST", gate_mode="original", beta_mode="logits",
                  gate_lower_bound=-5.0, output_dtype=torch.bfloat16, chunk=64, device="cpu",
                  name="random", normalize_qk=True) -> Workload:
    """Draw one workload. Draw order is fixed so a seed pins every tensor."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    lengths = [int(x) for x in lengths]
    T = sum(lengths)
    B = len(lengths)
    f32 = dict(dtype=torch.float32, device=device, generator=g)

    q = torch.randn(T, num_k_heads, dk, **f32)
    k = torch.randn(T, num_k_heads, dk, **f32)
    if normalize_qk:
        q = _l2_rows(q)
        k = _l2_rows(k)
    v = torch.randn(T, num_v_heads, dv, **f32)
    q, k, v = q.to(qkv_dtype), k.to(qkv_dtype), v.to(qkv_dtype)
    raw_gate = torch.randn(T, num_v_heads, dk, **f32) * raw_std
    beta_logits = torch.randn(T, num_v_heads, **f32) * beta_std + beta_mean
    lo, hi = a_log_range
    a_log = torch.rand(num_v_heads, **f32) * (hi - lo) + lo
    dt_bias = torch.randn(num_v_heads, dk, **f32) * dt_bias_std
    if max_slots is None:
        max_slots = B
    if state_indices is None:
        state_indices = torch.arange(B, dtype=torch.int32, device=device)
    shape = (max_slots, num_v_heads, dk, dv) if state_layout == "K_FIRST" else (max_slots, num_v_heads, dv, dk)
    state_pool = torch.randn(*shape, **f32) * state_std
    cu = torch.zeros(B + 1, dtype=torch.int64)
    cu[1:] = torch.tensor(lengths, dtype=torch.int64).cumsum(0)
    return Workload(name=name, q=q, k=k, v=v, raw_gate=raw_gate, beta_logits=beta_logits,
                    a_log=a_log, dt_bias=dt_bias, cu_seqlens=cu.to(torch.int32).to(device),
                    state_pool=state_pool, state_indices=state_indices.to(torch.int32).to(device),
                    gate_mode=gate_mode, beta_mode=beta_mode, state_layout=state_layout,
                    gate_lower_bound=gate_lower_bound, output_dtype=output_dtype, chunk=chunk,
                    seed=int(seed))


# --------------------------------------------------------------------------------------------
# The five named workloads (shapes and distributions as stated for each).
# --------------------------------------------------------------------------------------------

WORKLOADS = (
    "tiny_fp32_T64_d16",
    "single_T4096_H16",
    "varlen8_H32_vfirst",
    "long_T131072_H32_cp16",
    "batch64_T2048_H16_safe",
    "batch4_T2048_H32",  # one wave of 128 chains, inputs 404 MB (> L2): the profiling case
    "long_T16384_H32_cp2",  # context-parallel profiling case: 2 segments of 8192, inputs 420 MB
    "decode_B256_H32",  # single-token step: 256 sequences x 32 heads, pool 537 MB (> L2)
    "decode_B64_H16_safe",  # single-token step on the large-batch prefill's pool shape, safe gate
)


def make(name: str, device="cpu", seed: Optional[int] = None) -> Workload:
    """Build a named workload; the default seed is the workload's index in ``WORKLOADS``."""
    idx = WORKLOADS.index(name)
    s = idx if seed is None else seed
    if name == "tiny_fp32_T64_d16":
        w = random_inputs([64], 1, 1, 16, 16, seed=s, qkv_dtype=torch.float32, dt_bias_std=0.0,
                          state_std=0.0, output_dtype=torch.float32, chunk=16, device=device,
                          name=name)
    elif name == "single_T4096_H16":
        w = random_inputs([4096], 16, 16, 128, 128, seed=s, state_std=0.0, device=device, name=name)
    elif name == "varlen8_H32_vfirst":
        g = torch.Generator().manual_seed(1000 + s)
        lengths = torch.randint(1, 8193, (8,), generator=g).tolist()
        idxs = torch.randperm(16, generator=g)[:8].to(torch.int32)
        w = random_inputs(lengths, 32, 32, 128, 128, seed=s, state_std=0.1, max_slots=16,
                          state_indices=idxs, state_layout="V_FIRST", device=device, name=name)
    elif name == "long_T131072_H32_cp16":
        w = random_inputs([131072], 32, 32, 128, 128, seed=s, state_std=0.1, device=device, name=name)
        w.seg_offsets = (torch.arange(17, dtype=torch.int32) * 8192).to(device)
    elif name == "batch64_T2048_H16_safe":
        w = random_inputs([2048] * 64, 16, 16, 128, 128, seed=s, raw_std=2.0, beta_mean=2.0,
                          beta_std=1.0, state_std=0.1, gate_mode="safe", gate_lower_bound=-5.0,
                          device=device, name=name)
    elif name == "batch4_T2048_H32":
        w = random_inputs([2048] * 4, 32, 32, 128, 128, seed=s, state_std=0.1, device=device, name=name)
    elif name == "long_T16384_H32_cp2":
        w = random_inputs([16384], 32, 32, 128, 128, seed=s, state_std=0.1, device=device, name=name)
        w.seg_offsets = (torch.arange(3, dtype=torch.int32) * 8192).to(device)
    elif name == "decode_B256_H32":
        g = torch.Generator().manual_seed(1000 + s)
        idxs = torch.randperm(256, generator=g).to(torch.int32)
        w = random_inputs([1] * 256, 32, 32, 128, 128, seed=s, state_std=0.1, max_slots=256,
                          state_indices=idxs, device=device, name=name)
        w.notes["decode"] = True
    elif name == "decode_B64_H16_safe":
        w = random_inputs([1] * 64, 16, 16, 128, 128, seed=s, raw_std=2.0, beta_mean=2.0, beta_std=1.0,
                          state_std=0.1, gate_mode="safe", gate_lower_bound=-5.0, state_layout="V_FIRST",
                          device=device, name=name)
        w.notes["decode"] = True
    else:  # pragma: no cover
        raise KeyError(name)
    return w


def segment_offsets(total: int, num_segments: int, device="cpu") -> torch.Tensor:
    """Equal split of [0,total) into num_segments pieces (last one takes the remainder)."""
    base = total // num_segments
    offs = [i * base for i in range(num_segments)] + [total]
    return torch.tensor(offs, dtype=torch.int32, device=device)
