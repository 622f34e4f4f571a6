"""Context parallelism across GPUs: one long sequence, one token range per rank.

"KDA Context Parallelism" (Theory; Compose segments in sequence order; Incoming and outgoing
states): a stretch of the sequence is summarised by the affine map F(S) = M S + U, and the
maps, applied in sequence order, give every stretch its incoming state without replaying the
tokens before it.  Across ranks that is:

  1. every rank reduces its own range to one map (M_r, U_r)  -- kernels, all ranks in parallel
  2. one all-gather of the maps in rank order                  -- the only exchange (NCCL)
  3. every rank scans the world's maps from the initial state  -- a tiny kernel, redundantly
  4. every rank finishes its range from incoming[r]            -- kernels

Per rank and head the exchange moves one 128x128 transition and one 128x128 contribution (fp32,
128 KiB); nothing else crosses between GPUs.  The ranges are contiguous and in rank order:
rank r holds tokens [starts[r], starts[r+1]) of the sequence (``rank_ranges`` cuts them).

``ops`` selects the three per-rank steps; the default is this package's CUDA binding, which has
no CPU path.  Tests pass other implementations of the same three calls to check the exchange
and the ordering on CPU ranks.
"""
from __future__ import annotations

import contextlib

import torch
import torch.distributed as dist

__all__ = ["rank_ranges", "exchange_summaries", "context_parallel_prefill"]


def rank_ranges(T: int, world: int, chunk: int = 64) -> list[tuple[int, int]]:
    """Contiguous token ranges [start, end) of a T-token sequence, one per rank, in rank order.

    Boundaries are chunk-aligned (except the sequence's end) and the chunk counts differ by at most
    one, the earlier ranks taking the extra chunks; with fewer chunks than ranks the last ranks get
    empty ranges.
    """
    if T < 0 or world < 1 or chunk < 1:
        raise ValueError("T >= 0, world >= 1 and chunk >= 1 are required")
    nch = (T + chunk - 1) // chunk
    base, extra = divmod(nch, world)
    out, c = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        s, e = min(c * chunk, T), min((c + n) * chunk, T)
        out.append((s, e))
        c += n
    return out


def exchange_summaries(range_transition: torch.Tensor, range_contribution: torch.Tensor, group=None):
    """All-gather every rank's map in rank order: ([world, Hv, dk, dk], [world, Hv, <state>]).

    One collective per tensor into a preallocated buffer (a flat all-gather, which NCCL and gloo
    both take); the result is identical on every rank.
    """
    world = dist.get_world_size(group)
    outs = []
    for t in (range_transition, range_contribution):
        t = t.contiguous()
        buf = torch.empty((world * t.shape[0], *t.shape[1:]), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(buf, t, group=group)
        outs.append(buf.view(world, *t.shape))
    return outs[0], outs[1]


def _binding():
    import kimi_delta_attention_23_b200 as kda
    return kda


def context_parallel_prefill(q, k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, initial_state,
                             out=None, *, group=None, output_dtype=None, gate_mode="original",
                             beta_mode="logits", state_layout="K_FIRST", gate_lower_bound=-5.0,
                             device_status=None, stream=None, ops=None):
    """This rank's share of the context-parallel prefill of one sequence split across ``group``.

    q, k, v, raw_gate, beta_logits: this rank's token range (rows [starts[r], starts[r+1]) of the
    sequence; any length, including 0); seg_offsets: the range's own segment boundaries (device
    int32, 0 .. T_r); initial_state [Hv, <state>]: the sequence's initial state, the same on every
    rank.  Every rank must call this with the same head counts, layout and initial state.

    Returns dict(out [T_r, Hv, 128], final_state (the sequence's, on every rank), range_incoming,
    range_outgoing, and the range's segments' incoming_states, outgoing_states,
    transition_matrices, local_contributions).
    """
    ops = _binding() if ops is None else ops
    rank = dist.get_rank(group)
    if output_dtype is None:
        output_dtype = v.dtype if out is None else out.dtype
    kw = dict(gate_mode=gate_mode, beta_mode=beta_mode, state_layout=state_layout,
              gate_lower_bound=gate_lower_bound, device_status=device_status, stream=stream)
    ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
    with ctx:
        s = ops.kda_context_parallel_range_summary(q, k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets,
                                                   **kw)
        M_all, U_all = exchange_summaries(s["range_transition"], s["range_contribution"], group)
        scan = ops.kda_context_parallel(M_all, U_all, initial_state, state_layout=state_layout, stream=stream)
        range_in = scan["incoming_states"][rank].contiguous()
        f = ops.kda_context_parallel_range_finish(range_in, s["workspace"], seg_offsets, q.shape[0], out,
                                                  output_dtype=output_dtype, state_layout=state_layout,
                                                  device_status=device_status, stream=stream)
    f["final_state"] = scan["final_state"]
    f["range_incoming"] = range_in
    return f

