"""Context parallelism across ranks, on CPU: gloo ranks, each holding one token range of a
sequence, exchange their range maps through ``distributed.exchange_summaries`` (a real
all-gather); the three per-rank steps run on the fp64 oracle here (there is no GPU), so these
tests pin the cut into ranges, the exchange order and which incoming state each rank takes
against the oracle's straight token-by-token pass over the whole sequence."""
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import kda_workloads as W
import oracle
from kimi_delta_attention_23_b200 import distributed as D


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """The per-rank calls of ``context_parallel_prefill``, computed by the oracle."""

    def kda_context_parallel_range_summary(self, q, k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, *,
                                           gate_mode, beta_mode, state_layout, gate_lower_bound,
                                           device_status=None, stream=None):
        kw = dict(gate_mode=gate_mode, beta_mode=beta_mode, state_layout=state_layout,
                  gate_lower_bound=gate_lower_bound)
        M, U = oracle.kda_segment_summary(k, v, raw_gate, beta_logits, a_log, dt_bias,
                                          np.array([0, q.shape[0]], np.int32), **kw)
        ws = {"inputs": (q, k, v, raw_gate, beta_logits, a_log, dt_bias), "kw": kw}
        return {"range_transition": torch.from_numpy(M[0]), "range_contribution": torch.from_numpy(U[0]),
                "workspace": ws}

    def kda_context_parallel(self, M, U, initial_state, *, state_layout, stream=None):
        r = oracle.kda_affine_scan(M.numpy(), U.numpy(), initial_state.double().numpy(), state_layout=state_layout)
        return {key: torch.from_numpy(val) for key, val in r.items()}

    def kda_context_parallel_range_finish(self, range_incoming, workspace, seg_offsets, tokens, out=None, *,
                                          output_dtype, state_layout, device_status=None, stream=None):
        q, k, v, raw_gate, beta_logits, a_log, dt_bias = workspace["inputs"]
        kw = workspace["kw"]
        S = range_incoming.numpy()
        o, pool = oracle.kda_forward(q, k, v, raw_gate, beta_logits, a_log, dt_bias, np.array([0, tokens], np.int32),
                                     S[None], np.array([0], np.int32), **kw)
        M, U = oracle.kda_segment_summary(k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets.numpy(), **kw)
        sc = oracle.kda_affine_scan(M, U, S, state_layout=state_layout)
        return {"out": torch.from_numpy(o), "range_outgoing": torch.from_numpy(pool[0]),
                "incoming_states": torch.from_numpy(sc["incoming_states"]),
                "outgoing_states": torch.from_numpy(sc["outgoing_states"]),
                "transition_matrices": torch.from_numpy(M), "local_contributions": torch.from_numpy(U)}


def _case(T, layout):
    return W.random_inputs([T], 2, 4, 16, 16, seed=T + 7, qkv_dtype=torch.float32, output_dtype=torch.float32,
                           state_std=0.3, state_layout=layout)


def _local_segments(n, parts):
    # the range's own cut: `parts` pieces of uneven length (empty ones allowed)
    cuts = [0] + [int(n * f) for f in (0.3, 0.55, 0.9)[: parts - 1]] + [n]
    return torch.tensor(cuts, dtype=torch.int32)


def _rank_main(rank, world, port, T, chunk, layout, out):
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        w = _case(T, layout)
        s, e = D.rank_ranges(T, world, chunk)[rank]
        sl = slice(s, e)
        res = D.context_parallel_prefill(w.q[sl], w.k[sl], w.v[sl], w.raw_gate[sl], w.beta_logits[sl], w.a_log,
                                         w.dt_bias, _local_segments(e - s, 3), w.state_pool[0],
                                         state_layout=layout, ops=OracleOps())
        got = {key: (val.numpy() if isinstance(val, torch.Tensor) else val) for key, val in res.items()}
        got["range"] = (s, e)
        out[rank] = got  # one assignment: the manager's dict keeps no change made inside a value
    finally:
        dist.destroy_process_group()


def _run(world, T, chunk, layout):
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, port, T, chunk, layout, out), nprocs=world, start_method="spawn",
                       join=True)
    return [dict(out[r]) for r in range(world)]


def _rel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


@pytest.mark.parametrize("world,T,chunk,layout", [(2, 150, 16, "K_FIRST"), (3, 150, 16, "V_FIRST"),
                                                  (3, 20, 16, "K_FIRST")])
def test_ranks_reproduce_the_straight_pass(world, T, chunk, layout):
    res = _run(world, T, chunk, layout)
    w = _case(T, layout)
    o_ref, p_ref = oracle.kda_forward(w.q, w.k, w.v, w.raw_gate, w.beta_logits, w.a_log, w.dt_bias, w.cu_seqlens,
                                      w.state_pool, w.state_indices, state_layout=layout)
    assert [r["range"] for r in res] == D.rank_ranges(T, world, chunk)
    out = np.concatenate([r["out"] for r in res], axis=0)
    assert out.shape == o_ref.shape
    assert _rel(out, o_ref) < 1e-10
    for r in res:
        assert _rel(r["final_state"], p_ref[0]) < 1e-10  # the sequence's final state on every rank
        s, e = r["range"]
        # the state entering the range is the straight pass's state after token s - 1
        _, p_s = oracle.kda_forward(w.q[:s], w.k[:s], w.v[:s], w.raw_gate[:s], w.beta_logits[:s], w.a_log,
                                    w.dt_bias, np.array([0, s], np.int32), w.state_pool, w.state_indices,
                                    state_layout=layout)
        assert _rel(r["range_incoming"], p_s[0]) < 1e-10
        # segments inside the range continue from it: their first incoming state is the range's
        assert _rel(r["incoming_states"][0], r["range_incoming"]) < 1e-12
    for a, b in zip(res, res[1:]):
        assert _rel(b["range_incoming"], a["range_outgoing"]) < 1e-10


def test_exchange_gathers_in_rank_order():
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_exchange_main, args=(3, port, out), nprocs=3, start_method="spawn", join=True)
    for r in range(3):
        M_all, U_all = out[r]
        assert M_all.shape == (3, 2, 4, 4) and U_all.shape == (3, 2, 4, 5)
        for src in range(3):
            assert np.all(M_all[src] == src + 1) and np.all(U_all[src] == -(src + 1))


def _exchange_main(rank, world, port, out):
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    try:
        M = torch.full((2, 4, 4), float(rank + 1))
        U = torch.full((2, 4, 5), -float(rank + 1))
        M_all, U_all = D.exchange_summaries(M, U)
        out[rank] = (M_all.numpy(), U_all.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,world,chunk", [(0, 1, 64), (1, 1, 64), (131072, 8, 64), (150, 3, 16), (20, 3, 16),
                                           (64 * 7 + 5, 4, 64), (63, 2, 64)])
def test_rank_ranges_cover_the_sequence_in_order(T, world, chunk):
    rr = D.rank_ranges(T, world, chunk)
    assert len(rr) == world and rr[0][0] == 0 and rr[-1][1] == T
    for (s0, e0), (s1, e1) in zip(rr, rr[1:]):
        assert e0 == s1
    chunks = [(e - s + chunk - 1) // chunk for s, e in rr]
    assert max(chunks) - min(chunks) <= 1
    assert chunks == sorted(chunks, reverse=True)  # earlier ranks take the extra chunks
    for s, e in rr:
        assert (s % chunk == 0 or s == T) and (e % chunk == 0 or e == T) and s <= e


def test_rank_ranges_rejects_bad_arguments():
    with pytest.raises(ValueError):
        D.rank_ranges(-1, 2)
    with pytest.raises(ValueError):
        D.rank_ranges(10, 0)
