"""The benchmark's roofline accounting on the CPU: the algorithmic bytes and FLOPs per launch
against figures worked out by hand from their definitions (per token-head: q, k, v, the fp32
gate row, beta and the output; per chain: the fp32 state read and written once), the step
roofline's arithmetic, and the rule that a recorded DRAM traffic figure is reported only while
the sources it was measured on are unchanged."""
import json
import os
import types

import pytest
import torch

import bench


def workload(T, Hv, Hk=None, batch=1, qkv=torch.bfloat16, out=torch.bfloat16):
    """The fields the accounting reads, without allocating the inputs."""
    return types.SimpleNamespace(total_tokens=T, num_v_heads=Hv, num_k_heads=Hk or Hv, batch=batch,
                                 dk=128, dv=128, q=torch.empty(0, dtype=qkv), output_dtype=out)


def test_prefill_bytes_per_token_head_and_chain():
    # q, k: 2 x 128 x 2 B; v: 128 x 2 B; gate row: 128 x 4 B; beta: 4 B; output: 128 x 2 B
    per_token_head = 2 * 128 * 2 + 128 * 2 + 128 * 4 + 4 + 128 * 2
    assert per_token_head == 1540
    per_chain = 2 * 128 * 128 * 4  # the state read and written once
    w = workload(131072, 16, batch=64)
    assert bench.chunk_fwd_bytes(w, w.batch) == 1540 * 131072 * 16 + 64 * 16 * per_chain == 3363831808


def test_grouped_heads_read_q_and_k_once_per_key_head():
    w = workload(1000, 8, Hk=2)
    expected = 1000 * 8 * ((2 * 128 * 2) / 4 + 128 * 2 + 128 * 4 + 4 + 128 * 2) + 8 * 2 * 128 * 128 * 4
    assert bench.chunk_fwd_bytes(w, 1) == expected


def test_fp32_inputs_and_outputs_count_four_bytes():
    w = workload(64, 1, qkv=torch.float32, out=torch.float32)
    assert bench.chunk_fwd_bytes(w, 1, dk=16, dv=16) == 64 * (2 * 16 * 4 + 16 * 4 + 16 * 4 + 4 + 16 * 4) + 2 * 16 * 16 * 4


def test_decode_bytes_per_sequence_head():
    w = workload(256, 32, batch=256)
    assert bench.decode_bytes(w) == 256 * 32 * (1540 + 2 * 128 * 128 * 4)
    assert 1540 + 2 * 128 * 128 * 4 == 132612


def test_segment_build_bytes_of_the_long_step():
    # the method's bytes of the build over 32 pieces: q, k, v, gate, beta in (1284 B per
    # token-head), each piece-head's M and U out; then the scan reads M, U and writes the
    # incoming and outgoing states.  The two bf16 readouts per token-head (512 B) are the
    # design's intermediate and are counted apart.
    w = workload(131072, 32)
    th = 131072 * 32
    summaries = 32 * 32 * 2 * 128 * 128 * 4
    expected = th * 1284 + summaries + summaries + 32 * 32 * 2 * 128 * 128 * 4
    assert bench.segment_build_bytes(w, 32) == expected == 5788139520
    assert bench.segment_build_intermediate_bytes(w) == th * 512 == 2147483648


def test_apply_bytes():
    w = workload(131072, 32)
    assert bench.apply_bytes(w, 32) == 131072 * 32 * (512 + 256) + 32 * 32 * 128 * 128 * 4


def test_flops_per_token_head():
    # 6 d^2 (three d x d products) + 5 C d + C^2 / 3 at C = 64, d = 128
    w = workload(1, 1)
    assert bench.chunk_fwd_flops(w) == pytest.approx(6 * 128 * 128 + 5 * 64 * 128 + 64 * 64 / 3)
    assert bench.chunk_fwd_flops(w) == pytest.approx(140629.33, rel=1e-6)


@pytest.mark.parametrize("segments", [0, 16])
def test_step_roofline_takes_the_slower_bound(segments):
    w = workload(131072, 32, batch=1)
    pk = {"hbm_gbs": 6552.0, "bf16_tflops": 1590.0, "source": "measured"}
    r = bench.step_roofline(w, 5.0, segments, pk)
    nbytes = bench.chunk_fwd_bytes(w, 1) + (2 * segments * 32 * 3 * 128 * 128 * 4 if segments else 0)
    assert r["algorithmic_bytes"] == nbytes
    assert r["hbm_ms"] == pytest.approx(nbytes / 6552e9 * 1e3)
    assert r["tensor_ms"] == pytest.approx(bench.chunk_fwd_flops(w) / 1590e12 * 1e3)
    assert r["bound"] == "hbm" and r["roofline_ms"] == r["hbm_ms"]  # 91 FLOP per byte: below the ridge
    assert r["frac"] == pytest.approx(r["roofline_ms"] / 5.0)
    assert r["gbs"] == pytest.approx(nbytes / 5e-3 / 1e9)


def test_recorded_traffic_only_while_the_sources_are_unchanged(tmp_path, monkeypatch):
    csrc = tmp_path / "kimi_delta_attention_23_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "a.cu").write_text("one kernel\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", {"k": ["a.cu"]})
    record = {"k": {"dram_bytes_per_launch": 123.0, "source_hash": bench.kernel_source_hash("k")}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(record))
    assert bench.recorded_traffic("k") == 123.0
    assert bench.recorded_traffic("other") is None
    (csrc / "a.cu").write_text("the kernel changed\n")
    assert bench.recorded_traffic("k") is None


def test_committed_traffic_records_name_known_kernels():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    assert set(d) <= set(bench.KERNEL_SOURCES)
    for e in d.values():
        assert e["dram_bytes_per_launch"] > 0 and len(e["source_hash"]) == 16 and e["from"]
