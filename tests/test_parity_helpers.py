"""The GPU tests' parity measures, on the CPU: an error confined to one short sequence or one
head is caught by the per-chain bound even where the whole-tensor error is within tolerance."""
import numpy as np
import pytest

import parity


@pytest.fixture(autouse=True)
def _keep_records_clean():
    # these cases plant errors on purpose; they stay out of the run's parity summary
    n0 = len(parity.RECORDS)
    yield
    del parity.RECORDS[n0:]


def test_error_in_a_one_token_sequence_is_caught_per_chain():
    rng = np.random.default_rng(0)
    cu = [0, 300, 301, 430, 494, 494, 1005]  # lengths 300, 1, 129, 64, 0, 511
    ref = rng.normal(size=(1005, 2, 128))
    x = ref.copy()
    x[300, 1] *= 1.2  # 20 % off on the one-token sequence's second head
    assert parity.rel_l2(x, ref) < 1e-2
    with pytest.raises(AssertionError, match="seq 1 head 1"):
        parity.check_rows("planted", x, ref, 1e-2, cu=cu)


def test_per_chain_errors_skip_empty_sequences_and_match_by_hand():
    ref = np.ones((5, 1, 4))
    x = ref.copy()
    x[3:5] *= 1.5
    errs, seqs = parity.row_chain_errors(x, ref, [0, 3, 3, 5])
    assert seqs == [0, 2]
    assert errs[0, 0] == 0.0 and errs[1, 0] == pytest.approx(0.5)


def test_state_blocks_are_chains_per_slot_and_head():
    rng = np.random.default_rng(1)
    ref = rng.normal(size=(4, 8, 16, 16))
    x = ref.copy()
    x[2, 5] += 0.05 * np.abs(ref[2, 5]).mean()
    whole, worst = parity.check_states("ok", x, ref, 1e-1)
    assert worst > whole
    with pytest.raises(AssertionError, match="block 2,5"):
        parity.check_states("planted", x, ref, 1e-2)


def test_decayed_transitions_are_compared_against_the_floor():
    ref = np.zeros((2, 1, 8, 8))
    ref[0, 0] = np.eye(8)
    ref[1, 0] = 1e-30 * np.eye(8)  # decayed far below anything it could change
    x = ref.copy()
    x[1, 0] = 0.0
    parity.check_maps("decayed", x, ref, 1e-2)
    x[0, 0, 0, 0] = 1.1
    with pytest.raises(AssertionError):
        parity.check_maps("planted", x, ref, 1e-2)


def test_summary_names_the_worst_chain():
    n0 = len(parity.RECORDS)
    ref = np.ones((10, 1, 4))
    parity.check_rows("summary case", ref * 1.001, ref, 1e-2, cu=[0, 4, 10])
    lines = parity.summary_lines()
    assert len(parity.RECORDS) == n0 + 1
    assert any("summary case" in ln and "seq" in ln for ln in lines)
