"""The exclusive scan in log depth (KDA_SCAN_LOGDEPTH, through the C ABI) against the fp64
oracle's scan and against the sequential scan on the GPU.

"KDA Context Parallelism" (Compose segments in sequence order) notes that the composition is
associative; the log-depth form composes prefixes (P_i <- P_i o P_{i - 2^l}) and applies them to
the initial state.  Both GPU scans keep fp32 accuracy (three-term tf32 products), so the
tolerance is the scan tests' 1e-5 relative L2, per (segment, head) block as well as whole.
"""
import numpy as np
import pytest
import torch

import kimi_delta_attention_23_b200 as kda
import oracle
import parity

pytestmark = pytest.mark.gpu

TOL = 1e-5


def maps(N, H, dv, layout, seed):
    # transitions with spectral radius about 1/2, as a decaying segment's are (a product of many
    # stays inside fp32's range); contributions and the initial state O(1)
    rng = np.random.default_rng(seed)
    M = rng.normal(size=(N, H, 128, 128)) / (2 * np.sqrt(128))
    st = (128, dv) if layout == "K_FIRST" else (dv, 128)
    U = rng.normal(size=(N, H, *st))
    S0 = rng.normal(size=(H, *st))
    return M, U, S0


def cu(x):
    return torch.tensor(x, dtype=torch.float32, device="cuda")


@pytest.mark.parametrize("N", [1, 2, 17, 128])
@pytest.mark.parametrize("H,dv,layout", [(1, 128, "K_FIRST"), (3, 64, "V_FIRST")])
def test_logdepth_scan_matches_the_oracle_and_the_sequential_scan(cuda_device, N, H, dv, layout):
    M, U, S0 = maps(N, H, dv, layout, seed=N + H)
    ref = oracle.kda_affine_scan(M, U, S0, state_layout=layout)
    log = kda.kda_context_parallel(cu(M), cu(U), cu(S0), state_layout=layout, method="logdepth")
    seq = kda.kda_context_parallel(cu(M), cu(U), cu(S0), state_layout=layout, method="sequential")
    torch.cuda.synchronize()
    for key in ("incoming_states", "outgoing_states", "final_state"):
        parity.check_states(f"log-depth scan: {key}", log[key], ref[key], TOL)
        assert parity.rel_l2(log[key], seq[key]) <= TOL, key


def test_auto_choice_takes_log_depth_for_one_head_and_many_segments(cuda_device):
    N, H = 256, 1
    assert kda.kda_scan_logdepth_preferred(N, H, 128)
    assert not kda.kda_scan_logdepth_preferred(4, 32, 128)
    M, U, S0 = maps(N, H, 128, "K_FIRST", seed=7)
    ref = oracle.kda_affine_scan(M, U, S0)
    res = kda.kda_context_parallel(cu(M), cu(U), cu(S0), method="auto")
    torch.cuda.synchronize()
    for key in ("incoming_states", "outgoing_states", "final_state"):
        parity.check_states(f"log-depth scan (auto): {key}", res[key], ref[key], TOL)


def test_logdepth_needs_128_wide_keys(cuda_device):
    M, U, S0 = (torch.zeros(s, device="cuda") for s in ((3, 1, 16, 16), (3, 1, 16, 16), (1, 16, 16)))
    with pytest.raises(ValueError, match="dk = 128"):
        kda.kda_context_parallel(M, U, S0, method="logdepth")
