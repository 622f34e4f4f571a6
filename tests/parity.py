"""Parity measures shared by the GPU tests.

Every comparison with the fp64 oracle is made two ways:
  * the relative L2 error over the whole tensor (the tolerance's definition), and
  * the relative L2 error of every (sequence, head) chain on its own -- its output rows, or its
    state block -- so that an error confined to a short sequence or to one head cannot hide
    under the norm of the rest.
Both must be within the tolerance.  Each figure is recorded (test id, label, whole-tensor
error, worst chain and where it is) and ``tests/conftest.py`` prints the worst figures per
label at the end of the run.

Transition matrices M decay towards zero over a long segment (with the workloads' gates a
few hundred tokens take them below fp32's range); there a relative error says nothing, so
``check_maps`` divides a chain's error by the larger of its own norm and a floor of 1e-20
times the identity's norm: a transition that small changes no fp32 state it is applied to.
"""
from __future__ import annotations

import os

import numpy as np

RECORDS: list[dict] = []


def _np(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, np.float64)


def rel_l2(x, ref) -> float:
    x, ref = _np(x), _np(ref)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def _record(label, whole, worst, where, tol, chains):
    RECORDS.append({"test": os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0], "label": label,
                    "whole": whole, "worst": worst, "where": where, "tol": tol, "chains": chains})


def row_chain_errors(x, ref, cu):
    """Per (sequence, head) relative L2 of token-major rows [T, H, d]: sequence b owns rows
    cu[b]..cu[b+1]-1.  Returns (errors [B', H], sequence index of each row of errors); empty
    sequences have no rows and no entry."""
    x, ref = _np(x), _np(ref)
    cu = [int(c) for c in _np(cu).astype(np.int64)]
    d2 = ((x - ref) ** 2).sum(axis=-1)  # [T, H]
    r2 = (ref ** 2).sum(axis=-1)
    errs, seqs = [], []
    for b in range(len(cu) - 1):
        s, e = cu[b], cu[b + 1]
        if e <= s:
            continue
        num, den = d2[s:e].sum(axis=0), r2[s:e].sum(axis=0)
        errs.append(np.sqrt(num) / np.where(den > 0, np.sqrt(den), 1.0))
        seqs.append(b)
    return (np.array(errs) if errs else np.zeros((0, x.shape[1]))), seqs


def check_rows(label, x, ref, tol, cu=None):
    """Output rows [T, H, d] (cu: the sequences' row offsets; None = one sequence)."""
    x, ref = _np(x), _np(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    if cu is None:
        cu = [0, x.shape[0]]
    whole = rel_l2(x, ref)
    errs, seqs = row_chain_errors(x, ref, cu)
    worst, where = 0.0, None
    if errs.size:
        i, h = np.unravel_index(int(np.argmax(errs)), errs.shape)
        worst, where = float(errs[i, h]), f"seq {seqs[i]} head {h}"
    _record(label, whole, worst, where, tol, int(errs.size))
    assert whole <= tol, f"{label}: whole-tensor rel L2 {whole:.3e} > {tol}"
    assert worst <= tol, f"{label}: chain ({where}) rel L2 {worst:.3e} > {tol}"
    return whole, worst


def _block_errors(x, ref, floor=0.0):
    d = np.sqrt(((x - ref) ** 2).sum(axis=(-2, -1)))
    n = np.sqrt((ref ** 2).sum(axis=(-2, -1)))
    return d / np.maximum(np.where(n > 0, n, 1.0), floor)


def check_states(label, x, ref, tol, floor=0.0):
    """State-like blocks [..., H, a, b] (pool slots, segments' U / incoming / outgoing, final
    states): one chain per leading index and head."""
    x, ref = _np(x), _np(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    whole = rel_l2(x, ref)
    errs = _block_errors(x, ref, floor)
    worst, where = 0.0, None
    if errs.size:
        idx = np.unravel_index(int(np.argmax(errs)), errs.shape)
        worst, where = float(errs[idx]), "block " + ",".join(str(int(i)) for i in idx)
    _record(label, whole, worst, where, tol, int(errs.size))
    assert whole <= tol, f"{label}: whole-tensor rel L2 {whole:.3e} > {tol}"
    assert worst <= tol, f"{label}: chain ({where}) rel L2 {worst:.3e} > {tol}"
    return whole, worst


def check_maps(label, x, ref, tol):
    """Transition matrices [N, H, dk, dk]: per (segment, head), relative to the larger of the
    block's norm and 1e-20 times the identity's norm."""
    ref_n = _np(ref)
    floor = 1e-20 * np.sqrt(ref_n.shape[-1])
    return check_states(label, x, ref_n, tol, floor=floor)


# the named workloads: their labels are always listed, whatever their rank
WORKLOADS = ("tiny_fp32_T64_d16", "single_T4096_H16", "varlen8_H32_vfirst", "long_T131072_H32",
             "batch64_T2048_H16_safe", "decode_B256_H32", "decode_B64_H16_safe", "bf16 small[1]")


def summary_lines(max_lines=16):
    """The worst whole-tensor and per-chain figures per label (labels name a workload or a
    case and the quantity), worst ratio to the tolerance first, then every label of a named
    workload."""
    by = {}
    for r in RECORDS:
        e = by.setdefault(r["label"], {"whole": 0.0, "worst": 0.0, "where": None, "tol": r["tol"], "n": 0,
                                       "chains": 0, "test": r["test"]})
        e["n"] += 1
        e["chains"] += r["chains"]
        e["whole"] = max(e["whole"], r["whole"])
        if r["worst"] >= e["worst"]:
            e["worst"], e["where"], e["test"] = r["worst"], r["where"], r["test"]
        e["tol"] = max(e["tol"], r["tol"])
    rows = sorted(by.items(), key=lambda kv: -max(kv[1]["worst"], kv[1]["whole"]) / kv[1]["tol"])
    out = [f"parity vs the fp64 oracle: {len(RECORDS)} checks, {sum(e['chains'] for e in by.values())} "
           f"chains; worst per label (whole tensor / worst chain, tolerance):"]
    shown = rows[:max_lines] + [kv for kv in rows[max_lines:] if any(n in kv[0] for n in WORKLOADS)]
    for label, e in shown:
        out.append(f"  {label:<44s} {e['whole']:.2e} / {e['worst']:.2e} ({e['where']}) tol {e['tol']:.0e}")
    if len(rows) > len(shown):
        out.append(f"  ... {len(rows) - len(shown)} more labels, all below the first {max_lines} ratios")
    return out
