"""The C-ABI library loads here (no GPU) and exports every symbol include/kda.h declares; host-side
argument checks return their error codes before any CUDA call."""
import ctypes
import os
import re

import pytest

import kimi_delta_attention_23_b200 as kda
from kimi_delta_attention_23_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return re.findall(r"KDA_API\s+[\w\s\*]+?\b(kda_\w+)\s*\(", text)


def test_header_declares_the_boundary():
    names = set(declared_symbols())
    assert {"kda_chunk_fwd", "kda_segment_summarize_and_scan", "kda_workspace_size", "kda_status_string",
            "kda_version"} <= names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {kda.LIB_PATH}").read()
    exported = set(re.findall(r"\bT (kda_\w+)", out))
    assert set(declared_symbols()) <= exported


def test_status_strings_and_version(lib):
    for code in range(7):
        s = kda.kda_status_string(code)
        assert s.startswith("KDA_")
    assert kda.kda_status_string(99) == "KDA_ERR_UNKNOWN"
    assert lib.kda_version() >= 100
    assert kda.kda_workspace_size(1000, 2, 4, 4, 128, 128) == 0


def _chunk(lib, **over):
    args = dict(q=1, k=1, v=1, qkv=1, raw=1, beta=1, a_log=1, dt_bias=1, cu=1, batch=1, T=16, Hk=2, Hv=4,
                dk=128, dv=128, pool=1, slots=4, idx=1, out=1, out_dtype=1, flags=0)
    args.update(over)
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731  (never dereferenced: checks fail first)
    return lib.kda_chunk_fwd(p(args["q"]), p(args["k"]), p(args["v"]), args["qkv"], p(args["raw"]),
                             p(args["beta"]), p(args["a_log"]), p(args["dt_bias"]), p(args["cu"]), args["batch"],
                             args["T"], args["Hk"], args["Hv"], args["dk"], args["dv"], p(args["pool"]),
                             args["slots"], p(args["idx"]), p(args["out"]), args["out_dtype"], args["flags"],
                             -5.0, None, 0, None, None)


@pytest.mark.parametrize("over,code", [
    (dict(batch=-1), 1), (dict(T=-3), 1), (dict(Hk=0), 1), (dict(Hv=5), 1), (dict(dk=0), 1),
    (dict(slots=0), 1), (dict(flags=1 << 12), 1), (dict(flags=kda.SEG_SCAN_ONLY), 1), (dict(q=0), 1),
    (dict(pool=0), 1), (dict(idx=0), 1), (dict(cu=0), 1), (dict(out=0), 1), (dict(a_log=0), 1),
    (dict(qkv=7), 2), (dict(out_dtype=9), 2),
    (dict(qkv=0, out_dtype=1, Hv=2, Hk=2, dk=16, dv=16), 2),       # fp32 inputs need fp32 output
    (dict(qkv=0, out_dtype=0, dk=256, dv=16, Hv=2, Hk=2), 2),      # head dims beyond the kernels
    (dict(dk=64, dv=128), 2),                                       # bf16 fast path is dk = dv = 128
])
def test_chunk_fwd_host_checks(lib, over, code):
    assert _chunk(lib, **over) == code


def test_empty_batch_is_a_no_op(lib):
    assert _chunk(lib, batch=0, T=0) == 0


def _seg(lib, **over):
    args = dict(k=1, v=1, kv=1, raw=1, beta=1, a_log=1, dt_bias=1, T=64, Hk=2, Hv=2, dk=128, dv=128, offs=1,
                N=4, init=1, M=1, U=1, inc=1, outg=1, fin=1, q=0, rm=0, ru=0, flags=0)
    args.update(over)
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    return lib.kda_segment_summarize_and_scan(
        p(args["k"]), p(args["v"]), args["kv"], p(args["raw"]), p(args["beta"]), p(args["a_log"]),
        p(args["dt_bias"]), args["T"], args["Hk"], args["Hv"], args["dk"], args["dv"], p(args["offs"]),
        args["N"], p(args["init"]), p(args["M"]), p(args["U"]), p(args["inc"]), p(args["outg"]),
        p(args["fin"]), p(args["q"]), p(args["rm"]), p(args["ru"]), args["flags"], -5.0, None, 0, None, None)


@pytest.mark.parametrize("over,code", [
    (dict(N=0), 1), (dict(Hv=0), 1), (dict(init=0), 1), (dict(M=0), 1), (dict(U=0), 1), (dict(inc=0), 1),
    (dict(outg=0), 1), (dict(fin=0), 1), (dict(flags=1 << 20), 1), (dict(offs=0), 1), (dict(k=0), 1),
    (dict(Hk=3), 1), (dict(dk=129), 2), (dict(kv=5), 2),
    (dict(q=16), 1), (dict(q=16, rm=16), 1),                        # readouts need q and both outputs
    (dict(q=16, rm=16, ru=16, flags=kda.SEG_SCAN_ONLY), 1),
    (dict(q=16, rm=16, ru=16, kv=0), 2),                            # readouts only on the bf16 fast path
])
def test_segment_host_checks(lib, over, code):
    assert _seg(lib, **over) == code


def test_binding_refuses_cpu_tensors():
    import torch
    w = torch.zeros(4, 1, 16)
    with pytest.raises(ValueError, match="CUDA"):
        kda.kda_chunk_fwd(w, w, w, torch.zeros(4, 1, 16), torch.zeros(4, 1), torch.zeros(1), torch.zeros(1, 16),
                          torch.zeros(2, dtype=torch.int32), torch.zeros(1, 1, 16, 16),
                          torch.zeros(1, dtype=torch.int32))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback of any kind: without the built library the binding refuses to load
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(ImportError, match="not built"):
        kda.load_library()


def test_context_parallel_host_checks(lib):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    # apply: null pointers, dv != 128
    assert lib.kda_context_parallel_apply(None, p(16), p(16), p(16), 2, 64, 2, 128, p(16), 1, 0, None, None) == 1
    assert lib.kda_context_parallel_apply(p(16), p(16), p(16), p(16), 2, 64, 2, 64, p(16), 1, 0, None, None) == 2
    assert lib.kda_context_parallel_apply(p(16), p(16), p(16), p(16), 0, 64, 2, 128, p(16), 1, 0, None, None) == 1
    # prefill: workspace too small, fp32 inputs unsupported
    args = [p(16)] * 3 + [1] + [p(16)] * 4 + [64, 2, 2, 128, 128, p(16), 2, p(16), p(16), 1] + [p(16)] * 5 + [0, -5.0]
    assert lib.kda_context_parallel_prefill(*args, p(256), 16, None, None) == 3
    args_f32 = list(args)
    args_f32[3] = 0
    assert lib.kda_context_parallel_prefill(*args_f32, p(256), 1 << 30, None, None) == 2
    assert kda.kda_context_parallel_workspace_size(100, 4, 128) == 2 * 100 * 4 * 128 * 2


def test_piece_calls_host_checks(lib):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    assert lib.kda_context_parallel_piece_offsets(None, 2, 2, p(16), None) == 1
    assert lib.kda_context_parallel_piece_offsets(p(16), 0, 2, p(16), None) == 1
    assert lib.kda_context_parallel_piece_offsets(p(16), 2, 0, p(16), None) == 1
    args = [p(16)] * 4 + [2, 2, 2, 128, 128] + [p(16)] * 4 + [0, None]
    bad_null = list(args)
    bad_null[0] = None
    assert lib.kda_segment_compose(*bad_null) == 1
    bad_pieces = list(args)
    bad_pieces[5] = 0
    assert lib.kda_segment_compose(*bad_pieces) == 1
    bad_dims = list(args)
    bad_dims[7] = 256
    assert lib.kda_segment_compose(*bad_dims) == 2


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="the split depends on the device's SM count")
def test_without_a_device_nothing_is_split():
    # no CUDA device here: one piece per segment, the preferred workspace is the minimum
    assert kda.kda_context_parallel_pieces(1 << 17, 16, 32) == 1
    assert kda.kda_context_parallel_workspace_preferred(1 << 17, 16, 32, 128) == \
        kda.kda_context_parallel_workspace_size(1 << 17, 32, 128)


def _decode(lib, **over):
    args = dict(q=1, k=1, v=1, qkv=1, raw=1, beta=1, a_log=1, dt_bias=1, batch=3, Hk=2, Hv=4, dk=128, dv=128,
                pool=1, slots=4, idx=1, out=1, out_dtype=1, flags=0)
    args.update(over)
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731  (never dereferenced: checks fail first)
    return lib.kda_decode(p(args["q"]), p(args["k"]), p(args["v"]), args["qkv"], p(args["raw"]), p(args["beta"]),
                          p(args["a_log"]), p(args["dt_bias"]), args["batch"], args["Hk"], args["Hv"], args["dk"],
                          args["dv"], p(args["pool"]), args["slots"], p(args["idx"]), p(args["out"]),
                          args["out_dtype"], args["flags"], -5.0, None, None)


@pytest.mark.parametrize("over,code", [
    (dict(batch=-1), 1), (dict(Hk=0), 1), (dict(Hv=5), 1), (dict(dk=0), 1), (dict(dv=-2), 1), (dict(slots=0), 1),
    (dict(flags=kda.FUSED), 1), (dict(flags=kda.SEG_SCAN_ONLY), 1), (dict(flags=1 << 9), 1), (dict(q=0), 1),
    (dict(v=0), 1), (dict(raw=0), 1), (dict(pool=0), 1), (dict(idx=0), 1), (dict(out=0), 1), (dict(dt_bias=0), 1),
    (dict(qkv=5), 2), (dict(out_dtype=3), 2),
    (dict(qkv=0, out_dtype=1), 2),                                  # fp32 inputs need fp32 output
    (dict(dk=129), 2), (dict(dv=256), 2),                           # head dims beyond the kernel
])
def test_decode_host_checks(lib, over, code):
    assert _decode(lib, **over) == code


def test_decode_empty_batch_is_a_no_op(lib):
    assert _decode(lib, batch=0, q=0, k=0, v=0, raw=0, beta=0, out=0) == 0


def test_host_pipelined_prefill_host_checks(lib):
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731

    def call(segment=1024, qkv=1, final=16, flags=0, ws=256, ws_bytes=16, out_dtype=1):
        return lib.kda_prefill_host_pipelined(p(16), p(16), p(16), qkv, p(16), p(16), p(16), p(16), 4096, 2, 2, 128,
                                              128, p(16), p(16), out_dtype, p(final), segment, flags, -5.0, p(ws),
                                              ws_bytes, None, None)
    assert call(segment=100) == 1          # not a multiple of 64
    assert call(segment=0) == 1
    assert call(final=0) == 1              # null final state
    assert call(flags=1 << 4) == 1         # a segment-call flag
    assert call(qkv=0) == 2                # fp32 q/k/v bind no kernel here
    assert call() == 3                     # workspace too small
    need = kda.kda_prefill_host_workspace_size(4096, 2, 2, segment_tokens=1024)
    assert need >= 4096 * 2 * 128 * (2 + 2) + 4096 * 2 * 128 * (2 + 4 + 2)
    assert call(ws=256 + 8, ws_bytes=need) == 3  # workspace not 256-byte aligned
    assert kda.kda_prefill_host_workspace_size(4096, 2, 2, segment_tokens=100) == 0


def test_token_counts_beyond_int32_are_refused(lib):
    # token offsets are int32 (as cu_seqlens): larger counts are refused before any size arithmetic
    p = lambda x: ctypes.c_void_p(x) if x else None  # noqa: E731
    big = (1 << 31)
    assert _chunk(lib, T=big) == 1
    assert _seg(lib, T=big) == 1
    args = [p(16)] * 3 + [1] + [p(16)] * 4 + [big, 2, 2, 128, 128, p(16), 2, p(16), p(16), 1] + [p(16)] * 5 + \
        [0, -5.0]
    assert lib.kda_context_parallel_prefill(*args, p(256), 1 << 40, None, None) == 1
    fn = lib.kda_context_parallel_prefill_static
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    fn.restype = ctypes.c_int
    fn.argtypes = [vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, i64, i32, i32, i32, i32, vp, i32, vp, vp, ctypes.c_int,
                   vp, vp, vp, vp, vp, ctypes.c_uint32, ctypes.c_float, vp, vp]
    assert fn(*args, None, None) == 1
    assert lib.kda_context_parallel_apply(p(16), p(16), p(16), p(16), 2, big, 2, 128, p(16), 1, 0, None, None) == 1
    # the sizes say that no workspace can serve such a call
    assert kda.kda_context_parallel_workspace_size(big, 32, 128) == 2 ** 64 - 1
    assert kda.kda_context_parallel_workspace_preferred(big, 16, 32, 128) == 2 ** 64 - 1


def test_logdepth_scan_sizes_and_host_checks(lib):
    # two sets of every segment's prefix map: 2 * N * H * (128 * 128 + 128 * dv) floats
    assert kda.kda_scan_workspace_size(17, 3, 128, 64) == 2 * 17 * 3 * (128 * 128 + 128 * 64) * 4
    assert kda.kda_scan_workspace_size(17, 3, 64, 64) == 0    # dk must be 128
    assert kda.kda_scan_workspace_size(17, 3, 128, 48) == 0   # dv a multiple of 32
    assert lib.kda_scan_logdepth_preferred(1, 4, 128) == 0    # one segment: nothing to compose
    # forced without a workspace, or where it cannot run: refused before any launch
    assert _seg(lib, flags=kda.SEG_SCAN_ONLY | kda.SCAN_LOGDEPTH) == 3            # KDA_ERR_WORKSPACE
    assert _seg(lib, flags=kda.SEG_SCAN_ONLY | kda.SCAN_LOGDEPTH, dk=64) == 2     # KDA_ERR_UNSUPPORTED


def test_python_constants_match_the_header():
    """The binding's flag and status constants are the header's values."""
    text = open(HEADER).read()

    def enum_value(name):
        m = re.search(rf"\b{name}\s*=\s*(1u\s*<<\s*(\d+)|\d+)", text)
        assert m, name
        return (1 << int(m.group(2))) if m.group(2) else int(m.group(1))

    for py, c in (("GATE_SAFE", "KDA_GATE_SAFE"), ("BETA_PROB", "KDA_BETA_PROB"),
                  ("STATE_V_FIRST", "KDA_STATE_V_FIRST"), ("FUSED", "KDA_FUSED"),
                  ("SEG_SCAN_ONLY", "KDA_SEG_SCAN_ONLY"), ("FORCE_SIMT", "KDA_FORCE_SIMT"),
                  ("READOUT_HEAD_MAJOR", "KDA_READOUT_HEAD_MAJOR"), ("SCAN_LOGDEPTH", "KDA_SCAN_LOGDEPTH"),
                  ("DEBUG_WITHHOLD_HANDOFF", "KDA_DEBUG_WITHHOLD_HANDOFF"),
                  ("ERR_DEVICE_CHECK", "KDA_ERR_DEVICE_CHECK"), ("ERR_DEVICE_TIMEOUT", "KDA_ERR_DEVICE_TIMEOUT")):
        assert getattr(kda, py) == enum_value(c), (py, c)
    assert kda.kda_status_string(kda.ERR_DEVICE_TIMEOUT).startswith("KDA_ERR_DEVICE_TIMEOUT")
