"""Python binding of libkda.so, the sm_100a KDA prefill library (argument marshalling only).

Every step of the computation runs in the CUDA kernels behind the C ABI in ``include/kda.h``;
this module only turns torch tensors into pointers and extents.  PyTorch supplies device
memory and streams.  There is no CPU path: if ``libkda.so`` is missing, every call raises.

Public calls (same names as the C ABI):
  kda_chunk_fwd(...)                      chunk-parallel prefill, mutates state_pool in place
  kda_decode(...)                         one token per sequence, mutates state_pool in place
  kda_segment_summarize_and_scan(...)     segment (M_i, U_i) summaries + exclusive scan
  kda_context_parallel(M, U, initial)     the scan alone, returning exactly incoming_states,
                                          outgoing_states and final_state
  kda_context_parallel_prefill(...)       the context-parallel prefill of one long sequence
  kda_prefill_host_pipelined(...)         kda_chunk_fwd on one sequence in pinned host memory, the
                                          copies pipelined with the kernels in segments
  kda_context_parallel_range_summary(...) one rank's token range of a sequence as one map
  kda_context_parallel_range_finish(...)  that range's outputs from the state entering it
                                          (``distributed.context_parallel_prefill`` joins the
                                          two across ranks with one all-gather)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["kda_chunk_fwd", "kda_decode", "kda_segment_summarize_and_scan", "kda_context_parallel",
           "kda_context_parallel_apply", "kda_context_parallel_prefill", "kda_context_parallel_workspace_size",
           "kda_context_parallel_workspace_preferred", "kda_context_parallel_pieces",
           "kda_context_parallel_piece_offsets", "kda_segment_compose", "kda_context_parallel_range_workspace_size",
           "kda_context_parallel_range_summary", "kda_context_parallel_range_finish", "kda_prefill_host_pipelined",
           "kda_prefill_host_workspace_size", "kda_workspace_size",
           "kda_status_string", "load_library", "KdaError", "LIB_PATH"]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

# flag bits of include/kda.h
GATE_SAFE = 1 << 0
BETA_PROB = 1 << 1
STATE_V_FIRST = 1 << 2
FUSED = 1 << 3
SEG_SCAN_ONLY = 1 << 4
FORCE_SIMT = 1 << 5
READOUT_HEAD_MAJOR = 1 << 6
SCAN_LOGDEPTH = 1 << 7
DEBUG_WITHHOLD_HANDOFF = 1 << 8  # test hook: see include/kda.h
# device_status values (kda_status_t in include/kda.h) that callers test for
ERR_DEVICE_CHECK = 5
ERR_DEVICE_TIMEOUT = 6

_F32, _BF16 = 0, 1
_DTYPES = {torch.float32: _F32, torch.bfloat16: _BF16}

_lib = None


class KdaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {kda_status_string(code)} (status {code})")


def load_library():
    """Load libkda.so (built in-tree by ``build.py``); raise loudly if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkda.so is not built at {LIB_PATH}; run kimi_delta_attention_23_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    i32, i64, u32, f32, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32, ctypes.c_float, ctypes.c_size_t
    lib.kda_chunk_fwd.restype = ctypes.c_int
    lib.kda_chunk_fwd.argtypes = [vp, vp, vp, ctypes.c_int, fp, fp, fp, fp, ip, i32, i64, i32, i32, i32,
                                  i32, fp, i32, ip, vp, ctypes.c_int, u32, f32, vp, sz, ip, vp]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_decode.argtypes = [vp, vp, vp, ctypes.c_int, fp, fp, fp, fp, i32, i32, i32, i32, i32, fp, i32, ip,
                               vp, ctypes.c_int, u32, f32, ip, vp]
    lib.kda_segment_summarize_and_scan.restype = ctypes.c_int
    lib.kda_segment_summarize_and_scan.argtypes = [vp, vp, ctypes.c_int, fp, fp, fp, fp, i64, i32, i32,
                                                   i32, i32, ip, i32, fp, fp, fp, fp, fp, fp, vp, vp, vp, u32,
                                                   f32, vp, sz, ip, vp]
    lib.kda_context_parallel_apply.restype = ctypes.c_int
    lib.kda_context_parallel_apply.argtypes = [vp, vp, fp, ip, i32, i64, i32, i32, vp, ctypes.c_int, u32, ip, vp]
    lib.kda_context_parallel_prefill.restype = ctypes.c_int
    lib.kda_context_parallel_prefill.argtypes = [vp, vp, vp, ctypes.c_int, fp, fp, fp, fp, i64, i32, i32, i32, i32,
                                                 ip, i32, fp, vp, ctypes.c_int, fp, fp, fp, fp, fp, u32, f32, vp, sz,
                                                 ip, vp]
    lib.kda_context_parallel_workspace_size.restype = sz
    lib.kda_context_parallel_workspace_size.argtypes = [i64, i32, i32]
    lib.kda_context_parallel_piece_offsets.restype = ctypes.c_int
    lib.kda_context_parallel_piece_offsets.argtypes = [ip, i32, i32, ip, vp]
    lib.kda_context_parallel_pieces.restype = i32
    lib.kda_context_parallel_pieces.argtypes = [i64, i32, i32]
    lib.kda_segment_compose.restype = ctypes.c_int
    lib.kda_segment_compose.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, u32, vp]
    lib.kda_context_parallel_workspace_preferred.restype = sz
    lib.kda_context_parallel_workspace_preferred.argtypes = [i64, i32, i32, i32]
    lib.kda_context_parallel_range_workspace_size.restype = sz
    lib.kda_context_parallel_range_workspace_size.argtypes = [i64, i32, i32, i32]
    lib.kda_context_parallel_range_summary.restype = ctypes.c_int
    lib.kda_context_parallel_range_summary.argtypes = [vp, vp, vp, ctypes.c_int, fp, fp, fp, fp, i64, i32, i32,
                                                       i32, i32, ip, i32, fp, fp, u32, f32, vp, sz, ip, vp]
    lib.kda_context_parallel_range_finish.restype = ctypes.c_int
    lib.kda_context_parallel_range_finish.argtypes = [i64, i32, i32, i32, i32, fp, vp, ctypes.c_int, fp, fp, fp,
                                                      fp, fp, u32, vp, sz, ip, vp]
    lib.kda_prefill_host_workspace_size.restype = sz
    lib.kda_prefill_host_workspace_size.argtypes = [i64, i32, i32, ctypes.c_int, i64]
    lib.kda_prefill_host_pipelined.restype = ctypes.c_int
    lib.kda_prefill_host_pipelined.argtypes = [vp, vp, vp, ctypes.c_int, fp, fp, fp, fp, i64, i32, i32, i32, i32, fp,
                                               vp, ctypes.c_int, fp, i64, u32, f32, vp, sz, ip, vp]
    lib.kda_workspace_size.restype = sz
    lib.kda_workspace_size.argtypes = [i64, i32, i32, i32, i32, i32, i32, u32]
    lib.kda_scan_workspace_size.restype = sz
    lib.kda_scan_workspace_size.argtypes = [i32, i32, i32, i32]
    lib.kda_scan_logdepth_preferred.restype = i32
    lib.kda_scan_logdepth_preferred.argtypes = [i32, i32, i32]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_version.restype = i32
    lib.kda_version.argtypes = []
    _lib = lib
    return lib


def kda_status_string(code: int) -> str:
    return load_library().kda_status_string(int(code)).decode()


def kda_workspace_size(total_tokens, batch, num_k_heads, num_v_heads, dk, dv, num_segments=0, flags=0) -> int:
    return int(load_library().kda_workspace_size(total_tokens, batch, num_k_heads, num_v_heads, dk, dv,
                                                 num_segments, flags))


def _flags(gate_mode, beta_mode, state_layout, use_computebound=False, force_simt=False, scan_only=False):
    if gate_mode not in ("original", "safe"):
        raise ValueError(f"gate_mode must be 'original' or 'safe', got {gate_mode!r}")
    if beta_mode not in ("logits", "probability"):
        raise ValueError(f"beta_mode must be 'logits' or 'probability', got {beta_mode!r}")
    if state_layout not in ("K_FIRST", "V_FIRST"):
        raise ValueError(f"state_layout must be 'K_FIRST' or 'V_FIRST', got {state_layout!r}")
    f = 0
    f |= GATE_SAFE if gate_mode == "safe" else 0
    f |= BETA_PROB if beta_mode == "probability" else 0
    f |= STATE_V_FIRST if state_layout == "V_FIRST" else 0
    f |= FUSED if use_computebound else 0
    f |= FORCE_SIMT if force_simt else 0
    f |= SEG_SCAN_ONLY if scan_only else 0
    return f


def _readout_flags(readout_layout):
    if readout_layout not in ("token_major", "head_major"):
        raise ValueError(f"readout_layout must be 'token_major' or 'head_major', got {readout_layout!r}")
    return READOUT_HEAD_MAJOR if readout_layout == "head_major" else 0


def _readout_shape(T, Hv, dv, readout_layout):
    return (Hv, T, dv) if readout_layout == "head_major" else (T, Hv, dv)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str, dtype=None, device=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor (got {t.device}); there is no CPU path")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t, name, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


class _Owned:
    """Device tensors a wrapper allocates itself (results and scratch).

    PyTorch's caching allocator ties a block to the stream that was current when it was
    allocated.  The kernels run on ``stream``; when that is another stream, every such tensor is
    marked as in use there (``record_stream``), so that its memory goes to other work only after
    the kernels on ``stream`` are done with it -- the scratch a wrapper drops at return as much as
    a result the caller frees later."""

    def __init__(self, stream, device):
        self.stream, self.device, self.tensors = stream, device, []

    def empty(self, *shape, **kw):
        t = torch.empty(*shape, **kw)
        self.tensors.append(t)
        return t

    def keep(self, t, original=None):
        # a temporary made from a caller's tensor (.contiguous() and the like); the caller's own
        # tensor is left alone
        if original is None or t.data_ptr() != original.data_ptr():
            self.tensors.append(t)
        return t

    def launched(self):
        if self.stream is None or self.stream == torch.cuda.current_stream(self.device):
            return
        for t in self.tensors:
            if t.numel() and t.device.type == "cuda":
                t.record_stream(self.stream)


def kda_chunk_fwd(q, k, v, raw_gate, beta_logits, a_log, dt_bias, cu_seqlens, state_pool, state_indices,
                  out=None, *, output_dtype=None, use_computebound=False, gate_mode="original",
                  beta_mode="logits", state_layout="K_FIRST", gate_lower_bound=-5.0, force_simt=False,
                  workspace=None, device_status=None, stream=None, _debug_flags=0):
    """Chunk-parallel KDA prefill (``max.nn.state_space.kda_chunk`` semantics).

    Shapes: q,k [T,Hk,dk]; v [T,Hv,dv]; raw_gate [T,Hv,dk] f32; beta_logits [T,Hv] f32;
    a_log [Hv] f32; dt_bias [Hv,dk] f32; cu_seqlens [B+1] i32; state_pool [slots,Hv,dk,dv]
    (K_FIRST) or [slots,Hv,dv,dk] (V_FIRST) f32, mutated in place; state_indices [B] i32.
    Returns out [T,Hv,dv] in ``output_dtype`` (default: the dtype of v).  ``workspace`` (uint8
    CUDA tensor) enables the split route for batches of few or uneven sequences; it is
    allocated at kda_workspace_size bytes when not given (pass an empty tensor to disable).
    ``_debug_flags`` is OR-ed into the call's flags (tests pass ``DEBUG_WITHHOLD_HANDOFF``).
    """
    lib = load_library()
    dev = q.device
    own = _Owned(stream, dev)
    _dev(q, "q", device=dev)
    if q.dtype not in _DTYPES:
        raise ValueError("q/k/v must be float32 or bfloat16")
    T, Hk, dk = q.shape
    _dev(k, "k", q.dtype, dev)
    _shape(k, "k", (T, Hk, dk))
    _dev(v, "v", q.dtype, dev)
    if v.dim() != 3 or v.shape[0] != T:
        raise ValueError(f"v has shape {tuple(v.shape)}, expected [{T}, Hv, dv]")
    Hv, dv = v.shape[1], v.shape[2]
    _shape(_dev(raw_gate, "raw_gate", torch.float32, dev), "raw_gate", (T, Hv, dk))
    _shape(_dev(beta_logits, "beta_logits", torch.float32, dev), "beta_logits", (T, Hv))
    _shape(_dev(a_log, "a_log", torch.float32, dev), "a_log", (Hv,))
    _shape(_dev(dt_bias, "dt_bias", torch.float32, dev), "dt_bias", (Hv, dk))
    _dev(cu_seqlens, "cu_seqlens", torch.int32, dev)
    B = cu_seqlens.numel() - 1
    _shape(_dev(state_indices, "state_indices", torch.int32, dev), "state_indices", (B,))
    _dev(state_pool, "state_pool", torch.float32, dev)
    blk = (Hv, dk, dv) if state_layout == "K_FIRST" else (Hv, dv, dk)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != blk:
        raise ValueError(f"state_pool has shape {tuple(state_pool.shape)}, expected [slots, {blk}]")
    if output_dtype is None:
        output_dtype = v.dtype if out is None else out.dtype
    if output_dtype not in _DTYPES:
        raise ValueError("output_dtype must be float32 or bfloat16")
    if out is None:
        out = own.empty((T, Hv, dv), dtype=output_dtype, device=dev)
    _shape(_dev(out, "out", output_dtype, dev), "out", (T, Hv, dv))
    if device_status is not None:
        _shape(_dev(device_status, "device_status", torch.int32, dev), "device_status", (1,))
    flags = _flags(gate_mode, beta_mode, state_layout, use_computebound, force_simt) | int(_debug_flags)
    if workspace is None:
        need = 0
        if q.dtype == torch.bfloat16 and not force_simt:
            with torch.cuda.device(dev):
                need = kda_workspace_size(T, B, Hk, Hv, dk, dv, 0, flags)
        workspace = own.empty(need, dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8, dev)
    rc = lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(raw_gate), _ptr(beta_logits),
                           _ptr(a_log), _ptr(dt_bias), _ptr(cu_seqlens), B, T, Hk, Hv, dk, dv,
                           _ptr(state_pool), state_pool.shape[0], _ptr(state_indices), _ptr(out),
                           _DTYPES[output_dtype], flags, float(gate_lower_bound),
                           _ptr(workspace) if workspace.numel() else None, workspace.numel(),
                           _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_chunk_fwd")
    return out


def kda_decode(q, k, v, raw_gate, beta_logits, a_log, dt_bias, state_pool, state_indices, out=None, *,
               output_dtype=None, gate_mode="original", beta_mode="logits", state_layout="K_FIRST",
               gate_lower_bound=-5.0, device_status=None, stream=None):
    """One KDA step for one token of each sequence (the kda_decode path of kda_chunk's recurrence).

    Shapes: q,k [B,Hk,dk]; v [B,Hv,dv]; raw_gate [B,Hv,dk] f32; beta_logits [B,Hv] f32; a_log [Hv];
    dt_bias [Hv,dk]; state_pool [slots,Hv,dk,dv] (K_FIRST) or [slots,Hv,dv,dk] (V_FIRST) f32,
    mutated in place; state_indices [B] i32.  Returns out [B,Hv,dv] in ``output_dtype``.
    """
    lib = load_library()
    dev = q.device
    own = _Owned(stream, dev)
    _dev(q, "q", device=dev)
    if q.dtype not in _DTYPES:
        raise ValueError("q/k/v must be float32 or bfloat16")
    if q.dim() != 3:
        raise ValueError(f"q has shape {tuple(q.shape)}, expected [B, Hk, dk]")
    B, Hk, dk = q.shape
    _shape(_dev(k, "k", q.dtype, dev), "k", (B, Hk, dk))
    _dev(v, "v", q.dtype, dev)
    if v.dim() != 3 or v.shape[0] != B:
        raise ValueError(f"v has shape {tuple(v.shape)}, expected [{B}, Hv, dv]")
    Hv, dv = v.shape[1], v.shape[2]
    _shape(_dev(raw_gate, "raw_gate", torch.float32, dev), "raw_gate", (B, Hv, dk))
    _shape(_dev(beta_logits, "beta_logits", torch.float32, dev), "beta_logits", (B, Hv))
    _shape(_dev(a_log, "a_log", torch.float32, dev), "a_log", (Hv,))
    _shape(_dev(dt_bias, "dt_bias", torch.float32, dev), "dt_bias", (Hv, dk))
    _shape(_dev(state_indices, "state_indices", torch.int32, dev), "state_indices", (B,))
    _dev(state_pool, "state_pool", torch.float32, dev)
    blk = (Hv, dk, dv) if state_layout == "K_FIRST" else (Hv, dv, dk)
    if state_pool.dim() != 4 or tuple(state_pool.shape[1:]) != blk:
        raise ValueError(f"state_pool has shape {tuple(state_pool.shape)}, expected [slots, {blk}]")
    if output_dtype is None:
        output_dtype = v.dtype if out is None else out.dtype
    if output_dtype not in _DTYPES:
        raise ValueError("output_dtype must be float32 or bfloat16")
    if out is None:
        out = own.empty((B, Hv, dv), dtype=output_dtype, device=dev)
    _shape(_dev(out, "out", output_dtype, dev), "out", (B, Hv, dv))
    if device_status is not None:
        _shape(_dev(device_status, "device_status", torch.int32, dev), "device_status", (1,))
    flags = _flags(gate_mode, beta_mode, state_layout)
    rc = lib.kda_decode(_ptr(q), _ptr(k), _ptr(v), _DTYPES[q.dtype], _ptr(raw_gate), _ptr(beta_logits), _ptr(a_log),
                        _ptr(dt_bias), B, Hk, Hv, dk, dv, _ptr(state_pool), state_pool.shape[0],
                        _ptr(state_indices), _ptr(out), _DTYPES[output_dtype], flags, float(gate_lower_bound),
                        _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_decode")
    return out


def kda_segment_summarize_and_scan(k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, initial_state,
                                   *, M=None, U=None, incoming=None, outgoing=None, final_state=None,
                                   q=None, readout_m=None, readout_u=None, readout_layout="token_major",
                                   scan_only=False, gate_mode="original", beta_mode="logits", state_layout="K_FIRST",
                                   gate_lower_bound=-5.0, workspace=None, scan_logdepth=False, device_status=None,
                                   stream=None):
    """Segment summaries (M_i, U_i) of one sequence and the exclusive scan over them.

    Returns dict(incoming_states, outgoing_states, final_state, transition_matrices,
    local_contributions[, readout_m, readout_u]); the segment axis leads every stack.  With
    ``scan_only`` the given M and U are inputs and are not written.  With ``q`` (bf16, 128-wide
    heads) the build also returns each token's readouts through the transition and of the
    contribution, the inputs of ``kda_context_parallel_apply``: [T, Hv, 128] each, or [Hv, T, 128]
    with ``readout_layout="head_major"`` (every head's rows contiguous; the apply reads them faster).
    ``workspace`` (uint8 CUDA tensor of kda_scan_workspace_size bytes) lets the scan run in log
    depth where that is expected to finish first; ``scan_logdepth`` forces the log-depth form.
    """
    lib = load_library()
    dev = initial_state.device
    own = _Owned(stream, dev)
    _dev(initial_state, "initial_state", torch.float32, dev)
    Hv = initial_state.shape[0]
    N = seg_offsets.numel() - 1
    if scan_only:
        if M is None or U is None:
            raise ValueError("scan_only needs M and U")
        dk = M.shape[-1]
        dv = U.shape[-1] if state_layout == "K_FIRST" else U.shape[-2]
        kv_dtype, T, Hk = _F32, 0, Hv
    else:
        _dev(k, "k", None, dev)
        if k.dtype not in _DTYPES:
            raise ValueError("k/v must be float32 or bfloat16")
        T, Hk, dk = k.shape
        _dev(v, "v", k.dtype, dev)
        dv = v.shape[2]
        _shape(v, "v", (T, Hv, dv))
        _shape(_dev(raw_gate, "raw_gate", torch.float32, dev), "raw_gate", (T, Hv, dk))
        _shape(_dev(beta_logits, "beta_logits", torch.float32, dev), "beta_logits", (T, Hv))
        _shape(_dev(a_log, "a_log", torch.float32, dev), "a_log", (Hv,))
        _shape(_dev(dt_bias, "dt_bias", torch.float32, dev), "dt_bias", (Hv, dk))
        kv_dtype = _DTYPES[k.dtype]
    _dev(seg_offsets, "seg_offsets", torch.int32, dev) if not scan_only else None
    st = (dk, dv) if state_layout == "K_FIRST" else (dv, dk)
    _shape(initial_state, "initial_state", (Hv, *st))

    def buf(t, name, shape):
        if t is None:
            return own.empty(shape, dtype=torch.float32, device=dev)
        _shape(_dev(t, name, torch.float32, dev), name, shape)
        return t

    M = buf(M, "M", (N, Hv, dk, dk))
    U = buf(U, "U", (N, Hv, *st))
    incoming = buf(incoming, "incoming", (N, Hv, *st))
    outgoing = buf(outgoing, "outgoing", (N, Hv, *st))
    final_state = buf(final_state, "final_state", (Hv, *st))
    if q is not None:
        _shape(_dev(q, "q", torch.bfloat16, dev), "q", (T, Hk, dk))
        rshape = _readout_shape(T, Hv, dv, readout_layout)
        if readout_m is None:
            readout_m = own.empty(rshape, dtype=torch.bfloat16, device=dev)
        if readout_u is None:
            readout_u = own.empty(rshape, dtype=torch.bfloat16, device=dev)
        _shape(_dev(readout_m, "readout_m", torch.bfloat16, dev), "readout_m", rshape)
        _shape(_dev(readout_u, "readout_u", torch.bfloat16, dev), "readout_u", rshape)
    flags = _flags(gate_mode, beta_mode, state_layout, scan_only=scan_only)
    if q is not None:
        flags |= _readout_flags(readout_layout)
    if scan_logdepth:
        flags |= SCAN_LOGDEPTH
    if workspace is not None:
        _dev(workspace, "workspace", torch.uint8, dev)
    rc = lib.kda_segment_summarize_and_scan(
        _ptr(k) if not scan_only else None, _ptr(v) if not scan_only else None, kv_dtype,
        _ptr(raw_gate) if not scan_only else None, _ptr(beta_logits) if not scan_only else None,
        _ptr(a_log) if not scan_only else None, _ptr(dt_bias) if not scan_only else None, T, Hk, Hv, dk, dv,
        _ptr(seg_offsets) if not scan_only else None, N, _ptr(initial_state), _ptr(M), _ptr(U),
        _ptr(incoming), _ptr(outgoing), _ptr(final_state), _ptr(q), _ptr(readout_m), _ptr(readout_u), flags,
        float(gate_lower_bound), _ptr(workspace) if workspace is not None and workspace.numel() else None,
        workspace.numel() if workspace is not None else 0, _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_segment_summarize_and_scan")
    res = {"incoming_states": incoming, "outgoing_states": outgoing, "final_state": final_state,
           "transition_matrices": M, "local_contributions": U}
    if q is not None:
        res["readout_m"], res["readout_u"] = readout_m, readout_u
    return res


def kda_context_parallel_apply(readout_m, readout_u, incoming, seg_offsets, out=None, *, output_dtype=torch.bfloat16,
                               readout_layout="token_major", state_layout="K_FIRST", device_status=None, stream=None):
    """out_t = readout_m[t] . S_in(segment of t) + readout_u[t] for every token (readouts [T, Hv, 128],
    or [Hv, T, 128] with ``readout_layout="head_major"``; out [T, Hv, 128] either way)."""
    lib = load_library()
    dev = incoming.device
    own = _Owned(stream, dev)
    _dev(readout_m, "readout_m", torch.bfloat16, dev)
    rflags = _readout_flags(readout_layout)
    if readout_layout == "head_major":
        Hv, T, dv = readout_m.shape
    else:
        T, Hv, dv = readout_m.shape
    _shape(_dev(readout_u, "readout_u", torch.bfloat16, dev), "readout_u", _readout_shape(T, Hv, dv, readout_layout))
    _dev(incoming, "incoming", torch.float32, dev)
    _dev(seg_offsets, "seg_offsets", torch.int32, dev)
    N = seg_offsets.numel() - 1
    if out is None:
        out = own.empty((T, Hv, dv), dtype=output_dtype, device=dev)
    _shape(_dev(out, "out", None, dev), "out", (T, Hv, dv))
    rc = lib.kda_context_parallel_apply(_ptr(readout_m), _ptr(readout_u), _ptr(incoming), _ptr(seg_offsets), N, T,
                                        Hv, dv, _ptr(out), _DTYPES[out.dtype],
                                        _flags("original", "logits", state_layout) | rflags,
                                        _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_context_parallel_apply")
    return out


def kda_context_parallel(transition_matrices, local_contributions, initial_state, *, state_layout="K_FIRST",
                         method="auto", stream=None):
    """The exclusive affine scan alone ("KDA Context Parallelism", Requirements).

    transition_matrices (N, dk, dk), local_contributions (N, dk, dv), initial_state (dk, dv),
    fp32 CUDA tensors (a leading head axis after N is also accepted).  Returns a dict with
    exactly incoming_states, outgoing_states and final_state; no input is written.
    ``method``: "sequential" (one step per segment), "logdepth" (the composition in log depth,
    dk = 128 only) or "auto" (log depth where the library expects it to finish first).
    """
    M, U, S0 = transition_matrices, local_contributions, initial_state
    if M.dtype != torch.float32:
        raise ValueError("the scan kernel computes in float32; pass float32 tensors")
    if M.dim() < 3:
        raise ValueError("at least one segment is required: transition_matrices is (N, dk, dk)")
    squeeze = M.dim() == 3
    if squeeze:
        M, U, S0 = M.unsqueeze(1), U.unsqueeze(1), S0.unsqueeze(0)
    if M.shape[0] < 1:
        raise ValueError("at least one segment is required")
    if method not in ("auto", "sequential", "logdepth"):
        raise ValueError(f"unknown scan method {method!r}")
    own = _Owned(stream, S0.device)
    Mc, Uc, Sc = own.keep(M.contiguous(), M), own.keep(U.contiguous(), U), own.keep(S0.contiguous(), S0)
    N, H, dk = M.shape[0], M.shape[1], M.shape[-1]
    dv = U.shape[-1] if state_layout == "K_FIRST" else U.shape[-2]
    ws = None
    if method == "logdepth" or (method == "auto" and kda_scan_logdepth_preferred(N, H, dv, device=S0.device)):
        need = kda_scan_workspace_size(N, H, dk, dv)
        if need == 0 and method == "logdepth":
            raise ValueError("the log-depth scan needs dk = 128 and dv a multiple of 32 up to 128")
        ws = own.empty(need, dtype=torch.uint8, device=S0.device) if need else None
    res = kda_segment_summarize_and_scan(None, None, None, None, None, None,
                                         torch.zeros(M.shape[0] + 1, dtype=torch.int32), Sc,
                                         M=Mc, U=Uc, scan_only=True, state_layout=state_layout, workspace=ws,
                                         scan_logdepth=method == "logdepth", stream=stream)
    own.launched()
    out = {k: res[k] for k in ("incoming_states", "outgoing_states", "final_state")}
    if squeeze:
        out = {"incoming_states": out["incoming_states"][:, 0], "outgoing_states": out["outgoing_states"][:, 0],
               "final_state": out["final_state"][0]}
    return out


def kda_scan_workspace_size(num_segments, num_v_heads, dk=128, dv=128) -> int:
    """Workspace bytes of the log-depth scan (0 where it does not apply)."""
    return int(load_library().kda_scan_workspace_size(num_segments, num_v_heads, dk, dv))


def kda_scan_logdepth_preferred(num_segments, num_v_heads, dv=128, device=None) -> bool:
    """Whether the log-depth scan is expected to finish first on ``device`` (default: current)."""
    lib = load_library()
    if device is not None and torch.device(device).type == "cuda":
        with torch.cuda.device(device):
            return bool(lib.kda_scan_logdepth_preferred(num_segments, num_v_heads, dv))
    return bool(lib.kda_scan_logdepth_preferred(num_segments, num_v_heads, dv))


def kda_context_parallel_workspace_size(T, num_v_heads, dv=128) -> int:
    return int(load_library().kda_context_parallel_workspace_size(T, num_v_heads, dv))


def kda_context_parallel_pieces(T, num_segments, num_v_heads) -> int:
    """Pieces per segment the context-parallel prefill builds on the current device."""
    return int(load_library().kda_context_parallel_pieces(T, num_segments, num_v_heads))


def kda_context_parallel_piece_offsets(seg_offsets, pieces, *, out=None, stream=None):
    """Chunk-aligned boundaries of ``pieces`` pieces per segment (device int32 [N*pieces + 1])."""
    lib = load_library()
    dev = seg_offsets.device
    own = _Owned(stream, dev)
    _dev(seg_offsets, "seg_offsets", torch.int32, dev)
    N = seg_offsets.numel() - 1
    if out is None:
        out = own.empty(N * pieces + 1, dtype=torch.int32, device=dev)
    _shape(_dev(out, "out", torch.int32, dev), "out", (N * pieces + 1,))
    rc = lib.kda_context_parallel_piece_offsets(_ptr(seg_offsets), N, pieces, _ptr(out), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_context_parallel_piece_offsets")
    return out


def kda_segment_compose(M_pieces, U_pieces, incoming_pieces, final_state, pieces, *, M=None, U=None,
                        incoming=None, outgoing=None, state_layout="K_FIRST", stream=None):
    """Segment summaries (and incoming/outgoing states) composed from those of their pieces.

    Returns dict(transition_matrices, local_contributions, incoming_states, outgoing_states).
    """
    lib = load_library()
    dev = M_pieces.device
    own = _Owned(stream, dev)
    _dev(M_pieces, "M_pieces", torch.float32, dev)
    NP, Hv, dk = M_pieces.shape[0], M_pieces.shape[1], M_pieces.shape[2]
    if NP % pieces:
        raise ValueError("the piece count must divide the number of pieces")
    N = NP // pieces
    st = tuple(U_pieces.shape[2:])
    dv = st[1] if state_layout == "K_FIRST" else st[0]
    _shape(_dev(U_pieces, "U_pieces", torch.float32, dev), "U_pieces", (NP, Hv, *st))
    _dev(incoming_pieces, "incoming_pieces", torch.float32, dev)
    if incoming_pieces.shape[0] < NP or tuple(incoming_pieces.shape[1:]) != (Hv, *st):
        raise ValueError("incoming_pieces must be [>= N*pieces, Hv, <state>]")
    _shape(_dev(final_state, "final_state", torch.float32, dev), "final_state", (Hv, *st))

    def buf(t, name, shape):
        if t is None:
            return own.empty(shape, dtype=torch.float32, device=dev)
        _shape(_dev(t, name, torch.float32, dev), name, shape)
        return t

    M = buf(M, "M", (N, Hv, dk, dk))
    U = buf(U, "U", (N, Hv, *st))
    incoming = buf(incoming, "incoming", (N, Hv, *st))
    outgoing = buf(outgoing, "outgoing", (N, Hv, *st))
    rc = lib.kda_segment_compose(_ptr(M_pieces), _ptr(U_pieces), _ptr(incoming_pieces), _ptr(final_state), N,
                                 pieces, Hv, dk, dv, _ptr(M), _ptr(U), _ptr(incoming), _ptr(outgoing),
                                 _flags("original", "logits", state_layout), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_segment_compose")
    return {"transition_matrices": M, "local_contributions": U, "incoming_states": incoming,
            "outgoing_states": outgoing}


def kda_context_parallel_workspace_preferred(T, num_segments, num_v_heads, dv=128) -> int:
    return int(load_library().kda_context_parallel_workspace_preferred(T, num_segments, num_v_heads, dv))


def kda_context_parallel_prefill(q, k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, initial_state,
                                 out=None, *, final_state=None, M=None, U=None, incoming=None, outgoing=None,
                                 workspace=None, output_dtype=None, gate_mode="original", beta_mode="logits",
                                 state_layout="K_FIRST", gate_lower_bound=-5.0, device_status=None, stream=None):
    """Context-parallel prefill of one sequence (bf16 q/k/v, dk = dv = 128) cut at seg_offsets.

    Returns dict(out, final_state, incoming_states, outgoing_states, transition_matrices,
    local_contributions).  ``workspace`` (uint8 CUDA tensor of at least
    kda_context_parallel_workspace_size bytes) is allocated when not given, at the preferred size
    (kda_context_parallel_workspace_preferred: enough to build the segments as pieces).
    """
    lib = load_library()
    dev = q.device
    own = _Owned(stream, dev)
    _dev(q, "q", torch.bfloat16, dev)
    T, Hk, dk = q.shape
    _shape(_dev(k, "k", torch.bfloat16, dev), "k", (T, Hk, dk))
    _dev(v, "v", torch.bfloat16, dev)
    Hv, dv = v.shape[1], v.shape[2]
    _shape(v, "v", (T, Hv, dv))
    _shape(_dev(raw_gate, "raw_gate", torch.float32, dev), "raw_gate", (T, Hv, dk))
    _shape(_dev(beta_logits, "beta_logits", torch.float32, dev), "beta_logits", (T, Hv))
    _shape(_dev(a_log, "a_log", torch.float32, dev), "a_log", (Hv,))
    _shape(_dev(dt_bias, "dt_bias", torch.float32, dev), "dt_bias", (Hv, dk))
    _dev(seg_offsets, "seg_offsets", torch.int32, dev)
    N = seg_offsets.numel() - 1
    st = (dk, dv) if state_layout == "K_FIRST" else (dv, dk)
    _shape(_dev(initial_state, "initial_state", torch.float32, dev), "initial_state", (Hv, *st))
    if output_dtype is None:
        output_dtype = v.dtype if out is None else out.dtype
    if out is None:
        out = own.empty((T, Hv, dv), dtype=output_dtype, device=dev)
    _shape(_dev(out, "out", output_dtype, dev), "out", (T, Hv, dv))

    def buf(t, name, shape):
        if t is None:
            return own.empty(shape, dtype=torch.float32, device=dev)
        _shape(_dev(t, name, torch.float32, dev), name, shape)
        return t

    final_state = buf(final_state, "final_state", (Hv, *st))
    M = buf(M, "M", (N, Hv, dk, dk))
    U = buf(U, "U", (N, Hv, *st))
    incoming = buf(incoming, "incoming", (N, Hv, *st))
    outgoing = buf(outgoing, "outgoing", (N, Hv, *st))
    if workspace is None:
        with torch.cuda.device(dev):
            pref = kda_context_parallel_workspace_preferred(T, N, Hv, dv)
        workspace = own.empty(max(pref, 1), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8, dev)
    flags = _flags(gate_mode, beta_mode, state_layout)
    rc = lib.kda_context_parallel_prefill(_ptr(q), _ptr(k), _ptr(v), _BF16, _ptr(raw_gate), _ptr(beta_logits),
                                          _ptr(a_log), _ptr(dt_bias), T, Hk, Hv, dk, dv, _ptr(seg_offsets), N,
                                          _ptr(initial_state), _ptr(out), _DTYPES[output_dtype], _ptr(final_state),
                                          _ptr(M), _ptr(U), _ptr(incoming), _ptr(outgoing), flags,
                                          float(gate_lower_bound), _ptr(workspace), workspace.numel(),
                                          _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_context_parallel_prefill")
    return {"out": out, "final_state": final_state, "incoming_states": incoming, "outgoing_states": outgoing,
            "transition_matrices": M, "local_contributions": U}


def kda_context_parallel_range_workspace_size(T, num_segments, num_v_heads, dv=128) -> int:
    """Workspace bytes of the two per-rank calls on the current device."""
    return int(load_library().kda_context_parallel_range_workspace_size(T, num_segments, num_v_heads, dv))


def _token_ptr(t, T):
    # a range without tokens passes no token pointers
    return _ptr(t) if T > 0 else None


def kda_context_parallel_range_summary(q, k, v, raw_gate, beta_logits, a_log, dt_bias, seg_offsets, *,
                                       range_transition=None, range_contribution=None, workspace=None,
                                       gate_mode="original", beta_mode="logits", state_layout="K_FIRST",
                                       gate_lower_bound=-5.0, device_status=None, stream=None):
    """One rank's token range (bf16 q/k/v, dk = dv = 128, cut at seg_offsets) as ONE affine map.

    Returns dict(range_transition [Hv,128,128], range_contribution [Hv,<state>], workspace); the
    workspace carries the range's readouts and pieces to kda_context_parallel_range_finish.
    """
    lib = load_library()
    dev = q.device
    own = _Owned(stream, dev)
    _dev(q, "q", torch.bfloat16, dev)
    T, Hk, dk = q.shape
    _shape(_dev(k, "k", torch.bfloat16, dev), "k", (T, Hk, dk))
    _dev(v, "v", torch.bfloat16, dev)
    Hv, dv = v.shape[1], v.shape[2]
    _shape(v, "v", (T, Hv, dv))
    _shape(_dev(raw_gate, "raw_gate", torch.float32, dev), "raw_gate", (T, Hv, dk))
    _shape(_dev(beta_logits, "beta_logits", torch.float32, dev), "beta_logits", (T, Hv))
    _shape(_dev(a_log, "a_log", torch.float32, dev), "a_log", (Hv,))
    _shape(_dev(dt_bias, "dt_bias", torch.float32, dev), "dt_bias", (Hv, dk))
    _dev(seg_offsets, "seg_offsets", torch.int32, dev)
    N = seg_offsets.numel() - 1
    st = (dk, dv) if state_layout == "K_FIRST" else (dv, dk)
    if range_transition is None:
        range_transition = own.empty((Hv, dk, dk), dtype=torch.float32, device=dev)
    _shape(_dev(range_transition, "range_transition", torch.float32, dev), "range_transition", (Hv, dk, dk))
    if range_contribution is None:
        range_contribution = own.empty((Hv, *st), dtype=torch.float32, device=dev)
    _shape(_dev(range_contribution, "range_contribution", torch.float32, dev), "range_contribution", (Hv, *st))
    if workspace is None:
        with torch.cuda.device(dev):
            need = kda_context_parallel_range_workspace_size(T, max(N, 1), Hv, dv)
        workspace = own.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", torch.uint8, dev)
    rc = lib.kda_context_parallel_range_summary(
        _token_ptr(q, T), _token_ptr(k, T), _token_ptr(v, T), _BF16, _token_ptr(raw_gate, T),
        _token_ptr(beta_logits, T), _ptr(a_log), _ptr(dt_bias), T, Hk, Hv, dk, dv, _ptr(seg_offsets), N,
        _ptr(range_transition), _ptr(range_contribution), _flags(gate_mode, beta_mode, state_layout),
        float(gate_lower_bound), _ptr(workspace), workspace.numel(), _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_context_parallel_range_summary")
    return {"range_transition": range_transition, "range_contribution": range_contribution, "workspace": workspace}


def kda_context_parallel_range_finish(range_incoming, workspace, seg_offsets, tokens, out=None, *,
                                      output_dtype=torch.bfloat16, range_outgoing=None, M=None, U=None,
                                      incoming=None, outgoing=None, state_layout="K_FIRST", device_status=None,
                                      stream=None):
    """A range's outputs and per-segment states from the state entering it (range_incoming
    [Hv,<state>] fp32) and the workspace that kda_context_parallel_range_summary filled.

    Returns dict(out, range_outgoing, incoming_states, outgoing_states, transition_matrices,
    local_contributions) for the range's own segments.
    """
    lib = load_library()
    dev = range_incoming.device
    own = _Owned(stream, dev)
    _dev(range_incoming, "range_incoming", torch.float32, dev)
    Hv, st = range_incoming.shape[0], tuple(range_incoming.shape[1:])
    dk = dv = 128
    _shape(range_incoming, "range_incoming", (Hv, dk, dv))
    _dev(workspace, "workspace", torch.uint8, dev)
    _dev(seg_offsets, "seg_offsets", torch.int32, dev)
    N = seg_offsets.numel() - 1
    T = int(tokens)
    if out is None:
        out = own.empty((T, Hv, dv), dtype=output_dtype, device=dev)
    _shape(_dev(out, "out", output_dtype, dev), "out", (T, Hv, dv))

    def buf(t, name, shape):
        if t is None:
            return own.empty(shape, dtype=torch.float32, device=dev)
        _shape(_dev(t, name, torch.float32, dev), name, shape)
        return t

    range_outgoing = buf(range_outgoing, "range_outgoing", (Hv, *st))
    M = buf(M, "M", (N, Hv, dk, dk))
    U = buf(U, "U", (N, Hv, *st))
    incoming = buf(incoming, "incoming", (N, Hv, *st))
    outgoing = buf(outgoing, "outgoing", (N, Hv, *st))
    rc = lib.kda_context_parallel_range_finish(
        T, Hv, dk, dv, N, _ptr(range_incoming), _token_ptr(out, T), _DTYPES[output_dtype], _ptr(range_outgoing),
        _ptr(M), _ptr(U), _ptr(incoming), _ptr(outgoing), _flags("original", "logits", state_layout),
        _ptr(workspace), workspace.numel(), _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_context_parallel_range_finish")
    return {"out": out, "range_outgoing": range_outgoing, "incoming_states": incoming, "outgoing_states": outgoing,
            "transition_matrices": M, "local_contributions": U}


def kda_prefill_host_workspace_size(T, num_k_heads, num_v_heads, output_dtype=torch.bfloat16,
                                    segment_tokens=8192) -> int:
    return int(load_library().kda_prefill_host_workspace_size(T, num_k_heads, num_v_heads, _DTYPES[output_dtype],
                                                              segment_tokens))


def _host(t, name, dtype=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device.type != "cpu":
        raise ValueError(f"{name} must be a host (CPU) tensor, got {t.device}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() and not t.is_pinned():  # (an empty tensor has no storage to pin)
        raise ValueError(f"{name} must be in pinned host memory (tensor.pin_memory()) for the copies to overlap")
    return t


def kda_prefill_host_pipelined(q, k, v, raw_gate, beta_logits, a_log, dt_bias, initial_state, out=None, *,
                               final_state=None, segment_tokens=8192, workspace=None, output_dtype=None,
                               gate_mode="original", beta_mode="logits", state_layout="K_FIRST",
                               gate_lower_bound=-5.0, device_status=None, stream=None, device=None):
    """kda_chunk_fwd's prefill of ONE sequence held in pinned host memory (bf16 q/k/v,
    dk = dv = 128), the copies pipelined with the kernels in segments of ``segment_tokens``.

    Every tensor argument is a pinned CPU tensor (``workspace`` and ``device_status`` excepted:
    device).  Returns dict(out, final_state), host tensors that are complete once ``stream``
    (default: the device's current stream) has been synchronised.
    """
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    own = _Owned(stream, dev)
    _host(q, "q", torch.bfloat16)
    T, Hk, dk = q.shape
    _shape(_host(k, "k", torch.bfloat16), "k", (T, Hk, dk))
    _host(v, "v", torch.bfloat16)
    Hv, dv = v.shape[1], v.shape[2]
    _shape(v, "v", (T, Hv, dv))
    _shape(_host(raw_gate, "raw_gate", torch.float32), "raw_gate", (T, Hv, dk))
    _shape(_host(beta_logits, "beta_logits", torch.float32), "beta_logits", (T, Hv))
    _shape(_host(a_log, "a_log", torch.float32), "a_log", (Hv,))
    _shape(_host(dt_bias, "dt_bias", torch.float32), "dt_bias", (Hv, dk))
    st = (dk, dv) if state_layout == "K_FIRST" else (dv, dk)
    _shape(_host(initial_state, "initial_state", torch.float32), "initial_state", (Hv, *st))
    if output_dtype is None:
        output_dtype = v.dtype if out is None else out.dtype
    if out is None:
        out = torch.empty((T, Hv, dv), dtype=output_dtype, pin_memory=True)
    _shape(_host(out, "out", output_dtype), "out", (T, Hv, dv))
    if final_state is None:
        final_state = torch.empty((Hv, *st), dtype=torch.float32, pin_memory=True)
    _shape(_host(final_state, "final_state", torch.float32), "final_state", (Hv, *st))
    with torch.cuda.device(dev):
        if workspace is None:
            need = kda_prefill_host_workspace_size(T, Hk, Hv, output_dtype, segment_tokens)
            if need == 0:
                raise ValueError("segment_tokens must be a positive multiple of 64")
            workspace = own.empty(need, dtype=torch.uint8, device=dev)
        _dev(workspace, "workspace", torch.uint8, dev)
        rc = lib.kda_prefill_host_pipelined(
            _ptr(q), _ptr(k), _ptr(v), _BF16, _ptr(raw_gate), _ptr(beta_logits), _ptr(a_log), _ptr(dt_bias), T,
            Hk, Hv, dk, dv, _ptr(initial_state), _ptr(out), _DTYPES[output_dtype], _ptr(final_state),
            int(segment_tokens), _flags(gate_mode, beta_mode, state_layout), float(gate_lower_bound),
            _ptr(workspace), workspace.numel(), _ptr(device_status), _stream(stream, dev))
    own.launched()
    if rc != 0:
        raise KdaError(rc, "kda_prefill_host_pipelined")
    return {"out": out, "final_state": final_state}
