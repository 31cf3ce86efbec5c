"""B200 chunked causal linear attention (the LASP / LASP-2 hot path).

A thin ctypes binding over ``liblasp.so``, whose C ABI is declared in
``include/lasp.h``. Every function here has the name of its C entry point and
only marshals arguments: torch tensors supply device pointers and sizes, the
current CUDA stream is passed along, and a non-zero status raises
:class:`LaspError`. All arithmetic runs in the library's CUDA kernels; there is
no CPU path. If the library has not been built, the first call raises.

Token tensors are contiguous [B, N, H, d] (float32 or bfloat16, all the same);
state arrays are contiguous float32 [B, N/C, H, d, d] or [B, H, d, d]; decay is
a float32 [H] device tensor or None (lambda = 1).
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "LaspError", "library_path", "lasp_fwd", "lasp_bwd", "lasp_fwd_states", "lasp_fwd_finish", "lasp_bwd_states",
    "lasp_bwd_finish", "lasp_chunk_states", "lasp_chunk_dstates",
    "lasp_chunk_out", "lasp_chunk_grads", "lasp_bwd_noalloc",
    "lasp_state_prefix", "lasp_check_device_status", "lasp_set_wait_limit_ns", "lasp_wait_probe",
    "lasp_status_string", "lasp_version", "lasp_trace_enable", "lasp_trace_read", "lasp_kernel_name",
    "lasp_segment_tokens", "lasp_bidir_workspace_floats", "lasp_bidir_state_offset", "lasp_bidir_fwd",
    "lasp_bidir_bwd", "lasp_gla_cache_floats", "lasp_gla_chunk_states", "lasp_gla_state_prefix", "lasp_gla_fwd",
    "lasp_gla_bwd", "lasp_softmax_fwd", "lasp_softmax_bwd", "lasp_fwd_states_part", "lasp_fwd_finish_part",
    "lasp_bwd_states_part", "lasp_bwd_finish_part", "lasp_parts_ok",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "liblasp.so")
_lib = None
_lock = threading.Lock()

LASP_F32, LASP_BF16 = 0, 1
_STATUS = ["LASP_OK", "LASP_ERR_INVALID_ARG", "LASP_ERR_UNSUPPORTED", "LASP_ERR_MISALIGNED",
           "LASP_ERR_CUDA", "LASP_ERR_TIMEOUT"]


class LaspError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = _STATUS[status] if 0 <= status < len(_STATUS) else f"status {status}"
        super().__init__(f"{where}: {name}")


def library_path() -> str:
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"{_LIB_PATH} is missing: build it with `python -m sequence_linear_attention_b200.build`")
            lib = ctypes.CDLL(_LIB_PATH)
            P, I, L, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
            lib.lasp_fwd.argtypes = [P, P, P, P, P, I, I, L, I, I, I, P, P, P]
            lib.lasp_bwd.argtypes = [P, P, P, P, P, P, P, P, I, I, L, I, I, I, P, P, P, P, P, P]
            lib.lasp_fwd_states.argtypes = [P, P, P, I, I, L, I, I, I, P, P, P]
            lib.lasp_fwd_finish.argtypes = [P, P, P, P, P, I, I, L, I, I, I, P, P, P]
            lib.lasp_bwd_states.argtypes = [P, P, P, I, I, L, I, I, I, P, P, P]
            lib.lasp_bwd_finish.argtypes = [P, P, P, P, P, P, P, P, I, I, L, I, I, I, P, P, P, P, P]
            lib.lasp_chunk_states.argtypes = [P, P, P, P, P, I, I, L, I, I, I, P]
            lib.lasp_chunk_dstates.argtypes = [P, P, P, P, I, I, L, I, I, I, P]
            lib.lasp_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, I, I, L, I, I, I, P, P, P, P]
            lib.lasp_chunk_out.argtypes = [P, P, P, P, P, P, I, I, L, I, I, I, P]
            lib.lasp_chunk_grads.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, L, I, I, I, P]
            lib.lasp_state_prefix.argtypes = [P, P, P, P, P, I, I, I, I, L, I, P]
            lib.lasp_check_device_status.argtypes = [P, ctypes.POINTER(I)]
            lib.lasp_set_wait_limit_ns.argtypes = [U64]
            lib.lasp_wait_probe.argtypes = [P]
            lib.lasp_trace_enable.argtypes = [I]
            lib.lasp_trace_read.argtypes = [P, P, I]
            lib.lasp_kernel_name.argtypes = [I]
            lib.lasp_kernel_name.restype = ctypes.c_char_p
            lib.lasp_segment_tokens.argtypes = [L, I, I, I]
            lib.lasp_bidir_workspace_floats.argtypes = [I, I, L, I, I]
            lib.lasp_bidir_workspace_floats.restype = L
            lib.lasp_bidir_state_offset.argtypes = [I, I, L, I, I]
            lib.lasp_bidir_state_offset.restype = L
            lib.lasp_bidir_fwd.argtypes = [P, P, P, P, I, I, L, I, I, P, P]
            lib.lasp_bidir_bwd.argtypes = [P, P, P, P, P, P, P, I, I, L, I, I, P, P, P]
            lib.lasp_gla_cache_floats.argtypes = [I, I, L, I, I]
            lib.lasp_gla_cache_floats.restype = L
            lib.lasp_gla_chunk_states.argtypes = [P, P, P, P, P, I, I, L, I, I, I, I, P]
            lib.lasp_gla_state_prefix.argtypes = [P, P, P, P, P, I, I, I, I, I, P]
            lib.lasp_gla_fwd.argtypes = [P, P, P, P, P, I, I, L, I, I, I, P, P, P]
            lib.lasp_gla_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, L, I, I, I, P, P, P, P, P]
            lib.lasp_fwd_states_part.argtypes = [P, P, P, I, I, L, I, I, I, P, P, I, I, P]
            lib.lasp_fwd_finish_part.argtypes = [P, P, P, P, P, I, I, L, I, I, I, P, P, I, I, P]
            lib.lasp_bwd_states_part.argtypes = [P, P, P, I, I, L, I, I, I, P, P, I, I, P]
            lib.lasp_bwd_finish_part.argtypes = [P, P, P, P, P, P, P, P, I, I, L, I, I, I, P, P, P, P, I, I, P]
            lib.lasp_parts_ok.argtypes = [L, I, I, I]
            lib.lasp_parts_ok.restype = I
            F = ctypes.c_float
            lib.lasp_softmax_fwd.argtypes = [P, P, P, P, P, I, I, L, L, L, I, F, I, P]
            lib.lasp_softmax_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, L, L, L, I, F, I, P]
            lib.lasp_status_string.argtypes = [I]
            lib.lasp_status_string.restype = ctypes.c_char_p
            for f in (lib.lasp_fwd, lib.lasp_bwd, lib.lasp_fwd_states, lib.lasp_fwd_finish, lib.lasp_bwd_states,
                      lib.lasp_bwd_finish, lib.lasp_chunk_states, lib.lasp_chunk_dstates,
                      lib.lasp_chunk_out, lib.lasp_chunk_grads, lib.lasp_bwd_noalloc,
                      lib.lasp_state_prefix, lib.lasp_check_device_status, lib.lasp_set_wait_limit_ns,
                      lib.lasp_wait_probe, lib.lasp_version, lib.lasp_trace_enable, lib.lasp_trace_read,
                      lib.lasp_segment_tokens, lib.lasp_bidir_fwd, lib.lasp_bidir_bwd,
                      lib.lasp_gla_chunk_states, lib.lasp_gla_state_prefix, lib.lasp_gla_fwd,
                      lib.lasp_gla_bwd, lib.lasp_softmax_fwd, lib.lasp_softmax_bwd, lib.lasp_fwd_states_part,
                      lib.lasp_fwd_finish_part, lib.lasp_bwd_states_part, lib.lasp_bwd_finish_part):
                f.restype = I
            _lib = lib
    return _lib


# ----------------------------------------------------------------- marshalling
def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream, like):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream(like.device).cuda_stream


def _dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return LASP_F32
    if t.dtype == torch.bfloat16:
        return LASP_BF16
    raise TypeError(f"token tensors must be float32 or bfloat16, got {t.dtype}")


def _tokens(*ts):
    ref = ts[0]
    if ref.dim() != 4:
        raise ValueError("token tensors must be [B, N, H, d]")
    for t in ts:
        if t is None:
            continue
        if tuple(t.shape) != tuple(ref.shape) or t.dtype != ref.dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError("token tensors must be contiguous CUDA tensors of one shape and dtype")
    B, N, H, d = ref.shape
    return B, N, H, d, _dtype_code(ref)


def _check(status, where):
    if status != 0:
        raise LaspError(status, where)


# ---------------------------------------------------------------- entry points
def lasp_fwd(q, k, v, decay, o, C, state_cache, init_state=None, stream=None):
    """o = causal linear attention of (q, k, v); state_cache receives P_c. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _check(_load().lasp_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o), B, H, N, d, C, dt,
                            _ptr(state_cache), _ptr(init_state), _stream(stream, q)), "lasp_fwd")


def lasp_bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, init_state=None,
             dstate_in=None, dinit_state=None, stream=None):
    """dq, dk, dv of sum(o * dout); dstate_ws receives R_c. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                            B, H, N, d, C, dt, _ptr(state_cache), _ptr(dstate_ws), _ptr(init_state),
                            _ptr(dstate_in), _ptr(dinit_state), _stream(stream, q)), "lasp_bwd")


def lasp_fwd_states(k, v, decay, C, state_cache, total=None, stream=None):
    """First part of lasp_fwd: its states into state_cache and, if given, their
    decayed total (the LASP-2 shard state). See lasp.h."""
    B, N, H, d, dt = _tokens(k, v)
    _check(_load().lasp_fwd_states(_ptr(k), _ptr(v), _ptr(decay), B, H, N, d, C, dt, _ptr(state_cache), _ptr(total),
                                   _stream(stream, k)), "lasp_fwd_states")


def lasp_fwd_finish(q, k, v, decay, o, C, state_cache, init_state=None, stream=None):
    """Rest of lasp_fwd on a cache lasp_fwd_states filled: prefix from init_state, output. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _check(_load().lasp_fwd_finish(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o), B, H, N, d, C, dt,
                                   _ptr(state_cache), _ptr(init_state), _stream(stream, q)), "lasp_fwd_finish")


def lasp_bwd_states(q, dout, decay, C, dstate_ws, total=None, stream=None):
    """First part of lasp_bwd: its gradient states into dstate_ws and, if given,
    their decayed total (the LASP-2 shard gradient state). See lasp.h."""
    B, N, H, d, dt = _tokens(q, dout)
    _check(_load().lasp_bwd_states(_ptr(q), _ptr(dout), _ptr(decay), B, H, N, d, C, dt, _ptr(dstate_ws), _ptr(total),
                                   _stream(stream, q)), "lasp_bwd_states")


def lasp_bwd_finish(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in=None, dinit_state=None,
                    stream=None):
    """Rest of lasp_bwd on a workspace lasp_bwd_states filled: suffix from dstate_in, dq, dk, dv. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_bwd_finish(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                   B, H, N, d, C, dt, _ptr(state_cache), _ptr(dstate_ws), _ptr(dstate_in),
                                   _ptr(dinit_state), _stream(stream, q)), "lasp_bwd_finish")


def lasp_fwd_states_part(k, v, decay, C, state_cache, total, part, nparts, stream=None):
    """lasp_fwd_states for part `part` of `nparts` of the (b, h) pairs. See lasp.h."""
    B, N, H, d, dt = _tokens(k, v)
    _check(_load().lasp_fwd_states_part(_ptr(k), _ptr(v), _ptr(decay), B, H, N, d, C, dt, _ptr(state_cache),
                                        _ptr(total), part, nparts, _stream(stream, k)), "lasp_fwd_states_part")


def lasp_fwd_finish_part(q, k, v, decay, o, C, state_cache, init_state, part, nparts, stream=None):
    """lasp_fwd_finish for part `part` of `nparts` of the (b, h) pairs. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _check(_load().lasp_fwd_finish_part(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o), B, H, N, d, C, dt,
                                        _ptr(state_cache), _ptr(init_state), part, nparts, _stream(stream, q)),
           "lasp_fwd_finish_part")


def lasp_bwd_states_part(q, dout, decay, C, dstate_ws, total, part, nparts, stream=None):
    """lasp_bwd_states for part `part` of `nparts` of the (b, h) pairs. See lasp.h."""
    B, N, H, d, dt = _tokens(q, dout)
    _check(_load().lasp_bwd_states_part(_ptr(q), _ptr(dout), _ptr(decay), B, H, N, d, C, dt, _ptr(dstate_ws),
                                        _ptr(total), part, nparts, _stream(stream, q)), "lasp_bwd_states_part")


def lasp_bwd_finish_part(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in, dinit_state, part,
                         nparts, stream=None):
    """lasp_bwd_finish for part `part` of `nparts` of the (b, h) pairs. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_bwd_finish_part(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dk),
                                        _ptr(dv), B, H, N, d, C, dt, _ptr(state_cache), _ptr(dstate_ws),
                                        _ptr(dstate_in), _ptr(dinit_state), part, nparts, _stream(stream, q)),
           "lasp_bwd_finish_part")


def lasp_parts_ok(N, C, d, dtype):
    """1 when the part calls accept nparts > 1 for these sizes. See lasp.h."""
    return int(_load().lasp_parts_ok(N, C, d, dtype))


def lasp_bwd_noalloc(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_in=None, dinit_state=None,
                     stream=None):
    """lasp_bwd for callers that cannot allocate: the gradient-state workspace is
    a fixed array inside the library (see lasp.h for its limit and sharing rules)."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dk),
                                    _ptr(dv), B, H, N, d, C, dt, _ptr(state_cache), _ptr(dstate_in),
                                    _ptr(dinit_state), _stream(stream, q)), "lasp_bwd_noalloc")


def lasp_chunk_states(q, k, v, decay, M, C, stream=None):
    """M[b, c, h] = sum_j lambda^(C-1-j) k_j^T v_j. See lasp.h."""
    B, N, H, d, dt = _tokens(k, v)
    _check(_load().lasp_chunk_states(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(M), B, H, N, d, C, dt,
                                     _stream(stream, k)), "lasp_chunk_states")


def lasp_chunk_dstates(q, dout, decay, dM, C, stream=None):
    """dM[b, c, h] = sum_j lambda^(j+1) q_j^T do_j. See lasp.h."""
    B, N, H, d, dt = _tokens(q, dout)
    _check(_load().lasp_chunk_dstates(_ptr(q), _ptr(dout), _ptr(decay), _ptr(dM), B, H, N, d, C, dt,
                                      _stream(stream, q)), "lasp_chunk_dstates")


def lasp_chunk_out(q, k, v, decay, P, o, C, stream=None):
    """The output step alone: o from (q, k, v) and the chunk-entering states P. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _check(_load().lasp_chunk_out(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(P), _ptr(o), B, H, N, d, C, dt,
                                  _stream(stream, q)), "lasp_chunk_out")


def lasp_chunk_grads(q, k, v, dout, decay, P, R, dq, dk, dv, C, stream=None):
    """The dQ/dK/dV step alone, from the states P and R. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_chunk_grads(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(decay), _ptr(P), _ptr(R),
                                    _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, C, dt, _stream(stream, q)),
           "lasp_chunk_grads")


def lasp_state_prefix(M, Mprefix, decay, C, init=None, total=None, reverse=False, stream=None):
    """Exclusive decayed prefix (or suffix) over chunk states [B, T, H, d, d]. See lasp.h."""
    if M.dim() != 5:
        raise ValueError("M must be [B, T, H, d, d]")
    B, T, H, d, _ = M.shape
    _check(_load().lasp_state_prefix(_ptr(M), _ptr(Mprefix), _ptr(decay), _ptr(init), _ptr(total),
                                     B, T, H, d, int(C), int(bool(reverse)), _stream(stream, M)),
           "lasp_state_prefix")


def lasp_bidir_workspace_floats(B, H, N, d, dtype=LASP_BF16):
    """Floats of the workspace lasp_bidir_fwd / lasp_bidir_bwd need (0 if unsupported). See lasp.h."""
    return int(_load().lasp_bidir_workspace_floats(B, H, N, d, dtype))


def lasp_bidir_state_offset(B, H, N, d, dtype=LASP_BF16):
    """Offset (floats) of the fp32 total state [B, H, d, d] inside the workspace. See lasp.h."""
    return int(_load().lasp_bidir_state_offset(B, H, N, d, dtype))


def lasp_bidir_fwd(q, k, v, o, ws, stream=None):
    """o = q (k^T v) per (b, h), the bidirectional (unmasked) form; ws receives M. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _check(_load().lasp_bidir_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, H, N, d, dt, _ptr(ws),
                                  _stream(stream, q)), "lasp_bidir_fwd")


def lasp_bidir_bwd(q, k, v, dout, dq, dk, dv, ws, dws, stream=None):
    """dq, dk, dv of sum(o * dout) for lasp_bidir_fwd; dws receives dM. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _check(_load().lasp_bidir_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                  B, H, N, d, dt, _ptr(ws), _ptr(dws), _stream(stream, q)), "lasp_bidir_bwd")


def _gates(like, *gs):
    """The float32 [B, N, H, d] log-gate tensors of the gated calls."""
    import torch
    for g in gs:
        if g is None:
            continue
        if (tuple(g.shape) != tuple(like.shape) or g.dtype != torch.float32 or not g.is_contiguous()
                or not g.is_cuda):
            raise ValueError("gate tensors must be contiguous float32 CUDA tensors shaped like q")


def lasp_gla_cache_floats(B, H, N, d, C):
    """Floats of the state cache of the gated calls (-1 if unsupported). See lasp.h."""
    return int(_load().lasp_gla_cache_floats(B, H, N, d, C))


def lasp_gla_chunk_states(x, y, g, M, C, gsum=None, kind=0, stream=None):
    """Gated chunk states: kind 0 from (k, v), kind 1 from (q, dout); gsum the chunk log-gate totals. See lasp.h."""
    B, N, H, d, dt = _tokens(x, y)
    _gates(x, g)
    _check(_load().lasp_gla_chunk_states(_ptr(x), _ptr(y), _ptr(g), _ptr(M), _ptr(gsum), B, H, N, d, C, dt,
                                         int(kind), _stream(stream, x)), "lasp_gla_chunk_states")


def lasp_gla_state_prefix(M, Mprefix, gsum, init=None, total=None, reverse=False, stream=None):
    """Exclusive scan over gated chunk states with a diagonal decay exp(gsum_c) per chunk. See lasp.h."""
    if M.dim() != 5:
        raise ValueError("M must be [B, T, H, d, d]")
    B, T, H, d, _ = M.shape
    _check(_load().lasp_gla_state_prefix(_ptr(M), _ptr(Mprefix), _ptr(gsum), _ptr(init), _ptr(total), B, T, H, d,
                                         int(bool(reverse)), _stream(stream, M)), "lasp_gla_state_prefix")


def lasp_gla_fwd(q, k, v, g, o, C, state_cache, init_state=None, stream=None):
    """o for the gated recurrence kv_s = diag(exp(g_s)) kv_{s-1} + k_s^T v_s. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, o)
    _gates(q, g)
    _check(_load().lasp_gla_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), B, H, N, d, C, dt, _ptr(state_cache),
                                _ptr(init_state), _stream(stream, q)), "lasp_gla_fwd")


def lasp_gla_bwd(q, k, v, g, dout, dq, dk, dv, dg, C, state_cache, dstate_ws, dstate_in=None, dinit_state=None,
                 stream=None):
    """dq, dk, dv, dg of sum(o * dout) for lasp_gla_fwd. See lasp.h."""
    B, N, H, d, dt = _tokens(q, k, v, dout, dq, dk, dv)
    _gates(q, g, dg)
    _check(_load().lasp_gla_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dg), B, H, N, d, C, dt, _ptr(state_cache), _ptr(dstate_ws), _ptr(dstate_in),
                                _ptr(dinit_state), _stream(stream, q)), "lasp_gla_bwd")


def lasp_check_device_status(stream=None, device=None):
    """(status, site): synchronizes the stream, returns and clears the device status word."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream(device).cuda_stream
    site = ctypes.c_int(0)
    st = _load().lasp_check_device_status(s if isinstance(s, int) else s.cuda_stream, ctypes.byref(site))
    return st, site.value


def lasp_set_wait_limit_ns(limit_ns: int):
    _check(_load().lasp_set_wait_limit_ns(int(limit_ns)), "lasp_set_wait_limit_ns")


def lasp_wait_probe(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream().cuda_stream
    _check(_load().lasp_wait_probe(s if isinstance(s, int) else s.cuda_stream), "lasp_wait_probe")


def lasp_trace_enable(capacity: int):
    """Bracket each library kernel launch with CUDA events (up to `capacity`); 0 turns it off."""
    _check(_load().lasp_trace_enable(int(capacity)), "lasp_trace_enable")


def lasp_trace_read(capacity: int = 4096):
    """[(kernel_name, milliseconds)] of the launches recorded since the last read."""
    ids = (ctypes.c_int * capacity)()
    ms = (ctypes.c_float * capacity)()
    n = _load().lasp_trace_read(ids, ms, capacity)
    if n < 0:
        raise LaspError(-n, "lasp_trace_read")
    return [(lasp_kernel_name(ids[i]), float(ms[i])) for i in range(n)]


def lasp_kernel_name(kernel_id: int) -> str:
    return _load().lasp_kernel_name(int(kernel_id)).decode()


def lasp_segment_tokens(N: int, C: int, d: int, dtype_code: int) -> int:
    """Segment length lasp_fwd uses (see lasp.h)."""
    return int(_load().lasp_segment_tokens(int(N), int(C), int(d), int(dtype_code)))


def lasp_status_string(status: int) -> str:
    return _load().lasp_status_string(int(status)).decode()


def lasp_version() -> int:
    return int(_load().lasp_version())


# ------------------------------------------------------------ softmax attention
def _softmax_shapes(q, k, *rest_q):
    """(B, H, Nq, Nk, d, dtype) of queries [B, Nq, H, d] against keys [B, Nk, H, d]."""
    Bq, Nq, Hq, dq_ = _tokens(q, *rest_q)[:4]
    B, Nk, H, d, dt = _tokens(k)
    if (Bq, Hq, dq_) != (B, H, d) or q.dtype != k.dtype:
        raise ValueError("queries and keys must share B, H, d and dtype")
    return B, H, Nq, Nk, d, dt


def _rows(t, B, H, Nq):
    if t is not None and (tuple(t.shape) != (B, H, Nq) or t.dtype.itemsize != 4 or not t.is_contiguous()):
        raise ValueError("lse and delta must be contiguous float32 [B, H, Nq]")


def lasp_softmax_fwd(q, k, v, o, lse, q_offset=0, scale=None, stream=None):
    """Causal softmax attention of queries at positions q_offset + i against
    keys / values at 0..Nk-1; o [B, Nq, H, d], lse [B, H, Nq]. See lasp.h."""
    B, H, Nq, Nk, d, dt = _softmax_shapes(q, k, o)
    _tokens(k, v)
    _rows(lse, B, H, Nq)
    scale = float(d) ** -0.5 if scale is None else float(scale)
    _check(_load().lasp_softmax_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, q_offset, d,
                                    scale, dt, _stream(stream, q)), "lasp_softmax_fwd")


def lasp_softmax_bwd(q, k, v, o, lse, dout, dq, dk, dv, delta, q_offset=0, scale=None, stream=None):
    """dq, dk, dv of sum(o * dout) for lasp_softmax_fwd; delta [B, H, Nq] is a
    workspace. See lasp.h."""
    B, H, Nq, Nk, d, dt = _softmax_shapes(q, k, o, dout, dq)
    _tokens(k, v, dk, dv)
    _rows(lse, B, H, Nq)
    _rows(delta, B, H, Nq)
    scale = float(d) ** -0.5 if scale is None else float(scale)
    _check(_load().lasp_softmax_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                    _ptr(dv), _ptr(delta), B, H, Nq, Nk, q_offset, d, scale, dt,
                                    _stream(stream, q)), "lasp_softmax_bwd")
