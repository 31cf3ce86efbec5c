"""fp64 CPU oracle for causal linear attention with per-head decay (LASP / LASP-2).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. It shares no code with ``sequence_linear_attention_b200`` and never
imports it; the CUDA library never calls into it.

The arithmetic lives in ``lasp_oracle.c`` (plain C, double precision, one loop
nest per definition); this module compiles it with gcc on first use and wraps
it with ctypes. Each wrapper states the passage it follows:

* :func:`fwd` -- LASP page, section 3.2, Eq. 4-6 (token recurrence).
* :func:`bwd` -- LASP page, section 3.2, Eq. 12-13 (reverse recurrence).
* :func:`chunk_states` -- LASP page, Eq. 10 / Algorithm 2 (forward memory
  state of one chunk) and Eq. 20 / Algorithm 3 (gradient state); LASP-2 review
  page, "The reading": M_t summarises chunk t.
* :func:`state_scan` -- LASP-2 review page, "Core claim": prefix sum of the
  gathered states (forward), suffix sum of dM_t (backward); decay lambda^C per
  chunk from LASP Eq. 10 / Eq. 20.
* :func:`state_snapshots` -- LASP page, section 3.4 "KV State Caching": the
  chunk-boundary states of the recurrences.
* :func:`bidir_fwd`, :func:`bidir_bwd` -- the bidirectional (unmasked) form:
  LASP page, section 3.1, Eq. 3 right product Q (K^T V) without Norm; LASP-2
  review page, "Summary": the unmasked variant gathers all chunk states and
  every chunk computes Q_t M_{1:T}, and the backward the same with dM.
* :func:`softmax_fwd`, :func:`softmax_bwd` -- the softmax-attention layers of
  the hybrid model: LASP-2 review page, "Summary" (LASP-2H applies the same
  AllGather pattern to standard attention, gathering K_t and V_t); standard
  causal softmax attention with a query offset into the gathered keys, and its
  gradients by the chain rule through the softmax.
* :func:`gla_fwd`, :func:`gla_bwd`, :func:`gla_chunk_states`,
  :func:`gla_state_scan`, :func:`gla_state_snapshots` -- the gated form (a
  decay per token and key feature): LASP page, Appendix A.4, Eq. 24 with the
  GLA / GateLoop row of Table 5 (oscillation g_t 1^T), the gate passed as its
  natural log; gradients by the chain rule on that recurrence.

Inputs are float32 arrays shaped [B, N, H, d] (any strides, feature axis
contiguous). Values that came from bf16 are exact in float32 and double, so the
oracle sees exactly what the GPU sees. Outputs are float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lasp_oracle.c")
_LIB = os.path.join(_HERE, "liblasp_oracle.so")
_CFLAGS = ["-O3", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off", "-std=c11"]
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile lasp_oracle.c into liblasp_oracle.so (portable x86-64 code)."""
    stale = (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_P = ctypes.c_void_p
_L = ctypes.c_long
_I = ctypes.c_int


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_fwd.argtypes = [_P, _P, _P, _L, _L, _L, _P, _P, _P, _L, _L, _L, _P, _I, _L, _I, _I]
            lib.oracle_bwd.argtypes = [_P, _P, _P, _P, _L, _L, _L, _P, _P, _P,
                                       _P, _P, _P, _L, _L, _L, _P, _I, _L, _I, _I]
            lib.oracle_chunk_states.argtypes = [_P, _P, _L, _L, _L, _P, _P, _I, _L, _I, _I, _L, _I]
            lib.oracle_state_scan.argtypes = [_P, _P, _P, _P, _P, _I, _L, _I, _I, _L, _I]
            lib.oracle_state_snapshots.argtypes = [_P, _P, _L, _L, _L, _P, _P, _P, _I, _L, _I, _I, _L, _I]
            lib.oracle_bidir_fwd.argtypes = [_P, _P, _P, _L, _L, _L, _P, _L, _L, _L, _P, _I, _L, _I, _I]
            lib.oracle_bidir_bwd.argtypes = [_P, _P, _P, _P, _L, _L, _L, _P, _P, _P, _L, _L, _L, _P,
                                             _I, _L, _I, _I]
            lib.oracle_gla_fwd.argtypes = [_P, _P, _P, _P, _L, _L, _L, _P, _P, _L, _L, _L, _P, _I, _L, _I, _I]
            lib.oracle_gla_bwd.argtypes = [_P, _P, _P, _P, _P, _L, _L, _L, _P, _P,
                                           _P, _P, _P, _P, _L, _L, _L, _P, _I, _L, _I, _I]
            lib.oracle_gla_chunk_states.argtypes = [_P, _P, _P, _L, _L, _L, _P, _P, _I, _L, _I, _I, _L, _I]
            lib.oracle_gla_state_scan.argtypes = [_P, _P, _P, _P, _P, _I, _L, _I, _I, _I]
            lib.oracle_gla_state_snapshots.argtypes = [_P, _P, _P, _L, _L, _L, _P, _P, _I, _L, _I, _I, _L, _I]
            _D = ctypes.c_double
            lib.oracle_softmax_fwd.argtypes = [_P, _L, _L, _L, _P, _P, _L, _L, _L, _P, _L, _L, _L, _P,
                                               _I, _L, _L, _L, _I, _I, _D]
            lib.oracle_softmax_bwd.argtypes = [_P, _L, _L, _L, _P, _P, _L, _L, _L, _P, _P, _L, _L, _L, _P, _P,
                                               _L, _L, _L, _I, _L, _L, _L, _I, _I, _D]
            lib.oracle_num_threads.restype = _I
            for f in (lib.oracle_fwd, lib.oracle_bwd, lib.oracle_chunk_states,
                      lib.oracle_state_scan, lib.oracle_state_snapshots, lib.oracle_bidir_fwd,
                      lib.oracle_bidir_bwd, lib.oracle_gla_fwd, lib.oracle_gla_bwd,
                      lib.oracle_gla_chunk_states, lib.oracle_gla_state_scan,
                      lib.oracle_gla_state_snapshots, lib.oracle_softmax_fwd, lib.oracle_softmax_bwd):
                f.restype = None
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all cores)."""
    return int(_load().oracle_num_threads())


def _view(x: np.ndarray, same_as: np.ndarray | None = None):
    """(pointer, sb, sn, sh) in elements for a [B, N, H, d] float32 view."""
    if x.dtype != np.float32 or x.ndim != 4 or x.strides[3] != 4:
        raise ValueError("token tensors must be float32 [B, N, H, d] with a contiguous feature axis")
    if same_as is not None and (x.shape != same_as.shape or x.strides != same_as.strides):
        raise ValueError("token tensors must share shape and strides")
    sb, sn, sh, _ = (s // 4 for s in x.strides)
    return x.ctypes.data, sb, sn, sh


def _lam(lam, H):
    if lam is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(lam, dtype=np.float64).reshape(H))
    return a, a.ctypes.data


def _state(x, shape):
    if x is None:
        return None, None
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    if a.shape != shape:
        raise ValueError(f"state must have shape {shape}, got {a.shape}")
    return a, a.ctypes.data


def _ptr(a):
    return None if a is None else a.ctypes.data


def fwd(q, k, v, lam=None, init=None, want_final=False):
    """o_s = q_s kv_s with kv_s = lam*kv_{s-1} + k_s^T v_s (LASP Eq. 4-6).

    ``lam``: per-head decay [H] or None (lambda = 1). ``init``: [B, H, d, d]
    state entering token 0, or None. Returns o (float64 [B, N, H, d]) and, if
    ``want_final``, the state after the last token as well.
    """
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    _view(k, q), _view(v, q)
    la, pl = _lam(lam, H)
    ia, pi = _state(init, (B, H, d, d))
    o = np.empty((B, N, H, d), np.float64)
    fin = np.empty((B, H, d, d), np.float64) if want_final else None
    _load().oracle_fwd(pq, k.ctypes.data, v.ctypes.data, sb, sn, sh, pl, pi,
                       o.ctypes.data, N * H * d, H * d, d, _ptr(fin), B, N, H, d)
    return (o, fin) if want_final else o


def bwd(q, k, v, do, lam=None, init=None, dstate_in=None, want_dinit=False):
    """Gradients of sum(o * do) by the reverse recurrence (LASP Eq. 12-13).

    ``dstate_in``: [B, H, d, d] gradient state entering the last token from
    beyond the sequence end (0 if None). Returns dq, dk, dv (float64
    [B, N, H, d]) and, if ``want_dinit``, the gradient w.r.t. ``init``.
    """
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    for t in (k, v, do):
        _view(t, q)
    la, pl = _lam(lam, H)
    ia, pi = _state(init, (B, H, d, d))
    fa, pf = _state(dstate_in, (B, H, d, d))
    dq = np.empty((B, N, H, d), np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    dinit = np.empty((B, H, d, d), np.float64) if want_dinit else None
    _load().oracle_bwd(pq, k.ctypes.data, v.ctypes.data, do.ctypes.data, sb, sn, sh, pl, pi, pf,
                       dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, N * H * d, H * d, d,
                       _ptr(dinit), B, N, H, d)
    return (dq, dk, dv, dinit) if want_dinit else (dq, dk, dv)


def chunk_states(a, b, lam, C, kind=0):
    """Per-chunk states M [B, T, H, d, d] from their definition.

    kind 0: M_c = sum_t lam^(C-1-t) a_t^T b_t with (a, b) = (k, v)  (LASP Eq. 10).
    kind 1: M_c = sum_t lam^(t+1)   a_t^T b_t with (a, b) = (q, do) (LASP Eq. 20).
    """
    B, N, H, d = a.shape
    if N % C:
        raise ValueError("C must divide N")
    pa, sb, sn, sh = _view(a)
    _view(b, a)
    la, pl = _lam(lam, H)
    M = np.empty((B, N // C, H, d, d), np.float64)
    _load().oracle_chunk_states(pa, b.ctypes.data, sb, sn, sh, pl, M.ctypes.data, B, N, H, d, C, kind)
    return M


def state_scan(M, lam, C, init=None, reverse=False):
    """Exclusive decayed prefix (reverse=False) or suffix (reverse=True) scan.

    prefix: P_0 = init, P_c = lam^C P_{c-1} + M_{c-1}; total = lam^C P_{T-1} + M_{T-1}
    suffix: R_{T-1} = init, R_c = lam^C R_{c+1} + M_{c+1}; total = lam^C R_0 + M_0
    Returns (P, total) in float64.
    """
    M = np.ascontiguousarray(np.asarray(M, dtype=np.float64))
    B, T, H, d, _ = M.shape
    la, pl = _lam(lam, H)
    ia, pi = _state(init, (B, H, d, d))
    P = np.empty_like(M)
    tot = np.empty((B, H, d, d), np.float64)
    _load().oracle_state_scan(M.ctypes.data, P.ctypes.data, pl, pi, tot.ctypes.data,
                              B, T, H, d, C, int(bool(reverse)))
    return P, tot


def state_snapshots(a, b, lam, C, init=None, kind=0):
    """Chunk-boundary states of the token recurrences, [B, T, H, d, d].

    kind 0, (a, b) = (k, v): P_c = kv_{cC-1}, the state entering chunk c.
    kind 1, (a, b) = (q, do): R_c = gradient state chunk c receives from the
    tokens after it; ``init`` is then the gradient state entering from beyond
    the sequence end.
    """
    B, N, H, d = a.shape
    if N % C:
        raise ValueError("C must divide N")
    pa, sb, sn, sh = _view(a)
    _view(b, a)
    la, pl = _lam(lam, H)
    ia, pi = _state(init, (B, H, d, d))
    P = np.empty((B, N // C, H, d, d), np.float64)
    _load().oracle_state_snapshots(pa, b.ctypes.data, sb, sn, sh, pl, pi, P.ctypes.data,
                                   B, N, H, d, C, kind)
    return P


def bidir_fwd(q, k, v, want_state=False):
    """Bidirectional (unmasked) output o_s = q_s M with M = sum_s k_s^T v_s
    (LASP Eq. 3 right product, no Norm, no decay). Returns o (float64
    [B, N, H, d]) and, if ``want_state``, M [B, H, d, d]."""
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    _view(k, q), _view(v, q)
    o = np.empty((B, N, H, d), np.float64)
    M = np.empty((B, H, d, d), np.float64) if want_state else None
    _load().oracle_bidir_fwd(pq, k.ctypes.data, v.ctypes.data, sb, sn, sh, o.ctypes.data, N * H * d, H * d, d,
                             _ptr(M), B, N, H, d)
    return (o, M) if want_state else o


def bidir_bwd(q, k, v, do, want_state=False):
    """Gradients of sum(o * do) for :func:`bidir_fwd`: dq = do M^T,
    dk = v dM^T, dv = k dM with dM = sum_s q_s^T do_s. Returns dq, dk, dv
    (float64 [B, N, H, d]) and, if ``want_state``, dM [B, H, d, d]."""
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    for t in (k, v, do):
        _view(t, q)
    dq = np.empty((B, N, H, d), np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    dM = np.empty((B, H, d, d), np.float64) if want_state else None
    _load().oracle_bidir_bwd(pq, k.ctypes.data, v.ctypes.data, do.ctypes.data, sb, sn, sh, dq.ctypes.data,
                             dk.ctypes.data, dv.ctypes.data, N * H * d, H * d, d, _ptr(dM), B, N, H, d)
    return (dq, dk, dv, dM) if want_state else (dq, dk, dv)


# ------------------------------------------------------------------ gated form
def gla_fwd(q, k, v, g, init=None, want_final=False):
    """Gated recurrence (LASP Appendix A.4, Eq. 24; Table 5, GLA / GateLoop):
    S_s = diag(exp(g_s)) S_{s-1} + k_s^T v_s, o_s = q_s S_s.

    ``g``: float32 [B, N, H, d], the natural log of the gate of each token and
    key feature (same shape and strides as q). ``init``: [B, H, d, d] or None.
    Returns o (float64 [B, N, H, d]) and, if ``want_final``, the last state.
    """
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    for t in (k, v, g):
        _view(t, q)
    ia, pi = _state(init, (B, H, d, d))
    o = np.empty((B, N, H, d), np.float64)
    fin = np.empty((B, H, d, d), np.float64) if want_final else None
    _load().oracle_gla_fwd(pq, k.ctypes.data, v.ctypes.data, g.ctypes.data, sb, sn, sh, pi,
                           o.ctypes.data, N * H * d, H * d, d, _ptr(fin), B, N, H, d)
    return (o, fin) if want_final else o


def gla_bwd(q, k, v, g, do, init=None, dstate_in=None, want_dinit=False):
    """Gradients of sum(o * do) for :func:`gla_fwd` by the chain rule on the
    recurrence: dq, dk, dv and dg (the gradient with respect to the log-gate),
    all float64 [B, N, H, d], and, if ``want_dinit``, the gradient with
    respect to ``init``. ``dstate_in``: [B, H, d, d] gradient with respect to
    the state after the last token (0 if None).
    """
    B, N, H, d = q.shape
    pq, sb, sn, sh = _view(q)
    for t in (k, v, g, do):
        _view(t, q)
    ia, pi = _state(init, (B, H, d, d))
    fa, pf = _state(dstate_in, (B, H, d, d))
    dq = np.empty((B, N, H, d), np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    dg = np.empty_like(dq)
    dinit = np.empty((B, H, d, d), np.float64) if want_dinit else None
    _load().oracle_gla_bwd(pq, k.ctypes.data, v.ctypes.data, g.ctypes.data, do.ctypes.data, sb, sn, sh, pi, pf,
                           dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, dg.ctypes.data, N * H * d, H * d, d,
                           _ptr(dinit), B, N, H, d)
    return (dq, dk, dv, dg, dinit) if want_dinit else (dq, dk, dv, dg)


def gla_chunk_states(x, y, g, C, kind=0):
    """Gated per-chunk states [B, T, H, d, d] and chunk log-gate totals
    [B, T, H, d], from their definition.

    kind 0, (x, y) = (k, v): M_c = sum_t diag(exp(sum of g over t+1..C-1)) x_t^T y_t.
    kind 1, (x, y) = (q, do): M_c = sum_t diag(exp(sum of g over 0..t)) x_t^T y_t.
    """
    B, N, H, d = x.shape
    if N % C:
        raise ValueError("C must divide N")
    px, sb, sn, sh = _view(x)
    _view(y, x), _view(g, x)
    M = np.empty((B, N // C, H, d, d), np.float64)
    gs = np.empty((B, N // C, H, d), np.float64)
    _load().oracle_gla_chunk_states(px, y.ctypes.data, g.ctypes.data, sb, sn, sh, M.ctypes.data, gs.ctypes.data,
                                    B, N, H, d, C, kind)
    return M, gs


def gla_state_scan(M, gsum, init=None, reverse=False):
    """Exclusive scan over gated chunk states; a step through chunk c scales
    row i by exp(gsum[c, i]). Returns (P, total) in float64 (see the C file)."""
    M = np.ascontiguousarray(np.asarray(M, dtype=np.float64))
    B, T, H, d, _ = M.shape
    gs = np.ascontiguousarray(np.asarray(gsum, dtype=np.float64))
    if gs.shape != (B, T, H, d):
        raise ValueError("gsum must be [B, T, H, d]")
    ia, pi = _state(init, (B, H, d, d))
    P = np.empty_like(M)
    tot = np.empty((B, H, d, d), np.float64)
    _load().oracle_gla_state_scan(M.ctypes.data, gs.ctypes.data, P.ctypes.data, pi, tot.ctypes.data,
                                  B, T, H, d, int(bool(reverse)))
    return P, tot


def gla_state_snapshots(x, y, g, C, init=None, kind=0):
    """Chunk-boundary states of the gated recurrences, [B, T, H, d, d]:
    kind 0 (k, v): the state entering each chunk; kind 1 (q, do): the gradient
    state each chunk receives from the tokens after it (``init`` = dstate_in)."""
    B, N, H, d = x.shape
    if N % C:
        raise ValueError("C must divide N")
    px, sb, sn, sh = _view(x)
    _view(y, x), _view(g, x)
    ia, pi = _state(init, (B, H, d, d))
    P = np.empty((B, N // C, H, d, d), np.float64)
    _load().oracle_gla_state_snapshots(px, y.ctypes.data, g.ctypes.data, sb, sn, sh, pi, P.ctypes.data,
                                       B, N, H, d, C, kind)
    return P


# ------------------------------------------------------------ softmax attention
def _tok_view(x: np.ndarray):
    if x.dtype != np.float32 or x.ndim != 4 or x.strides[3] != 4:
        raise ValueError("token tensors must be float32 [B, N, H, d] with a contiguous feature axis")
    sb, sn, sh, _ = (s // 4 for s in x.strides)
    return x.ctypes.data, sb, sn, sh


def softmax_fwd(q, k, v, q_offset=0, scale=None):
    """Causal softmax attention of queries q [B, Nq, H, d] at global positions
    q_offset + i against keys / values k, v [B, Nk, H, d] at positions
    0..Nk-1: o_i = sum_{j <= q_offset + i} softmax_j(scale q_i . k_j) v_j, and
    lse_i, the natural log of the softmax denominator (with the scores as
    given, no shift). scale defaults to d^-1/2. Returns o (float64
    [B, Nq, H, d]) and lse (float64 [B, H, Nq])."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    if k.shape != v.shape or k.strides != v.strides or k.shape[0] != B or k.shape[2:] != (H, d):
        raise ValueError("k and v must be [B, Nk, H, d] views with the same strides")
    if q_offset < 0 or q_offset + Nq > Nk:
        raise ValueError("the queries must sit inside the keys: q_offset + Nq <= Nk")
    scale = float(d) ** -0.5 if scale is None else float(scale)
    pq, qb, qn, qh = _tok_view(q)
    pk, kb, kn, kh = _tok_view(k)
    pv = _tok_view(v)[0]
    o = np.empty((B, Nq, H, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    _load().oracle_softmax_fwd(pq, qb, qn, qh, pk, pv, kb, kn, kh, o.ctypes.data, Nq * H * d, H * d, d,
                               lse.ctypes.data, B, Nq, Nk, q_offset, H, d, scale)
    return o, lse


def softmax_bwd(q, k, v, do, q_offset=0, scale=None):
    """Gradients of sum(o * do) for :func:`softmax_fwd` with respect to q
    ([B, Nq, H, d]) and k, v ([B, Nk, H, d]; keys no query reaches get zero).
    do shares q's shape and strides. Returns dq, dk, dv as float64."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    if k.shape != v.shape or k.strides != v.strides or k.shape[0] != B or k.shape[2:] != (H, d):
        raise ValueError("k and v must be [B, Nk, H, d] views with the same strides")
    if do.shape != q.shape or do.strides != q.strides:
        raise ValueError("do must share q's shape and strides")
    if q_offset < 0 or q_offset + Nq > Nk:
        raise ValueError("the queries must sit inside the keys: q_offset + Nq <= Nk")
    scale = float(d) ** -0.5 if scale is None else float(scale)
    pq, qb, qn, qh = _tok_view(q)
    pk, kb, kn, kh = _tok_view(k)
    pv = _tok_view(v)[0]
    pd = _tok_view(do)[0]
    dq = np.empty((B, Nq, H, d), np.float64)
    dk = np.empty((B, Nk, H, d), np.float64)
    dv = np.empty_like(dk)
    _load().oracle_softmax_bwd(pq, qb, qn, qh, pk, pv, kb, kn, kh, pd, dq.ctypes.data, Nq * H * d, H * d, d,
                               dk.ctypes.data, dv.ctypes.data, Nk * H * d, H * d, d, B, Nq, Nk, q_offset, H, d, scale)
    return dq, dk, dv
