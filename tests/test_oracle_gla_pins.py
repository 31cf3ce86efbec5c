"""Pins for the gated oracle (a decay per token and key feature).

The gated form is the GLA / GateLoop row of Table 5 in Appendix A.4 of the
LASP page (Eq. 24: m_t = o_t m_{t-1} + e_t i_t^T with o_t = g_t 1^T). The
oracle's gated functions are checked here against things other than
themselves: the constant-gate special case (which is the decayed recurrence of
section 3.2, a separate function of the oracle), the quadratic form written
out in numpy, central finite differences for every gradient, the identity
that ties the log-gate gradient to q . dq - k . dk, chunk states + scans
against token-by-token snapshots, the shard decomposition, and a chunk-by-chunk
restatement of the algorithm the CUDA kernels follow.
"""
import numpy as np
import pytest

import oracle


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _problem(seed, B=2, N=40, H=3, d=8, quant=None, gate_scale=0.3):
    rng = np.random.default_rng(seed)

    def r(shape):
        x = rng.standard_normal(shape)
        if quant:
            x = np.round(x * quant) / quant
        return x.astype(np.float32)

    q, k, v, do = (r((B, N, H, d)) for _ in range(4))
    # log-gates <= 0 of varied size per feature, on a 1/256 grid (exact in float32)
    g = -np.round(rng.uniform(0.0, gate_scale, (B, N, H, d)) * 256) / 256
    return q, k, v, g.astype(np.float32), do


# ------------------------------------------------------- constant-gate case
def test_constant_gate_is_the_decayed_recurrence():
    """g_s[i] = log(lambda_h) everywhere reduces Eq. 24 to LASP Eq. 5 (Table 5,
    row TNL / RetNet: oscillation lambda J); the oracle's decayed functions are
    separate code, and with lambda = exp(a) in double the two agree bit for bit."""
    q, k, v, _, do = _problem(3, B=2, N=24, H=3, d=6)
    B, N, H, d = q.shape
    a = np.array([-1 / 32, -1 / 4, 0.0], np.float32)
    lam = np.exp(a.astype(np.float64))
    g = np.ascontiguousarray(np.broadcast_to(a[None, None, :, None], q.shape), dtype=np.float32)
    rng = np.random.default_rng(33)
    init = rng.standard_normal((B, H, d, d))
    dsin = rng.standard_normal((B, H, d, d))
    o1, f1 = oracle.gla_fwd(q, k, v, g, init=init, want_final=True)
    o2, f2 = oracle.fwd(q, k, v, lam, init=init, want_final=True)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(f1, f2)
    dq1, dk1, dv1, _, di1 = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dsin, want_dinit=True)
    dq2, dk2, dv2, di2 = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=dsin, want_dinit=True)
    for x, y in ((dq1, dq2), (dk1, dk2), (dv1, dv2), (di1, di2)):
        np.testing.assert_array_equal(x, y)


def test_zero_gate_is_plain_linear_attention():
    """log-gate 0 (gate 1) is ordinary linear attention (Table 5, row Linear
    Attention: oscillation J): the prefix sum of outer products."""
    q, k, v, _, _ = _problem(4, B=1, N=12, H=2, d=4)
    g = np.zeros_like(q)
    o = oracle.gla_fwd(q, k, v, g)
    kv = np.cumsum(np.einsum("bnhi,bnhj->bnhij", k.astype(np.float64), v.astype(np.float64)), axis=1)
    ref = np.einsum("bnhi,bnhij->bnhj", q.astype(np.float64), kv)
    assert _rel(o, ref) < 1e-13


# ------------------------------------------------------------ quadratic form
def _quadratic(q, k, v, g, init=None):
    """o_t = sum_{s<=t} sum_i q_t[i] k_s[i] exp(sum_{r=s+1}^{t} g_r[i]) v_s
             + sum_i q_t[i] exp(sum_{r=0}^{t} g_r[i]) init[i, :]."""
    q, k, v, g = (x.astype(np.float64) for x in (q, k, v, g))
    B, N, H, d = q.shape
    G = np.cumsum(g, axis=1)  # inclusive
    o = np.zeros((B, N, H, d))
    for t in range(N):
        for s in range(t + 1):
            w = np.exp(G[:, t] - G[:, s])  # [B, H, d]: gates r = s+1..t
            att = np.sum(q[:, t] * k[:, s] * w, axis=-1)  # [B, H]
            o[:, t] += att[..., None] * v[:, s]
        if init is not None:
            o[:, t] += np.einsum("bhi,bhij->bhj", q[:, t] * np.exp(G[:, t]), init)
    return o


@pytest.mark.parametrize("seed", [1, 2])
def test_recurrence_equals_quadratic_form(seed):
    q, k, v, g, _ = _problem(seed, B=2, N=20, H=2, d=5, gate_scale=1.0)
    init = np.random.default_rng(seed + 10).standard_normal((2, 2, 5, 5))
    assert _rel(oracle.gla_fwd(q, k, v, g), _quadratic(q, k, v, g)) < 1e-12
    assert _rel(oracle.gla_fwd(q, k, v, g, init=init), _quadratic(q, k, v, g, init)) < 1e-12


# -------------------------------------------------------- finite differences
def test_gradients_match_finite_differences():
    q, k, v, g, do = _problem(5, B=1, N=18, H=2, d=5, quant=64, gate_scale=0.5)
    B, N, H, d = q.shape
    rng = np.random.default_rng(55)
    init = np.round(rng.standard_normal((B, H, d, d)) * 64) / 64
    dsin = np.round(rng.standard_normal((B, H, d, d)) * 64) / 64
    dq, dk, dv, dg, dinit = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dsin, want_dinit=True)

    def loss(qq, kk, vv, gg, ii):
        o, fin = oracle.gla_fwd(qq, kk, vv, gg, init=ii, want_final=True)
        return float(np.sum(o * do) + np.sum(fin * dsin))

    idx = [tuple(int(rng.integers(0, s)) for s in q.shape) for _ in range(30)]
    # q, k, v enter the loss linearly: the central difference is exact up to rounding
    h = 1.0 / 64
    for grad, which in ((dq, 0), (dk, 1), (dv, 2)):
        for ix in idx:
            p = [q.copy(), k.copy(), v.copy()]
            m = [q.copy(), k.copy(), v.copy()]
            p[which][ix] += h
            m[which][ix] -= h
            fd = (loss(*p, g, init) - loss(*m, g, init)) / (2 * h)
            assert abs(fd - grad[ix]) <= 1e-9 * max(1.0, abs(grad[ix])), (which, ix)
    # the log-gate enters through exp: central difference error is O(h^2)
    hg = 2.0 ** -10
    for ix in idx:
        gp, gm = g.copy(), g.copy()
        gp[ix] += hg
        gm[ix] -= hg
        fd = (loss(q, k, v, gp, init) - loss(q, k, v, gm, init)) / (2 * hg)
        assert abs(fd - dg[ix]) <= 1e-5 * max(1.0, abs(dg[ix])), ix
    for _ in range(10):
        ix = tuple(int(rng.integers(0, s)) for s in init.shape)
        ip, im = init.copy(), init.copy()
        ip[ix] += h
        im[ix] -= h
        fd = (loss(q, k, v, g, ip) - loss(q, k, v, g, im)) / (2 * h)
        assert abs(fd - dinit[ix]) <= 1e-9 * max(1.0, abs(dinit[ix]))


def test_gate_gradient_identity():
    """With B_t = sum_{r<=t} g_r the output depends on the gates only through
    q_t exp(B_t), k_s exp(-B_s) and, for the last state, exp(B_{N-1}); so
    dg_s = sum_{t>=s} (q_t dq_t - k_t dk_t) + rowsum(dstate_in * S_{N-1}).
    The oracle computes dg from G_s and S_{s-1} instead."""
    q, k, v, g, do = _problem(6, B=2, N=30, H=2, d=6, gate_scale=0.6)
    B, N, H, d = q.shape
    rng = np.random.default_rng(66)
    init = rng.standard_normal((B, H, d, d))
    dsin = rng.standard_normal((B, H, d, d))
    dq, dk, dv, dg = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dsin)
    _, fin = oracle.gla_fwd(q, k, v, g, init=init, want_final=True)
    per_t = q.astype(np.float64) * dq - k.astype(np.float64) * dk
    rev = np.flip(np.cumsum(np.flip(per_t, axis=1), axis=1), axis=1)
    ref = rev + np.sum(dsin * fin, axis=-1)[:, None, :, :]
    assert _rel(dg, ref) < 1e-11


# ------------------------------------------------ chunk states and scans
@pytest.mark.parametrize("C", [1, 4, 8])
def test_chunk_states_and_scans_equal_snapshots(C):
    q, k, v, g, do = _problem(7, B=2, N=32, H=2, d=5, gate_scale=0.5)
    B, N, H, d = q.shape
    rng = np.random.default_rng(77)
    init = rng.standard_normal((B, H, d, d))
    dsin = rng.standard_normal((B, H, d, d))
    M, gs = oracle.gla_chunk_states(k, v, g, C, kind=0)
    np.testing.assert_allclose(gs, g.astype(np.float64).reshape(B, N // C, C, H, d).sum(axis=2), rtol=0, atol=1e-12)
    P, tot = oracle.gla_state_scan(M, gs, init=init)
    snap = oracle.gla_state_snapshots(k, v, g, C, init=init, kind=0)
    _, fin = oracle.gla_fwd(q, k, v, g, init=init, want_final=True)
    assert _rel(P, snap) < 1e-12
    assert _rel(tot, fin) < 1e-12
    dM, gs1 = oracle.gla_chunk_states(q, do, g, C, kind=1)
    np.testing.assert_array_equal(gs1, gs)
    R, dtot = oracle.gla_state_scan(dM, gs, init=dsin, reverse=True)
    rsnap = oracle.gla_state_snapshots(q, do, g, C, init=dsin, kind=1)
    *_, dinit = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dsin, want_dinit=True)
    assert _rel(R, rsnap) < 1e-12
    assert _rel(dtot, dinit) < 1e-12


def test_chunk_state_of_one_chunk_is_the_recurrence_from_zero():
    """With C = N, M_0 is the state after the last token started from zero, and
    the gradient state kind 1 is the dinit of a loss without dstate_in."""
    q, k, v, g, do = _problem(8, B=1, N=16, H=2, d=4)
    M, _ = oracle.gla_chunk_states(k, v, g, 16, kind=0)
    _, fin = oracle.gla_fwd(q, k, v, g, want_final=True)
    assert _rel(M[:, 0], fin) < 1e-13
    dM, _ = oracle.gla_chunk_states(q, do, g, 16, kind=1)
    *_, dinit = oracle.gla_bwd(q, k, v, g, do, want_dinit=True)
    assert _rel(dM[:, 0], dinit) < 1e-13


# ------------------------------------------------------ shard decomposition
@pytest.mark.parametrize("W", [2, 4])
def test_shard_decomposition_equals_unsplit(W):
    """LASP-2's split: each shard starts from the previous shard's last state;
    the backward chains dstate_in / dinit the other way."""
    q, k, v, g, do = _problem(9, B=1, N=32, H=2, d=4)
    L = 32 // W
    o_full = oracle.gla_fwd(q, k, v, g)
    dq_f, dk_f, dv_f, dg_f = oracle.gla_bwd(q, k, v, g, do)
    inits, st = [], None
    outs = []
    for w in range(W):
        sl = slice(w * L, (w + 1) * L)
        inits.append(st)
        o, st = oracle.gla_fwd(*(np.ascontiguousarray(x[:, sl]) for x in (q, k, v, g)), init=st, want_final=True)
        outs.append(o)
    assert _rel(np.concatenate(outs, axis=1), o_full) < 1e-12
    grads = [None] * W
    dsin = None
    for w in reversed(range(W)):
        sl = slice(w * L, (w + 1) * L)
        *gr, dsin = oracle.gla_bwd(*(np.ascontiguousarray(x[:, sl]) for x in (q, k, v, g, do)),
                                   init=inits[w], dstate_in=dsin, want_dinit=True)
        grads[w] = gr
    for i, full in enumerate((dq_f, dk_f, dv_f, dg_f)):
        assert _rel(np.concatenate([gr[i] for gr in grads], axis=1), full) < 1e-11


# ----------------------------------------- the chunked algorithm, restated
def _chunk_form(q, k, v, g, do, C, init=None, dstate_in=None):
    """The chunk algorithm the CUDA path uses, restated in numpy (float64).

    In chunk c with inclusive cumulative log-gates b_t = sum_{r<=t} g_r (from
    the chunk start) and entering state P_c:
      o_t  = (q_t * e^{b_t}) P_c + sum_{s<=t} (sum_i q_t[i] k_s[i] e^{b_t[i]-b_s[i]}) v_s
      P_{c+1} = diag(e^{b_end}) P_c + (k * e^{b_end - b})^T v.
    Backward with R_c, the gradient of the state leaving chunk c:
      dq = e^{b} * (dO P_c^T) + sum_s dA_ts k_s e^{b_t - b_s},    dA = (dO V^T) . causal
      dk = sum_t dA_ts q_t e^{b_t - b_s} + e^{b_end - b} * (V R_c^T)
      dv = A^T dO + (k * e^{b_end - b}) R_c
      dg = reverse cumsum over the chunk of (q dq - k dk), plus
           rowsum(R_c * S_end) on every token (S_end = P_{c+1})
      R_{c-1} = diag(e^{b_end}) R_c + (q * e^{b})^T dO.
    """
    f = lambda x: x.astype(np.float64)
    q, k, v, g, do = map(f, (q, k, v, g, do))
    B, N, H, d = q.shape
    T = N // C
    o = np.zeros_like(q)
    dq, dk, dv, dg = (np.zeros_like(q) for _ in range(4))
    dinit = np.zeros((B, H, d, d))
    mask = np.tril(np.ones((C, C)))
    for b in range(B):
        for h in range(H):
            P = np.zeros((d, d)) if init is None else init[b, h].copy()
            Ps = []
            for c in range(T):
                sl = slice(c * C, (c + 1) * C)
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                bc = np.cumsum(g[b, sl, h], axis=0)
                be = bc[-1]
                W = np.exp(bc[:, None, :] - bc[None, :, :])
                A = np.einsum("ti,si,tsi->ts", Q, K, W) * mask
                o[b, sl, h] = A @ V + (Q * np.exp(bc)) @ P
                Ps.append(P)
                P = np.exp(be)[:, None] * P + (K * np.exp(be - bc)).T @ V
            R = np.zeros((d, d)) if dstate_in is None else dstate_in[b, h].copy()
            for c in reversed(range(T)):
                sl = slice(c * C, (c + 1) * C)
                Q, K, V, dO = q[b, sl, h], k[b, sl, h], v[b, sl, h], do[b, sl, h]
                bc = np.cumsum(g[b, sl, h], axis=0)
                be = bc[-1]
                W = np.exp(bc[:, None, :] - bc[None, :, :])
                A = np.einsum("ti,si,tsi->ts", Q, K, W) * mask
                dA = (dO @ V.T) * mask
                Pc = Ps[c]
                dQ = np.exp(bc) * (dO @ Pc.T) + np.einsum("ts,si,tsi->ti", dA, K, W)
                dK = np.einsum("ts,ti,tsi->si", dA, Q, W) + np.exp(be - bc) * (V @ R.T)
                dV = A.T @ dO + (K * np.exp(be - bc)) @ R
                S_end = np.exp(be)[:, None] * Pc + (K * np.exp(be - bc)).T @ V
                per_t = Q * dQ - K * dK
                dG = np.flip(np.cumsum(np.flip(per_t, axis=0), axis=0), axis=0) + np.sum(R * S_end, axis=1)
                dq[b, sl, h], dk[b, sl, h], dv[b, sl, h], dg[b, sl, h] = dQ, dK, dV, dG
                R = np.exp(be)[:, None] * R + (Q * np.exp(bc)).T @ dO
            dinit[b, h] = R
    return o, dq, dk, dv, dg, dinit


@pytest.mark.parametrize("C", [1, 5, 8, 40])
def test_recurrence_equals_chunk_form(C):
    q, k, v, g, do = _problem(11, B=2, N=40, H=2, d=6, gate_scale=0.4)
    B, N, H, d = q.shape
    rng = np.random.default_rng(111)
    init = rng.standard_normal((B, H, d, d))
    dsin = rng.standard_normal((B, H, d, d))
    o, dq, dk, dv, dg, dinit = _chunk_form(q, k, v, g, do, C, init, dsin)
    assert _rel(o, oracle.gla_fwd(q, k, v, g, init=init)) < 1e-11
    ref = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dsin, want_dinit=True)
    for x, y in zip((dq, dk, dv, dg, dinit), ref):
        assert _rel(x, y) < 1e-10
