"""Pins for the fp64 oracle: each test ties it to something other than itself.

* Hand-worked example and closed forms (tests/golden/), LASP page Eq. 4-6, 12-13.
* The quadratic masked form, LASP page Eq. 2 (without Norm) with the decay mask
  of Algorithm 2 step 4, and its textbook gradients (Eq. 14, 17 and the dV
  intra form with one chunk covering the sequence).
* lambda = 1 is ordinary causal linear attention (LASP page, section 3.2:
  "choosing lambda = 1 yields the ordinary linear attention"): prefix sums of
  outer products with numpy.
* Central finite differences of L = sum(O * dO); L is linear in each of q, k, v
  and init, so the difference quotient is exact up to rounding.
* The chunk form of Algorithms 2 and 3 (Eq. 7-11, 14-23), restated here in
  numpy, for several chunk sizes.
* Shard invariance (LASP-2 decomposition): per-shard runs chained through the
  entering states equal the unsplit run.
"""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def _rand(rng, shape, quant=None):
    x = rng.standard_normal(shape)
    if quant:
        x = np.round(x * quant) / quant  # values exactly representable, for exact differences
    return x.astype(np.float32)


def _problem(seed, B=2, N=40, H=3, d=8, decayed=True, quant=None):
    rng = np.random.default_rng(seed)
    q, k, v, do = (_rand(rng, (B, N, H, d), quant) for _ in range(4))
    lam = rng.uniform(0.6, 1.0, H).astype(np.float32) if decayed else None
    return q, k, v, do, lam


# ---------------------------------------------------------------- golden files
def _read_golden(name):
    rows = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            rows.setdefault(key, []).append([float(x) for x in vals])
    return rows


def test_two_token_worked_example():
    g = _read_golden("two_token_worked_example.txt")
    lam = np.array([g["lambda"][0][0]], np.float32)
    t = {k: np.array(g[k], np.float32).reshape(1, 2, 1, 2) for k in ("q", "k", "v", "do")}
    o = oracle.fwd(t["q"], t["k"], t["v"], lam)
    dq, dk, dv = oracle.bwd(t["q"], t["k"], t["v"], t["do"], lam)
    for name, got in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_array_equal(got.reshape(2, 2), np.array(g[name]), err_msg=name)
    M = oracle.chunk_states(t["k"], t["v"], lam, C=2, kind=0)
    np.testing.assert_array_equal(M.reshape(2, 2), np.array(g["M"]))
    dM = oracle.chunk_states(t["q"], t["do"], lam, C=2, kind=1)
    np.testing.assert_array_equal(dM.reshape(2, 2), np.array(g["dM"]))


def test_unit_vector_closed_form():
    g = _read_golden("unit_vector_closed_form.txt")
    lam_v, N = g["lambda"][0][0], int(g["N"][0][0])
    e1 = np.zeros((1, N, 1, 4), np.float32)
    e1[..., 0] = 1.0
    lam = np.array([lam_v], np.float32)
    o = oracle.fwd(e1, e1, e1, lam)
    dq, dk, dv = oracle.bwd(e1, e1, e1, e1, lam)
    np.testing.assert_array_equal(o[0, :, 0, 0], g["o_e1"][0])
    np.testing.assert_array_equal(dq[0, :, 0, 0], g["o_e1"][0])
    np.testing.assert_array_equal(dk[0, :, 0, 0], g["dk_e1"][0])
    np.testing.assert_array_equal(dv[0, :, 0, 0], g["dk_e1"][0])
    assert not np.any(o[..., 1:]) and not np.any(dk[..., 1:])


@pytest.mark.parametrize("lam_v", [1.0, 0.9, 0.3])
def test_unit_vector_closed_form_formula(lam_v):
    N = 50
    e1 = np.zeros((1, N, 1, 4), np.float32)
    e1[..., 0] = 1.0
    lam = np.array([lam_v], np.float32)
    l = float(lam[0])
    s = np.arange(N)
    geo_in = (s + 1.0) if l == 1.0 else (1 - l ** (s + 1)) / (1 - l)
    geo_out = (N - s + 0.0) if l == 1.0 else (1 - l ** (N - s)) / (1 - l)
    o = oracle.fwd(e1, e1, e1, lam)
    dq, dk, dv = oracle.bwd(e1, e1, e1, e1, lam)
    assert _rel(o[0, :, 0, 0], geo_in) < 1e-14
    assert _rel(dq[0, :, 0, 0], geo_in) < 1e-14
    assert _rel(dk[0, :, 0, 0], geo_out) < 1e-14
    assert _rel(dv[0, :, 0, 0], geo_out) < 1e-14


# ------------------------------------------------------------ quadratic form
def _decay_mask(N, l):
    s = np.arange(N)
    diff = s[:, None] - s[None, :]
    return np.where(diff >= 0, float(l) ** np.maximum(diff, 0), 0.0)


def _quadratic(q, k, v, do, lam, init=None, dstate_in=None):
    """O = (Q K^T . D) V and its gradients, per (b, h), in float64."""
    B, N, H, d = q.shape
    o, dq, dk, dv = (np.zeros((B, N, H, d)) for _ in range(4))
    dinit = np.zeros((B, H, d, d))
    for b in range(B):
        for h in range(H):
            l = 1.0 if lam is None else float(lam[h])
            D = _decay_mask(N, l)
            Q, K, V, dO = (x[b, :, h, :].astype(np.float64) for x in (q, k, v, do))
            A = (Q @ K.T) * D
            dP = (dO @ V.T) * D
            o[b, :, h] = A @ V
            dq[b, :, h] = dP @ K
            dk[b, :, h] = dP.T @ Q
            dv[b, :, h] = A.T @ dO
            w_in = l ** (np.arange(N) + 1.0)            # weight of the entering state at token s
            w_out = l ** (N - 1.0 - np.arange(N))       # weight of the state entering from the end
            if init is not None:
                E = init[b, h]
                o[b, :, h] += w_in[:, None] * (Q @ E)
                dq[b, :, h] += w_in[:, None] * (dO @ E.T)
                dinit[b, h] = (Q * w_in[:, None]).T @ dO
            if dstate_in is not None:
                F = dstate_in[b, h]
                dk[b, :, h] += w_out[:, None] * (V @ F.T)
                dv[b, :, h] += w_out[:, None] * (K @ F)
                # the last state is lambda^N init + ..., and F is the gradient
                # of the later tokens' loss with respect to that state
                dinit[b, h] += l ** N * F
    return o, dq, dk, dv, dinit


@pytest.mark.parametrize("decayed", [False, True])
@pytest.mark.parametrize("seed", [1, 2])
def test_recurrence_equals_quadratic_form(decayed, seed):
    q, k, v, do, lam = _problem(seed, decayed=decayed)
    o = oracle.fwd(q, k, v, lam)
    dq, dk, dv = oracle.bwd(q, k, v, do, lam)
    ro, rdq, rdk, rdv, _ = _quadratic(q, k, v, do, lam)
    for got, ref in ((o, ro), (dq, rdq), (dk, rdk), (dv, rdv)):
        assert _rel(got, ref) < 1e-12


def test_entering_states_equal_quadratic_form():
    q, k, v, do, lam = _problem(3)
    B, N, H, d = q.shape
    rng = np.random.default_rng(33)
    init = rng.standard_normal((B, H, d, d))
    F = rng.standard_normal((B, H, d, d))
    o = oracle.fwd(q, k, v, lam, init=init)
    dq, dk, dv, dinit = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=F, want_dinit=True)
    ro, rdq, rdk, rdv, rdinit = _quadratic(q, k, v, do, lam, init=init, dstate_in=F)
    for got, ref in ((o, ro), (dq, rdq), (dk, rdk), (dv, rdv), (dinit, rdinit)):
        assert _rel(got, ref) < 1e-12


def test_lambda_one_is_prefix_sum_of_outer_products():
    q, k, v, do, _ = _problem(4, N=30, decayed=False)
    o = oracle.fwd(q, k, v, None)
    kv = np.cumsum(np.einsum("bnhi,bnhj->bnhij", k.astype(np.float64), v.astype(np.float64)), axis=1)
    ref = np.einsum("bnhi,bnhij->bnhj", q.astype(np.float64), kv)
    assert _rel(o, ref) < 1e-12
    # all-ones decay array is the same computation as "no decay"
    ones = np.ones(q.shape[2], np.float32)
    np.testing.assert_array_equal(oracle.fwd(q, k, v, ones), o)


# -------------------------------------------------------- finite differences
def test_gradients_match_finite_differences():
    q, k, v, do, lam = _problem(5, B=1, N=24, H=2, d=6, quant=64)
    B, N, H, d = q.shape
    rng = np.random.default_rng(55)
    init = np.round(rng.standard_normal((B, H, d, d)) * 64) / 64
    dq, dk, dv, dinit = oracle.bwd(q, k, v, do, lam, init=init, want_dinit=True)
    h = 1.0 / 64

    def loss(qq, kk, vv, ii):
        return float(np.sum(oracle.fwd(qq, kk, vv, lam, init=ii) * do))

    idx = [tuple(int(rng.integers(0, s)) for s in q.shape) for _ in range(40)]
    for grad, which in ((dq, 0), (dk, 1), (dv, 2)):
        for ix in idx:
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][ix] += h
            args_m[which][ix] -= h
            fd = (loss(*args_p, init) - loss(*args_m, init)) / (2 * h)
            assert abs(fd - grad[ix]) <= 1e-9 * max(1.0, abs(grad[ix])), (which, ix)
    for _ in range(10):
        ix = tuple(int(rng.integers(0, s)) for s in init.shape)
        ip, im = init.copy(), init.copy()
        ip[ix] += h
        im[ix] -= h
        fd = (loss(q, k, v, ip) - loss(q, k, v, im)) / (2 * h)
        assert abs(fd - dinit[ix]) <= 1e-9 * max(1.0, abs(dinit[ix]))


# ------------------------------------------------- chunk form (Algorithms 2-3)
def _chunk_form(q, k, v, do, lam, C):
    """Algorithms 2 and 3 of the LASP page, restated chunk by chunk in numpy.

    Page indices are 1-based: Lambda = diag(lambda^1..lambda^C), mask
    M_ij = lambda^(i-j) for i >= j.  KV_t is the state after chunk t, dKV_t
    the gradient state that includes chunk t (Algorithm 3 step 18).
    """
    B, N, H, d = q.shape
    T = N // C
    o, dq, dk, dv = (np.zeros((B, N, H, d)) for _ in range(4))
    for b in range(B):
        for h in range(H):
            l = 1.0 if lam is None else float(lam[h])
            Mask = _decay_mask(C, l)
            Lam = np.diag(l ** np.arange(1, C + 1.0))
            LamInvC = np.diag(l ** (C - np.arange(1, C + 1.0)))  # lambda^C Lambda^-1
            Qs, Ks, Vs, dOs = ([x[b, t * C:(t + 1) * C, h].astype(np.float64) for t in range(T)]
                               for x in (q, k, v, do))
            KV = [np.zeros((d, d))]  # KV[t] = state after t chunks
            for t in range(T):      # Algorithm 2
                intra = ((Qs[t] @ Ks[t].T) * Mask) @ Vs[t]          # step 9
                inter = Lam @ Qs[t] @ KV[t]                           # step 14
                o[b, t * C:(t + 1) * C, h] = intra + inter            # step 15
                KV.append(l ** C * KV[t] + (LamInvC @ Ks[t]).T @ Vs[t])  # step 16
            dKV = np.zeros((d, d))  # dKV_{t+1} while processing chunk t
            for t in reversed(range(T)):  # Algorithm 3
                dP = (dOs[t] @ Vs[t].T) * Mask
                dq_t = dP @ Ks[t] + Lam @ dOs[t] @ KV[t].T                      # steps 7, 8
                dk_t = dP.T @ Qs[t] + (LamInvC @ Vs[t]) @ dKV.T                  # steps 9, 14
                dv_t = ((Qs[t] @ Ks[t].T) * Mask).T @ dOs[t] + (LamInvC @ Ks[t]) @ dKV  # 10, 15
                dq[b, t * C:(t + 1) * C, h] = dq_t
                dk[b, t * C:(t + 1) * C, h] = dk_t
                dv[b, t * C:(t + 1) * C, h] = dv_t
                dKV = l ** C * dKV + (Lam @ Qs[t]).T @ dOs[t]                    # step 18
    return o, dq, dk, dv


@pytest.mark.parametrize("C", [1, 2, 8, 16, 48])
def test_recurrence_equals_chunk_form(C):
    q, k, v, do, lam = _problem(6, N=48)
    o = oracle.fwd(q, k, v, lam)
    dq, dk, dv = oracle.bwd(q, k, v, do, lam)
    co, cdq, cdk, cdv = _chunk_form(q, k, v, do, lam, C)
    for got, ref in ((o, co), (dq, cdq), (dk, cdk), (dv, cdv)):
        assert _rel(got, ref) < 1e-12


# ------------------------------------------------------ chunk states and scans
@pytest.mark.parametrize("C", [4, 16])
def test_chunk_states_undecayed_is_KtV(C):
    q, k, v, do, _ = _problem(7, N=32, decayed=False)
    M = oracle.chunk_states(k, v, None, C, kind=0)
    dM = oracle.chunk_states(q, do, None, C, kind=1)
    for c in range(32 // C):
        for h in range(q.shape[2]):
            Kc = k[0, c * C:(c + 1) * C, h].astype(np.float64)
            Vc = v[0, c * C:(c + 1) * C, h].astype(np.float64)
            assert _rel(M[0, c, h], Kc.T @ Vc) < 1e-13
            Qc = q[0, c * C:(c + 1) * C, h].astype(np.float64)
            dOc = do[0, c * C:(c + 1) * C, h].astype(np.float64)
            assert _rel(dM[0, c, h], Qc.T @ dOc) < 1e-13


def test_chunk_states_equal_recurrence_run_over_the_chunk():
    """M_c is the state after running Eq. 5 over chunk c from zero; dM_c is the
    gradient w.r.t. the state entering chunk c when the chunk runs alone."""
    q, k, v, do, lam = _problem(8, N=36)
    C = 12
    M = oracle.chunk_states(k, v, lam, C, kind=0)
    dM = oracle.chunk_states(q, do, lam, C, kind=1)
    for c in range(3):
        sl = slice(c * C, (c + 1) * C)
        qc, kc, vc, dc = (np.ascontiguousarray(x[:, sl]) for x in (q, k, v, do))
        _, fin = oracle.fwd(qc, kc, vc, lam, want_final=True)
        assert _rel(M[:, c], fin) < 1e-13
        zero = np.zeros_like(fin)
        *_, dinit = oracle.bwd(qc, kc, vc, dc, lam, init=zero, want_dinit=True)
        assert _rel(dM[:, c], dinit) < 1e-13


def test_state_scan_closed_forms():
    rng = np.random.default_rng(9)
    B, T, H, d, C = 2, 7, 3, 4, 5
    lam = np.array([1.0, 0.9, 0.5], np.float32)
    M = rng.standard_normal((B, T, H, d, d))
    P, tot = oracle.state_scan(M, lam, C)
    # lambda = 1: exclusive cumulative sum
    ex = np.concatenate([np.zeros_like(M[:, :1]), np.cumsum(M, axis=1)[:, :-1]], axis=1)
    assert _rel(P[:, :, 0], ex[:, :, 0]) < 1e-14
    assert _rel(tot[:, 0], M[:, :, 0].sum(axis=1)) < 1e-14
    # constant states: P_c = A (1 - g^c) / (1 - g), g = lambda^C
    A = rng.standard_normal((d, d))
    Mc = np.broadcast_to(A, (B, T, H, d, d)).copy()
    P2, _ = oracle.state_scan(Mc, lam, C)
    for h in (1, 2):
        g = float(lam[h]) ** C
        for c in range(T):
            assert _rel(P2[0, c, h], A * (1 - g ** c) / (1 - g)) < 1e-13 if c else not np.any(P2[0, 0, h])
    # reverse scan = forward scan of the reversed sequence of states
    R, rtot = oracle.state_scan(M, lam, C, reverse=True)
    Pr, ptot = oracle.state_scan(M[:, ::-1], lam, C)
    np.testing.assert_array_equal(R, Pr[:, ::-1])
    np.testing.assert_array_equal(rtot, ptot)
    # entering state: P_c gains lambda^(cC) * init
    init = rng.standard_normal((B, H, d, d))
    P3, _ = oracle.state_scan(M, lam, C, init=init)
    for h in range(H):
        for c in range(T):
            assert _rel(P3[:, c, h], P[:, c, h] + float(lam[h]) ** (C * c) * init[:, h]) < 1e-13


def test_scan_of_chunk_states_equals_recurrence_snapshots():
    """Two routes to the states the backward pass caches: Eq. 10 chunk states
    plus the LASP-2 prefix, against snapshots of the Eq. 5 recurrence; and the
    mirror for the gradient states (Eq. 20 + suffix vs. Eq. 13)."""
    q, k, v, do, lam = _problem(10, N=48)
    B, N, H, d = q.shape
    rng = np.random.default_rng(100)
    init = rng.standard_normal((B, H, d, d))
    F = rng.standard_normal((B, H, d, d))
    for C in (4, 16):
        P, tot = oracle.state_scan(oracle.chunk_states(k, v, lam, C, 0), lam, C, init=init)
        Ps = oracle.state_snapshots(k, v, lam, C, init=init, kind=0)
        assert _rel(P, Ps) < 1e-12
        _, fin = oracle.fwd(q, k, v, lam, init=init, want_final=True)
        assert _rel(tot, fin) < 1e-12
        R, rtot = oracle.state_scan(oracle.chunk_states(q, do, lam, C, 1), lam, C, init=F, reverse=True)
        Rs = oracle.state_snapshots(q, do, lam, C, init=F, kind=1)
        assert _rel(R, Rs) < 1e-12
        *_, dinit = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=F, want_dinit=True)
        assert _rel(rtot, dinit) < 1e-12


# ------------------------------------------------------------ shard invariance
@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_shard_decomposition_equals_unsplit(W):
    """LASP-2 on W virtual shards: shard states, a prefix (forward) or suffix
    (backward) over shards, then each shard's local pass with the entering
    state, equal the unsplit pass."""
    q, k, v, do, lam = _problem(11, B=1, N=64)
    B, N, H, d = q.shape
    L = N // W
    o = oracle.fwd(q, k, v, lam)
    dq, dk, dv = oracle.bwd(q, k, v, do, lam)
    E, _ = oracle.state_scan(oracle.chunk_states(k, v, lam, L, 0), lam, L)
    F, _ = oracle.state_scan(oracle.chunk_states(q, do, lam, L, 1), lam, L, reverse=True)
    for w in range(W):
        sl = slice(w * L, (w + 1) * L)
        qs, ks, vs, ds = (np.ascontiguousarray(x[:, sl]) for x in (q, k, v, do))
        ow = oracle.fwd(qs, ks, vs, lam, init=E[:, w])
        gw = oracle.bwd(qs, ks, vs, ds, lam, init=E[:, w], dstate_in=F[:, w])
        assert _rel(ow, o[:, sl]) < 1e-12
        for got, ref in zip(gw, (dq[:, sl], dk[:, sl], dv[:, sl])):
            assert _rel(got, ref) < 1e-12


def test_results_do_not_depend_on_thread_count():
    import subprocess
    import sys
    code = ("import numpy as np, oracle;"
            "r=np.random.default_rng(0);x=[r.standard_normal((1,64,2,40)).astype(np.float32) for _ in range(4)];"
            "lam=np.array([0.9,0.99],np.float32);"
            "o=oracle.fwd(*x[:3],lam);g=oracle.bwd(*x,lam);"
            "import hashlib;print(hashlib.sha256(b''.join(a.tobytes() for a in (o,)+g)).hexdigest())")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for n in ("1", "3"):
        env = dict(os.environ, OMP_NUM_THREADS=n, PYTHONPATH=root)
        outs.append(subprocess.run([sys.executable, "-c", code], env=env, check=True,
                                   capture_output=True, text=True).stdout.strip())
    assert outs[0] == outs[1]


# ------------------------------------------- bidirectional (unmasked) variant
def test_bidirectional_equals_left_product():
    """LASP Eq. 3: Q (K^T V) equals the left product (Q K^T) V, written with
    numpy matmuls in the other association; the gradients equal the textbook
    ones of the left product: dQ = dO V^T K, dK = (dO V^T)^T Q, dV = (Q K^T)^T dO."""
    q, k, v, do, _ = _problem(31, B=2, N=37, H=3, d=8, decayed=False)
    o, M = oracle.bidir_fwd(q, k, v, want_state=True)
    dq, dk, dv, dM = oracle.bidir_bwd(q, k, v, do, want_state=True)
    for b in range(2):
        for h in range(3):
            Q, K, V, D = (x[b, :, h, :].astype(np.float64) for x in (q, k, v, do))
            S, dP = Q @ K.T, D @ V.T
            assert _rel(o[b, :, h], S @ V) < 1e-13
            assert _rel(dq[b, :, h], dP @ K) < 1e-13
            assert _rel(dk[b, :, h], dP.T @ Q) < 1e-13
            assert _rel(dv[b, :, h], S.T @ D) < 1e-13
            assert _rel(M[b, h], K.T @ V) < 1e-13
            assert _rel(dM[b, h], Q.T @ D) < 1e-13


def test_bidirectional_is_causal_plus_anticausal_minus_diagonal():
    """Unmasked = the causal recurrence (lambda = 1) + the same recurrence run
    on the reversed sequence, minus the diagonal term counted twice; ties the
    bidirectional oracle to the token recurrence (LASP Eq. 4-6)."""
    q, k, v, do, _ = _problem(32, B=1, N=29, H=2, d=8, decayed=False)
    flip = lambda x: np.ascontiguousarray(x[:, ::-1])
    causal = oracle.fwd(q, k, v)
    anti = oracle.fwd(flip(q), flip(k), flip(v))[:, ::-1]
    diag = np.einsum("bnhi,bnhi->bnh", q.astype(np.float64), k.astype(np.float64))[..., None] * v
    assert _rel(oracle.bidir_fwd(q, k, v), causal + anti - diag) < 1e-12
    dq_c, dk_c, dv_c = oracle.bwd(q, k, v, do)
    dq_a, dk_a, dv_a = (g[:, ::-1] for g in oracle.bwd(flip(q), flip(k), flip(v), flip(do)))
    qd = q.astype(np.float64)
    kd, vd, dd = k.astype(np.float64), v.astype(np.float64), do.astype(np.float64)
    vdo = np.einsum("bnhi,bnhi->bnh", vd, dd)[..., None]   # diagonal term's gradients
    qk = np.einsum("bnhi,bnhi->bnh", qd, kd)[..., None]
    dq, dk, dv = oracle.bidir_bwd(q, k, v, do)
    assert _rel(dq, dq_c + dq_a - vdo * kd) < 1e-12
    assert _rel(dk, dk_c + dk_a - vdo * qd) < 1e-12
    assert _rel(dv, dv_c + dv_a - qk * dd) < 1e-12


def test_bidirectional_gradients_match_finite_differences():
    q, k, v, do, _ = _problem(33, B=1, N=20, H=2, d=6, decayed=False, quant=64)
    dq, dk, dv = oracle.bidir_bwd(q, k, v, do)
    h = 1.0 / 64
    rng = np.random.default_rng(34)

    def loss(qq, kk, vv):
        return float(np.sum(oracle.bidir_fwd(qq, kk, vv) * do))

    for grad, which in ((dq, 0), (dk, 1), (dv, 2)):
        for _ in range(30):
            ix = tuple(int(rng.integers(0, s)) for s in q.shape)
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][ix] += h
            args_m[which][ix] -= h
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[ix]) <= 1e-9 * max(1.0, abs(grad[ix])), (which, ix)
