"""Pins for the oracle's softmax attention (the standard attention layers a
hybrid model keeps; LASP-2 review page, "Summary": LASP-2H gathers K_t and V_t
for them): a hand-worked two-token example, torch's scaled-dot-product
attention in float64 with its autograd gradients (a library routine, with an
explicit mask for queries offset into the keys), the one-key and zero-query
closed forms, central differences, and the shard decomposition."""
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _rand(shape, seed, s=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * s).astype(np.float32)


def test_two_token_worked_example():
    q = np.array([1, 1], np.float32).reshape(1, 2, 1, 1)
    k = np.array([0, 1], np.float32).reshape(1, 2, 1, 1)
    v = np.array([1, 2], np.float32).reshape(1, 2, 1, 1)
    do = np.array([1, 1], np.float32).reshape(1, 2, 1, 1)
    o, lse = oracle.softmax_fwd(q, k, v, scale=1.0)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, scale=1.0)
    got = {"o": o.reshape(2), "lse": lse.reshape(2), "dq": dq.reshape(2), "dk": dk.reshape(2), "dv": dv.reshape(2)}
    n = 0
    with open(os.path.join(HERE, "golden", "softmax_two_token_example.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, t, val = line.split()
            assert got[name][int(t)] == pytest.approx(float(val), abs=1e-14), (name, t)
            n += 1
    assert n == 10


def _torch_reference(q, k, v, do, q_offset, scale):
    import torch
    t = lambda x: torch.from_numpy(x.astype(np.float64)).permute(0, 2, 1, 3).requires_grad_(True)
    Q, K, V = t(q), t(k), t(v)
    Nq, Nk = q.shape[1], k.shape[1]
    mask = (torch.arange(Nk)[None, :] <= (q_offset + torch.arange(Nq))[:, None])
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask, scale=scale)
    O.backward(torch.from_numpy(do.astype(np.float64)).permute(0, 2, 1, 3))
    s = torch.einsum("bhid,bhjd->bhij", Q.detach(), K.detach()) * scale
    lse = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
    back = lambda x: x.permute(0, 2, 1, 3).numpy()
    return back(O.detach()), lse.numpy(), back(Q.grad), back(K.grad), back(V.grad)


@pytest.mark.parametrize("B,H,Nq,Nk,q_offset,d,scale", [
    (2, 3, 37, 37, 0, 16, None), (1, 2, 20, 50, 30, 8, 0.7), (1, 1, 5, 64, 11, 32, None), (2, 1, 64, 64, 0, 128, None)])
def test_equals_torch_scaled_dot_product_attention(B, H, Nq, Nk, q_offset, d, scale):
    q, do = _rand((B, Nq, H, d), 1), _rand((B, Nq, H, d), 2)
    k, v = _rand((B, Nk, H, d), 3), _rand((B, Nk, H, d), 4)
    sc = d ** -0.5 if scale is None else scale
    ro, rlse, rdq, rdk, rdv = _torch_reference(q, k, v, do, q_offset, sc)
    o, lse = oracle.softmax_fwd(q, k, v, q_offset=q_offset, scale=scale)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, q_offset=q_offset, scale=scale)
    for got, ref in ((o, ro), (lse, rlse), (dq, rdq), (dk, rdk), (dv, rdv)):
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_one_key_closed_form():
    """One query, one key: the weight is 1, so o = v, lse = s, and only dv
    (= do) is non-zero."""
    q, k, v, do = (_rand((1, 1, 2, 8), s) for s in range(4))
    o, lse = oracle.softmax_fwd(q, k, v, scale=0.5)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, scale=0.5)
    np.testing.assert_allclose(o, v.astype(np.float64), rtol=0, atol=0)
    np.testing.assert_allclose(lse[0, :, 0], 0.5 * np.sum(q[0, 0] * k[0, 0].astype(np.float64), axis=-1), rtol=1e-14)
    assert not dq.any() and not dk.any()
    np.testing.assert_allclose(dv, do.astype(np.float64), rtol=0, atol=0)


def test_zero_queries_average_the_values():
    """q = 0: every visible key has the same weight, so o_i is the mean of
    v_0..v_{p_i}, lse_i = log(p_i + 1), dk = 0 and dv_j = sum_{i: p_i >= j} do_i / (p_i + 1)."""
    B, H, Nq, Nk, off, d = 1, 2, 9, 14, 5, 4
    q = np.zeros((B, Nq, H, d), np.float32)
    k, v, do = _rand((B, Nk, H, d), 5), _rand((B, Nk, H, d), 6), _rand((B, Nq, H, d), 7)
    o, lse = oracle.softmax_fwd(q, k, v, q_offset=off)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, q_offset=off)
    v64, do64 = v.astype(np.float64), do.astype(np.float64)
    for i in range(Nq):
        p = off + i
        np.testing.assert_allclose(o[:, i], v64[:, :p + 1].mean(axis=1), rtol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], np.log(p + 1.0), rtol=1e-14)
    assert not dk.any()
    ref_dv = np.zeros_like(dv)
    for i in range(Nq):
        ref_dv[:, :off + i + 1] += do64[:, i:i + 1] / (off + i + 1)
    np.testing.assert_allclose(dv, ref_dv, rtol=1e-13, atol=1e-15)


def test_central_differences():
    """dL/dx for L = sum(o * do), by central differences of the forward with
    exactly representable steps (2^-12) on float32 inputs."""
    B, H, Nq, Nk, off, d = 1, 1, 6, 9, 3, 4
    q, do = _rand((B, Nq, H, d), 8), _rand((B, Nq, H, d), 9)
    k, v = _rand((B, Nk, H, d), 10), _rand((B, Nk, H, d), 11)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do, q_offset=off, scale=0.8)
    L = lambda qq, kk, vv: float(np.sum(oracle.softmax_fwd(qq, kk, vv, q_offset=off, scale=0.8)[0] * do))
    h = 2.0 ** -12
    rng = np.random.default_rng(12)
    for x, g, name in ((q, dq, "q"), (k, dk, "k"), (v, dv, "v")):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in x.shape)
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": (xp, k, v), "k": (q, xp, v), "v": (q, k, xp)}[name]
            argm = {"q": (xm, k, v), "k": (q, xm, v), "v": (q, k, xm)}[name]
            fd = (L(*args) - L(*argm)) / (2 * h)
            assert fd == pytest.approx(g[idx], rel=1e-5, abs=1e-7), (name, idx)


def test_shards_equal_the_whole_sequence():
    """Rows of a query block at offset r L against the keys are the rows of
    the whole call, and the blocks' dk, dv add up to the whole call's."""
    B, H, W, L, d = 1, 2, 3, 7, 8
    N = W * L
    q, k, v, do = (_rand((B, N, H, d), 20 + s) for s in range(4))
    o, lse = oracle.softmax_fwd(q, k, v)
    dq, dk, dv = oracle.softmax_bwd(q, k, v, do)
    sdk, sdv = np.zeros_like(dk), np.zeros_like(dv)
    for r in range(W):
        sl = slice(r * L, (r + 1) * L)
        qs, dos = np.ascontiguousarray(q[:, sl]), np.ascontiguousarray(do[:, sl])
        o_r, lse_r = oracle.softmax_fwd(qs, k, v, q_offset=r * L)
        dq_r, dk_r, dv_r = oracle.softmax_bwd(qs, k, v, dos, q_offset=r * L)
        np.testing.assert_allclose(o_r, o[:, sl], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse_r, lse[:, :, sl], rtol=1e-13)
        np.testing.assert_allclose(dq_r, dq[:, sl], rtol=1e-12, atol=1e-14)
        assert not dk_r[:, (r + 1) * L:].any() and not dv_r[:, (r + 1) * L:].any()
        sdk += dk_r
        sdv += dv_r
    np.testing.assert_allclose(sdk, dk, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(sdv, dv, rtol=1e-12, atol=1e-14)
