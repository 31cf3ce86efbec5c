"""The gated form (a decay per token and key feature; LASP Appendix A.4, Eq. 24
with the GLA / GateLoop row of Table 5) through the C ABI against the oracle:
o, dq, dk, dv, dg, dinit, and the rows on their own (chunk states with their
log-gate totals, the diagonal-decay scans). Tolerance max|gpu - ref| / max|ref|
<= 1e-4 for fp32 inputs and 2e-2 for bf16 inputs (fp32 accumulation)."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import TOL_BF16, TOL_F32, host_f32, rel_err, to_device, to_host

pytestmark = pytest.mark.gpu


def _gates_device(g):
    import torch
    return torch.from_numpy(np.ascontiguousarray(g, np.float32)).cuda()


def _f32_device(x):
    import torch
    return None if x is None else torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda()


def _run(inp, g, C, init=None, dstate_in=None):
    import torch
    import sequence_linear_attention_b200 as lasp
    bf16 = inp["bf16"]
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    B, N, H, d = q.shape
    gd = _gates_device(g)
    cache = torch.empty(lasp.lasp_gla_cache_floats(B, H, N, d, C), dtype=torch.float32, device="cuda")
    ws = torch.empty(B * (N // C) * H * d * d, dtype=torch.float32, device="cuda")
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    dg = torch.empty_like(gd)
    dinit = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    init_t, din_t = _f32_device(init), _f32_device(dstate_in)
    lasp.lasp_gla_fwd(q, k, v, gd, o, C, cache, init_state=init_t)
    lasp.lasp_gla_bwd(q, k, v, gd, do, dq, dk, dv, dg, C, cache, ws, dstate_in=din_t, dinit_state=dinit)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    return dict(o=to_host(o), dq=to_host(dq), dk=to_host(dk), dv=to_host(dv), dg=dg.cpu().numpy(),
                dinit=dinit.cpu().numpy())


def _reference(inp, g, init=None, dstate_in=None):
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    o = oracle.gla_fwd(q, k, v, g, init=init)
    dq, dk, dv, dg, dinit = oracle.gla_bwd(q, k, v, g, do, init=init, dstate_in=dstate_in, want_dinit=True)
    return dict(o=o, dq=dq, dk=dk, dv=dv, dg=dg, dinit=dinit)


def _compare(got, ref, tol, keys=("o", "dq", "dk", "dv", "dg", "dinit")):
    errs = {n: rel_err(got[n], ref[n]) for n in keys}
    assert all(np.isfinite(list(errs.values()))), errs
    bad = {n: e for n, e in errs.items() if e > tol}
    assert not bad, errs


CASES = [
    # (B, N, H, d, C, bf16, tau, seed): several chunks each, a ragged chunk
    # count, the largest chunk, strong gates (tau = 1) and mild ones
    (1, 256, 2, 32, 16, False, 16.0, 2001),
    (2, 384, 2, 64, 128, False, 4.0, 2002),
    (1, 320, 3, 128, 64, False, 1.0, 2003),
    (2, 1024, 2, 128, 64, True, 16.0, 2004),
    (1, 640, 2, 128, 128, True, 2.0, 2005),
    (1, 192, 2, 128, 32, True, 1.0, 2006),
]


@pytest.mark.parametrize("B,N,H,d,C,bf16,tau,seed", CASES)
def test_gated_matches_oracle(B, N, H, d, C, bf16, tau, seed):
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=seed, bf16=bf16, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=seed, tau=tau)
    rng = np.random.default_rng(seed)
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got = _run(inp, g, C, init=init, dstate_in=dsin)
    ref = _reference(inp, g, init=init.astype(np.float64), dstate_in=dsin.astype(np.float64))
    _compare(got, ref, TOL_BF16 if bf16 else TOL_F32)


@pytest.mark.parametrize("bf16", [False, True])
def test_gated_without_boundary_states(bf16):
    B, N, H, d, C = 1, 512, 2, 128, 64
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2010, bf16=bf16, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2010)
    _compare(_run(inp, g, C), _reference(inp, g), TOL_BF16 if bf16 else TOL_F32)


def test_zero_gates_are_plain_linear_attention():
    """Log-gate 0 everywhere: the undecayed lasp_fwd / lasp_bwd path (a separate
    implementation) and the oracle agree with the gated path."""
    B, N, H, d, C = 1, 256, 2, 64, 64
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2011, bf16=False, decayed=False)
    g = np.zeros((B, N, H, d), np.float32)
    got = _run(inp, g, C)
    ref = _reference(inp, g)
    _compare(got, ref, TOL_F32)
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    assert rel_err(got["o"], oracle.fwd(q, k, v)) <= TOL_F32
    assert np.max(np.abs(got["dg"])) > 0


def test_constant_gate_matches_the_decayed_path():
    """g = log(lambda_h) per head is the decayed form of section 3.2: the gated
    path agrees with lasp_fwd / lasp_bwd run with that decay."""
    from gpu_helpers import run_fwd_bwd
    B, N, H, d, C = 1, 512, 4, 128, 64
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2012, bf16=False, decayed=True)
    lam = inp["lam"]
    g = np.ascontiguousarray(np.broadcast_to(np.log(lam)[None, None, :, None], (B, N, H, d)), dtype=np.float32)
    got = _run(inp, g, C)
    dec = run_fwd_bwd(inp, C)
    for n in ("o", "dq", "dk", "dv"):
        assert rel_err(got[n], to_host(dec[n])) <= TOL_F32, n


def test_strong_gates_forget_the_past():
    """Gates of about e^-30 per token: every state is negligible, so o_t is
    q_t (k_t^T v_t) up to e^-30 and nothing overflows or turns into NaN."""
    B, N, H, d, C = 1, 256, 2, 64, 64
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2013, bf16=False, decayed=False)
    g = np.full((B, N, H, d), -30.0, np.float32)
    got = _run(inp, g, C)
    ref = _reference(inp, g)
    _compare(got, ref, TOL_F32)
    q, k, v = (host_f32(inp, n) for n in ("q", "k", "v"))
    local = np.einsum("bnhi,bnhi->bnh", q.astype(np.float64), k)[..., None] * v
    assert rel_err(got["o"], local) <= TOL_F32


@pytest.mark.parametrize("C", [16, 32, 128])
def test_output_does_not_depend_on_chunk_size(C):
    B, N, H, d = 1, 512, 2, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2014, bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2014, tau=4.0)
    a, b = _run(inp, g, 64), _run(inp, g, C)
    for n in ("o", "dq", "dk", "dv", "dg"):
        assert rel_err(b[n], a[n]) <= TOL_BF16, n


@pytest.mark.parametrize("bf16", [False, True])
def test_rows_chunk_states_and_scans(bf16):
    """a1 / a4 / a2 / a5 of the gated form on their own: lasp_gla_chunk_states
    (both kinds, with the log-gate totals) and lasp_gla_state_prefix (both
    directions, with init and total) against the oracle's definitions."""
    import torch
    import sequence_linear_attention_b200 as lasp
    B, N, H, d, C = 2, 256, 2, 64, 32
    T = N // C
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2015, bf16=bf16, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2015, tau=2.0)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    gd = _gates_device(g)
    M = torch.empty((B, T, H, d, d), dtype=torch.float32, device="cuda")
    dM = torch.empty_like(M)
    gs = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    lasp.lasp_gla_chunk_states(k, v, gd, M, C, gsum=gs, kind=0)
    lasp.lasp_gla_chunk_states(q, do, gd, dM, C, kind=1)
    rng = np.random.default_rng(2015)
    init = rng.standard_normal((B, H, d, d)).astype(np.float32)
    P, R = torch.empty_like(M), torch.empty_like(M)
    tot, rtot = (torch.empty((B, H, d, d), dtype=torch.float32, device="cuda") for _ in range(2))
    lasp.lasp_gla_state_prefix(M, P, gs, init=_f32_device(init), total=tot)
    lasp.lasp_gla_state_prefix(dM, R, gs, init=_f32_device(init), total=rtot, reverse=True)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    qh, kh, vh, doh = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    M_ref, gs_ref = oracle.gla_chunk_states(kh, vh, g, C, kind=0)
    dM_ref, _ = oracle.gla_chunk_states(qh, doh, g, C, kind=1)
    tol = TOL_F32  # the states are fp32 sums of exact products either way
    assert rel_err(M.cpu().numpy(), M_ref) <= tol
    assert rel_err(dM.cpu().numpy(), dM_ref) <= tol
    assert rel_err(gs.cpu().numpy(), gs_ref) <= 1e-6
    P_ref, tot_ref = oracle.gla_state_scan(M_ref, gs_ref, init=init.astype(np.float64))
    R_ref, rtot_ref = oracle.gla_state_scan(dM_ref, gs_ref, init=init.astype(np.float64), reverse=True)
    for got, ref in ((P, P_ref), (tot, tot_ref), (R, R_ref), (rtot, rtot_ref)):
        assert rel_err(got.cpu().numpy(), ref) <= tol


# ------------------------------------------------ tensor-core path (bf16, d = 128, C = 128)
# the forward walks segments of up to 8 tiles: 1024 and 2048 tokens give 8-tile
# segments (one and two per head), 512 one 4-tile segment, 1152 three 3-tile
# segments, 1408 (11 tiles) eleven one-tile segments
@pytest.mark.parametrize("B,N,H,tau,seed", [(2, 1024, 2, 16.0, 2020), (1, 512, 3, 1.0, 2021), (1, 2048, 1, 4.0, 2022),
                                            (1, 1152, 2, 4.0, 2023), (2, 1408, 1, 2.0, 2024)])
def test_tensor_core_path_matches_oracle(B, N, H, tau, seed):
    d, C = 128, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=seed, bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=seed, tau=tau)
    rng = np.random.default_rng(seed)
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got = _run(inp, g, C, init=init, dstate_in=dsin)
    ref = _reference(inp, g, init=init.astype(np.float64), dstate_in=dsin.astype(np.float64))
    _compare(got, ref, TOL_BF16)


def test_tensor_core_path_with_more_segments_than_sms():
    """150 one-segment heads: the first CTAs walk a second segment after their
    first, so the backward's walk passes from a segment's first tile to the
    next segment's last (whose entering state comes from the scan again)."""
    B, N, H, d, C = 1, 1024, 150, 128, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2025, bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2025, tau=4.0)
    rng = np.random.default_rng(2025)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got = _run(inp, g, C, dstate_in=dsin)
    ref = _reference(inp, g, dstate_in=dsin.astype(np.float64))
    _compare(got, ref, TOL_BF16)


def test_tensor_core_rows_match_oracle():
    _rows_states(True, 128, 128)


def _rows_states(bf16, C, d):
    import torch
    import sequence_linear_attention_b200 as lasp
    B, N, H = 2, 512, 2
    T = N // C
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2023, bf16=bf16, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2023, tau=2.0)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    gd = _gates_device(g)
    M = torch.empty((B, T, H, d, d), dtype=torch.float32, device="cuda")
    dM = torch.empty_like(M)
    gs = torch.empty((B, T, H, d), dtype=torch.float32, device="cuda")
    lasp.lasp_gla_chunk_states(k, v, gd, M, C, gsum=gs, kind=0)
    lasp.lasp_gla_chunk_states(q, do, gd, dM, C, kind=1)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    qh, kh, vh, doh = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    M_ref, gs_ref = oracle.gla_chunk_states(kh, vh, g, C, kind=0)
    dM_ref, _ = oracle.gla_chunk_states(qh, doh, g, C, kind=1)
    # the tensor-core states round the gate-weighted operand to bf16
    assert rel_err(M.cpu().numpy(), M_ref) <= TOL_BF16
    assert rel_err(dM.cpu().numpy(), dM_ref) <= TOL_BF16
    assert rel_err(gs.cpu().numpy(), gs_ref) <= 1e-5


def _strong_gates(kind, B, N, H, d, seed):
    if kind == "const_ln0.1":
        return np.full((B, N, H, d), np.log(0.1), np.float32)
    if kind == "logsig_tau1":
        return lasp_inputs.make_log_gates(B, N, H, d, seed=seed, tau=1.0)
    # mild gates everywhere but one 128-token tile of the last head, whose
    # log-gates are -3 per token
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=seed, tau=16.0)
    g[:, 256:384, H - 1, :] = -3.0
    return g


@pytest.mark.parametrize("kind", ["const_ln0.1", "logsig_tau1", "one_tile"])
@pytest.mark.parametrize("C", [128, 64])
def test_tensor_core_call_with_strong_gates_matches_oracle(kind, C):
    """bf16 with d = 128 takes the tensor-core path, whose factorized intra-tile
    form holds while each half-tile's |log-gates| sum to at most 79. Constant
    gates of 0.1 (64 ln 0.1 = -147 per half-tile), log sigmoid(x) gates at
    tau = 1 and a single strong tile go beyond that: the forward's state
    kernel sees it and the call and its backward run the exact CUDA-core
    kernels instead. The results match the oracle and no status is recorded
    (LASP Appendix A.4, Eq. 24 defines these inputs like any other)."""
    B, N, H, d = 1, 512, 2, 128
    seed = 2040 + C
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=seed, bf16=True, decayed=False)
    g = _strong_gates(kind, B, N, H, d, seed)
    rng = np.random.default_rng(seed)
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got = _run(inp, g, C, init=init, dstate_in=dsin)  # asserts a clean device status
    ref = _reference(inp, g, init=init.astype(np.float64), dstate_in=dsin.astype(np.float64))
    _compare(got, ref, TOL_BF16)


def test_mild_gates_leave_the_exact_kernels_idle():
    """With gates inside the factorized range the exact CUDA-core kernels a
    tensor-core call also launches return at once: each takes a small part of
    the tensor-core kernel it stands in for."""
    import sequence_linear_attention_b200 as lasp
    B, N, H, d, C = 1, 4096, 4, 128, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2050, bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2050, tau=16.0)
    _run(inp, g, C)
    lasp.lasp_trace_enable(64)
    try:
        _run(inp, g, C)
        trace = lasp.lasp_trace_read(64)
    finally:
        lasp.lasp_trace_enable(0)
    ms = dict(trace)
    names = [n for n, _ in trace]
    assert names == ["gla_segment_states_tc", "gla_segment_scan", "gla_out_tc", "gla_states_exact",
                     "gla_scan_exact", "gla_out_exact", "gla_segment_states_tc", "gla_segment_scan", "gla_bwd_tc",
                     "gla_states_exact", "gla_scan_exact", "gla_bwd_exact"], names
    assert ms["gla_out_exact"] < 0.5 * ms["gla_out_tc"], trace
    assert ms["gla_bwd_exact"] < 0.5 * ms["gla_bwd_tc"], trace


@pytest.mark.parametrize("C", [16, 32, 64])
def test_tensor_core_path_chunks_dividing_the_tile(C):
    """C < 128 on the tensor cores: 128-token tiles span 128/C chunks, with the
    states at tile boundaries only (in the slots of the tiles' first and last
    chunks); against the oracle with entering states and dstate_in."""
    B, N, H, d = 1, 768, 2, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=2030 + C, bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=2030 + C, tau=4.0)
    rng = np.random.default_rng(C)
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    got = _run(inp, g, C, init=init, dstate_in=dsin)
    ref = _reference(inp, g, init=init.astype(np.float64), dstate_in=dsin.astype(np.float64))
    _compare(got, ref, TOL_BF16)


def test_bench_size_sampled_heads():
    """The gated bench configuration (B1 H16 N65536 d128 C128, bf16, gates
    log(sigmoid(x))/16) run on the GPU as bench.py times it; two whole heads
    (every position) of o, dq, dk, dv and dg against the oracle."""
    import torch
    import sequence_linear_attention_b200 as lasp
    w = lasp_inputs.WORKLOADS["decayed_bf16_N64K"]
    B, N, H, d, C = w["B"], w["N"], w["H"], w["d"], 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=w["seed"], bf16=True, decayed=False)
    g = lasp_inputs.make_log_gates(B, N, H, d, seed=w["seed"])
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    gd = _gates_device(g)
    cache = torch.empty(lasp.lasp_gla_cache_floats(B, H, N, d, C), dtype=torch.float32, device="cuda")
    ws = torch.empty(B * (N // C) * H * d * d, dtype=torch.float32, device="cuda")
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    dg = torch.empty_like(gd)
    lasp.lasp_gla_fwd(q, k, v, gd, o, C, cache)
    lasp.lasp_gla_bwd(q, k, v, gd, do, dq, dk, dv, dg, C, cache, ws)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    heads = [3, 14]
    got = {n: to_host(t)[:, :, heads] for n, t in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv))}
    got["dg"] = dg.cpu().numpy()[:, :, heads]
    sub = lambda x: np.ascontiguousarray(x[:, :, heads])
    qh, kh, vh, doh = (sub(host_f32(inp, n)) for n in ("q", "k", "v", "do"))
    gh = sub(g)
    ref = {"o": oracle.gla_fwd(qh, kh, vh, gh)}
    ref["dq"], ref["dk"], ref["dv"], ref["dg"] = oracle.gla_bwd(qh, kh, vh, gh, doh)
    _compare(got, ref, TOL_BF16, keys=("o", "dq", "dk", "dv", "dg"))
