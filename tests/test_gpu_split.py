"""lasp_fwd and lasp_bwd in the two parts that the LASP-2 exchange separates
(lasp_*_states, then lasp_*_finish): the parts together give exactly what the
whole call gives, on the tensor-core walk path and on the per-chunk path; the
totals they return are the oracle's final state (forward) and the gradient of
the initial state (backward), and zero for an empty sequence."""
import numpy as np
import pytest

import oracle
from gpu_helpers import decay_device, rel_err, to_device, to_host, tol
from sequence_linear_attention_b200 import inputs as lasp_inputs

pytestmark = pytest.mark.gpu

# (B, N, H, d, C, bf16): walk path at C = 128 and C = 64; per-chunk path (fp32)
CASES = [(2, 2048, 3, 128, 128, True), (1, 1024, 2, 128, 64, True), (1, 512, 2, 64, 64, False)]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}N{c[1]}H{c[2]}d{c[3]}C{c[4]}{'bf16' if c[5] else 'f32'}")
def test_parts_equal_the_whole_call(case):
    import torch
    import sequence_linear_attention_b200 as lasp
    B, N, H, d, C, bf16 = case
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=4100 + N, bf16=bf16, decayed=True)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    rng = np.random.default_rng(4200 + N)
    init = torch.from_numpy((rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)).cuda()
    dsin = torch.from_numpy((rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)).cuda()
    shape = (B, N // C, H, d, d)
    # whole calls
    o1, dq1, dk1, dv1 = (torch.empty_like(q) for _ in range(4))
    P1, R1 = torch.empty(shape, device="cuda"), torch.empty(shape, device="cuda")
    din1 = torch.empty((B, H, d, d), device="cuda")
    lasp.lasp_fwd(q, k, v, decay, o1, C, P1, init_state=init)
    lasp.lasp_bwd(q, k, v, decay, do, dq1, dk1, dv1, C, P1, R1, dstate_in=dsin, dinit_state=din1)
    # in parts
    o2, dq2, dk2, dv2 = (torch.empty_like(q) for _ in range(4))
    P2, R2 = torch.empty(shape, device="cuda"), torch.empty(shape, device="cuda")
    din2, tf, tb = (torch.empty((B, H, d, d), device="cuda") for _ in range(3))
    lasp.lasp_fwd_states(k, v, decay, C, P2, total=tf)
    lasp.lasp_fwd_finish(q, k, v, decay, o2, C, P2, init_state=init)
    lasp.lasp_bwd_states(q, do, decay, C, R2, total=tb)
    lasp.lasp_bwd_finish(q, k, v, decay, do, dq2, dk2, dv2, C, P2, R2, dstate_in=dsin, dinit_state=din2)
    st, _ = lasp.lasp_check_device_status()
    assert st == 0
    for a, b in ((o1, o2), (dq1, dq2), (dk1, dk2), (dv1, dv2), (din1, din2)):
        assert torch.equal(a, b)
    # the totals from a zero start: the final state, and the initial state's gradient
    f = {n: lasp_inputs.as_f32(inp[n], bf16) for n in ("q", "k", "v", "do")}
    _, final = oracle.fwd(f["q"], f["k"], f["v"], inp["lam"], want_final=True)
    *_, dinit = oracle.bwd(f["q"], f["k"], f["v"], f["do"], inp["lam"], want_dinit=True)
    assert rel_err(to_host(tf), final) <= tol(bf16)
    assert rel_err(to_host(tb), dinit) <= tol(bf16)


def test_empty_sequence_gives_zero_totals():
    import torch
    import sequence_linear_attention_b200 as lasp
    B, H, d, C = 2, 3, 128, 128
    x = torch.empty((B, 0, H, d), dtype=torch.bfloat16, device="cuda")
    cache = torch.empty(0, device="cuda")
    tf = torch.full((B, H, d, d), 7.0, device="cuda")
    tb = torch.full((B, H, d, d), 7.0, device="cuda")
    lasp.lasp_fwd_states(x, x, None, C, cache, total=tf)
    lasp.lasp_bwd_states(x, x, None, C, cache, total=tb)
    st, _ = lasp.lasp_check_device_status()
    assert st == 0
    assert not torch.any(tf) and not torch.any(tb)


@pytest.mark.parametrize("nparts", [2, 3, 6])
def test_pair_parts_equal_the_whole_call(nparts):
    """The four split calls restricted to parts of the (b, h) pairs (b-major),
    run part after part as LASP-2's overlapped exchange runs them, give the
    whole calls' results bit for bit, totals included."""
    import torch
    import sequence_linear_attention_b200 as lasp
    B, N, H, d, C = 2, 2048, 3, 128, 128
    assert lasp.lasp_parts_ok(N, C, d, lasp.LASP_BF16) == 1
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=4300, bf16=True, decayed=True)
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    rng = np.random.default_rng(4301)
    init = torch.from_numpy((rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)).cuda()
    dsin = torch.from_numpy((rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)).cuda()
    shape = (B, N // C, H, d, d)
    res = []
    for parts in (1, nparts):
        o, dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(4))
        P, R = torch.empty(shape, device="cuda"), torch.empty(shape, device="cuda")
        tf, tb, din = (torch.full((B, H, d, d), float("nan"), device="cuda") for _ in range(3))
        for p in range(parts):
            lasp.lasp_fwd_states_part(k, v, decay, C, P, tf, p, parts)
        for p in range(parts):
            lasp.lasp_fwd_finish_part(q, k, v, decay, o, C, P, init, p, parts)
        for p in range(parts):
            lasp.lasp_bwd_states_part(q, do, decay, C, R, tb, p, parts)
        for p in range(parts):
            lasp.lasp_bwd_finish_part(q, k, v, decay, do, dq, dk, dv, C, P, R, dsin, din, p, parts)
        st, _ = lasp.lasp_check_device_status()
        assert st == 0
        res.append((o, dq, dk, dv, tf, tb, din))
    for a, b in zip(*res):
        assert torch.equal(a, b)
    # parts beyond the pairs, or on sizes the walks do not take, are refused
    with pytest.raises(lasp.LaspError):
        lasp.lasp_fwd_states_part(k, v, decay, C, P, tf, 0, B * H + 1)
    q32 = torch.zeros((1, 256, 2, 64), device="cuda")
    with pytest.raises(lasp.LaspError) as e:
        lasp.lasp_fwd_states_part(q32, q32, None, 64, torch.empty((1, 4, 2, 64, 64), device="cuda"), None, 0, 2)
    assert e.value.status == 2
