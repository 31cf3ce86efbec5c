"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs. Metric per tensor: max|gpu - ref| / max|ref|;
bar 1e-4 for fp32 inputs, 2e-2 for bf16 inputs with fp32 accumulation."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import (decay_device, host_f32, rel_err, run_fwd_bwd, run_states, to_device, to_host, tol)

pytestmark = pytest.mark.gpu


def _oracle_all(inp, C, init=None, dstate_in=None):
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    lam = inp["lam"]
    o = oracle.fwd(q, k, v, lam, init=init)
    dq, dk, dv, dinit = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=dstate_in, want_dinit=True)
    P = oracle.state_snapshots(k, v, lam, C, init=init, kind=0)
    R = oracle.state_snapshots(q, do, lam, C, init=dstate_in, kind=1)
    return dict(o=o, dq=dq, dk=dk, dv=dv, P=P, R=R, dinit=dinit)


def _compare(gpu, ref, bf16, names=("o", "dq", "dk", "dv")):
    errs = {n: rel_err(to_host(gpu[n]), ref[n]) for n in names}
    bad = {n: e for n, e in errs.items() if not e <= tol(bf16)}
    assert not bad, f"errors above {tol(bf16)}: {bad} (all: {errs})"
    return errs


SMALL = [
    # (B, H, N, d, C, bf16, decayed)
    (1, 2, 256, 32, 64, False, False),   # the tiny fp32 workload
    (1, 2, 256, 32, 64, False, True),
    (2, 3, 256, 128, 128, False, True),  # fp32, d = 128
    (2, 3, 384, 128, 128, True, True),   # several 128-token tiles
    (1, 4, 320, 128, 64, True, True),    # N not a multiple of 128
    (3, 5, 256, 128, 32, True, False),   # odd B and H
    (1, 2, 192, 128, 16, True, True),
    (2, 2, 224, 64, 32, True, True),     # d = 64 (per-chunk tensor-core kernels, ragged tile)
    (2, 3, 640, 64, 128, True, True),    # d = 64, several tiles
    (1, 2, 512, 64, 64, True, False),    # d = 64, two chunks per tile
    (1, 2, 512, 64, 256, True, True),    # d = 64, chunks of two tiles (tensor-core states only)
    (1, 3, 96, 32, 16, True, True),      # d = 32 (per-chunk tensor-core kernels, ragged tile)
    (2, 2, 384, 32, 64, True, True),     # d = 32, several tiles
    (1, 3, 256, 32, 128, True, False),
    (1, 2, 96, 64, 24, True, True),      # C not a multiple of 16
    (1, 2, 128, 128, 128, True, True),   # a single chunk
    (2, 2, 64, 64, 1, False, True),      # C = 1: pure inter-chunk
    (1, 2, 2048, 128, 128, True, True),  # forward walk over two 1024-token segments
    (2, 3, 1536, 128, 256, True, True),  # chunks of two tiles (both walks)
    (1, 2, 2048, 128, 256, True, False),  # two 1024-token segments of four such chunks
    (1, 2, 1024, 128, 512, True, False),
    (2, 150, 1024, 128, 128, True, True),  # more segments than SMs: each CTA walks several
    (2, 3, 1152, 128, 128, True, True),    # three segments of three tiles
    (1, 4, 2048, 128, 128, True, False),   # walks without decay
    (1, 3, 2048, 128, 64, True, True),     # walks with chunks that divide the tile
    (2, 2, 1280, 128, 32, True, True),
    (1, 2, 384, 128, 16, True, False),
]


@pytest.mark.parametrize("B,H,N,d,C,bf16,decayed", SMALL)
def test_small_shapes_against_oracle(B, H, N, d, C, bf16, decayed):
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=7 + N + d + C, bf16=bf16, decayed=decayed)
    gpu = run_fwd_bwd(inp, C)
    ref = _oracle_all(inp, C)
    _compare(gpu, ref, bf16)
    # the chunk-entering states P_c and R_c, through the state entry points
    _compare(run_states(inp, C, gpu["P"], gpu["R"]), ref, bf16, names=("P", "R"))


@pytest.mark.parametrize("bf16,N,C", [(False, 256, 64), (True, 256, 64), (True, 2048, 128)])
def test_entering_states_against_oracle(bf16, N, C):
    """init_state (the forward state entering token 0) and dstate_in (the
    gradient state entering from beyond the end), plus dinit_state."""
    B, H, d = 2, 3, 128 if bf16 else 32
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=77, bf16=bf16, decayed=True)
    rng = np.random.default_rng(78)
    init = (rng.standard_normal((B, H, d, d)) * 0.2).astype(np.float32)
    din = (rng.standard_normal((B, H, d, d)) * 0.2).astype(np.float32)
    gpu = run_fwd_bwd(inp, C, init=init, dstate_in=din, want_dinit=True)
    ref = _oracle_all(inp, C, init=init.astype(np.float64), dstate_in=din.astype(np.float64))
    _compare(gpu, ref, bf16, names=("o", "dq", "dk", "dv", "dinit"))
    _compare(run_states(inp, C, gpu["P"], gpu["R"], init=init, dstate_in=din), ref, bf16, names=("P", "R"))


def test_chunk_size_invariance():
    """The output does not depend on the chunk size (it is a regrouping of the
    same sums, LASP Eq. 8 and Eq. 10)."""
    inp = lasp_inputs.make_inputs(1, 512, 4, 128, seed=91, bf16=True, decayed=True)
    b = run_fwd_bwd(inp, 128)
    for C in (32, 64, 256):  # walks with chunks inside a tile; forward walk + per-chunk backward
        a = run_fwd_bwd(inp, C)
        for n in ("o", "dq", "dk", "dv"):
            assert rel_err(to_host(a[n]), to_host(b[n]).astype(np.float64)) <= tol(True), (C, n)


def test_no_decay_equals_all_ones_bitwise():
    import torch
    inp = lasp_inputs.make_inputs(1, 256, 2, 128, seed=92, bf16=True, decayed=False)
    a = run_fwd_bwd(inp, 64, decay_override=None)
    b = run_fwd_bwd(inp, 64, decay_override=np.ones(2, np.float32))
    for n in ("o", "dq", "dk", "dv"):
        assert torch.equal(a[n], b[n]), n


def test_state_entry_points_against_oracle():
    """lasp_chunk_states, lasp_chunk_dstates and lasp_state_prefix on their own."""
    import torch
    import sequence_linear_attention_b200 as lasp
    B, H, N, d, C = 2, 3, 512, 128, 128
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=93, bf16=True, decayed=True)
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    T = N // C
    M = torch.empty((B, T, H, d, d), dtype=torch.float32, device="cuda")
    dM = torch.empty_like(M)
    lasp.lasp_chunk_states(None, k, v, decay, M, C)
    lasp.lasp_chunk_dstates(q, do, decay, dM, C)
    kf, vf, qf, df = (host_f32(inp, n) for n in ("k", "v", "q", "do"))
    assert rel_err(to_host(M), oracle.chunk_states(kf, vf, inp["lam"], C, 0)) <= tol(True)
    assert rel_err(to_host(dM), oracle.chunk_states(qf, df, inp["lam"], C, 1)) <= tol(True)
    # the scan alone, on fp32 states: out of place and in place, both directions
    rng = np.random.default_rng(94)
    Mh = rng.standard_normal((B, 37, H, d, d)).astype(np.float32)
    init = rng.standard_normal((B, H, d, d)).astype(np.float32)
    for reverse in (False, True):
        for Cs in (128, 32768):
            Md = torch.from_numpy(Mh).cuda()
            P = torch.empty_like(Md)
            tot = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
            lasp.lasp_state_prefix(Md, P, decay, Cs, init=torch.from_numpy(init).cuda(), total=tot,
                                   reverse=reverse)
            rP, rtot = oracle.state_scan(Mh, inp["lam"], Cs, init=init, reverse=reverse)
            assert rel_err(to_host(P), rP) <= tol(False)
            assert rel_err(to_host(tot), rtot) <= tol(False)
            lasp.lasp_state_prefix(Md, Md, decay, Cs, reverse=reverse)  # in place, no init
            rP0, _ = oracle.state_scan(Mh, inp["lam"], Cs, reverse=reverse)
            assert rel_err(to_host(Md), rP0) <= tol(False)
    st, _ = lasp.lasp_check_device_status()
    assert st == 0


def test_outputs_stay_inside_their_buffers():
    """Guard regions around every output, the state cache and the workspace
    keep their sentinel bytes; every output element is written."""
    import torch
    import sequence_linear_attention_b200 as lasp
    B, H, N, d, C = 1, 3, 320, 128, 64
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=95, bf16=True, decayed=True)
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    G = 4096  # guard elements on each side (8 KiB of bf16, 16 KiB of fp32)

    def guarded(n, dtype):
        buf = torch.full((n + 2 * G,), float("nan"), dtype=dtype, device="cuda")
        return buf, buf[G:G + n]

    n_tok, n_st = B * N * H * d, B * (N // C) * H * d * d
    bufs = {}
    for name in ("o", "dq", "dk", "dv"):
        bufs[name] = guarded(n_tok, torch.bfloat16)
    for name in ("P", "R"):
        bufs[name] = guarded(n_st, torch.float32)
    view = {n: b[1].view(B, N, H, d) if n in ("o", "dq", "dk", "dv") else b[1].view(B, N // C, H, d, d)
            for n, b in bufs.items()}
    lasp.lasp_fwd(q, k, v, decay, view["o"], C, view["P"])
    lasp.lasp_bwd(q, k, v, decay, do, view["dq"], view["dk"], view["dv"], C, view["P"], view["R"])
    torch.cuda.synchronize()
    for name, (buf, _) in bufs.items():
        assert torch.isnan(buf[:G]).all() and torch.isnan(buf[-G:]).all(), name
        if name in ("o", "dq", "dk", "dv"):
            assert not torch.isnan(buf[G:-G]).any(), name


def test_invalid_decay_is_recorded():
    import torch
    import sequence_linear_attention_b200 as lasp
    inp = lasp_inputs.make_inputs(1, 128, 2, 64, seed=96, bf16=True, decayed=False)
    k, v = to_device(inp["k"], True), to_device(inp["v"], True)
    M = torch.empty((1, 1, 2, 64, 64), dtype=torch.float32, device="cuda")
    bad = torch.tensor([0.5, 1.5], dtype=torch.float32, device="cuda")
    lasp.lasp_chunk_states(None, k, v, bad, M, 128)
    st, site = lasp.lasp_check_device_status()
    assert st == 1 and site == 1  # LASP_ERR_INVALID_ARG at the decay check
    assert lasp.lasp_check_device_status()[0] == 0  # reading clears it


def test_wait_that_runs_out_reports_timeout():
    """A barrier nobody arrives on: the bounded wait gives up, records
    LASP_ERR_TIMEOUT, and the context stays usable."""
    import torch
    import sequence_linear_attention_b200 as lasp
    lasp.lasp_set_wait_limit_ns(2_000_000)  # 2 ms
    try:
        lasp.lasp_wait_probe()
        st, site = lasp.lasp_check_device_status()
    finally:
        lasp.lasp_set_wait_limit_ns(2_000_000_000)
    assert st == 5 and site == 2
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum()) == 8.0  # the context still works
