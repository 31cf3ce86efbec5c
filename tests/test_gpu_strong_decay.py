"""GPU parity at strong decays: lambda_h in {0.5, 0.1, 1e-3} and a mixed
per-head array [1, 0.99, 0.5, 1e-3], on every ungated path.

The method takes lambda as any predefined constant (LASP paper, section 3.2,
after Eq. 5); the workloads' own rates start at 0.96875, where no decay power
underflows. Here lambda^{127-j}, lambda^128 and lambda^{i+1} reach zero
inside one tile, and the walks' mask weights, built by a running product,
run down to zero with them. Each case is compared with the fp64 oracle on the
same seeded inputs, per tensor, max|gpu - ref| / max|ref| <= 2e-2 (bf16) or
1e-4 (fp32)."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import decay_device, host_f32, rel_err, run_fwd_bwd, run_states, to_device, to_host, tol

pytestmark = pytest.mark.gpu

LAMBDAS = {
    "0.5": [0.5] * 4,
    "0.1": [0.1] * 4,
    "1e-3": [1e-3] * 4,
    "mixed": [1.0, 0.99, 0.5, 1e-3],
}

# (B, N, d, C, bf16): which kernels each shape takes (asserted in test_gpu_paths.py)
PATHS = {
    "walks_C128": (1, 2048, 128, 128, True),   # segment walks, two 1024-token segments
    "walks_C64": (2, 1024, 128, 64, True),     # walks with chunks that divide the tile
    "per_chunk_tc": (1, 320, 128, 64, True),   # ragged tile: per-chunk tensor-core kernels
    "per_chunk_tc_d64": (1, 384, 64, 128, True),  # d = 64 on the per-chunk tensor-core kernels
    "per_chunk_tc_d32": (1, 256, 32, 64, True),   # d = 32 on the per-chunk tensor-core kernels
    "simt_f32_d64": (1, 256, 64, 64, False),   # CUDA cores, fp32
    "bf16_C256": (1, 1024, 128, 256, True),    # walks with chunks of two tiles
    "bf16_C512": (1, 1024, 128, 512, True),    # forward walk, CUDA-core backward
}


def _inputs(path, lam_name, seed):
    B, N, d, C, bf16 = PATHS[path]
    inp = lasp_inputs.make_inputs(B, N, 4, d, seed=seed, bf16=bf16, decayed=False)
    inp["lam"] = np.asarray(LAMBDAS[lam_name], np.float32)
    return inp, C, bf16


def _oracle_all(inp, C, init=None, dstate_in=None):
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    lam = inp["lam"]
    o = oracle.fwd(q, k, v, lam, init=init)
    dq, dk, dv, dinit = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=dstate_in, want_dinit=True)
    P = oracle.state_snapshots(k, v, lam, C, init=init, kind=0)
    R = oracle.state_snapshots(q, do, lam, C, init=dstate_in, kind=1)
    return dict(o=o, dq=dq, dk=dk, dv=dv, P=P, R=R, dinit=dinit)


def _check(gpu, ref, bf16, names):
    errs = {n: rel_err(to_host(gpu[n]), ref[n]) for n in names}
    bad = {n: e for n, e in errs.items() if not (e <= tol(bf16))}
    assert not bad, f"errors above {tol(bf16)}: {bad} (all: {errs})"


@pytest.mark.parametrize("lam_name", sorted(LAMBDAS))
@pytest.mark.parametrize("path", sorted(PATHS))
def test_strong_decay_against_oracle(path, lam_name):
    inp, C, bf16 = _inputs(path, lam_name, seed=5100 + sorted(PATHS).index(path) * 10
                           + sorted(LAMBDAS).index(lam_name))
    B, N, d = inp["q"].shape[0], inp["q"].shape[1], inp["q"].shape[3]
    rng = np.random.default_rng(5200 + sorted(PATHS).index(path))
    init = (rng.standard_normal((B, 4, d, d)) * 0.2).astype(np.float32)
    din = (rng.standard_normal((B, 4, d, d)) * 0.2).astype(np.float32)
    gpu = run_fwd_bwd(inp, C, init=init, dstate_in=din, want_dinit=True)
    ref = _oracle_all(inp, C, init=init.astype(np.float64), dstate_in=din.astype(np.float64))
    _check(gpu, ref, bf16, ("o", "dq", "dk", "dv", "dinit"))
    # P_c and R_c through the state entry points (chunk states + scans)
    _check(run_states(inp, C, gpu["P"], gpu["R"], init=init, dstate_in=din), ref, bf16, ("P", "R"))


@pytest.mark.parametrize("lam_name", sorted(LAMBDAS))
def test_strong_decay_without_entering_states(lam_name):
    """The walks with no init_state / dstate_in (the zero-start branches)."""
    inp, C, bf16 = _inputs("walks_C128", lam_name, seed=5300 + sorted(LAMBDAS).index(lam_name))
    gpu = run_fwd_bwd(inp, C)
    ref = _oracle_all(inp, C)
    _check(gpu, ref, bf16, ("o", "dq", "dk", "dv"))


@pytest.mark.parametrize("lam_name", sorted(LAMBDAS))
@pytest.mark.parametrize("bf16,d,C", [(True, 128, 128), (True, 128, 64), (True, 64, 64), (True, 32, 128),
                                      (False, 64, 32)])
def test_state_entry_points_at_strong_decay(lam_name, bf16, d, C):
    """lasp_chunk_states, lasp_chunk_dstates and lasp_state_prefix (with an
    entering state and the total) on their own, against the oracle's
    definitions (LASP Eq. 10 and Eq. 20; the prefix / suffix of the LASP-2
    review, "The reading")."""
    import torch
    import sequence_linear_attention_b200 as lasp
    B, H, N = 2, 4, 512
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=5400 + C + d, bf16=bf16, decayed=False)
    lam = np.asarray(LAMBDAS[lam_name], np.float32)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    decay = decay_device(lam)
    T = N // C
    M = torch.empty((B, T, H, d, d), dtype=torch.float32, device="cuda")
    dM = torch.empty_like(M)
    lasp.lasp_chunk_states(None, k, v, decay, M, C)
    lasp.lasp_chunk_dstates(q, do, decay, dM, C)
    kf, vf, qf, df = (host_f32(inp, n) for n in ("k", "v", "q", "do"))
    rM = oracle.chunk_states(kf, vf, lam, C, 0)
    rdM = oracle.chunk_states(qf, df, lam, C, 1)
    assert rel_err(to_host(M), rM) <= tol(bf16)
    assert rel_err(to_host(dM), rdM) <= tol(bf16)
    rng = np.random.default_rng(5500 + C)
    init = rng.standard_normal((B, H, d, d)).astype(np.float32)
    for reverse, S, rS in ((False, M, rM), (True, dM, rdM)):
        out = torch.empty_like(S)
        tot = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
        lasp.lasp_state_prefix(S, out, decay, C, init=torch.from_numpy(init).cuda(), total=tot, reverse=reverse)
        # the scan is fp32 arithmetic on fp32 states: compare with the oracle's
        # scan of the GPU's own chunk states at the fp32 bar
        Sh = to_host(S)
        ref_p, ref_tot = oracle.state_scan(Sh, lam, C, init=init, reverse=reverse)
        assert rel_err(to_host(out), ref_p) <= tol(False), reverse
        assert rel_err(to_host(tot), ref_tot) <= tol(False), reverse
        # and end to end against the oracle's definition from the tokens
        ref_e2e, _ = oracle.state_scan(rS, lam, C, init=init, reverse=reverse)
        assert rel_err(to_host(out), ref_e2e) <= tol(bf16), reverse
    st, site = lasp.lasp_check_device_status()
    assert st == 0, (st, site)
