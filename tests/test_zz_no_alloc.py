"""lasp_bwd_noalloc, the backward entry point for callers that cannot allocate
device memory (it keeps its gradient-state workspace in a fixed array inside
the library). Called through the C ABI, it must give exactly what lasp_bwd
gives (the same kernels run on the same inputs), call after call, since every
call reuses the same array; and both must match the fp64 oracle.

This file is collected last on purpose, so that a run that stops at the first
failure has run every other test before it."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import decay_device, host_f32, rel_err, to_device, to_host, tol

pytestmark = pytest.mark.gpu

# (seed, B, H, N, d, C, bf16, lam): lam is "workload" (the per-head rates),
# None (no decay) or a list of per-head rates
CASES = [
    (11, 1, 4, 1024, 128, 128, True, "workload"),       # segment-walk branch
    (12, 2, 3, 640, 128, 64, True, None),               # walk branch, chunks inside the tile
    (14, 1, 2, 320, 128, 64, True, "workload"),         # per-chunk tensor-core branch (ragged tile)
    (15, 1, 2, 256, 64, 64, False, "workload"),         # per-chunk CUDA-core branch, fp32
    (16, 1, 4, 1024, 128, 128, True, [1.0, 0.99, 0.5, 1e-3]),  # strong decays on the walk
    (17, 1, 2, 1024, 128, 256, True, "workload"),       # walk branch with chunks of two tiles
    (18, 2, 3, 640, 64, 128, True, "workload"),         # per-chunk tensor-core branch, d = 64
    (19, 1, 2, 384, 32, 64, True, [0.5, 1e-3]),         # per-chunk tensor-core branch, d = 32, strong decays
]


def _problem(seed, B, H, N, d, C, bf16, lam):
    import torch
    import sequence_linear_attention_b200 as lasp
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=seed, bf16=bf16, decayed=lam == "workload")
    if isinstance(lam, list):
        inp["lam"] = np.asarray(lam, np.float32)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    o = torch.empty_like(q)
    P = torch.empty((B, N // C, H, d, d), dtype=torch.float32, device="cuda")
    lasp.lasp_fwd(q, k, v, decay, o, C, P)
    return inp, (q, k, v, do, decay, P)


def _both(dev, C, dstate_in):
    """lasp_bwd with its own workspace, then lasp_bwd_noalloc into NaN-filled
    outputs; returns both sets of (dq, dk, dv, dinit)."""
    import torch
    import sequence_linear_attention_b200 as lasp
    q, k, v, do, decay, P = dev
    B, _, H, d = q.shape
    ref = [torch.empty_like(q) for _ in range(3)]
    ws = torch.empty_like(P)
    dinit_ref = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    lasp.lasp_bwd(q, k, v, decay, do, *ref, C, P, ws, dstate_in=dstate_in, dinit_state=dinit_ref)
    got = [torch.full_like(q, float("nan")) for _ in range(3)]
    dinit = torch.full_like(dinit_ref, float("nan"))
    lasp.lasp_bwd_noalloc(q, k, v, decay, do, *got, C, P, dstate_in=dstate_in, dinit_state=dinit)
    st, site = lasp.lasp_check_device_status()
    assert st == 0, (st, site)
    return got + [dinit], ref + [dinit_ref]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"s{c[0]}")
def test_noalloc_backward_equals_lasp_bwd_on_consecutive_calls(case):
    """Bit for bit against lasp_bwd, twice in a row (the second call finds the
    first call's gradient states in the shared array), with and without a
    gradient state entering from beyond the end; and against the oracle."""
    import torch
    seed, B, H, N, d, C, bf16, lam = case
    inp, dev = _problem(*case)
    rng = np.random.default_rng(seed + 100)
    din = (rng.standard_normal((B, H, d, d)) * 0.2).astype(np.float32)
    for dstate_in in (None, torch.from_numpy(din).cuda(), None):
        got, ref = _both(dev, C, dstate_in)
        for name, g, r in zip(("dq", "dk", "dv", "dinit"), got, ref):
            assert torch.equal(g, r), (name, dstate_in is not None)
    # the last call (no dstate_in) against the oracle
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    rdq, rdk, rdv, rdinit = oracle.bwd(q, k, v, do, inp["lam"], want_dinit=True)
    for name, g, r in zip(("dq", "dk", "dv", "dinit"), got, (rdq, rdk, rdv, rdinit)):
        assert rel_err(to_host(g), r) <= tol(bf16), name


def test_noalloc_backward_rejects_problems_beyond_its_workspace():
    import torch
    import sequence_linear_attention_b200 as lasp
    # 1 x 16 heads x 64 chunks = 1024 states of 64 KiB: 64 MiB, beyond the 32 MiB array
    _, (q, k, v, do, decay, P) = _problem(13, 1, 16, 8192, 128, 128, True, "workload")
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    with pytest.raises(lasp.LaspError) as e:
        lasp.lasp_bwd_noalloc(q, k, v, decay, do, dq, dk, dv, 128, P)
    assert e.value.status == 2  # LASP_ERR_UNSUPPORTED
