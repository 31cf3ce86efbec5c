"""lasp_bwd_noalloc, the backward entry point for callers that cannot allocate
device memory (it keeps its gradient-state workspace in a fixed array inside
the library). Called through the C ABI, it must give what lasp_bwd gives,
call after call, since every call reuses the same array.

This file is collected last on purpose, so that a run that stops at the first
failure has run every other test before it."""
import numpy as np
import pytest

from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import decay_device, rel_err, to_device, to_host, tol

pytestmark = pytest.mark.gpu


def _problem(seed, B, H, N, C, decayed):
    import torch
    import sequence_linear_attention_b200 as lasp
    inp = lasp_inputs.make_inputs(B, N, H, 128, seed=seed, bf16=True, decayed=decayed)
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    o = torch.empty_like(q)
    P = torch.empty((B, N // C, H, 128, 128), dtype=torch.float32, device="cuda")
    lasp.lasp_fwd(q, k, v, decay, o, C, P)
    return q, k, v, do, decay, P


def test_noalloc_backward_matches_lasp_bwd_on_consecutive_calls():
    import torch
    import sequence_linear_attention_b200 as lasp
    # two different problems in a row, both inside the fixed workspace
    for seed, (B, H, N, C, decayed) in ((11, (1, 4, 1024, 128, True)), (12, (2, 3, 640, 64, False))):
        q, k, v, do, decay, P = _problem(seed, B, H, N, C, decayed)
        ref = [torch.empty_like(q) for _ in range(3)]
        ws = torch.empty_like(P)
        dinit_ref = torch.empty((B, H, 128, 128), dtype=torch.float32, device="cuda")
        lasp.lasp_bwd(q, k, v, decay, do, *ref, C, P, ws, dinit_state=dinit_ref)
        got = [torch.full_like(q, float("nan")) for _ in range(3)]
        dinit = torch.full_like(dinit_ref, float("nan"))
        lasp.lasp_bwd_noalloc(q, k, v, decay, do, *got, C, P, dinit_state=dinit)
        st, site = lasp.lasp_check_device_status()
        assert st == 0, (st, site)
        for g, r in zip(got + [dinit], ref + [dinit_ref]):
            assert rel_err(to_host(g), to_host(r).astype(np.float64)) <= tol(True)


def test_noalloc_backward_rejects_problems_beyond_its_workspace():
    import sequence_linear_attention_b200 as lasp
    # 1 x 8 x 1024 / 128 = 64 states fit; 16 heads x 64 chunks = 1024 states do not
    q, k, v, do, decay, P = _problem(13, 1, 16, 8192, 128, True)
    import torch
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    with pytest.raises(lasp.LaspError) as e:
        lasp.lasp_bwd_noalloc(q, k, v, decay, do, dq, dk, dv, 128, P)
    assert e.value.status == 2  # LASP_ERR_UNSUPPORTED
