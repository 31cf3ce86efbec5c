"""The bidirectional (unmasked) form through the C ABI against the oracle:
o = q (k^T v) and its gradients (LASP Eq. 3; the LASP-2 page's unmasked
variant), bf16 inputs, tolerance max|gpu - ref| / max|ref| <= 2e-2; the total
states M and dM (fp32, read from the workspace) against the oracle's."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import TOL_BF16, host_f32, rel_err, to_device, to_host

pytestmark = pytest.mark.gpu


def _run(inp):
    import torch
    import sequence_linear_attention_b200 as lasp
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    B, N, H, d = q.shape
    nws = lasp.lasp_bidir_workspace_floats(B, H, N, d)
    off = lasp.lasp_bidir_state_offset(B, H, N, d)
    ws = torch.empty(nws, dtype=torch.float32, device="cuda")
    dws = torch.empty_like(ws)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lasp.lasp_bidir_fwd(q, k, v, o, ws)
    lasp.lasp_bidir_bwd(q, k, v, do, dq, dk, dv, ws, dws)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    M = ws[off:off + B * H * d * d].view(B, H, d, d)
    dM = dws[off:off + B * H * d * d].view(B, H, d, d)
    return dict(o=o, dq=dq, dk=dk, dv=dv, M=M, dM=dM)


def _check(gpu, inp, heads=None):
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    if heads is not None:
        q, k, v, do = (np.ascontiguousarray(x[:, :, heads]) for x in (q, k, v, do))
    o, M = oracle.bidir_fwd(q, k, v, want_state=True)
    dq, dk, dv, dM = oracle.bidir_bwd(q, k, v, do, want_state=True)
    ref = dict(o=o, dq=dq, dk=dk, dv=dv, M=M, dM=dM)
    errs = {}
    for n, r in ref.items():
        g = to_host(gpu[n])
        g = g[:, :, heads] if (heads is not None and g.ndim == 4 and n not in ("M", "dM")) else g
        g = g[:, heads] if (heads is not None and n in ("M", "dM")) else g
        errs[n] = rel_err(g, r)
    # states are fp32 sums of exact bf16 products; outputs are rounded to bf16
    bad = {n: e for n, e in errs.items() if e > (1e-4 if n in ("M", "dM") else TOL_BF16)}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("B,H,N", [(1, 2, 128), (2, 3, 384), (1, 2, 2048), (2, 150, 256), (1, 1, 3072)])
def test_bidirectional_small_shapes_against_oracle(B, H, N):
    inp = lasp_inputs.make_inputs(B, N, H, 128, seed=300 + N + H, bf16=True, decayed=False)
    _check(_run(inp), inp)


def test_bidirectional_bench_size_sampled_heads():
    inp = lasp_inputs.make_inputs(1, 65536, 16, 128, seed=1002, bf16=True, decayed=False)
    _check(_run(inp), inp, heads=[0, 11])


def test_bidirectional_kernels_and_unsupported_sizes():
    import torch
    import sequence_linear_attention_b200 as lasp
    inp = lasp_inputs.make_inputs(1, 512, 2, 128, seed=310, bf16=True, decayed=False)
    lasp.lasp_trace_enable(64)
    try:
        _run(inp)
        names = [n for n, _ in lasp.lasp_trace_read(64)]
    finally:
        lasp.lasp_trace_enable(0)
    assert names == ["segment_states_tc", "bidir_total", "bidir_apply_tc",
                     "segment_states_tc", "bidir_total", "bidir_apply_tc", "bidir_apply_tc", "bidir_apply_tc"], names
    x = torch.zeros((1, 200, 2, 128), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros(1 << 20, dtype=torch.float32, device="cuda")
    with pytest.raises(lasp.LaspError):
        lasp.lasp_bidir_fwd(x, x, x, torch.empty_like(x), ws)
