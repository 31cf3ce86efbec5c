"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library through its C ABI, and compare with the oracle per tensor with
max|gpu - ref| / max|ref|."""
from __future__ import annotations

import numpy as np

from sequence_linear_attention_b200 import inputs as lasp_inputs

# Tolerances: max|gpu - ref| / max|ref| per tensor, for fp32 inputs (fp32
# arithmetic) and for bf16 inputs with fp32 accumulation.
TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol(bf16: bool) -> float:
    return TOL_BF16 if bf16 else TOL_F32


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = float(np.max(np.abs(ref))) if ref.size else 0.0
    num = float(np.max(np.abs(got - ref))) if ref.size else 0.0
    if den == 0.0:
        return num
    return num / den


def to_device(x: np.ndarray, bf16: bool):
    import torch
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_host(t) -> np.ndarray:
    import torch
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return lasp_inputs.bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))
    return t.float().cpu().numpy()


def decay_device(lam):
    import torch
    return None if lam is None else torch.from_numpy(np.asarray(lam, np.float32)).cuda()


def host_f32(inp: dict, name: str) -> np.ndarray:
    return lasp_inputs.as_f32(inp[name], inp["bf16"])


_KEEP = object()


def run_fwd_bwd(inp: dict, C: int, init=None, dstate_in=None, want_dinit=False, decay_override=_KEEP):
    """Runs lasp_fwd and lasp_bwd on the device; returns a dict of device tensors."""
    import torch
    import sequence_linear_attention_b200 as lasp
    bf16 = inp["bf16"]
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    B, N, H, d = q.shape
    lam = inp["lam"] if decay_override is _KEEP else decay_override
    decay = decay_device(lam)
    T = N // C
    o = torch.empty_like(q)
    cache = torch.empty((B, T, H, d, d), dtype=torch.float32, device="cuda")
    init_t = None if init is None else torch.from_numpy(np.asarray(init, np.float32)).cuda()
    din_t = None if dstate_in is None else torch.from_numpy(np.asarray(dstate_in, np.float32)).cuda()
    lasp.lasp_fwd(q, k, v, decay, o, C, cache, init_state=init_t)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty_like(cache)
    dinit = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda") if want_dinit else None
    lasp.lasp_bwd(q, k, v, decay, do, dq, dk, dv, C, cache, ws, init_state=init_t, dstate_in=din_t,
                  dinit_state=dinit)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    return dict(o=o, dq=dq, dk=dk, dv=dv, P=cache, R=ws, dinit=dinit)


def run_states(inp: dict, C: int, P, R, init=None, dstate_in=None):
    """P_c and R_c through the exposed state entry points (lasp_chunk_states /
    lasp_chunk_dstates, then lasp_state_prefix forward / reverse), into the
    given [B, N/C, H, d, d] fp32 device buffers."""
    import torch
    import sequence_linear_attention_b200 as lasp
    bf16 = inp["bf16"]
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    init_t = None if init is None else torch.from_numpy(np.asarray(init, np.float32)).cuda()
    din_t = None if dstate_in is None else torch.from_numpy(np.asarray(dstate_in, np.float32)).cuda()
    lasp.lasp_chunk_states(None, k, v, decay, P, C)
    lasp.lasp_state_prefix(P, P, decay, C, init=init_t)
    lasp.lasp_chunk_dstates(q, do, decay, R, C)
    lasp.lasp_state_prefix(R, R, decay, C, init=din_t, reverse=True)
    status, site = lasp.lasp_check_device_status()
    assert status == 0, (status, site)
    return dict(P=P, R=R)
