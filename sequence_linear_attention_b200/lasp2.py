"""LASP-2 sequence parallelism: one shard of every sequence per rank.

Rank r of a group of W ranks holds tokens [r L, (r + 1) L) of each sequence, as
contiguous [B, L, H, d] tensors. The exchange between shards is one AllGather
of d x d states per direction (LASP-2, "The reading" and its backward pass):

forward
  1. the shard's memory state, M_r = sum_j lambda^{L-1-j} k_j^T v_j
     (LASP Eq. 10 with the shard as one chunk): the first part of the
     single-device forward, whose segment states it sums with their decays;
  2. AllGather of M_0 .. M_{W-1};
  3. the state entering the shard, by the decayed prefix over the shards
     before it: E_0 = the sequence's initial state, E_r = lambda^L E_{r-1} + M_{r-1};
  4. the rest of the single-device forward of the shard (its prefix over the
     segment states already in the cache, then the output) from E_r.

backward
  1. the shard's gradient state, dM_r = sum_j lambda^{j+1} q_j^T do_j
     (LASP Eq. 20 with the shard as one chunk), likewise the first part of the
     single-device backward;
  2. AllGather of dM_0 .. dM_{W-1};
  3. the gradient state entering the shard's last token from the shards after
     it, by the decayed suffix: G_{W-1} = the gradient w.r.t. the sequence's
     final state, G_r = lambda^L G_{r+1} + dM_{r+1};
  4. the rest of the single-device backward of the shard from G_r.

No state is computed twice: the segment states stay in the state cache
(forward) or the gradient-state workspace (backward) for the second part. The
scans over the W gathered states run in the library's scan kernel (the
gathered [W, B, H, d, d] array is the [1, W, B*H, d, d] chunk-state array of
one sequence whose B*H "heads" carry the decays of the H heads B times). All
arithmetic runs in the library's kernels; torch.distributed moves the states.
The payload of each AllGather is W * B * H * d * d fp32 values (1 MiB per rank
at B = 1, H = 16, d = 128), so the exchange is latency-bound on NVLink.

Each function takes the same tensors as the single-device call, plus the
process group (default: the world group). ``kernels`` replaces the device
kernels by an object with the same five methods (see ``DeviceKernels``); the
library's own are the default and the only ones used outside tests.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import lasp_bwd_finish, lasp_bwd_states, lasp_fwd_finish, lasp_fwd_states, lasp_state_prefix

__all__ = ["DeviceKernels", "lasp2_fwd", "lasp2_bwd"]


class DeviceKernels:
    """The library's kernels, through its C ABI, in the shape this module calls
    them. The shard states are the first parts of the single-device forward and
    backward calls (their segment states, in the cache or workspace, and the
    decayed total); the rest of those calls reuses the segment states."""

    @staticmethod
    def shard_state(k, v, decay, M, C, state_cache):
        lasp_fwd_states(k, v, decay, C, state_cache, total=M)

    @staticmethod
    def shard_dstate(q, dout, decay, dM, C, dstate_ws):
        lasp_bwd_states(q, dout, decay, C, dstate_ws, total=dM)

    @staticmethod
    def state_prefix(M, out, decay, L, init, total, reverse):
        lasp_state_prefix(M, out, decay, L, init=init, total=total, reverse=reverse)

    @staticmethod
    def fwd(q, k, v, decay, o, C, state_cache, init_state):
        lasp_fwd_finish(q, k, v, decay, o, C, state_cache, init_state=init_state)

    @staticmethod
    def bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in):
        lasp_bwd_finish(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in=dstate_in)


def _group_shape(x, group):
    if x.dim() != 4:
        raise ValueError("shard tensors must be [B, L, H, d]")
    B, L, H, d = x.shape
    if L < 1:
        raise ValueError("every rank needs a non-empty shard")
    return dist.get_world_size(group), dist.get_rank(group), B, L, H, d


def _all_gather(out, x, group):
    # NCCL gathers device memory straight into the [W, ...] buffer. Other
    # backends (gloo) gather host copies into the list of the buffer's W slices.
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, x, group=group)
    elif out.is_cuda:
        host = torch.empty(out.shape, dtype=out.dtype)
        dist.all_gather(list(host.unbind(0)), x.cpu(), group=group)
        out.copy_(host)
    else:
        dist.all_gather(list(out.unbind(0)), x, group=group)


def _scan_over_shards(kern, gathered, decay, L, init, total, reverse):
    """Exclusive decayed scan over the W gathered [B, H, d, d] states; returns
    the [W, B, H, d, d] scan, writes the total (if given)."""
    W, B, H, d, _ = gathered.shape
    flat = lambda t: None if t is None else t.reshape(1, B * H, d, d)
    rep = None if decay is None else decay.repeat(B)
    out = torch.empty_like(gathered)
    kern.state_prefix(gathered.view(1, W, B * H, d, d), out.view(1, W, B * H, d, d), rep, L,
                      flat(init), flat(total), reverse)
    return out


def _check_state(t, B, H, d, like, name):
    if t is None:
        return
    if (tuple(t.shape) != (B, H, d, d) or t.dtype != torch.float32 or not t.is_contiguous()
            or t.device != like.device):
        raise ValueError(f"{name} must be a contiguous float32 [B, H, d, d] tensor on the shard's device")


def lasp2_fwd(q, k, v, decay, o, C, state_cache, init_state=None, final_state=None, group=None, kernels=None):
    """Forward pass of this rank's shard (see the module docstring).

    q, k, v, o: [B, L, H, d] shard tensors; C, state_cache: as for the
    single-device forward on [B, L, H, d] (the cache holds the shard's chunk
    states for ``lasp2_bwd``). init_state: float [B, H, d, d] entering the
    sequence's first token, or None; the same tensor on every rank (rank 0's
    is the one that counts). final_state: float [B, H, d, d] or None, receives
    the state after the sequence's last token, on every rank.
    Returns the state entering this shard, float [B, H, d, d].
    """
    kern = kernels or DeviceKernels
    W, r, B, L, H, d = _group_shape(q, group)
    _check_state(init_state, B, H, d, q, "init_state")
    _check_state(final_state, B, H, d, q, "final_state")
    M = torch.empty((B, 1, H, d, d), dtype=torch.float32, device=q.device)
    kern.shard_state(k, v, decay, M.view(B, H, d, d), C, state_cache)
    gathered = torch.empty((W, B, H, d, d), dtype=torch.float32, device=q.device)
    _all_gather(gathered, M.view(B, H, d, d), group)
    entering = _scan_over_shards(kern, gathered, decay, L, init_state, final_state, False)[r]
    kern.fwd(q, k, v, decay, o, C, state_cache, entering)
    return entering


def lasp2_bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in=None, dinit_state=None,
              group=None, kernels=None):
    """Backward pass of this rank's shard (see the module docstring): dq, dk, dv
    of sum(o * dout) over the whole sequence, for this shard's tokens.

    state_cache: the cache ``lasp2_fwd`` wrote on this rank. dstate_ws: as for
    the single-device backward on [B, L, H, d]. dstate_in: float [B, H, d, d]
    gradient w.r.t. the state after the sequence's last token, or None; the same
    tensor on every rank. dinit_state: float [B, H, d, d] or None, receives the
    gradient w.r.t. the sequence's initial state, on every rank.
    Returns the gradient state entering this shard's last token.
    """
    kern = kernels or DeviceKernels
    W, r, B, L, H, d = _group_shape(q, group)
    _check_state(dstate_in, B, H, d, q, "dstate_in")
    _check_state(dinit_state, B, H, d, q, "dinit_state")
    dM = torch.empty((B, 1, H, d, d), dtype=torch.float32, device=q.device)
    kern.shard_dstate(q, dout, decay, dM.view(B, H, d, d), C, dstate_ws)
    gathered = torch.empty((W, B, H, d, d), dtype=torch.float32, device=q.device)
    _all_gather(gathered, dM.view(B, H, d, d), group)
    incoming = _scan_over_shards(kern, gathered, decay, L, dstate_in, dinit_state, True)[r]
    kern.bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, incoming)
    return incoming
