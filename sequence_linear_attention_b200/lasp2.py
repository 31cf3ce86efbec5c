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

Overlap (LASP-2 review page, "Core claim": the AllGather of fixed-size
states runs alongside computation). The (b, h) pairs are split into parts
(two by default, where both segment walks run and there are at least two
pairs): part p's shard states are gathered asynchronously (NCCL's stream)
while part p + 1's shard states are computed, and each part's scan over the
shards and its output start as soon as its own gather lands, so the gather of
the last part runs under the output of the ones before. No kernel waits on a
collective inside itself; the streams order them.

Each function takes the same tensors as the single-device call, plus the
process group (default: the world group). ``kernels`` replaces the device
kernels by an object with the same five methods (see ``DeviceKernels``); the
library's own are the default and the only ones used outside tests. ``parts``
overrides the number of parts.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (LASP_BF16, LASP_F32, lasp_bwd_finish_part, lasp_bwd_states_part, lasp_fwd_finish_part,
               lasp_fwd_states_part, lasp_parts_ok, lasp_state_prefix)

__all__ = ["DeviceKernels", "lasp2_fwd", "lasp2_bwd", "default_parts"]


class DeviceKernels:
    """The library's kernels, through its C ABI, in the shape this module calls
    them. The shard states are the first parts of the single-device forward and
    backward calls (their segment states, in the cache or workspace, and the
    decayed total); the rest of those calls reuses the segment states. Every
    call works on part `part` of `nparts` of the (b, h) pairs."""

    @staticmethod
    def shard_state(k, v, decay, M, C, state_cache, part, nparts):
        lasp_fwd_states_part(k, v, decay, C, state_cache, M, part, nparts)

    @staticmethod
    def shard_dstate(q, dout, decay, dM, C, dstate_ws, part, nparts):
        lasp_bwd_states_part(q, dout, decay, C, dstate_ws, dM, part, nparts)

    @staticmethod
    def state_prefix(M, out, decay, L, init, total, reverse):
        lasp_state_prefix(M, out, decay, L, init=init, total=total, reverse=reverse)

    @staticmethod
    def fwd(q, k, v, decay, o, C, state_cache, init_state, part, nparts):
        lasp_fwd_finish_part(q, k, v, decay, o, C, state_cache, init_state, part, nparts)

    @staticmethod
    def bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in, part, nparts):
        lasp_bwd_finish_part(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in, None, part,
                             nparts)


def default_parts(q, C, world=2):
    """Two parts where there is an exchange to hide (more than one rank), both
    segment walks run on the shard and it has at least two (b, h) pairs; else
    one (at one rank the split only adds launches and a second wave tail:
    3.4% slower on the 2M-token workload)."""
    B, L, H, d = q.shape
    dt = LASP_BF16 if q.dtype == torch.bfloat16 else LASP_F32
    return 2 if world > 1 and B * H >= 2 and q.is_cuda and lasp_parts_ok(L, C, d, dt) else 1


def _group_shape(x, group):
    if x.dim() != 4:
        raise ValueError("shard tensors must be [B, L, H, d]")
    B, L, H, d = x.shape
    if L < 1:
        raise ValueError("every rank needs a non-empty shard")
    return dist.get_world_size(group), dist.get_rank(group), B, L, H, d


class _Done:
    def wait(self):
        pass


def _all_gather(out, x, group):
    """Gathers x from every rank into the [W, ...] buffer out; returns a handle
    whose wait() orders later work on the current stream after the gather.
    NCCL gathers device memory straight into the buffer, asynchronously on its
    own stream; other backends (gloo) gather host copies, synchronously."""
    if dist.get_backend(group) == "nccl":
        return dist.all_gather_into_tensor(out, x, group=group, async_op=True)
    if out.is_cuda:
        host = torch.empty(out.shape, dtype=out.dtype)
        dist.all_gather(list(host.unbind(0)), x.cpu(), group=group)
        out.copy_(host)
    else:
        dist.all_gather(list(out.unbind(0)), x, group=group)
    return _Done()


def _bounds(B, H, nparts):
    bh = B * H
    return [bh * p // nparts for p in range(nparts + 1)]


def _pairs(t, bh0, bh1):
    """Pairs bh0 .. bh1 - 1 of a [B, H, d, d] state (or None), as [1, n, d, d]."""
    if t is None:
        return None
    d = t.shape[-1]
    return t.reshape(-1, d, d)[bh0:bh1].unsqueeze(0)


def _exchange(kern, states_fn, finish_fn, decay, L, init, total, reverse, B, H, d, W, r, nparts, device, group):
    """The exchange of one direction: per part, the shard states (states_fn),
    an asynchronous gather, then the scan over the W shards and the rest of the
    call (finish_fn) once that part's gather has landed. Returns the states
    entering this shard, [B, H, d, d]."""
    M = torch.empty((B, H, d, d), dtype=torch.float32, device=device)
    bounds = _bounds(B, H, nparts)
    handles, bufs = [], []
    for p in range(nparts):
        states_fn(M, p)
        bh0, bh1 = bounds[p], bounds[p + 1]
        buf = torch.empty((W, bh1 - bh0, d, d), dtype=torch.float32, device=device)
        handles.append(_all_gather(buf, M.view(B * H, d, d)[bh0:bh1], group))
        bufs.append(buf)
    # the decay of every (b, h) pair; a part's slice is copied, since the ABI
    # takes 16-byte-aligned pointers only
    rep = None if decay is None else decay.repeat(B)
    entering = torch.empty((B, H, d, d), dtype=torch.float32, device=device)
    for p in range(nparts):
        handles[p].wait()
        bh0, bh1 = bounds[p], bounds[p + 1]
        n = bh1 - bh0
        out = torch.empty_like(bufs[p])
        # the W gathered states of these pairs as one sequence of W chunks with n heads
        kern.state_prefix(bufs[p].view(1, W, n, d, d), out.view(1, W, n, d, d),
                          None if rep is None else rep[bh0:bh1].clone(), L, _pairs(init, bh0, bh1),
                          _pairs(total, bh0, bh1), reverse)
        entering.view(B * H, d, d)[bh0:bh1].copy_(out[r])
        finish_fn(entering, p)
    return entering


def _check_state(t, B, H, d, like, name):
    if t is None:
        return
    if (tuple(t.shape) != (B, H, d, d) or t.dtype != torch.float32 or not t.is_contiguous()
            or t.device != like.device):
        raise ValueError(f"{name} must be a contiguous float32 [B, H, d, d] tensor on the shard's device")


def lasp2_fwd(q, k, v, decay, o, C, state_cache, init_state=None, final_state=None, group=None, kernels=None,
              parts=None):
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
    nparts = parts or (default_parts(q, C, W) if kernels is None else 1)
    return _exchange(kern, lambda M, p: kern.shard_state(k, v, decay, M, C, state_cache, p, nparts),
                     lambda E, p: kern.fwd(q, k, v, decay, o, C, state_cache, E, p, nparts),
                     decay, L, init_state, final_state, False, B, H, d, W, r, nparts, q.device, group)


def lasp2_bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in=None, dinit_state=None,
              group=None, kernels=None, parts=None):
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
    nparts = parts or (default_parts(q, C, W) if kernels is None else 1)
    return _exchange(kern, lambda dM, p: kern.shard_dstate(q, dout, decay, dM, C, dstate_ws, p, nparts),
                     lambda G, p: kern.bwd(q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, G, p, nparts),
                     decay, L, dstate_in, dinit_state, True, B, H, d, W, r, nparts, q.device, group)
