"""LASP-2H: the softmax-attention layers of a hybrid model under LASP-2's
sequence split (LASP-2 review page, "Summary" and abstract: the same AllGather
pattern applied to standard attention layers, gathering K_t and V_t).

Rank r of a group of W ranks holds tokens [r L, (r + 1) L) of each sequence, as
contiguous [B, L, H, d] tensors, like ``lasp2``.

forward
  1. AllGather of every rank's K and V shard into [B, W L, H, d] buffers (the
     ranks before r supply the keys its queries see; the later ones' are not
     read);
  2. causal softmax attention of the shard's queries, at positions r L + i,
     against the gathered keys (``lasp_softmax_fwd`` with q_offset = r L).

backward
  1. the same call's gradients: dq for the shard's queries, and partial dk, dv
     for every gathered key (zero for keys after the shard);
  2. a reduce-scatter (sum) of the partial dk, dv: each rank receives the sum
     over all ranks for its own keys.

The payloads are 2 W B L H d bf16 values per gather and per reduce-scatter
(the keys and values of the whole sequence), unlike linear attention's fixed
d x d states. All arithmetic runs in the library's kernels; torch.distributed
moves the tensors. Each collective works on one batch row at a time, so that
every rank's block is contiguous.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import lasp_softmax_bwd, lasp_softmax_fwd

__all__ = ["DeviceKernels", "lasp2h_fwd", "lasp2h_bwd", "gathered_like"]


class DeviceKernels:
    """The library's softmax-attention kernels through the C ABI."""

    @staticmethod
    def fwd(q, k_all, v_all, o, lse, q_offset, scale):
        lasp_softmax_fwd(q, k_all, v_all, o, lse, q_offset=q_offset, scale=scale)

    @staticmethod
    def bwd(q, k_all, v_all, o, lse, dout, dq, dk_all, dv_all, delta, q_offset, scale):
        lasp_softmax_bwd(q, k_all, v_all, o, lse, dout, dq, dk_all, dv_all, delta, q_offset=q_offset, scale=scale)


def _shape(x, group):
    if x.dim() != 4:
        raise ValueError("shard tensors must be [B, L, H, d]")
    B, L, H, d = x.shape
    if L < 1:
        raise ValueError("every rank needs a non-empty shard")
    return dist.get_world_size(group), dist.get_rank(group), B, L, H, d


def gathered_like(x, group=None):
    """An empty [B, W L, H, d] buffer for the gathered keys or values of the
    shard tensor x."""
    W, _, B, L, H, d = _shape(x, group)
    return torch.empty((B, W * L, H, d), dtype=x.dtype, device=x.device)


def _gather_rows(out, x, group):
    # batch row by batch row: rank r's [L, H, d] lands at rows r L.. of out[b]
    nccl = dist.get_backend(group) == "nccl"
    W = dist.get_world_size(group)
    for b in range(x.shape[0]):
        if nccl:
            dist.all_gather_into_tensor(out[b], x[b], group=group)
        else:  # gloo: host copies, gathered into the W slices of the row
            host = torch.empty(out[b].shape, dtype=out.dtype)
            dist.all_gather(list(host.chunk(W, 0)), x[b].cpu().contiguous(), group=group)
            out[b].copy_(host)


def _reduce_scatter_rows(out, full, group):
    # the sum over ranks of full[b], rank r keeping rows r L .. (r + 1) L
    nccl = dist.get_backend(group) == "nccl"
    W, r = dist.get_world_size(group), dist.get_rank(group)
    L = out.shape[1]
    for b in range(out.shape[0]):
        if nccl:
            dist.reduce_scatter_tensor(out[b], full[b], group=group)
        else:  # gloo has no reduce-scatter: a sum over all rows, then this rank's
            host = full[b].cpu().float()
            dist.all_reduce(host, group=group)
            out[b].copy_(host[r * L:(r + 1) * L])


def _check_rows(t, B, H, L, like, name):
    if (tuple(t.shape) != (B, H, L) or t.dtype != torch.float32 or not t.is_contiguous()
            or t.device != like.device):
        raise ValueError(f"{name} must be a contiguous float32 [B, H, L] tensor on the shard's device")


def lasp2h_fwd(q, k, v, o, lse, k_all, v_all, scale=None, group=None, kernels=None):
    """Forward of this rank's shard: o [B, L, H, d] and lse [B, H, L] (natural
    log, kept for the backward). k_all, v_all: [B, W L, H, d] buffers
    (``gathered_like``) that receive the gathered keys and values; pass them
    to ``lasp2h_bwd`` unchanged. scale defaults to d^-1/2."""
    kern = kernels or DeviceKernels
    W, r, B, L, H, d = _shape(q, group)
    _check_rows(lse, B, H, L, q, "lse")
    _gather_rows(k_all, k, group)
    _gather_rows(v_all, v, group)
    kern.fwd(q, k_all, v_all, o, lse, r * L, scale)


def lasp2h_bwd(q, o, lse, dout, dq, dk, dv, k_all, v_all, scale=None, group=None, kernels=None):
    """Backward of this rank's shard: dq, dk, dv [B, L, H, d] of sum(o * dout)
    over the whole sequence, for this shard's tokens (dk, dv summed over the
    ranks whose queries see them). k_all, v_all: what ``lasp2h_fwd`` gathered."""
    kern = kernels or DeviceKernels
    W, r, B, L, H, d = _shape(q, group)
    _check_rows(lse, B, H, L, q, "lse")
    dk_all, dv_all = torch.empty_like(k_all), torch.empty_like(v_all)
    delta = torch.empty_like(lse)
    kern.bwd(q, k_all, v_all, o, lse, dout, dq, dk_all, dv_all, delta, r * L, scale)
    _reduce_scatter_rows(dk, dk_all, group)
    _reduce_scatter_rows(dv, dv_all, group)
