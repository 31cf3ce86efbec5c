"""Seeded synthetic inputs for chunked causal linear attention.

This module is the one piece shared by the CUDA path's tests/benchmark and the
CPU oracle: it draws the random tensors and does nothing else. It holds none of
the method's arithmetic.

Recipe (the workloads of the LASP / LASP-2 pages are Linear-Llama3 and TNL
layers with head dimension 128; no data set or trained weight is used):

* q, k, v: i.i.d. standard normal, times d^-1/2; dO: i.i.d. standard normal.
* One independent stream per tensor, in the order q, k, v, dO, derived from
  ``numpy.random.SeedSequence(seed)``; each tensor is drawn in blocks of
  ``_BLOCK`` elements, block i from the i-th child of that stream, so the values
  do not depend on how many threads draw them.
* Samples are float64, scaled, cast to float32 (round to nearest even), then,
  for bf16 workloads, rounded to bf16 (round to nearest even) and returned as
  the raw 16-bit patterns (``numpy.uint16``).
* Per-head decay lambda_h = 1 - 2^-(5 + 8h/H), h = 0..H-1, as float32; the
  undecayed workloads use lambda = 1.
* Gated workloads (a log-gate per token and key feature): g = log(sigmoid(x)) / tau
  with x i.i.d. standard normal from a fifth stream, tau = 16 by default (gates
  mostly in 0.9-1.0; tau = 1 gives strong gates), float32 [B, N, H, d].
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_BLOCK = 1 << 22
_NAMES = ("q", "k", "v", "do")


def decay_rates(H: int) -> np.ndarray:
    """lambda_h = 1 - 2^-(5 + 8h/H) for h = 0..H-1, float32 [H]."""
    h = np.arange(H, dtype=np.float64)
    return (1.0 - np.exp2(-(5.0 + 8.0 * h / H))).astype(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return the 16-bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _draw(child: np.random.SeedSequence, n: int, scale: float, bf16: bool, out: np.ndarray, off: int):
    g = np.random.Generator(np.random.PCG64(child))
    x = g.standard_normal(n, dtype=np.float64)
    if scale != 1.0:
        x *= scale
    x32 = x.astype(np.float32)
    out[off:off + n] = f32_to_bf16_bits(x32) if bf16 else x32


def draw_tensor(seed: int, index: int, shape, scale: float, bf16: bool, threads: int | None = None):
    """Tensor ``index`` (0=q, 1=k, 2=v, 3=dO) of the stream rooted at ``seed``."""
    n = int(np.prod(shape))
    stream = np.random.SeedSequence(seed).spawn(len(_NAMES))[index]
    nblk = (n + _BLOCK - 1) // _BLOCK
    children = stream.spawn(nblk)
    out = np.empty(n, np.uint16 if bf16 else np.float32)
    threads = threads or min(32, os.cpu_count() or 1)
    with ThreadPoolExecutor(max_workers=threads) as ex:
        futs = [ex.submit(_draw, children[i], min(_BLOCK, n - i * _BLOCK), scale, bf16, out, i * _BLOCK)
                for i in range(nblk)]
        for f in futs:
            f.result()
    return out.reshape(shape)


def draw_tensor_rows(seed: int, index: int, shape, scale: float, bf16: bool, row0: int, rows: int):
    """Rows row0 .. row0 + rows - 1 (axis 1) of the [B, N, H, d] tensor that
    :func:`draw_tensor` draws for the same arguments, drawing only the blocks
    that hold them (a shard of a long sequence without the rest of it)."""
    B, N, H, d = shape
    n = B * N * H * d
    stream = np.random.SeedSequence(seed).spawn(len(_NAMES))[index]
    children = stream.spawn((n + _BLOCK - 1) // _BLOCK)
    row = H * d
    out = np.empty((B, rows * row), np.uint16 if bf16 else np.float32)

    def part(b, i, lo, hi):
        m = min(_BLOCK, n - i * _BLOCK)
        blk = np.empty(m, out.dtype)
        _draw(children[i], m, scale, bf16, blk, 0)
        a, z = max(lo, i * _BLOCK), min(hi, i * _BLOCK + m)
        out[b, a - lo:z - lo] = blk[a - i * _BLOCK:z - i * _BLOCK]

    with ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1)) as ex:
        futs = []
        for b in range(B):
            lo, hi = (b * N + row0) * row, (b * N + row0 + rows) * row
            futs += [ex.submit(part, b, i, lo, hi) for i in range(lo // _BLOCK, (hi + _BLOCK - 1) // _BLOCK)]
        for f in futs:
            f.result()
    return out.reshape(B, rows, H, d)


def make_shard_inputs(B: int, N: int, H: int, d: int, seed: int, row0: int, rows: int, bf16: bool = True,
                      decayed: bool = True, with_grad: bool = True) -> dict:
    """:func:`make_inputs` restricted to the token rows row0 .. row0 + rows - 1
    of every sequence (one rank's shard in sequence parallelism)."""
    out = {}
    for i, name in enumerate(_NAMES):
        if name == "do" and not with_grad:
            continue
        scale = 1.0 if name == "do" else float(d) ** -0.5
        out[name] = draw_tensor_rows(seed, i, (B, N, H, d), scale, bf16, row0, rows)
    out["lam"] = decay_rates(H) if decayed else None
    out["bf16"] = bf16
    return out


def make_log_gates(B: int, N: int, H: int, d: int, seed: int, tau: float = 16.0) -> np.ndarray:
    """Log-gates log(sigmoid(x)) / tau, float32 [B, N, H, d], x from stream 4 of ``seed``."""
    shape = (B, N, H, d)
    n = int(np.prod(shape))
    stream = np.random.SeedSequence(seed).spawn(len(_NAMES) + 1)[len(_NAMES)]
    nblk = (n + _BLOCK - 1) // _BLOCK
    out = np.empty(n, np.float32)
    for i, child in enumerate(stream.spawn(nblk)):
        m = min(_BLOCK, n - i * _BLOCK)
        x = np.random.Generator(np.random.PCG64(child)).standard_normal(m, dtype=np.float64)
        out[i * _BLOCK:i * _BLOCK + m] = (-np.logaddexp(0.0, -x) / tau).astype(np.float32)
    return out.reshape(shape)


def make_inputs(B: int, N: int, H: int, d: int, seed: int, bf16: bool = True,
                decayed: bool = True, with_grad: bool = True) -> dict:
    """q, k, v (and dO) in the [B, N, H, d] token-major layout, plus lambda [H] or None.

    bf16 workloads return uint16 bit patterns; fp32 workloads return float32.
    """
    shape = (B, N, H, d)
    out = {}
    for i, name in enumerate(_NAMES):
        if name == "do" and not with_grad:
            continue
        scale = 1.0 if name == "do" else float(d) ** -0.5
        out[name] = draw_tensor(seed, i, shape, scale, bf16)
    out["lam"] = decay_rates(H) if decayed else None
    out["bf16"] = bf16
    return out


def make_attention_inputs(B: int, Nq: int, Nk: int, H: int, d: int, seed: int, bf16: bool = True) -> dict:
    """Inputs of a softmax-attention layer: q and dO [B, Nq, H, d], k and v
    [B, Nk, H, d], i.i.d. standard normal (the layer's own scale, d^-1/2 by
    default, multiplies the scores), drawn like :func:`make_inputs` from the
    streams of ``seed`` (q, k, v, dO), rounded to bf16 for bf16 workloads."""
    out = {"q": draw_tensor(seed, 0, (B, Nq, H, d), 1.0, bf16), "k": draw_tensor(seed, 1, (B, Nk, H, d), 1.0, bf16),
           "v": draw_tensor(seed, 2, (B, Nk, H, d), 1.0, bf16), "do": draw_tensor(seed, 3, (B, Nq, H, d), 1.0, bf16),
           "bf16": bf16}
    return out


def as_f32(x: np.ndarray, bf16: bool) -> np.ndarray:
    """The float32 values a tensor from :func:`make_inputs` holds."""
    return bf16_bits_to_f32(x) if bf16 else np.ascontiguousarray(x, dtype=np.float32)


# The five workloads, by what they are. Seeds are 1000 + position in this list.
WORKLOADS = {
    "tiny_fp32": dict(B=1, H=2, N=256, d=32, C=64, bf16=False, decayed=False, seed=1000),
    "basic_bf16_N8K": dict(B=4, H=16, N=8192, d=128, C=64, bf16=True, decayed=False, seed=1001),
    "decayed_bf16_N64K": dict(B=1, H=16, N=65536, d=128, C=128, bf16=True, decayed=True, seed=1002),
    "long_bf16_N1M": dict(B=1, H=16, N=1048576, d=128, C=128, bf16=True, decayed=False, seed=1003),
    "shards_bf16_N2M": dict(B=1, H=8, N=2097152, d=128, C=128, bf16=True, decayed=True, seed=1004,
                            W=64),
}
