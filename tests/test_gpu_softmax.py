"""The softmax-attention layers of a hybrid model (LASP-2 review page,
"Summary": LASP-2H applies the AllGather pattern to standard attention,
gathering K_t and V_t) through the C ABI against the fp64 oracle: o, lse and
the gradients dq, dk, dv, on one sequence (q_offset = 0) and on a block of
queries against gathered keys (q_offset > 0), with ragged tiles. Tolerance
max|gpu - ref| / max|ref| <= 2e-2 per tensor (bf16 inputs, fp32 accumulation),
as for the linear-attention path."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import TOL_BF16, rel_err, to_device, to_host

pytestmark = pytest.mark.gpu


def _run(inp, q_offset, scale=None, backward=True):
    import torch
    import sequence_linear_attention_b200 as lasp
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    B, Nq, H, d = q.shape
    o = torch.full_like(q, float("nan"))
    lse = torch.full((B, H, Nq), float("nan"), dtype=torch.float32, device="cuda")
    lasp.lasp_softmax_fwd(q, k, v, o, lse, q_offset=q_offset, scale=scale)
    out = dict(o=o, lse=lse)
    if backward:
        dq = torch.full_like(q, float("nan"))
        dk, dv = torch.full_like(k, float("nan")), torch.full_like(v, float("nan"))
        delta = torch.empty_like(lse)
        lasp.lasp_softmax_bwd(q, k, v, o, lse, do, dq, dk, dv, delta, q_offset=q_offset, scale=scale)
        out.update(dq=dq, dk=dk, dv=dv)
    st, site = lasp.lasp_check_device_status()
    assert st == 0, (st, site)
    return {n: (to_host(t) if t.dtype != torch.float32 else t.cpu().numpy()) for n, t in out.items()}


def _reference(inp, q_offset, scale=None, backward=True):
    f = {n: lasp_inputs.as_f32(inp[n], True) for n in ("q", "k", "v", "do")}
    o, lse = oracle.softmax_fwd(f["q"], f["k"], f["v"], q_offset=q_offset, scale=scale)
    ref = dict(o=o, lse=lse)
    if backward:
        ref["dq"], ref["dk"], ref["dv"] = oracle.softmax_bwd(f["q"], f["k"], f["v"], f["do"], q_offset=q_offset,
                                                             scale=scale)
    return ref


def _compare(got, ref, names):
    errs = {n: rel_err(got[n], ref[n]) for n in names}
    assert all(np.isfinite(list(errs.values()))), errs
    bad = {n: e for n, e in errs.items() if not e <= TOL_BF16}
    assert not bad, f"errors above {TOL_BF16}: {bad} (all: {errs})"


CASES = [
    # (B, H, Nq, Nk, q_offset): one sequence, then query blocks against gathered keys
    (1, 2, 128, 128, 0),     # one tile
    (2, 3, 384, 384, 0),     # several tiles
    (1, 2, 320, 320, 0),     # ragged last tile
    (1, 1, 1, 1, 0),         # a single token
    (1, 2, 1536, 1536, 0),   # twelve key tiles per late query tile
    (1, 2, 256, 640, 384),   # a rank's queries against the keys of all ranks up to its own
    (2, 2, 300, 500, 200),   # offset and sizes off the tile grid
    (1, 2, 128, 1024, 128),  # keys beyond the last query: never attended, zero gradients
]


@pytest.mark.parametrize("B,H,Nq,Nk,q_offset", CASES)
def test_softmax_attention_matches_oracle(B, H, Nq, Nk, q_offset):
    inp = lasp_inputs.make_attention_inputs(B, Nq, Nk, H, 128, seed=6000 + Nq + Nk + q_offset)
    got = _run(inp, q_offset)
    ref = _reference(inp, q_offset)
    _compare(got, ref, ("o", "lse", "dq", "dk", "dv"))
    if Nk > q_offset + Nq:
        assert not np.any(got["dk"][:, q_offset + Nq:]) and not np.any(got["dv"][:, q_offset + Nq:])


def test_growing_scores_rescale_the_running_output():
    """Keys scaled up along the sequence: each later key tile holds larger
    scores than any before, so every row's running maximum keeps growing and
    the kernel rescales O in TMEM many times."""
    B, H, N = 1, 2, 1024
    inp = lasp_inputs.make_attention_inputs(B, N, N, H, 128, seed=6100)
    k = lasp_inputs.as_f32(inp["k"], True) * (1.0 + np.arange(N, dtype=np.float32) / 64.0)[None, :, None, None]
    inp["k"] = lasp_inputs.f32_to_bf16_bits(k)
    got = _run(inp, 0)
    ref = _reference(inp, 0)
    _compare(got, ref, ("o", "lse", "dq", "dk", "dv"))


def test_scale_argument():
    inp = lasp_inputs.make_attention_inputs(1, 256, 256, 2, 128, seed=6200)
    got = _run(inp, 0, scale=0.3)
    ref = _reference(inp, 0, scale=0.3)
    _compare(got, ref, ("o", "lse", "dq", "dk", "dv"))


def test_shards_equal_the_whole_sequence():
    """LASP-2H on one device: the queries of each of W shards against the
    keys gathered up to the shard's end give the rows of the whole-sequence
    call, and the shards' dk, dv summed over the shards give its dk, dv."""
    B, H, W, L = 1, 2, 4, 256
    N = W * L
    inp = lasp_inputs.make_attention_inputs(B, N, N, H, 128, seed=6300)
    whole = _run(inp, 0)
    dk = np.zeros_like(whole["dk"], dtype=np.float64)
    dv = np.zeros_like(dk)
    for r in range(W):
        sl = slice(r * L, (r + 1) * L)
        part = dict(inp, q=np.ascontiguousarray(inp["q"][:, sl]), do=np.ascontiguousarray(inp["do"][:, sl]))
        got = _run(part, r * L)
        for n in ("o", "dq"):
            assert rel_err(got[n], whole[n][:, sl]) <= TOL_BF16, (r, n)
        assert rel_err(got["lse"], whole["lse"][:, :, sl]) <= 1e-5, r
        dk += got["dk"]
        dv += got["dv"]
    assert rel_err(dk, whole["dk"]) <= TOL_BF16
    assert rel_err(dv, whole["dv"]) <= TOL_BF16


def test_unsupported_and_invalid_sizes():
    import torch
    import sequence_linear_attention_b200 as lasp
    q = torch.zeros((1, 128, 2, 64), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, 2, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(lasp.LaspError) as e:
        lasp.lasp_softmax_fwd(q, q, q, q, lse)
    assert e.value.status == 2  # d = 64: unsupported
    q = torch.zeros((1, 128, 2, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((1, 100, 2, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lasp.LaspError) as e:
        lasp.lasp_softmax_fwd(q, k, k, q, lse)
    assert e.value.status == 1  # the queries reach past the keys


def test_bench_size_sampled_rows_and_sums():
    """The bench configuration (B1 H16 N65536 d128, causal, standard-normal
    inputs) as bench.py --softmax runs it. The oracle checks sampled query
    rows of o, lse and dq of two heads (a block of rows at its offset into the
    keys), and dk, dv for their last 128 keys (every query that sees them lies
    in the block of the last 128 queries). Over all keys two sums hold exactly:
    sum_j dv_j = sum_i do_i (each row of attention weights sums to 1) and
    sum_j dk_j = 0 (each row of ds sums to 0), per head and feature."""
    import torch
    import sequence_linear_attention_b200 as lasp
    w = lasp_inputs.WORKLOADS["decayed_bf16_N64K"]
    B, N, H, d = w["B"], w["N"], w["H"], w["d"]
    inp = lasp_inputs.make_attention_inputs(B, N, N, H, d, seed=w["seed"])
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    delta = torch.empty_like(lse)
    lasp.lasp_softmax_fwd(q, k, v, o, lse)
    lasp.lasp_softmax_bwd(q, k, v, o, lse, do, dq, dk, dv, delta)
    st, site = lasp.lasp_check_device_status()
    assert st == 0, (st, site)
    f = {n: lasp_inputs.as_f32(inp[n], True) for n in ("q", "k", "v", "do")}
    go, gdq, gdk, gdv = (to_host(t) for t in (o, dq, dk, dv))
    glse = lse.cpu().numpy()
    heads = [5, 12]  # two sampled heads for the oracle (its cost grows with N^2 per head)
    hk, hv = f["k"][:, :, heads], f["v"][:, :, heads]
    tail = 128
    # query blocks at the start, in the middle (off the tile grid) and at the end
    for r0, n in ((0, 96), (30001, 64), (N - tail, tail)):
        qs = np.ascontiguousarray(f["q"][:, r0:r0 + n][:, :, heads])
        dos = np.ascontiguousarray(f["do"][:, r0:r0 + n][:, :, heads])
        ro, rl = oracle.softmax_fwd(qs, hk, hv, q_offset=r0)
        assert rel_err(go[:, r0:r0 + n][:, :, heads], ro) <= TOL_BF16, r0
        assert rel_err(glse[:, heads, r0:r0 + n], rl) <= TOL_BF16, r0
        if r0 == N - tail:
            rdq, rdk, rdv = oracle.softmax_bwd(qs, hk, hv, dos, q_offset=r0)
            assert rel_err(gdq[:, r0:][:, :, heads], rdq) <= TOL_BF16
            assert rel_err(gdk[:, r0:][:, :, heads], rdk[:, r0:]) <= TOL_BF16
            assert rel_err(gdv[:, r0:][:, :, heads], rdv[:, r0:]) <= TOL_BF16
    # every head: the sums over all keys
    sdv = gdv.astype(np.float64).sum(axis=1)
    sdo = f["do"].astype(np.float64).sum(axis=1)
    assert rel_err(sdv, sdo) <= TOL_BF16
    # sum_j dk_j = 0: against the size of the terms it sums
    sdk = np.abs(gdk.astype(np.float64).sum(axis=1))
    assert float(sdk.max()) <= TOL_BF16 * float(np.abs(gdk).sum(axis=1).max())
