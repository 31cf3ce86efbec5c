"""The five workloads at their full sizes, on the GPU, against the oracle.

Where the whole oracle would take too long (tens of billions of fp64 FLOPs per
head), the comparison samples whole heads: every output of the sampled (b, h)
pairs is compared, over the full sequence, together with the states P and R
of those heads at every chunk."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import decay_device, rel_err, run_fwd_bwd, run_states, to_device, to_host, tol

pytestmark = pytest.mark.gpu
W = lasp_inputs.WORKLOADS


def _head(inp, name, b, h):
    x = inp[name][b:b + 1, :, h:h + 1, :]
    return lasp_inputs.as_f32(np.ascontiguousarray(x), inp["bf16"])


def _check_heads(inp, gpu, C, heads):
    bf16 = inp["bf16"]
    errs = {}
    for b, h in heads:
        q, k, v, do = (_head(inp, n, b, h) for n in ("q", "k", "v", "do"))
        lam = None if inp["lam"] is None else inp["lam"][h:h + 1]
        ref = dict(o=oracle.fwd(q, k, v, lam))
        ref["dq"], ref["dk"], ref["dv"] = oracle.bwd(q, k, v, do, lam)
        ref["P"] = oracle.state_snapshots(k, v, lam, C, kind=0)
        ref["R"] = oracle.state_snapshots(q, do, lam, C, kind=1)
        for n, r in ref.items():
            g = gpu[n][b:b + 1, :, h:h + 1]
            errs[(b, h, n)] = rel_err(to_host(g), r)
    bad = {k: e for k, e in errs.items() if not e <= tol(bf16)}
    assert not bad, f"above {tol(bf16)}: {bad}"
    return errs


def _run(name, heads):
    w = W[name]
    inp = lasp_inputs.make_inputs(w["B"], w["N"], w["H"], w["d"], seed=w["seed"], bf16=w["bf16"],
                                  decayed=w["decayed"])
    gpu = run_fwd_bwd(inp, w["C"])
    # P_c and R_c through the state entry points, into the (now free) cache and workspace
    gpu.update(run_states(inp, w["C"], gpu["P"], gpu["R"]))
    return _check_heads(inp, gpu, w["C"], heads)


def test_tiny_fp32_all_heads():
    _run("tiny_fp32", [(0, 0), (0, 1)])


def test_basic_bf16_N8K_sampled_heads():
    _run("basic_bf16_N8K", [(0, 0), (1, 7), (3, 15)])


def test_decayed_bf16_N64K_sampled_heads():
    # the most and the least decayed heads
    _run("decayed_bf16_N64K", [(0, 0), (0, 15)])


def test_long_bf16_N1M_sampled_head():
    _run("long_bf16_N1M", [(0, 5)])


def test_shards_bf16_N2M_split_equals_unsplit():
    """LASP-2 on one GPU: W shards of L tokens. Shard states with C = L, an
    exclusive prefix over the shards, then each shard's forward with its
    entering state; the result equals the unsplit forward. A sampled head of
    two shards is also checked against the oracle."""
    import torch
    import sequence_linear_attention_b200 as lasp
    w = W["shards_bf16_N2M"]
    B, N, H, d, C, Wn = w["B"], w["N"], w["H"], w["d"], w["C"], w["W"]
    L = N // Wn
    inp = lasp_inputs.make_inputs(B, N, H, d, seed=w["seed"], bf16=True, decayed=True, with_grad=False)
    q, k, v = (to_device(inp[n], True) for n in ("q", "k", "v"))
    decay = decay_device(inp["lam"])
    o_full = torch.empty_like(q)
    cache = torch.empty((B, N // C, H, d, d), dtype=torch.float32, device="cuda")
    lasp.lasp_fwd(q, k, v, decay, o_full, C, cache)
    shard_states = torch.empty((B, Wn, H, d, d), dtype=torch.float32, device="cuda")
    lasp.lasp_chunk_states(None, k, v, decay, shard_states, L)
    lasp.lasp_state_prefix(shard_states, shard_states, decay, L)  # E_w, in place
    o_split = torch.empty_like(q)
    view = lambda t: t.view(B * Wn, L, H, d)
    lasp.lasp_fwd(view(q), view(k), view(v), decay, view(o_split), C, cache.view(B * Wn, L // C, H, d, d),
                  init_state=shard_states.view(B * Wn, H, d, d))
    st, _ = lasp.lasp_check_device_status()
    assert st == 0
    # split vs unsplit, compared on the device in fp32, one head at a time
    for h in range(H):
        a, b = o_split[:, :, h].float(), o_full[:, :, h].float()
        assert float((a - b).abs().max() / b.abs().max()) <= tol(True), h
    # sampled head against the oracle: shard states, prefix, local forward
    h = 3
    qh, kh, vh = (_head(inp, n, 0, h) for n in ("q", "k", "v"))
    lam = inp["lam"][h:h + 1]
    E, _ = oracle.state_scan(oracle.chunk_states(kh, vh, lam, L, 0), lam, L)
    assert rel_err(to_host(shard_states[:, :, h:h + 1]), E) <= tol(True)
    for s in (1, Wn - 1):
        sl = slice(s * L, (s + 1) * L)
        ref = oracle.fwd(np.ascontiguousarray(qh[:, sl]), np.ascontiguousarray(kh[:, sl]),
                         np.ascontiguousarray(vh[:, sl]), lam, init=E[:, s])
        assert rel_err(to_host(o_split[:, sl, h:h + 1]), ref) <= tol(True), s
