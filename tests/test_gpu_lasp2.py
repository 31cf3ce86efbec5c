"""LASP-2 sequence parallelism on the device: W processes share one GPU, each
holds one shard of the sequence and runs ``lasp2_fwd`` / ``lasp2_bwd`` through
the library's kernels; the shard states cross between them over gloo on the
host (the kernels of different processes never wait on one another). Their
shards, put together, must equal the single-device forward and backward over
the whole sequence and the oracle's, together with the final state and the
gradient of the initial state."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from gpu_helpers import decay_device, rel_err, to_device, to_host, tol

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

# (W, B, L, H, d, C, bf16, decayed): the tensor-core walks (bf16, d = 128) and
# the CUDA-core path (fp32); decayed is True (the workloads' per-head rates),
# or one lambda for every head
CASES = {
    "bf16_W2": (2, 2, 1024, 4, 128, 128, True, True),
    "bf16_W2_lam0.5": (2, 1, 1024, 4, 128, 128, True, 0.5),
    "bf16_W3_C64": (3, 1, 512, 2, 128, 64, True, True),
    "f32_W2": (2, 1, 256, 2, 64, 64, False, True),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(name):
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    W, B, L, H, d, C, bf16, decayed = CASES[name]
    inp = lasp_inputs.make_inputs(B, W * L, H, d, seed=3300 + sorted(CASES).index(name), bf16=bf16,
                                  decayed=decayed is True)
    if decayed is not True:
        inp["lam"] = np.full(H, decayed, np.float32)
    rng = np.random.default_rng(3400 + sorted(CASES).index(name))
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    dsin = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32)
    return inp, init, dsin


def _worker(rank, name, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    import sequence_linear_attention_b200 as lasp
    from sequence_linear_attention_b200 import lasp2
    W, B, L, H, d, C, bf16, decayed = CASES[name]
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=datetime.timedelta(seconds=60))
    try:
        inp, init, dsin = _inputs(name)
        sl = slice(rank * L, (rank + 1) * L)
        q, k, v, do = (to_device(np.ascontiguousarray(inp[n][:, sl]), bf16) for n in ("q", "k", "v", "do"))
        decay = decay_device(inp["lam"])
        init_t, dsin_t = (torch.from_numpy(x).cuda() for x in (init, dsin))
        o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
        cache = torch.empty((B, L // C, H, d, d), dtype=torch.float32, device="cuda")
        ws = torch.empty_like(cache)
        final = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
        dinit = torch.empty_like(final)
        lasp2.lasp2_fwd(q, k, v, decay, o, C, cache, init_state=init_t, final_state=final)
        lasp2.lasp2_bwd(q, k, v, decay, do, dq, dk, dv, C, cache, ws, dstate_in=dsin_t, dinit_state=dinit)
        st, site = lasp.lasp_check_device_status()
        out[rank] = dict(status=st, **{n: to_host(t) for n, t in dict(
            o=o, dq=dq, dk=dk, dv=dv, final=final, dinit=dinit).items()})
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", sorted(CASES))
def test_shards_on_one_gpu_equal_the_whole_sequence(name):
    import torch

    import oracle
    import sequence_linear_attention_b200 as lasp
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    W, B, L, H, d, C, bf16, decayed = CASES[name]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(name, _free_port(), out), nprocs=W, join=True, start_method="spawn")
        res = dict(out)
    # the whole sequence on one device
    inp, init, dsin = _inputs(name)
    q, k, v, do = (to_device(inp[n], bf16) for n in ("q", "k", "v", "do"))
    decay = decay_device(inp["lam"])
    init_t, dsin_t = (torch.from_numpy(x).cuda() for x in (init, dsin))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    cache = torch.empty((B, W * L // C, H, d, d), dtype=torch.float32, device="cuda")
    ws = torch.empty_like(cache)
    dinit = torch.empty((B, H, d, d), dtype=torch.float32, device="cuda")
    lasp.lasp_fwd(q, k, v, decay, o, C, cache, init_state=init_t)
    lasp.lasp_bwd(q, k, v, decay, do, dq, dk, dv, C, cache, ws, init_state=init_t, dstate_in=dsin_t,
                  dinit_state=dinit)
    whole = {n: to_host(t) for n, t in dict(o=o, dq=dq, dk=dk, dv=dv, dinit=dinit).items()}
    # and in the oracle
    f = {n: lasp_inputs.as_f32(inp[n], bf16) for n in ("q", "k", "v", "do")}
    ro, rfinal = oracle.fwd(f["q"], f["k"], f["v"], inp["lam"], init=init, want_final=True)
    rdq, rdk, rdv, rdinit = oracle.bwd(f["q"], f["k"], f["v"], f["do"], inp["lam"], init=init, dstate_in=dsin,
                                       want_dinit=True)
    ref = dict(o=ro, dq=rdq, dk=rdk, dv=rdv)
    bar = tol(bf16)
    for r in range(W):
        got = res[r]
        assert got["status"] == 0, r
        sl = slice(r * L, (r + 1) * L)
        for n in ("o", "dq", "dk", "dv"):
            assert rel_err(got[n], ref[n][:, sl]) <= bar, (r, n)
            assert rel_err(got[n], whole[n][:, sl]) <= bar, (r, n)
        # states as every state of a bf16 run: the decays scale bf16 operands
        assert rel_err(got["final"], rfinal) <= bar, r
        assert rel_err(got["dinit"], rdinit) <= bar, r
        assert rel_err(got["dinit"], whole["dinit"]) <= bar, r
