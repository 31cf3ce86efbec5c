"""LASP-2H on the device: W processes share one GPU, each holds one shard of
the sequence and runs ``lasp2h_fwd`` / ``lasp2h_bwd`` with the library's
softmax-attention kernels; K, V and the partial dK, dV cross between them over
gloo on the host (no kernel of one process waits on another's). Their shards
put together must equal the single-device call over the whole sequence and
the oracle, at the bf16 bar."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

from gpu_helpers import TOL_BF16, rel_err, to_device, to_host

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

# (W, B, L, H): bf16, d = 128; shards of whole tiles and of ragged ones
CASES = {"W2": (2, 1, 512, 2), "W3_ragged": (3, 2, 200, 2)}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(name):
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    W, B, L, H = CASES[name]
    return lasp_inputs.make_attention_inputs(B, W * L, W * L, H, 128, seed=3800 + sorted(CASES).index(name))


def _worker(rank, name, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    import sequence_linear_attention_b200 as lasp
    from sequence_linear_attention_b200 import lasp2h
    W, B, L, H = CASES[name]
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs(name)
        sl = slice(rank * L, (rank + 1) * L)
        q, k, v, do = (to_device(np.ascontiguousarray(inp[n][:, sl]), True) for n in ("q", "k", "v", "do"))
        o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
        lse = torch.empty((B, H, L), dtype=torch.float32, device="cuda")
        k_all, v_all = lasp2h.gathered_like(k), lasp2h.gathered_like(v)
        lasp2h.lasp2h_fwd(q, k, v, o, lse, k_all, v_all)
        lasp2h.lasp2h_bwd(q, o, lse, do, dq, dk, dv, k_all, v_all)
        st, site = lasp.lasp_check_device_status()
        out[rank] = dict(status=st, **{n: to_host(t) for n, t in dict(o=o, dq=dq, dk=dk, dv=dv).items()})
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
@pytest.mark.parametrize("name", sorted(CASES))
def test_shards_on_one_gpu_equal_the_whole_sequence(name):
    import torch

    import oracle
    import sequence_linear_attention_b200 as lasp
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    W, B, L, H = CASES[name]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(name, _free_port(), out), nprocs=W, join=True, start_method="spawn")
        res = dict(out)
    inp = _inputs(name)
    q, k, v, do = (to_device(inp[n], True) for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    lse = torch.empty((B, H, W * L), dtype=torch.float32, device="cuda")
    delta = torch.empty_like(lse)
    lasp.lasp_softmax_fwd(q, k, v, o, lse)
    lasp.lasp_softmax_bwd(q, k, v, o, lse, do, dq, dk, dv, delta)
    whole = {n: to_host(t) for n, t in dict(o=o, dq=dq, dk=dk, dv=dv).items()}
    f = {n: lasp_inputs.as_f32(inp[n], True) for n in ("q", "k", "v", "do")}
    ref = dict(o=oracle.softmax_fwd(f["q"], f["k"], f["v"])[0])
    ref["dq"], ref["dk"], ref["dv"] = oracle.softmax_bwd(f["q"], f["k"], f["v"], f["do"])
    for r in range(W):
        assert res[r]["status"] == 0, r
        sl = slice(r * L, (r + 1) * L)
        for n in ("o", "dq", "dk", "dv"):
            assert rel_err(res[r][n], ref[n][:, sl]) <= TOL_BF16, (r, n)
            assert rel_err(res[r][n], whole[n][:, sl]) <= TOL_BF16, (r, n)
