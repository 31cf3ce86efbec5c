"""LASP-2H (the softmax-attention layers under LASP-2's sequence split), the
rank logic on CPU: gloo ranks each hold one shard, gather K and V, and run
``lasp2h_fwd`` / ``lasp2h_bwd`` with the oracle in place of the device
kernels. Their shards put together must equal the oracle's whole-sequence
attention and gradients (dk, dv summed over the ranks by the reduce-scatter),
for W = 2 and 3, B = 1 and 2. A wrong query offset, a gather into the wrong
rows or a missing reduction fails it."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (W, B, L, H, d)
CASES = [(2, 1, 12, 2, 8), (3, 2, 8, 1, 4), (2, 2, 5, 3, 8)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case_inputs(i, W, B, L, H, d):
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    return lasp_inputs.make_attention_inputs(B, W * L, W * L, H, d, seed=3700 + i, bf16=False)


class _OracleKernels:
    @staticmethod
    def fwd(q, k_all, v_all, o, lse, q_offset, scale):
        import oracle
        import torch
        ro, rl = oracle.softmax_fwd(q.numpy(), k_all.numpy(), v_all.numpy(), q_offset=q_offset, scale=scale)
        o.copy_(torch.from_numpy(ro))
        lse.copy_(torch.from_numpy(rl))

    @staticmethod
    def bwd(q, k_all, v_all, o, lse, dout, dq, dk_all, dv_all, delta, q_offset, scale):
        import oracle
        import torch
        rdq, rdk, rdv = oracle.softmax_bwd(q.numpy(), k_all.numpy(), v_all.numpy(), dout.numpy(),
                                           q_offset=q_offset, scale=scale)
        dq.copy_(torch.from_numpy(rdq))
        dk_all.copy_(torch.from_numpy(rdk))
        dv_all.copy_(torch.from_numpy(rdv))


def _worker(rank, i, W, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch
    import torch.distributed as dist

    from sequence_linear_attention_b200 import lasp2h
    _, B, L, H, d = CASES[i]
    dist.init_process_group("gloo", rank=rank, world_size=W, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _case_inputs(i, *CASES[i])
        sl = slice(rank * L, (rank + 1) * L)
        q, k, v, do = (torch.from_numpy(np.ascontiguousarray(inp[n][:, sl])) for n in ("q", "k", "v", "do"))
        o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
        lse = torch.empty((B, H, L), dtype=torch.float32)
        k_all, v_all = lasp2h.gathered_like(k), lasp2h.gathered_like(v)
        lasp2h.lasp2h_fwd(q, k, v, o, lse, k_all, v_all, kernels=_OracleKernels)
        lasp2h.lasp2h_bwd(q, o, lse, do, dq, dk, dv, k_all, v_all, kernels=_OracleKernels)
        out[rank] = {n: t.numpy().copy() for n, t in dict(o=o, lse=lse, dq=dq, dk=dk, dv=dv).items()}
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("i", range(len(CASES)))
def test_shards_equal_the_whole_sequence(i):
    import oracle
    W, B, L, H, d = CASES[i]
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(i, W, _free_port(), out), nprocs=W, join=True, start_method="spawn")
        res = dict(out)
    inp = _case_inputs(i, *CASES[i])
    o, lse = oracle.softmax_fwd(inp["q"], inp["k"], inp["v"])
    dq, dk, dv = oracle.softmax_bwd(inp["q"], inp["k"], inp["v"], inp["do"])
    for r in range(W):
        sl = slice(r * L, (r + 1) * L)
        np.testing.assert_allclose(res[r]["o"], o[:, sl], rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(res[r]["lse"], lse[:, :, sl], rtol=1e-5, atol=1e-6)
        for n, ref in (("dq", dq), ("dk", dk), ("dv", dv)):
            np.testing.assert_allclose(res[r][n], ref[:, sl], rtol=1e-5, atol=1e-6, err_msg=f"rank {r} {n}")
