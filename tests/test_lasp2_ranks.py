"""LASP-2 sequence parallelism, the rank logic on CPU: gloo ranks each hold one
shard of the sequence and run ``lasp2_fwd`` / ``lasp2_bwd`` with the oracle in
place of the device kernels. Their shards, put together, must equal the
oracle's forward and backward over the whole sequence, with the initial state,
the final state and both boundary gradients, for W = 2 and W = 3, B = 1 and 2,
decayed and undecayed. This pins which gathered states enter which shard, the
direction of each scan and the per-head decays of a multi-sequence batch, with
the (b, h) pairs exchanged in one part, two, and one part per pair; the
device kernels themselves have their own parity tests."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (W, B, L, H, d, decayed, boundary states)
CASES = [
    (2, 1, 32, 2, 8, True, True),
    (2, 2, 24, 3, 8, False, False),
    (3, 2, 16, 2, 4, True, True),
    (3, 1, 8, 1, 4, True, False),
]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _case_inputs(i, W, B, L, H, d, decayed, boundary):
    from sequence_linear_attention_b200 import inputs as lasp_inputs
    inp = lasp_inputs.make_inputs(B, W * L, H, d, seed=3100 + i, bf16=False, decayed=decayed)
    rng = np.random.default_rng(3200 + i)
    init = (rng.standard_normal((B, H, d, d)) * 0.3).astype(np.float32) if boundary else None
    dsin = (rng.standard_normal((B, H, d, d)) * 0.3).astype(np.float32) if boundary else None
    return inp, init, dsin


class _OracleKernels:
    """The five kernel calls of the LASP-2 module, done by the oracle on CPU
    tensors, each writing only the (b, h) pairs of its part. The
    single-device forward keeps its initial state in the state cache, which is
    what the backward needs from it."""

    @staticmethod
    def _lam(decay):
        return None if decay is None else decay.double().numpy()

    @staticmethod
    def _pairs(B, H, part, nparts):
        return [(bh // H, bh % H) for bh in range(B * H * part // nparts, B * H * (part + 1) // nparts)]

    @classmethod
    def _states(cls, x, y, decay, M, kind, part, nparts):
        import oracle
        import torch
        B, L, H, _ = x.shape
        full = torch.from_numpy(oracle.chunk_states(x.numpy(), y.numpy(), cls._lam(decay), L, kind)[:, 0])
        for b, h in cls._pairs(B, H, part, nparts):
            M[b, h] = full[b, h]

    @classmethod
    def shard_state(cls, k, v, decay, M, C, scratch, part, nparts):
        cls._states(k, v, decay, M, 0, part, nparts)

    @classmethod
    def shard_dstate(cls, q, dout, decay, dM, C, scratch, part, nparts):
        cls._states(q, dout, decay, dM, 1, part, nparts)

    @classmethod
    def state_prefix(cls, M, out, decay, L, init, total, reverse):
        import oracle
        import torch
        P, tot = oracle.state_scan(M.double().numpy(), cls._lam(decay), L,
                                   init=None if init is None else init.double().numpy(), reverse=reverse)
        out.copy_(torch.from_numpy(P))
        if total is not None:
            total.copy_(torch.from_numpy(tot))

    @classmethod
    def fwd(cls, q, k, v, decay, o, C, state_cache, init_state, part, nparts):
        import oracle
        import torch
        B, L, H, _ = q.shape
        # pairs of later parts hold no entering state yet: zeros stand in, and
        # only this part's pairs are written
        init = torch.zeros_like(init_state)
        pairs = cls._pairs(B, H, part, nparts)
        for b, h in pairs:
            init[b, h] = init_state[b, h]
        full = torch.from_numpy(oracle.fwd(q.numpy(), k.numpy(), v.numpy(), cls._lam(decay),
                                           init=init.double().numpy()))
        for b, h in pairs:
            o[b, :, h] = full[b, :, h]
            state_cache[b, h] = init_state[b, h]

    @classmethod
    def bwd(cls, q, k, v, decay, dout, dq, dk, dv, C, state_cache, dstate_ws, dstate_in, part, nparts):
        import oracle
        import torch
        B, L, H, _ = q.shape
        pairs = cls._pairs(B, H, part, nparts)
        din = torch.zeros_like(dstate_in)
        for b, h in pairs:
            din[b, h] = dstate_in[b, h]
        g = oracle.bwd(q.numpy(), k.numpy(), v.numpy(), dout.numpy(), cls._lam(decay),
                       init=state_cache.double().numpy(), dstate_in=din.double().numpy())
        for t, x in zip((dq, dk, dv), g):
            for b, h in pairs:
                t[b, :, h] = torch.from_numpy(x)[b, :, h]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    from sequence_linear_attention_b200 import lasp2
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        for i, (W, B, L, H, d, decayed, boundary) in enumerate(CASES):
            if W != world:
                continue
            inp, init, dsin = _case_inputs(i, W, B, L, H, d, decayed, boundary)
            sl = slice(rank * L, (rank + 1) * L)
            q, k, v, do = (torch.from_numpy(np.ascontiguousarray(inp[n][:, sl])) for n in ("q", "k", "v", "do"))
            decay = None if inp["lam"] is None else torch.from_numpy(np.asarray(inp["lam"], np.float32))
            init_t = None if init is None else torch.from_numpy(init)
            dsin_t = None if dsin is None else torch.from_numpy(dsin)
            for parts in sorted({1, min(2, B * H), B * H}):
                o, dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(4))
                cache = torch.empty((B, H, d, d), dtype=torch.float32)
                final = torch.empty((B, H, d, d), dtype=torch.float32)
                dinit = torch.empty((B, H, d, d), dtype=torch.float32)
                entering = lasp2.lasp2_fwd(q, k, v, decay, o, L, cache, init_state=init_t, final_state=final,
                                           kernels=_OracleKernels, parts=parts)
                incoming = lasp2.lasp2_bwd(q, k, v, decay, do, dq, dk, dv, L, cache, None, dstate_in=dsin_t,
                                           dinit_state=dinit, kernels=_OracleKernels, parts=parts)
                out[(i, rank, parts)] = {n: t.numpy().copy() for n, t in dict(
                    o=o, dq=dq, dk=dk, dv=dv, final=final, dinit=dinit, entering=entering,
                    incoming=incoming).items()}
    finally:
        dist.destroy_process_group()


def _run_world(world):
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                           start_method="spawn")
        return dict(out)


def _rel(got, ref):
    den = float(np.max(np.abs(ref)))
    num = float(np.max(np.abs(got - ref)))
    return num / den if den > 0 else num


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
def test_shards_equal_the_whole_sequence(world):
    sys.path.insert(0, ROOT)
    import oracle
    res = _run_world(world)
    ran = 0
    for i, (W, B, L, H, d, decayed, boundary) in enumerate(CASES):
        if W != world:
            continue
        ran += 1
        inp, init, dsin = _case_inputs(i, W, B, L, H, d, decayed, boundary)
        q, k, v, do, lam = inp["q"], inp["k"], inp["v"], inp["do"], inp["lam"]
        o, final = oracle.fwd(q, k, v, lam, init=init, want_final=True)
        dq, dk, dv, dinit = oracle.bwd(q, k, v, do, lam, init=init, dstate_in=dsin, want_dinit=True)
        # states at the shard boundaries: entering shard r (after token rL - 1)
        # and the gradient entering shard r's last token from the tokens after it
        S = oracle.state_snapshots(k, v, lam, L, init=init, kind=0)
        G = oracle.state_snapshots(q, do, lam, L, init=dsin, kind=1)
        for r, parts in ((r, p) for r in range(W) for p in sorted({1, min(2, B * H), B * H})):
            got = res[(i, r, parts)]
            sl = slice(r * L, (r + 1) * L)
            for name, ref in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
                assert _rel(got[name], ref[:, sl]) <= 1e-5, (i, r, name)
            assert _rel(got["final"], final) <= 1e-5, (i, r)
            assert _rel(got["dinit"], dinit) <= 1e-5, (i, r)
            assert _rel(got["entering"], S[:, r]) <= 1e-5, (i, r)
            assert _rel(got["incoming"], G[:, r]) <= 1e-5, (i, r, parts)
    assert ran >= 2
