"""Randomized parity: shapes, chunk sizes, dtypes, decays and entering states
drawn from a fixed seed across what the library accepts (d in {32, 64, 128}, C
dividing N, fp32 and bf16, per-head decays from 1e-3 to 1, init_state and
dstate_in on or off). Each draw runs lasp_fwd and lasp_bwd through the C ABI
and is compared with the fp64 oracle per tensor, max|gpu - ref| / max|ref| <=
1e-4 (fp32) or 2e-2 (bf16). The draws reach the segment walks, the per-chunk
tensor-core kernels and the CUDA-core kernels in combinations the hand-picked
cases do not list (LASP paper, section 3.2: the output and its gradients do not
depend on C; lambda is any predefined constant)."""
import numpy as np
import pytest

import oracle
from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import host_f32, rel_err, run_fwd_bwd, to_host, tol

pytestmark = pytest.mark.gpu

NCASES = 96


def _draw(i: int):
    rng = np.random.default_rng([20261202, i])
    bf16 = bool(rng.random() < 0.75)
    d = int(rng.choice([32, 64, 128]))
    C = int(rng.choice([16, 32, 64, 128, 256] if bf16 else [1, 8, 16, 32, 64, 128]))
    T = int(rng.integers(1, 9))
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 5))
    kind = str(rng.choice(["none", "mild", "strong"]))
    lam = {"none": np.ones(H), "mild": rng.uniform(0.9, 1.0, H),
           "strong": 10.0 ** rng.uniform(-3.0, 0.0, H)}[kind].astype(np.float32)
    init = (rng.standard_normal((B, H, d, d)) * 0.2).astype(np.float32) if rng.random() < 0.5 else None
    din = (rng.standard_normal((B, H, d, d)) * 0.2).astype(np.float32) if rng.random() < 0.5 else None
    return dict(B=B, H=H, N=C * T, d=d, C=C, bf16=bf16, kind=kind, lam=lam, init=init, din=din,
                seed=3000 + i)


def _name(i: int) -> str:
    c = _draw(i)
    return (f"{i}-{'bf16' if c['bf16'] else 'f32'}-B{c['B']}H{c['H']}N{c['N']}d{c['d']}C{c['C']}-{c['kind']}"
            f"{'-init' if c['init'] is not None else ''}{'-din' if c['din'] is not None else ''}")


@pytest.mark.parametrize("i", range(NCASES), ids=_name)
def test_random_shapes_against_oracle(i):
    c = _draw(i)
    inp = lasp_inputs.make_inputs(c["B"], c["N"], c["H"], c["d"], seed=c["seed"], bf16=c["bf16"], decayed=False)
    inp["lam"] = c["lam"]
    gpu = run_fwd_bwd(inp, c["C"], init=c["init"], dstate_in=c["din"], want_dinit=True)
    q, k, v, do = (host_f32(inp, n) for n in ("q", "k", "v", "do"))
    init = None if c["init"] is None else c["init"].astype(np.float64)
    din = None if c["din"] is None else c["din"].astype(np.float64)
    ref = dict(o=oracle.fwd(q, k, v, c["lam"], init=init))
    ref["dq"], ref["dk"], ref["dv"], ref["dinit"] = oracle.bwd(q, k, v, do, c["lam"], init=init, dstate_in=din,
                                                               want_dinit=True)
    errs = {n: rel_err(to_host(gpu[n]), ref[n]) for n in ("o", "dq", "dk", "dv", "dinit")}
    bad = {n: e for n, e in errs.items() if not e <= tol(c["bf16"])}
    assert not bad, f"errors above {tol(c['bf16'])}: {bad} (all: {errs})"


# ---------------------------------------------------------------- softmax attention (LASP-2H layers)
def _softmax_draw(i: int):
    rng = np.random.default_rng([20261203, i])
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    Nq = int(rng.integers(1, 513))
    q_offset = int(rng.choice([0, 0, int(rng.integers(1, 400))]))
    Nk = q_offset + Nq + int(rng.choice([0, 0, int(rng.integers(1, 300))]))
    scale = None if rng.random() < 0.5 else float(rng.uniform(0.03, 0.2))
    return B, H, Nq, Nk, q_offset, scale, 4000 + i


@pytest.mark.parametrize("i", range(24),
                         ids=lambda i: "{}-B{}H{}Nq{}Nk{}off{}".format(i, *_softmax_draw(i)[:5]))
def test_random_softmax_shapes_against_oracle(i):
    """Causal softmax attention (bf16, d = 128) with random query counts,
    offsets into the gathered keys, keys beyond the last query and scales."""
    from test_gpu_softmax import _compare, _reference, _run
    B, H, Nq, Nk, q_offset, scale, seed = _softmax_draw(i)
    inp = lasp_inputs.make_attention_inputs(B, Nq, Nk, H, 128, seed=seed)
    _compare(_run(inp, q_offset, scale=scale), _reference(inp, q_offset, scale=scale),
             ("o", "lse", "dq", "dk", "dv"))


# ---------------------------------------------------------------- gated form
def _gated_draw(i: int):
    rng = np.random.default_rng([20261204, i])
    bf16 = bool(rng.random() < 0.7)
    d = 128 if (bf16 and rng.random() < 0.7) else int(rng.choice([32, 64, 128]))
    C = int(rng.choice([16, 32, 64, 128]))
    # N a multiple of 128 (the tensor-core path for bf16, d = 128) or any multiple of C
    N = 128 * int(rng.integers(1, 13)) if rng.random() < 0.7 else C * int(rng.integers(1, 9))
    B, H = int(rng.integers(1, 3)), int(rng.integers(1, 4))
    tau = float(rng.choice([1.0, 2.0, 4.0, 16.0]))
    init = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32) if rng.random() < 0.5 else None
    din = (rng.standard_normal((B, H, d, d)) * 0.1).astype(np.float32) if rng.random() < 0.5 else None
    return dict(B=B, H=H, N=N, d=d, C=C, bf16=bf16, tau=tau, init=init, din=din, seed=5000 + i)


def _gated_name(i: int) -> str:
    c = _gated_draw(i)
    return f"{i}-{'bf16' if c['bf16'] else 'f32'}-B{c['B']}H{c['H']}N{c['N']}d{c['d']}C{c['C']}-tau{c['tau']:g}"


@pytest.mark.parametrize("i", range(32), ids=_gated_name)
def test_random_gated_shapes_against_oracle(i):
    """The gated form (a decay per token and key feature) with random shapes,
    chunk sizes, gate strengths (log sigmoid(x) / tau; tau = 1 reaches the exact
    fallback's range) and entering states."""
    from test_gpu_gla import _compare, _reference, _run
    c = _gated_draw(i)
    inp = lasp_inputs.make_inputs(c["B"], c["N"], c["H"], c["d"], seed=c["seed"], bf16=c["bf16"], decayed=False)
    g = lasp_inputs.make_log_gates(c["B"], c["N"], c["H"], c["d"], seed=c["seed"], tau=c["tau"])
    got = _run(inp, g, c["C"], init=c["init"], dstate_in=c["din"])
    ref = _reference(inp, g, init=None if c["init"] is None else c["init"].astype(np.float64),
                     dstate_in=None if c["din"] is None else c["din"].astype(np.float64))
    _compare(got, ref, tol(c["bf16"]))


# ---------------------------------------------------------------- bidirectional form
def _bidir_draw(i: int):
    rng = np.random.default_rng([20261205, i])
    return int(rng.integers(1, 3)), int(rng.integers(1, 6)), 128 * int(rng.integers(1, 33)), 6000 + i


@pytest.mark.parametrize("i", range(12), ids=lambda i: "{}-B{}H{}N{}".format(i, *_bidir_draw(i)[:3]))
def test_random_bidirectional_shapes_against_oracle(i):
    """The unmasked form (bf16, d = 128) on random batch, head and token counts
    (one to thirty-two 128-token tiles: one or several segments)."""
    from test_gpu_bidir import _check, _run
    B, H, N, seed = _bidir_draw(i)
    inp = lasp_inputs.make_inputs(B, N, H, 128, seed=seed, bf16=True, decayed=False)
    _check(_run(inp), inp)
