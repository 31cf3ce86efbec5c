"""The C-ABI library without a GPU: it loads, exports every entry point that
include/lasp.h declares, and rejects bad arguments on the host before any
launch (these calls never reach the device, so they run on a CPU-only host)."""
import ctypes
import os
import re

import pytest

import sequence_linear_attention_b200 as lasp
from sequence_linear_attention_b200 import build as lasp_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lasp.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
F32, BF16 = 0, 1
A = 1 << 20  # a fake, 16-byte aligned device address; validation never dereferences it


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"LASP_API\s+[\w\s\*]+?\b(lasp_\w+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    lasp_build.build()
    return lasp._load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert {"lasp_fwd", "lasp_bwd", "lasp_chunk_states", "lasp_state_prefix"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lasp.lasp_status_string(0) == "LASP_OK"
    assert lasp.lasp_status_string(5) == "LASP_ERR_TIMEOUT"
    assert lasp.lasp_status_string(99) == "LASP_ERR_UNKNOWN"
    assert lasp.lasp_version() >= 100


def _fwd(lib, q=A, k=A, v=A, decay=None, o=A, B=1, H=2, N=256, d=32, C=64, dt=F32, cache=A, init=None):
    return lib.lasp_fwd(q, k, v, decay, o, B, H, N, d, C, dt, cache, init, None)


def _bwd(lib, B=1, H=2, N=256, d=32, C=64, dt=BF16, ptrs=None):
    p = dict(q=A, k=A, v=A, decay=None, do=A, dq=A, dk=A, dv=A, cache=A, ws=A, init=None, din=None, dinit=None)
    p.update(ptrs or {})
    return lib.lasp_bwd(p["q"], p["k"], p["v"], p["decay"], p["do"], p["dq"], p["dk"], p["dv"], B, H, N, d, C, dt,
                        p["cache"], p["ws"], p["init"], p["din"], p["dinit"], None)


def test_fwd_rejects_bad_sizes(lib):
    assert _fwd(lib, N=250) == INVALID          # C does not divide N
    assert _fwd(lib, C=0) == INVALID
    assert _fwd(lib, B=0) == INVALID
    assert _fwd(lib, H=0) == INVALID
    assert _fwd(lib, N=-64) == INVALID
    assert _fwd(lib, d=96) == UNSUPPORTED
    assert _fwd(lib, d=256) == UNSUPPORTED
    assert _fwd(lib, dt=7) == INVALID
    assert _fwd(lib, B=70000) == UNSUPPORTED


def test_fwd_rejects_bad_pointers(lib):
    assert _fwd(lib, q=None) == INVALID
    assert _fwd(lib, cache=None) == INVALID
    assert _fwd(lib, o=A + 8) == MISALIGNED
    assert _fwd(lib, decay=A + 4) == MISALIGNED
    assert _fwd(lib, init=A + 2) == MISALIGNED


def test_empty_sequence_launches_nothing(lib):
    # N = 0 is valid and returns before touching the device (no GPU here)
    assert _fwd(lib, N=0) == OK
    assert _bwd(lib, N=0) == OK
    assert lib.lasp_chunk_states(None, A, A, None, A, 1, 2, 0, 64, 16, BF16, None) == OK


def test_bwd_rejects_bad_arguments(lib):
    assert _bwd(lib, ptrs={"ws": None}) == INVALID
    assert _bwd(lib, ptrs={"dk": A + 1}) == MISALIGNED
    assert _bwd(lib, ptrs={"dinit": A + 12}) == MISALIGNED
    assert _bwd(lib, N=100, C=64) == INVALID


def test_state_prefix_rejects_bad_arguments(lib):
    f = lib.lasp_state_prefix
    assert f(A, A, None, None, None, 1, 4, 2, 64, 128, 2, None) == INVALID   # reverse must be 0 or 1
    assert f(A, A, None, None, None, 1, -1, 2, 64, 128, 0, None) == INVALID
    assert f(A, A, None, None, None, 1, 4, 2, 48, 128, 0, None) == UNSUPPORTED
    assert f(None, A, None, None, None, 1, 4, 2, 64, 128, 0, None) == INVALID
    assert f(A, A, None, None, None, 1, 4, 2, 64, 0, 0, None) == INVALID
    assert f(A, A + 4, None, None, None, 1, 4, 2, 64, 128, 0, None) == MISALIGNED
    assert f(None, None, None, None, None, 1, 0, 2, 64, 128, 0, None) == OK  # T = 0, nothing to write


def test_chunk_states_rejects_bad_arguments(lib):
    f = lib.lasp_chunk_states
    assert f(None, None, A, None, A, 1, 2, 256, 64, 64, BF16, None) == INVALID
    assert f(None, A, A, None, A, 1, 2, 256, 64, 48, BF16, None) == INVALID   # 48 does not divide 256
    assert f(None, A, A + 2, None, A, 1, 2, 256, 64, 64, BF16, None) == MISALIGNED
    g = lib.lasp_chunk_dstates
    assert g(A, None, None, A, 1, 2, 256, 64, 64, BF16, None) == INVALID


def test_binding_marshals_only(lib):
    import inspect
    src = inspect.getsource(lasp)
    # the binding never falls back to torch arithmetic or to the oracle
    for forbidden in ("oracle", "einsum", "matmul", "cumsum", "@"):
        assert forbidden not in src.replace("@property", ""), forbidden
    assert ctypes.CDLL(lasp.library_path())


def test_bidir_rejects_bad_arguments(lib):
    f = lib.lasp_bidir_fwd
    assert f(A, A, A, A, 1, 2, 256, 64, BF16, A, None) == UNSUPPORTED      # d = 64
    assert f(A, A, A, A, 1, 2, 256, 128, F32, A, None) == UNSUPPORTED      # fp32
    assert f(A, A, A, A, 1, 2, 200, 128, BF16, A, None) == UNSUPPORTED     # N not a multiple of 128
    assert f(A, A, A, A, 0, 2, 256, 128, BF16, A, None) == INVALID
    assert f(A, A, A, A, 1, 2, 0, 128, BF16, None, None) == OK             # nothing to do
    assert f(A, A, A, A, 1, 2, 256, 128, BF16, None, None) == INVALID      # no workspace
    assert f(A, A, A + 8, A, 1, 2, 256, 128, BF16, A, None) == MISALIGNED
    g = lib.lasp_bidir_bwd
    assert g(A, A, A, A, A, A, A, 1, 2, 256, 128, BF16, A, None, None) == INVALID
    assert g(A, A, A, A, A, A, A, 1, 2, 256, 32, BF16, A, A, None) == UNSUPPORTED
    assert lasp.lasp_bidir_workspace_floats(1, 2, 256, 64) == 0
    assert lasp.lasp_bidir_state_offset(1, 2, 256, 64) == -1
    # segment states, then the [B, H, d, d] total, then its bf16 tiles
    n = lasp.lasp_bidir_workspace_floats(2, 3, 2048, 128)
    off = lasp.lasp_bidir_state_offset(2, 3, 2048, 128)
    assert off == 2 * 2 * 3 * 128 * 128   # two 1024-token segments
    assert n == off + 2 * 3 * 128 * 128 + 2 * 3 * 128 * 128 // 2


def test_gated_calls_reject_bad_arguments(lib):
    f = lib.lasp_gla_fwd
    assert f(A, A, A, A, A, 1, 2, 512, 64, 256, BF16, A, None, None) == UNSUPPORTED   # C > 128
    assert f(A, A, A, A, A, 1, 2, 512, 96, 64, BF16, A, None, None) == UNSUPPORTED    # d = 96
    assert f(A, A, A, A, A, 1, 2, 500, 64, 64, BF16, A, None, None) == INVALID        # C does not divide N
    assert f(A, A, A, None, A, 1, 2, 512, 64, 64, BF16, A, None, None) == INVALID     # no gates
    assert f(A, A, A, A, A, 1, 2, 512, 64, 64, BF16, None, None, None) == INVALID     # no cache
    assert f(A, A, A, A + 4, A, 1, 2, 512, 64, 64, F32, A, None, None) == MISALIGNED
    assert f(A, A, A, A, A, 1, 2, 0, 64, 64, F32, None, None, None) == OK             # nothing to do
    g = lib.lasp_gla_bwd
    assert g(A, A, A, A, A, A, A, A, None, 1, 2, 512, 64, 64, F32, A, A, None, None, None) == INVALID  # no dg
    assert g(A, A, A, A, A, A, A, A, A, 1, 2, 512, 64, 64, F32, A, None, None, None, None) == INVALID  # no ws
    assert g(A, A, A, A, A, A, A, A, A, 1, 2, 512, 64, 256, F32, A, A, None, None, None) == UNSUPPORTED
    s = lib.lasp_gla_chunk_states
    assert s(A, A, A, A, None, 1, 2, 512, 64, 64, F32, 2, None) == INVALID             # kind
    assert s(A, A, A, A, A + 4, 1, 2, 512, 64, 64, F32, 0, None) == MISALIGNED         # gsum
    p = lib.lasp_gla_state_prefix
    assert p(A, A, None, None, None, 1, 4, 2, 64, 0, None) == INVALID                  # no gsum
    assert p(A, A, A, None, None, 1, 4, 2, 64, 2, None) == INVALID                     # reverse
    assert p(None, None, None, None, None, 1, 0, 2, 64, 0, None) == OK                 # T = 0, no total
    assert lasp.lasp_gla_cache_floats(2, 3, 512, 64, 64) == 2 * 8 * 3 * 64 * 66 + 4
    assert lasp.lasp_gla_cache_floats(2, 3, 512, 64, 256) == -1


def test_split_calls_reject_bad_arguments(lib):
    fs, ff = lib.lasp_fwd_states, lib.lasp_fwd_finish
    assert fs(A, A, None, 1, 2, 512, 96, 64, BF16, A, None, None) == UNSUPPORTED         # d = 96
    assert fs(A, A, None, 1, 2, 500, 64, 64, BF16, A, None, None) == INVALID             # C does not divide N
    assert fs(A, A, None, 1, 2, 512, 64, 64, F32, None, None, None) == INVALID           # no cache
    assert fs(A, A, None, 1, 2, 512, 64, 64, F32, A, A + 4, None) == MISALIGNED          # total
    assert fs(None, None, None, 1, 2, 0, 64, 64, F32, None, None, None) == OK            # nothing to do
    assert ff(A, A, A, None, None, 1, 2, 512, 64, 64, F32, A, None, None) == INVALID     # no output
    assert ff(A, A, A, None, A, 1, 2, 0, 64, 64, F32, None, None, None) == OK
    bs, bf = lib.lasp_bwd_states, lib.lasp_bwd_finish
    assert bs(A, None, None, 1, 2, 512, 64, 64, F32, A, None, None) == INVALID           # no dout
    assert bf(A, A, A, None, A, A, A, A, 1, 2, 512, 64, 64, F32, A, None, None, None, None) == INVALID  # no ws
    assert bf(A, A, A, None, A, A, A, A, 1, 2, 512, 64, 64, F32, A, A, A + 4, None, None) == MISALIGNED


def test_softmax_calls_reject_bad_arguments(lib):
    """LASP-2H's softmax-attention calls validate on the host: types and sizes
    the tensor cores do not take, a query without its own key (q_offset + Nq >
    Nk), a scale that is not a positive finite number, missing or misaligned
    buffers; and calls with nothing to do return before any launch."""
    inf, nan = float("inf"), float("nan")
    f = lib.lasp_softmax_fwd
    #      q  k  v  o  lse  B  H  Nq   Nk   off  d    scale  dtype
    assert f(A, A, A, A, A, 1, 2, 256, 256, 0, 64, 0.125, BF16, None) == UNSUPPORTED   # d = 64
    assert f(A, A, A, A, A, 1, 2, 256, 256, 0, 128, 0.125, F32, None) == UNSUPPORTED   # fp32
    assert f(A, A, A, A, A, 1, 2, 256, 256, 0, 128, 0.125, 7, None) == INVALID         # no such type
    assert f(A, A, A, A, A, 0, 2, 256, 256, 0, 128, 0.125, BF16, None) == INVALID      # B = 0
    assert f(A, A, A, A, A, 1, 2, 256, 200, 0, 128, 0.125, BF16, None) == INVALID      # keys short
    assert f(A, A, A, A, A, 1, 2, 128, 256, 129, 128, 0.125, BF16, None) == INVALID    # offset past Nk
    assert f(A, A, A, A, A, 1, 2, 128, 256, -1, 128, 0.125, BF16, None) == INVALID     # negative offset
    for bad in (0.0, -0.125, inf, nan):
        assert f(A, A, A, A, A, 1, 2, 256, 256, 0, 128, bad, BF16, None) == INVALID, bad
    assert f(A, A, A, A, None, 1, 2, 256, 256, 0, 128, 0.125, BF16, None) == INVALID   # no lse
    assert f(A, A + 8, A, A, A, 1, 2, 256, 256, 0, 128, 0.125, BF16, None) == MISALIGNED
    assert f(None, None, None, None, None, 1, 2, 0, 256, 0, 128, 0.125, BF16, None) == OK  # no query
    g = lib.lasp_softmax_bwd
    #      q  k  v  o  lse dout dq dk dv delta  B  H  Nq   Nk   off  d    scale  dtype
    assert g(A, A, A, A, A, A, A, A, A, A, 1, 2, 256, 256, 0, 64, 0.125, BF16, None) == UNSUPPORTED
    assert g(A, A, A, A, A, A, A, A, A, A, 1, 2, 256, 200, 0, 128, 0.125, BF16, None) == INVALID
    assert g(A, A, A, A, A, A, A, None, A, A, 1, 2, 256, 256, 0, 128, 0.125, BF16, None) == INVALID  # no dk
    assert g(A, A, A, A, A, A, A, A, A, None, 1, 2, 256, 256, 0, 128, 0.125, BF16, None) == INVALID  # no delta
    assert g(A, A, A, A, A, A, A, A, A + 4, A, 1, 2, 256, 256, 0, 128, 0.125, BF16, None) == MISALIGNED
    assert g(A, A, A, A, A, A, A, A, A, A, 1, 2, 256, 256, 0, 128, nan, BF16, None) == INVALID
    # no key and no query: nothing to write
    assert g(None, A, A, None, None, None, None, A, A, None, 1, 2, 0, 0, 0, 128, 0.125, BF16, None) == OK


def test_per_chunk_calls_reject_bad_arguments(lib):
    """lasp_chunk_out (row a3 on given states) and lasp_chunk_grads (row a6)."""
    f = lib.lasp_chunk_out
    #        q  k  v  decay  P     o  B  H  N    d   C   dtype
    assert f(A, A, A, None, A, A, 1, 2, 512, 96, 64, BF16, None) == UNSUPPORTED        # d = 96
    assert f(A, A, A, None, A, A, 1, 2, 500, 64, 64, BF16, None) == INVALID            # C does not divide N
    assert f(A, A, A, None, A, A, 1, 2, 512, 64, 64, 9, None) == INVALID               # no such type
    assert f(A, A, A, None, None, A, 1, 2, 512, 64, 64, BF16, None) == INVALID         # no states
    assert f(A, A, A, A + 4, A, A, 1, 2, 512, 64, 64, BF16, None) == MISALIGNED        # decay
    assert f(None, None, None, None, None, None, 1, 2, 0, 64, 64, BF16, None) == OK    # empty
    g = lib.lasp_chunk_grads
    #        q  k  v  dout decay P  R     dq dk dv     B  H  N    d   C   dtype
    assert g(A, A, A, A, None, A, None, A, A, A, 1, 2, 512, 64, 64, BF16, None) == INVALID     # no R
    assert g(A, A, A, A, None, A, A, A, A, A + 8, 1, 2, 512, 64, 64, BF16, None) == MISALIGNED
    assert g(A, A, A, A, None, A, A, A, A, A, 0, 2, 512, 64, 64, BF16, None) == INVALID        # B = 0
    assert g(None, None, None, None, None, None, None, None, None, None, 1, 2, 0, 64, 64, F32, None) == OK


def test_noalloc_backward_rejects_on_the_host(lib):
    """lasp_bwd_noalloc checks sizes, pointers and its fixed workspace's limit
    (B (N / C) H d^2 4 bytes within LASP_NOALLOC_SCRATCH_BYTES) before it looks
    up the workspace on the device."""
    f = lib.lasp_bwd_noalloc
    #      q  k  v  decay dout dq dk dv  B  H  N     d    C    dtype cache dstate_in dinit
    assert f(A, A, A, None, A, A, A, A, 1, 2, 512, 96, 64, BF16, A, None, None, None) == UNSUPPORTED
    assert f(A, A, A, None, A, A, A, A, 1, 2, 500, 64, 64, BF16, A, None, None, None) == INVALID
    assert f(A, A, A, None, A, A, A, A, 1, 2, 512, 64, 64, BF16, None, None, None, None) == INVALID  # no cache
    assert f(A, A, A, None, A, A, A, A, 1, 2, 512, 64, 64, BF16, A, A + 4, None, None) == MISALIGNED
    # 1 x 16 heads x 64 chunks of 128 x 128 fp32 states: 64 MiB, beyond the array
    assert f(A, A, A, None, A, A, A, A, 1, 16, 8192, 128, 128, BF16, A, None, None, None) == UNSUPPORTED
    assert f(None, None, None, None, None, None, None, None, 1, 2, 0, 64, 64, BF16, None, None, None,
             None) == OK


def test_part_calls_reject_bad_arguments(lib):
    """The split calls restricted to part `part` of `nparts` of the (b, h)
    pairs: 0 <= part < nparts <= B H, and nparts > 1 only where both walks run
    (lasp_parts_ok)."""
    ok = lib.lasp_parts_ok
    assert ok(65536, 128, 128, BF16) == 1
    assert ok(1024, 64, 128, BF16) == 1          # chunks that divide the tile
    assert ok(1024, 128, 64, BF16) == 0          # d = 64: per-chunk kernels
    assert ok(1024, 128, 128, F32) == 0
    assert ok(320, 64, 128, BF16) == 0           # a ragged tile
    assert ok(0, 128, 128, BF16) == 0
    fs = lib.lasp_fwd_states_part
    #         k  v  decay B  H  N     d    C    dtype cache total part nparts
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, A, None, 0, 0, None) == INVALID      # nparts = 0
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, A, None, 4, 4, None) == INVALID      # part = nparts
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, A, None, -1, 2, None) == INVALID
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, A, None, 0, 5, None) == INVALID      # nparts > B H
    assert fs(A, A, None, 1, 4, 1024, 64, 128, BF16, A, None, 0, 2, None) == UNSUPPORTED   # not parts_ok
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, None, None, 0, 2, None) == INVALID   # no cache
    assert fs(A, A, None, 1, 4, 1024, 128, 128, BF16, A, A + 4, 1, 2, None) == MISALIGNED  # total
    bf = lib.lasp_bwd_finish_part
    #         q  k  v  decay dout dq dk dv  B  H  N     d    C    dtype cache ws   din   dinit part nparts
    assert bf(A, A, A, None, A, A, A, A, 1, 4, 1024, 128, 128, BF16, A, None, None, None, 0, 2,
              None) == INVALID                                                           # no workspace
    assert bf(A, A, A, None, A, A, A, A, 1, 4, 1024, 128, 128, BF16, A, A, None, A + 8, 1, 2,
              None) == MISALIGNED                                                        # dinit_state
    assert bf(A, A, A, None, A, A, A, A, 1, 4, 1024, 128, 128, BF16, A, A, None, None, 2, 2,
              None) == INVALID                                                           # part = nparts


def test_kernel_names_and_segment_length(lib):
    """The trace's kernel names are stable (bench.py keys its byte model on
    them), and lasp_segment_tokens is host arithmetic: about 1024 tokens, a
    multiple of the tile and of the chunk that divides N, or C off the walks."""
    names = {lasp.lasp_kernel_name(i) for i in range(64)}
    for n in ("segment_states_tc", "segment_scan", "fwd_walk_tc", "bwd_walk_tc", "state_scan", "chunk_states_tc",
              "chunk_out_tc", "chunk_bwd_tc", "gla_bwd_tc", "softmax_dkdv_tc", "softmax_dq_tc", "softmax_fwd_tc"):
        assert n in names, n
    assert lasp.lasp_kernel_name(-1) == "unknown"
    seg = lasp.lasp_segment_tokens
    assert seg(65536, 128, 128, BF16) == 1024
    assert seg(1152, 128, 128, BF16) == 384      # nine tiles: three segments of three
    assert seg(256, 64, 128, BF16) == 256
    assert seg(320, 64, 128, BF16) == 64         # not a multiple of the tile: per chunk
    assert seg(256, 64, 32, F32) == 64
    assert seg(100, 64, 128, BF16) == 0          # C does not divide N


def test_the_header_serves_a_plain_c_program(tmp_path, lib):
    """include/lasp.h compiles as strict C99, and a C program linked against
    the library calls it without torch: host-side calls that return before any
    CUDA call (sizes, validation, names)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "client.c"
    src.write_text(r"""
#include <stdio.h>
#include "lasp.h"
int main(void) {
  printf("%d\n", lasp_version() > 0);
  printf("%s\n", lasp_status_string(LASP_ERR_UNSUPPORTED));
  printf("%d\n", lasp_fwd(0, 0, 0, 0, 0, 1, 2, 512, 96, 64, LASP_BF16, 0, 0, 0));         /* d = 96 */
  printf("%d\n", lasp_fwd_states(0, 0, 0, 1, 2, 500, 64, 64, LASP_F32, 0, 0, 0));        /* C does not divide N */
  printf("%lld\n", (long long)lasp_gla_cache_floats(2, 3, 512, 64, 64));
  printf("%d\n", lasp_segment_tokens(65536, 128, 128, LASP_BF16));
  return 0;
}
""")
    exe = tmp_path / "client"
    libdir = os.path.dirname(lasp.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), "-L", libdir, "-llasp", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out == ["1", "LASP_ERR_UNSUPPORTED", str(UNSUPPORTED), str(INVALID), str(2 * 8 * 3 * 64 * 66 + 4),
                   str(lasp.lasp_segment_tokens(65536, 128, 128, BF16))]
