"""Which kernels run: the library trace records every launch, so these tests
fail if a size silently takes another path (for example the CUDA-core kernels
where the tensor-core walk is expected)."""
import numpy as np
import pytest

from sequence_linear_attention_b200 import inputs as lasp_inputs
from gpu_helpers import run_fwd_bwd

pytestmark = pytest.mark.gpu


def _traced_names(inp, C):
    import sequence_linear_attention_b200 as lasp
    lasp.lasp_trace_enable(64)
    try:
        run_fwd_bwd(inp, C)
        return [n for n, _ in lasp.lasp_trace_read(64)]
    finally:
        lasp.lasp_trace_enable(0)


def test_bf16_d128_c128_runs_the_segment_walks():
    inp = lasp_inputs.make_inputs(1, 2048, 2, 128, seed=201, bf16=True, decayed=True)
    names = _traced_names(inp, 128)
    assert names == ["segment_states_tc", "segment_scan", "fwd_walk_tc",
                     "segment_states_tc", "segment_scan", "bwd_walk_tc"], names


def test_bf16_c64_runs_the_segment_walks():
    """Chunks that divide the 128-token tile walk too (the cache then holds each
    tile's entering state in the slot of the tile's first chunk)."""
    for C in (64, 32, 16):
        inp = lasp_inputs.make_inputs(1, 512, 2, 128, seed=202 + C, bf16=True, decayed=True)
        names = _traced_names(inp, C)
        assert names == ["segment_states_tc", "segment_scan", "fwd_walk_tc",
                         "segment_states_tc", "segment_scan", "bwd_walk_tc"], (C, names)


def test_bf16_c64_with_a_ragged_tile_runs_the_per_chunk_tensor_core_kernels():
    inp = lasp_inputs.make_inputs(1, 320, 2, 128, seed=202, bf16=True, decayed=True)
    names = _traced_names(inp, 64)
    assert names == ["chunk_states_tc", "state_scan", "chunk_out_tc",
                     "chunk_states_tc", "state_scan", "chunk_bwd_tc"], names


@pytest.mark.parametrize("d", [64, 32])
def test_bf16_small_heads_run_the_per_chunk_tensor_core_kernels(d):
    """d = 64 and 32: the tiles keep 128 features, zero past d."""
    for N, C in ((512, 128), (512, 64), (224, 32)):
        inp = lasp_inputs.make_inputs(1, N, 2, d, seed=205 + C + d, bf16=True, decayed=True)
        names = _traced_names(inp, C)
        assert names == ["chunk_states_tc", "state_scan", "chunk_out_tc",
                         "chunk_states_tc", "state_scan", "chunk_bwd_tc"], (d, N, C, names)


def test_bf16_chunks_off_the_16_grid_run_on_cuda_cores():
    inp = lasp_inputs.make_inputs(1, 96, 2, 64, seed=206, bf16=True, decayed=True)
    names = _traced_names(inp, 24)
    assert names == ["chunk_states_simt", "state_scan", "chunk_out_simt",
                     "chunk_states_simt", "state_scan", "chunk_bwd_simt"], names


def test_bf16_c256_runs_the_segment_walks():
    """Chunks of two tiles walk both ways: the forward leaves both tiles'
    entering states in the two halves of the chunk's cache slot."""
    inp = lasp_inputs.make_inputs(1, 1024, 2, 128, seed=203, bf16=True, decayed=True)
    names = _traced_names(inp, 256)
    assert names == ["segment_states_tc", "segment_scan", "fwd_walk_tc",
                     "segment_states_tc", "segment_scan", "bwd_walk_tc"], names


def test_bf16_c512_walks_forward_and_uses_cuda_cores_backward():
    inp = lasp_inputs.make_inputs(1, 1024, 2, 128, seed=203, bf16=True, decayed=True)
    names = _traced_names(inp, 512)
    assert names[:3] == ["segment_states_tc", "segment_scan", "fwd_walk_tc"], names
    assert names[3:] == ["chunk_states_tc", "state_scan", "chunk_bwd_simt"], names


def test_fp32_runs_on_cuda_cores():
    inp = lasp_inputs.make_inputs(1, 256, 2, 32, seed=204, bf16=False, decayed=False)
    names = _traced_names(inp, 64)
    assert names == ["chunk_states_simt", "state_scan", "chunk_out_simt",
                     "chunk_states_simt", "state_scan", "chunk_bwd_simt"], names


def test_segment_length():
    import sequence_linear_attention_b200 as lasp
    assert lasp.lasp_segment_tokens(65536, 128, 128, 1) == 1024
    assert lasp.lasp_segment_tokens(1152, 128, 128, 1) == 384   # 9 tiles: three segments of three
    assert lasp.lasp_segment_tokens(256, 64, 128, 1) == 256     # two tiles of four chunks
    assert lasp.lasp_segment_tokens(8192, 64, 128, 1) == 1024
    assert lasp.lasp_segment_tokens(320, 64, 128, 1) == 64      # N not a multiple of 128: per-chunk path
    assert lasp.lasp_segment_tokens(256, 64, 32, 0) == 64
    assert lasp.lasp_segment_tokens(100, 64, 128, 1) == 0       # C does not divide N
