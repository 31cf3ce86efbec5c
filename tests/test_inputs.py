"""The seeded input generator: a shard of a sequence drawn on its own holds the
same values as the same rows of the whole sequence."""
import numpy as np

from sequence_linear_attention_b200 import inputs as lasp_inputs


def test_shard_rows_equal_the_rows_of_the_whole_tensor(monkeypatch):
    monkeypatch.setattr(lasp_inputs, "_BLOCK", 1 << 10)  # shards then cross block edges
    for bf16 in (True, False):
        full = lasp_inputs.make_inputs(2, 96, 3, 8, seed=5, bf16=bf16)
        for row0, rows in ((0, 96), (0, 32), (32, 32), (40, 17), (95, 1)):
            shard = lasp_inputs.make_shard_inputs(2, 96, 3, 8, seed=5, row0=row0, rows=rows, bf16=bf16)
            for n in ("q", "k", "v", "do"):
                assert np.array_equal(shard[n], full[n][:, row0:row0 + rows]), (bf16, row0, rows, n)
            assert np.array_equal(shard["lam"], full["lam"])
