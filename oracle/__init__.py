"""CPU oracle of Echo's error-compensated 4-bit all-reduce.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check in
``__graft_entry__`` and by the CPU-baseline leg of ``bench.py``; never by
the product library.
"""
from .oracle import (SOURCE, CallResult, Oracle, Params, allreduce,  # noqa: F401
                     bf16_to_f32, build, compile_source, default, dequant,
                     f32_to_bf16, owner_of_columns, pack, quantize_group,
                     reduce_scatter, unpack)
