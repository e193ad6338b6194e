"""CPU oracle for the chunk-adaptive mixed-bitwidth KV cache path.

TEST INFRASTRUCTURE ONLY: used by tests, the smoke check and the benchmark's
CPU-baseline leg.  The library's data path never imports it.
"""
