"""libmqkv: chunk-adaptive mixed-bitwidth KV cache for B200 (sm_100a).

The data path lives in the C-ABI shared library libmqkv.so (CUDA kernels in
csrc/); `mqkv` is its thin Python binding and `workloads` draws the seeded
synthetic inputs.  Importing the package does not load the CUDA library.
"""
__all__ = ["mqkv", "workloads"]
