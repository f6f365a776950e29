"""SAS gated block-sparse causal attention for one B200 (sm_100a).

The compute path is libsas.so (CUDA kernels behind the C ABI in include/sas.h);
`gated_block_sparse_b200.sas` is its Python binding and
`gated_block_sparse_b200.inputs` the seeded synthetic workloads.
"""
__all__ = ["sas", "inputs", "build"]
