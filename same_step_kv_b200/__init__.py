"""same_step_kv_b200: same-step KV chunk attention for B200 (sm_100a).

The compute path is the C-ABI library libpv.so (CUDA kernels for sm_100a);
`same_step_kv_b200.pv` is its thin Python binding.  Importing this package
loads nothing; importing `same_step_kv_b200.pv` loads the library and raises
if it has not been built.
"""
__all__ = ["pv", "synth"]
