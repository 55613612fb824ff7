"""B200-native paged KV-cache decode attention (sm_100a CUDA behind a C ABI).

``paged_attention_decode_pkv_b200.pkv`` is the binding to the C-ABI library
``libpkv.so``; ``paged_attention_decode_pkv_b200.workloads`` makes seeded
synthetic inputs.  Importing the package itself loads nothing.
"""
__all__ = ["pkv", "workloads"]
