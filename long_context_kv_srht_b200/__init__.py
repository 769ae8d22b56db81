"""B200-native ParisKV KV-cache retrieval path.

The compute path is the C-ABI library ``libpariskv.so`` (hand-written sm_100a CUDA kernels);
``long_context_kv_srht_b200.pariskv`` is the thin Python binding over it. Importing this
package does not load the library; importing ``pariskv`` does, and fails loudly when it is
missing.
"""
__all__ = ["pariskv", "workload"]
