"""Attention over a cross-layer shared KV cache on B200 (sm_100a).

The product is the C library ``libkvshare.so`` (C ABI in ``include/kvshare.h``);
``cross_layer_kv_shared_b200.kvshare`` is its ctypes binding. Importing this
package does not load the library; importing ``.kvshare`` does, and fails
loudly if it has not been built.
"""
