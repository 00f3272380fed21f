"""Plain fp64 CPU oracle for attention over a cross-layer shared KV cache.

TEST INFRASTRUCTURE ONLY. This package is the slow, obviously correct
definition the CUDA path is checked against. Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it. It shares no code with ``cross_layer_kv_shared_b200`` (no kernels,
headers, helpers or constants) and never imports it.

Modules
-------
``kvshare_ref``  layer-map resolution, K/V reconstruction for the three
                 sharing forms, softmax attention (decode and causal prefill),
                 stored-byte counts.
``router_ref``   attention statistics of a decode step (per-head entropy and
                 peak, per-kv-head attention mass each cached token receives)
                 and the fp32 router score that feeds the rank rule.
``encode_ref``   the write side of the low-rank form for one new token: shared
                 coefficients (bf16) from the pair's basis, each layer's residual
                 coordinates, in a stated fp32 order; a calibration basis fit.
``quant_ref``    the write side of the low-rank form: per-token rank routing and
                 symmetric int8 quantisation with an fp16 per-token scale,
                 evaluated in fp32 with correctly rounded IEEE operations.

Every function is pinned by tests under ``tests/`` against closed forms,
invariants, a library routine (torch SDPA in fp64) or high-precision brute force.
"""
from . import encode_ref, kvshare_ref, quant_ref, router_ref  # noqa: F401
